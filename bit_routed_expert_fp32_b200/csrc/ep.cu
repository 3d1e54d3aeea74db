// Row kernels of expert parallelism (the layer's experts split over several GPUs): the
// gather that builds the dispatch buffer of token rows in routed (expert-major) order,
// and the gate-weighted combine of the expert output rows that come back.  The
// exchanges themselves are NCCL all-to-alls issued by the caller; these kernels only
// touch this GPU's memory.
//
// The pages mention running the engine on several consumer GPUs (molayo1419.me, "Delta
// Inference Engine", the multi-GPU paragraph); with experts partitioned over GPUs each
// token row travels to the GPUs that hold its selected experts and the outputs travel
// back, which is what these kernels bracket.
#include "kernels.h"

namespace moe {
namespace {

// dst[i][:] = src[index[i] / div][:], bf16 rows of H elements; one CTA per row.
__global__ void __launch_bounds__(128) gather_rows_kernel(int n, int H, const uint16_t* src, const int32_t* index,
                                                          int div, int n_src, uint16_t* dst, Ctrl* ctrl) {
    const int i = blockIdx.x;
    if (i >= n) return;
    const int r = __ldg(index + i) / div;
    if (r < 0 || r >= n_src) {                 // an index past the source: reported, row zeroed
        if (threadIdx.x == 0) report_error(ctrl, MOE_ERR_DEVICE_CHECK, kDetRange | 3);
        for (int c = threadIdx.x; c < H / 8; c += blockDim.x)
            reinterpret_cast<uint4*>(dst + (size_t)i * H)[c] = make_uint4(0, 0, 0, 0);
        return;
    }
    const uint4* s = reinterpret_cast<const uint4*>(src + (size_t)r * H);
    uint4* d = reinterpret_cast<uint4*>(dst + (size_t)i * H);
    for (int c = threadIdx.x; c < H / 8; c += blockDim.x) d[c] = __ldg(s + c);
}

// y[t][:] = sum_j g[t][j] * rows[inv_perm[t k + j]][:] (j ascending) + shared[t][:]: fp32
// rows (the experts' outputs as moe_forward returns them with MOE_OUT_F32), fp32 sums,
// stored as bf16; one thread per 4 consecutive outputs.
__global__ void __launch_bounds__(256) combine_pairs_kernel(int T, int k, int H, int n_rows, const float* rows,
                                                            const int32_t* inv_perm, const float* gates,
                                                            const float* shared, uint16_t* y, Ctrl* ctrl) {
    const int per_tok = H / 4;
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (size_t)T * per_tok) return;
    const int t = (int)(idx / per_tok), c4 = (int)(idx - (size_t)t * per_tok) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
        const int r = __ldg(inv_perm + (size_t)t * k + j);
        if (r < 0 || r >= n_rows) {                // reported, left out of the sum
            report_error(ctrl, MOE_ERR_DEVICE_CHECK, kDetRange | 4);
            continue;
        }
        const float g = __ldg(gates + (size_t)t * k + j);
        const float4 v = __ldg(reinterpret_cast<const float4*>(rows + (size_t)r * H + c4));
        acc.x = fmaf(g, v.x, acc.x);
        acc.y = fmaf(g, v.y, acc.y);
        acc.z = fmaf(g, v.z, acc.z);
        acc.w = fmaf(g, v.w, acc.w);
    }
    if (shared) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(shared + (size_t)t * H + c4));
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
    }
    uint2 o;
    o.x = (uint32_t)f32_to_bf16_bits(acc.x) | ((uint32_t)f32_to_bf16_bits(acc.y) << 16);
    o.y = (uint32_t)f32_to_bf16_bits(acc.z) | ((uint32_t)f32_to_bf16_bits(acc.w) << 16);
    *reinterpret_cast<uint2*>(y + (size_t)t * H + c4) = o;
}

}  // namespace

cudaError_t launch_gather_rows(int n, int H, const uint16_t* src, const int32_t* index, int div, int n_src,
                               uint16_t* dst, Ctrl* ctrl, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    gather_rows_kernel<<<n, 128, 0, s>>>(n, H, src, index, div, n_src, dst, ctrl);
    return cudaGetLastError();
}

cudaError_t launch_combine_pairs(int T, int k, int H, int n_rows, const float* rows, const int32_t* inv_perm,
                                 const float* gates, const float* shared, uint16_t* y, Ctrl* ctrl, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    const long long n = (long long)T * (H / 4);
    combine_pairs_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(T, k, H, n_rows, rows, inv_perm, gates, shared, y,
                                                                    ctrl);
    return cudaGetLastError();
}

}  // namespace moe
