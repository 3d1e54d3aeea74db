// Router: fp32 logits (a1), softmax + top-k + renormalised gates (a2), and the
// per-expert histogram / exclusive scan / permutation (a3).
//
// The pages only say that each token's router picks a few experts and that only
// those experts are read (ossradar.top, Xolotl README, "How it works, in one
// paragraph").  The computation is the plain DeepSeek-style softmax top-k router:
// L = x Wr^T + b; the k largest logits (ties to the lower id) in descending order;
// gates = softmax over the k selected logits, which equals p_sel / sum p_sel.
//
// Decode (T <= 64): one launch.  E/2 CTAs stream the 7.3 MB fp32 router (four warps
// per expert row), compute the Z tables of the gate/up dequantiser, and the last
// CTA to finish (atomic ticket) does top-k, histogram, scan and permutation.
// Prefill: a tiled fp32 GEMM for the logits, a top-k kernel whose last CTA scans the
// per-chunk histograms, and a scatter kernel that writes perm/inv_perm per chunk.
// Ordering inside an expert is token ascending, made deterministic by processing the
// flattened (token, slot) pairs in order with warp match/ballot ranks.
#include "kernels.h"

namespace moe {
namespace {

__device__ inline float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ inline float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ inline float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Top-k of one token's logits held by a warp: v[j] = logit of expert lane + 32 j
// (-inf padding).  Writes ids / gates for lanes < k.  Ties go to the lower id.
__device__ void warp_topk(float (&v)[8], int k, int lane, int32_t* ids_out, float* gates_out) {
    float my_sel = 0.f;
    int my_id = 0;
    float zmax = 0.f;
    for (int r = 0; r < k; ++r) {
        float bv = v[0];
        int bi = lane;
#pragma unroll
        for (int j = 1; j < 8; ++j) {
            if (v[j] > bv) {          // strict: equal values keep the lower id (j ascending)
                bv = v[j];
                bi = lane + 32 * j;
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ov > bv || (ov == bv && oi < bi)) {
                bv = ov;
                bi = oi;
            }
        }
        if (r == 0) zmax = bv;
        if (lane == r) {
            my_sel = bv;
            my_id = bi;
        }
        if ((bi & 31) == lane) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (j == (bi >> 5)) v[j] = -INFINITY;
        }
    }
    float ex = lane < k ? expf(my_sel - zmax) : 0.f;
    float sum = warp_sum(ex);
    if (lane < k) {
        ids_out[lane] = my_id;
        gates_out[lane] = ex / sum;
    }
}

__device__ void load_logits_row(const float* row, int E, int lane, float (&v)[8]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        int e = lane + 32 * j;
        v[j] = e < E ? ldcg_f32(row + e) : -INFINITY;
    }
}

// Exclusive scan of s_cnt[0..E) into s_off[0..E] by one warp (E <= 256).
__device__ void warp_scan_counts(const int* s_cnt, int* s_off, int E, int lane) {
    int loc[8];
    int sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        int e = lane * 8 + j;
        loc[j] = e < E ? s_cnt[e] : 0;
        sum += loc[j];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    int run = incl - sum;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        int e = lane * 8 + j;
        if (e < E) s_off[e] = run;
        run += loc[j];
    }
    if (lane == 31) s_off[E] = incl;
}

// Ranks the flattened pairs [0, n) (ids in s_ids) into positions starting at
// s_run[e]; writes perm / inv_perm.  One warp; pair order = (token, slot) order.
__device__ void warp_scatter(const int32_t* ids, int pair0, int n, int* s_run, int32_t* perm, int32_t* inv_perm,
                             int lane) {
    const unsigned lt = (1u << lane) - 1u;
    for (int base = 0; base < n; base += 32) {
        int i = base + lane;
        bool valid = i < n;
        int e = valid ? ids[i] : -1 - lane;
        unsigned mask = __match_any_sync(0xffffffffu, e);
        int rank = __popc(mask & lt);
        int first = valid ? s_run[e] : 0;
        __syncwarp();
        if (valid && rank == 0) s_run[e] = first + __popc(mask);
        __syncwarp();
        if (valid) {
            int pos = first + rank;
            perm[pos] = pair0 + i;
            inv_perm[pair0 + i] = pos;
        }
    }
}

// Active expert list: experts with a nonzero count (ascending), then shared experts.
__device__ void warp_active(const int* s_cnt, int E, int S, int32_t* active, Ctrl* ctrl, int T, int lane) {
    int n = 0;
    for (int base = 0; base < E; base += 32) {
        int e = base + lane;
        bool on = e < E && s_cnt[e] > 0;
        unsigned m = __ballot_sync(0xffffffffu, on);
        if (on) active[n + __popc(m & ((1u << lane) - 1u))] = e;
        n += __popc(m);
    }
    if (lane < S) active[n + lane] = E + lane;
    if (lane == 0) {
        ctrl->n_active = n + S;
        ctrl->routed_T = T;
    }
}

// ---------------------------------------------------------------- Z tables
// The gate/up expert kernel feeds the MMA with "base + c" values straight out of the
// code words (no per-pair subtraction) and starts every 64-wide group's accumulator
// at -Z.  For token t and group G (elements x_e, e = 0..63 of the group):
//   Bx = sum_e lo_base(e) x_e,  Hx = sum_e hi_base(e) x_e,  Sx = sum_e x_e,
// with lo_base / hi_base the magic bases the expert kernel uses for the pair that
// holds element e (pair p = (e % 16) / 2):  lo 64,32,8,16,4,64,16,4 and
// hi 512,256,128,64,32,16,8,8.  Then for code offset o:
//   Z_ternary = Bx + Sx,  Z_q2 = Bx + 1.5 Sx,  Z_q3 = Bx + Hx + 3.5 Sx.
// Stored negated as zx[format][T][G] (the MMA's accumulator input).
__device__ void compute_z(const RouteArgs& p, int t, int Gi, int lane) {
    constexpr float kLo[8] = {64.f, 32.f, 8.f, 16.f, 4.f, 64.f, 16.f, 4.f};
    constexpr float kHi[8] = {512.f, 256.f, 128.f, 64.f, 32.f, 16.f, 8.f, 8.f};
    const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(p.x + (size_t)t * p.H + Gi * 64) + lane);
    const float x0 = bf16lo(v), x1 = bf16hi(v);
    const float bl = kLo[lane & 7], bh = kHi[lane & 7];
    float bx = fmaf(bl, x0, bl * x1), hx = fmaf(bh, x0, bh * x1), sx = x0 + x1;
    bx = warp_sum(bx);
    hx = warp_sum(hx);
    sx = warp_sum(sx);
    if (lane == 0) {
        const int G = p.H / 64;
        const size_t i = (size_t)t * G + Gi, plane = (size_t)p.T * G;
        p.zx[i] = -(bx + sx);
        p.zx[plane + i] = -fmaf(1.5f, sx, bx);
        p.zx[2 * plane + i] = -fmaf(3.5f, sx, bx + hx);
    }
}

__global__ void __launch_bounds__(256) route_xz_kernel(RouteArgs p) {
    const int G = p.H / 64;
    const int warp = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (warp < p.T * G) compute_z(p, warp / G, warp % G, lane);
}

// ---------------------------------------------------------------- decode router
// 2 experts per CTA, 4 warps per expert row (one K quarter each), 7 float4 loads in
// flight per lane; then the Z tables; the last CTA does top-k and the permutation.
__global__ void __launch_bounds__(256) route_small_kernel(RouteArgs p) {
    constexpr int U = 7;
    __shared__ float s_part[8][kSmallT];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int el = warp >> 2, q = warp & 3;
    const int e = blockIdx.x * 2 + el;
    const int q4 = p.H / 16;                     // float4 per K quarter
    if (e < p.E) {
        const float4* w4 = reinterpret_cast<const float4*>(p.Wr + (size_t)e * p.H) + q * q4;
        for (int tb = 0; tb < p.T; tb += 8) {
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0.f;
            for (int i0 = lane; i0 < q4; i0 += 32 * U) {
                float4 w[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int i = i0 + 32 * u;
                    w[u] = i < q4 ? __ldg(w4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (tb + j >= p.T) break;
                    const uint2* xr = reinterpret_cast<const uint2*>(p.x + (size_t)(tb + j) * p.H) + q * q4;
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int i = i0 + 32 * u;
                        if (i < q4) {
                            const uint2 xv = __ldg(xr + i);
                            acc[j] = fmaf(w[u].x, bf16lo(xv.x), acc[j]);
                            acc[j] = fmaf(w[u].y, bf16hi(xv.x), acc[j]);
                            acc[j] = fmaf(w[u].z, bf16lo(xv.y), acc[j]);
                            acc[j] = fmaf(w[u].w, bf16hi(xv.y), acc[j]);
                        }
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float v = warp_sum(acc[j]);
                if (lane == 0 && tb + j < p.T) s_part[warp][tb + j] = v;
            }
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 2 * p.T; i += blockDim.x) {
        const int l = i / p.T, t = i - l * p.T, ee = blockIdx.x * 2 + l;
        if (ee < p.E) {
            const float v = (s_part[4 * l][t] + s_part[4 * l + 1][t]) + (s_part[4 * l + 2][t] + s_part[4 * l + 3][t]);
            p.logits[(size_t)t * p.E + ee] = v + (p.bias ? p.bias[ee] : 0.f);
        }
    }
    {
        const int G = p.H / 64;
        for (int pr = blockIdx.x * 8 + warp; pr < p.T * G; pr += gridDim.x * 8) compute_z(p, pr / G, pr % G, lane);
    }
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&p.ctrl->route_ticket, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    __shared__ int32_t s_ids[kSmallT * 16];
    __shared__ int s_cnt[256];
    __shared__ int s_off[257];
    // top-k per token: warp w takes tokens w, w+8, ...
    for (int t = warp; t < p.T; t += 8) {
        float v[8];
        load_logits_row(p.logits + (size_t)t * p.E, p.E, lane, v);
        warp_topk(v, p.k, lane, p.r.topk_ids + (size_t)t * p.k, p.r.topk_w + (size_t)t * p.k);
        __syncwarp();
        if (lane < p.k) s_ids[t * p.k + lane] = p.r.topk_ids[(size_t)t * p.k + lane];
    }
    for (int i = threadIdx.x; i < 256; i += blockDim.x) s_cnt[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < p.T * p.k; i += blockDim.x) atomicAdd(&s_cnt[s_ids[i]], 1);
    __syncthreads();
    if (warp == 0) {
        warp_scan_counts(s_cnt, s_off, p.E, lane);
        __syncwarp();
        for (int i = lane; i < p.E; i += 32) {
            p.r.counts[i] = s_cnt[i];
            p.r.offsets[i] = s_off[i];
        }
        if (lane == 0) p.r.offsets[p.E] = s_off[p.E];
        __syncwarp();
        // s_off doubles as the running position per expert
        warp_scatter(s_ids, 0, p.T * p.k, s_off, p.r.perm, p.r.inv_perm, lane);
        warp_active(s_cnt, p.E, p.S, p.active, p.ctrl, p.T, lane);
        if (lane == 0) p.ctrl->route_ticket = 0;
    }
}

// ---------------------------------------------------------------- prefill router
constexpr int GBM = 64, GBN = 64, GBK = 32;

__global__ void __launch_bounds__(256) route_logits_gemm_kernel(RouteArgs p) {
    __shared__ float xs[GBK][GBM + 4];
    __shared__ float ws[GBK][GBN + 4];
    const int tid = threadIdx.x;
    const int t0 = blockIdx.x * GBM, e0 = blockIdx.y * GBN;
    const int ty = tid >> 4, tx = tid & 15;
    float acc[4][4] = {};
    const int lr = tid >> 2, lc = (tid & 3) * 8;
    for (int h0 = 0; h0 < p.H; h0 += GBK) {
        {
            int t = t0 + lr;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (t < p.T) v = __ldg(reinterpret_cast<const uint4*>(p.x + (size_t)t * p.H + h0 + lc));
            xs[lc + 0][lr] = bf16lo(v.x);
            xs[lc + 1][lr] = bf16hi(v.x);
            xs[lc + 2][lr] = bf16lo(v.y);
            xs[lc + 3][lr] = bf16hi(v.y);
            xs[lc + 4][lr] = bf16lo(v.z);
            xs[lc + 5][lr] = bf16hi(v.z);
            xs[lc + 6][lr] = bf16lo(v.w);
            xs[lc + 7][lr] = bf16hi(v.w);
            int e = e0 + lr;
            float4 a = make_float4(0, 0, 0, 0), b = a;
            if (e < p.E) {
                const float4* src = reinterpret_cast<const float4*>(p.Wr + (size_t)e * p.H + h0 + lc);
                a = __ldg(src);
                b = __ldg(src + 1);
            }
            ws[lc + 0][lr] = a.x;
            ws[lc + 1][lr] = a.y;
            ws[lc + 2][lr] = a.z;
            ws[lc + 3][lr] = a.w;
            ws[lc + 4][lr] = b.x;
            ws[lc + 5][lr] = b.y;
            ws[lc + 6][lr] = b.z;
            ws[lc + 7][lr] = b.w;
        }
        __syncthreads();
        // two-level sum: each 32-wide K slice is summed on its own, then added to the
        // running total, so rounding grows with H/32 additions rather than H
        float part[4][4] = {};
#pragma unroll 8
        for (int kk = 0; kk < GBK; ++kk) {
            float4 a = *reinterpret_cast<const float4*>(&xs[kk][ty * 4]);
            float4 b = *reinterpret_cast<const float4*>(&ws[kk][tx * 4]);
            float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) part[i][j] = fmaf(av[i], bv[j], part[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] += part[i][j];
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int t = t0 + ty * 4 + i;
        if (t >= p.T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int e = e0 + tx * 4 + j;
            if (e < p.E) p.logits[(size_t)t * p.E + e] = acc[i][j] + (p.bias ? p.bias[e] : 0.f);
        }
    }
}

__global__ void __launch_bounds__(256) route_topk_kernel(RouteArgs p) {
    __shared__ int s_cnt[256];
    __shared__ int s_last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) s_cnt[i] = 0;
    __syncthreads();
    const int tend = min(p.T, (c + 1) * kChunk);
    for (int t = c * kChunk + warp; t < tend; t += 8) {
        float v[8];
        load_logits_row(p.logits + (size_t)t * p.E, p.E, lane, v);
        warp_topk(v, p.k, lane, p.r.topk_ids + (size_t)t * p.k, p.r.topk_w + (size_t)t * p.k);
        __syncwarp();
        if (lane < p.k) atomicAdd(&s_cnt[p.r.topk_ids[(size_t)t * p.k + lane]], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) p.hist[(size_t)c * p.E + e] = s_cnt[e];
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&p.ctrl->topk_ticket, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // last CTA: per-expert exclusive scan over chunks, totals, offsets, chunk bases
    const int nchunks = gridDim.x;
    __shared__ int s_off[257];
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
        int run = 0;
        for (int q = 0; q < nchunks; ++q) {
            int* h = p.hist + (size_t)q * p.E + e;
            int v = __ldcg(h);
            *h = run;
            run += v;
        }
        s_cnt[e] = run;
    }
    __syncthreads();
    if (warp == 0) warp_scan_counts(s_cnt, s_off, p.E, lane);
    __syncthreads();
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
        p.r.counts[e] = s_cnt[e];
        p.r.offsets[e] = s_off[e];
        for (int q = 0; q < nchunks; ++q) p.hist[(size_t)q * p.E + e] += s_off[e];
    }
    if (threadIdx.x == 0) p.r.offsets[p.E] = s_off[p.E];
    if (warp == 0) {
        warp_active(s_cnt, p.E, p.S, p.active, p.ctrl, p.T, lane);
        if (lane == 0) p.ctrl->topk_ticket = 0;
    }
}

__global__ void __launch_bounds__(32) route_scatter_kernel(RouteArgs p) {
    __shared__ int s_run[256];
    const int c = blockIdx.x, lane = threadIdx.x;
    for (int e = lane; e < p.E; e += 32) s_run[e] = p.hist[(size_t)c * p.E + e];
    __syncwarp();
    const int t0 = c * kChunk, t1 = min(p.T, t0 + kChunk);
    warp_scatter(p.r.topk_ids + (size_t)t0 * p.k, t0 * p.k, (t1 - t0) * p.k, s_run, p.r.perm, p.r.inv_perm, lane);
}

}  // namespace

cudaError_t launch_route(const RouteArgs& a, cudaStream_t s) {
    if (a.T <= kSmallT) {
        route_small_kernel<<<(a.E + 1) / 2, 256, 0, s>>>(a);
        return cudaGetLastError();
    }
    const int zwarps = a.T * (a.H / 64);
    route_xz_kernel<<<(zwarps + 7) / 8, 256, 0, s>>>(a);
    dim3 g1((a.T + GBM - 1) / GBM, (a.E + GBN - 1) / GBN);
    route_logits_gemm_kernel<<<g1, 256, 0, s>>>(a);
    const int nchunks = (a.T + kChunk - 1) / kChunk;
    route_topk_kernel<<<nchunks, 256, 0, s>>>(a);
    route_scatter_kernel<<<nchunks, 32, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
