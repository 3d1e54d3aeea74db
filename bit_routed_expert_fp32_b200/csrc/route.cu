// Router: fp32 logits, softmax + top-k + renormalised gates, and the per-expert
// histogram / exclusive scan / permutation.
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
// Prefill: a tensor-core logits GEMM (fp32 router split exactly into three bf16
// pieces), a top-k kernel whose last CTA scans the per-chunk histograms, and a
// scatter kernel that writes perm/inv_perm per chunk.
// Ordering inside an expert is token ascending, made deterministic by processing the
// flattened (token, slot) pairs in order with warp match/ballot ranks.
#include "kernels.h"
#include "operands.cuh"

namespace moe {
namespace {

__device__ inline float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ inline float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Double-float sums (a value is hi + lo, two fp32 numbers) with the exact two-sum
// (Knuth: s = a + b and the rounding error of that addition, both in fp32): the
// relative error of a sum of n terms is about n 2^-48 of the sum of their magnitudes.
// The decode router forms each thread's share of a logit (28 products of an fp32
// weight and a bf16 token) with fp32 fmas and adds the shares across the CTA in
// double-float, so the logit carries the rounding of 28-term partial sums only, at
// fp32 arithmetic rates (the fp64 units of this part are a small fraction of its fp32
// ones, and a double-float product costs a dozen fp32 operations).
struct Df {
    float hi, lo;
};
// (explicitly rounded operations: the compiler must not fuse or reorder them)
__device__ __forceinline__ void two_sum(float a, float b, float& s, float& err) {
    s = __fadd_rn(a, b);
    const float bp = __fsub_rn(s, a);
    err = __fadd_rn(__fsub_rn(a, __fsub_rn(s, bp)), __fsub_rn(b, bp));
}
__device__ __forceinline__ Df df_add(Df a, Df b) {
    Df r;
    float err;
    two_sum(a.hi, b.hi, r.hi, err);
    r.lo = __fadd_rn(__fadd_rn(a.lo, b.lo), err);
    return r;
}
// Kahan's compensated sum: a.hi the sum, a.lo minus the compensation (the low-order
// part the next addition must still add).
__device__ __forceinline__ void kahan_add(Df& a, float v) {
    const float y = __fadd_rn(v, a.lo);
    const float t = __fadd_rn(a.hi, y);
    a.lo = __fsub_rn(y, __fsub_rn(t, a.hi));
    a.hi = t;
}
// every lane ends with the same sum (the exact two-sum is symmetric in its arguments)
__device__ inline Df warp_sum_df(Df v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        Df w;
        w.hi = __shfl_xor_sync(0xffffffffu, v.hi, o);
        w.lo = __shfl_xor_sync(0xffffffffu, v.lo, o);
        v = df_add(v, w);
    }
    return v;
}

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
// An id outside [0, E) (only possible with caller-given routing, which reports it) takes
// no position; its pair's inv_perm entry is set to 0 so that readers stay in bounds.
// dedup_k > 0 (caller-given routing, k = dedup_k): an id that an earlier slot of the same
// token already holds is left out as an invalid one is (the range starts on a token).
__device__ void warp_scatter(const int32_t* ids, int pair0, int n, int* s_run, int32_t* perm, int32_t* inv_perm,
                             int lane, int E, int dedup_k = 0) {
    const unsigned lt = (1u << lane) - 1u;
    for (int base = 0; base < n; base += 32) {
        int i = base + lane;
        int e = i < n ? ids[i] : -1;
        bool valid = i < n && e >= 0 && e < E;
        if (valid && dedup_k > 1) {
            const int sl = (pair0 + i) % dedup_k;
            for (int j = 0; j < sl; ++j)
                if (ids[i - sl + j] == e) valid = false;
        }
        if (i < n && !valid) inv_perm[pair0 + i] = 0;
        if (!valid) e = -1 - lane;
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

__global__ void __launch_bounds__(256) route_xz_kernel(RouteArgs p) {
    if (blockIdx.x == 0 && threadIdx.x == 0) {          // no expert pass of this workspace runs now
        p.ctrl->work[0] = 0;
        p.ctrl->work[1] = 0;
    }
    const int G8 = 8 * ((p.H / 64 + 7) / 8);
    const int warp = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (p.ops && warp < p.T * G8) {
        const OperandArgs o{p.T, p.H, p.x, p.zx, p.iq, p.ctrl};
        compute_z(o, warp / G8, warp % G8, lane);
        if (p.iq) compute_iq(o, warp / G8, warp % G8, lane);
    }
}

// ---------------------------------------------------------------- decode router
// Top-k of one token by one warp with 32-bit reductions: lane l holds the logits of
// experts 8l .. 8l+7 (v[j], -inf padding) as order-preserving keys; each round takes
// the largest key over the warp (redux.sync), the lowest lane holding it and, inside
// that lane, the lowest j, so equal logits go to the lower expert id.  Writes ids and
// renormalised gates for slots < k to ids_out / gates_out and to s_ids (shared).
__device__ inline uint32_t order_key(float f) {
    const uint32_t b = f == 0.f ? 0u : __float_as_uint(f);          // -0 and +0 are equal
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ void warp_topk_redux(const float (&v)[8], int k, int lane, int32_t* ids_out, float* gates_out,
                                int32_t* s_ids) {
    uint32_t key[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) key[j] = v[j] == -INFINITY ? 0u : order_key(v[j]);
    float my_sel = 0.f, top = 0.f;
    int my_id = 0;
    for (int r = 0; r < k; ++r) {
        uint32_t bk = key[0];
        int bj = 0;
#pragma unroll
        for (int j = 1; j < 8; ++j)
            if (key[j] > bk) {              // strict: an equal key keeps the lower j
                bk = key[j];
                bj = j;
            }
        const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
        const int wl = __ffs(__ballot_sync(0xffffffffu, bk == m)) - 1;
        const int wj = __shfl_sync(0xffffffffu, bj, wl);
        float val = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j == bj) val = v[j];
        val = __shfl_sync(0xffffffffu, val, wl);
        if (r == 0) top = val;
        if (lane == r) {
            my_sel = val;
            my_id = 8 * wl + wj;
        }
        if (lane == wl) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (j == wj) key[j] = 0u;
        }
    }
    const float ex = lane < k ? expf(my_sel - top) : 0.f;
    const float sum = warp_sum(ex);
    if (lane < k) {
        ids_out[lane] = my_id;
        gates_out[lane] = ex / sum;
        s_ids[lane] = my_id;
    }
}

// One CTA per expert row: 8 warps hold the whole fp32 row in registers (one load
// each, all in flight at once) and form its logit for every token, the tokens staged
// kRouteTB at a time in shared memory (one coalesced load of all of them, then
// shared-memory reads: a token's elements reach every thread without a chain of
// global-memory round trips); then the Z tables; the last CTA to finish (atomic
// ticket) does top-k, histogram, scan and the permutation.
constexpr int kRouteVec = 7;                           // float4 of the row per thread (H <= 7168)
constexpr int kRouteTB = 4;                            // tokens staged per round
constexpr int kRouteSlice = 256 * kRouteVec * 4;       // row elements per pass (7168)
constexpr size_t kRouteSmem = (size_t)kRouteTB * kRouteSlice * 2;   // 57,344 B

__global__ void __launch_bounds__(256) route_small_kernel(RouteArgs p) {
    griddep_launch_dependents();        // one wave of CTAs: the expert pass may start launching
    if (blockIdx.x == 0 && threadIdx.x == 0) {          // no expert pass of this workspace runs now
        p.ctrl->work[0] = 0;
        p.ctrl->work[1] = 0;
    }
    // fp32 fma partial sums of 28 products per thread, added across the CTA in
    // double-float (Df): the logit carries only the partial sums' rounding (tokens with
    // large outliers make long fp32 sums lose the bits that separate close logits)
    extern __shared__ __align__(16) uint8_t route_smem[];
    uint2* xs = reinterpret_cast<uint2*>(route_smem);   // [kRouteTB][kRouteSlice / 4]
    __shared__ Df s_part[8][kSmallT];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x;
    const int n4 = p.H / 4;                                        // float4 per row
    const float4* w4 = reinterpret_cast<const float4*>(p.Wr + (size_t)e * p.H);
    for (int i0 = 0; i0 < n4; i0 += 256 * kRouteVec) {
        float4 w[kRouteVec];
#pragma unroll
        for (int u = 0; u < kRouteVec; ++u) {
            const int i = i0 + threadIdx.x + 256 * u;
            w[u] = i < n4 ? __ldg(w4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (i0 == 0 && p.ops) {
            // the decode operands of (token, group) pairs, one per warp: formed while the
            // router row's loads are in flight
            const int G8 = 8 * ((p.H / 64 + 7) / 8);
            for (int pr = blockIdx.x * 8 + warp; pr < p.T * G8; pr += gridDim.x * 8) {
                const OperandArgs o{p.T, p.H, p.x, p.zx, p.iq, p.ctrl};
                compute_z(o, pr / G8, pr % G8, lane);
                if (p.iq) compute_iq(o, pr / G8, pr % G8, lane);
            }
        }
        const int n_el = min(kRouteSlice, p.H - 4 * i0);            // elements of this pass
        for (int tb = 0; tb < p.T; tb += kRouteTB) {
            const int nt = min(kRouteTB, p.T - tb);
            // stage tokens tb .. tb+nt-1, elements 4 i0 .. 4 i0 + n_el (8 per uint4)
            for (int q = threadIdx.x; q < nt * (n_el / 8); q += 256) {
                const int j = q / (n_el / 8), c = q - j * (n_el / 8);
                reinterpret_cast<uint4*>(xs)[j * (kRouteSlice / 8) + c] =
                    __ldg(reinterpret_cast<const uint4*>(p.x + (size_t)(tb + j) * p.H + 4 * i0) + c);
            }
            __syncthreads();
            float acc[kRouteTB];
#pragma unroll
            for (int j = 0; j < kRouteTB; ++j) acc[j] = 0.f;
#pragma unroll
            for (int u = 0; u < kRouteVec; ++u) {
                const int il = threadIdx.x + 256 * u;                // float4 index within the pass
                if (i0 + il < n4) {
#pragma unroll
                    for (int j = 0; j < kRouteTB; ++j) {
                        if (j < nt) {
                            const uint2 xv = xs[j * (kRouteSlice / 4) + il];
                            acc[j] = __fmaf_rn(w[u].x, bf16lo(xv.x), acc[j]);
                            acc[j] = __fmaf_rn(w[u].y, bf16hi(xv.x), acc[j]);
                            acc[j] = __fmaf_rn(w[u].z, bf16lo(xv.y), acc[j]);
                            acc[j] = __fmaf_rn(w[u].w, bf16hi(xv.y), acc[j]);
                        }
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < kRouteTB; ++j) {
                if (j >= nt) break;
                const Df v = warp_sum_df(Df{acc[j], 0.f});
                if (lane == 0) s_part[warp][tb + j] = i0 == 0 ? v : df_add(s_part[warp][tb + j], v);
            }
            __syncthreads();                                         // xs is refilled next round
        }
    }
    __syncthreads();
    for (int t = threadIdx.x; t < p.T; t += blockDim.x) {
        Df v = s_part[0][t];
#pragma unroll
        for (int w = 1; w < 8; ++w) v = df_add(v, s_part[w][t]);
        // the bias and the one final rounding (a few fp64 operations per logit)
        p.logits[(size_t)t * p.E + e] = (float)((double)v.hi + (double)v.lo + (p.bias ? (double)p.bias[e] : 0.0));
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
    for (int i = threadIdx.x; i < 256; i += blockDim.x) s_cnt[i] = 0;
    // top-k per token: warp w takes tokens w, w+8, ...
    for (int t = warp; t < p.T; t += 8) {
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int ee = 8 * lane + j;
            v[j] = ee < p.E ? ldcg_f32(p.logits + (size_t)t * p.E + ee) : -INFINITY;
        }
        warp_topk_redux(v, p.k, lane, p.r.topk_ids + (size_t)t * p.k, p.r.topk_w + (size_t)t * p.k,
                        s_ids + t * p.k);
    }
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
        warp_scatter(s_ids, 0, p.T * p.k, s_off, p.r.perm, p.r.inv_perm, lane, p.E);
        if (lane == 0) p.ctrl->route_ticket = 0;
    } else if (warp == 1) {
        warp_active(s_cnt, p.E, p.S, p.active, p.ctrl, p.T, lane);
    }
}

// ---------------------------------------------------------------- prefill router
// Router logits for many tokens on the tensor cores.  x is bf16 (exact); the fp32
// router weight is split exactly into three bf16 pieces w = w1 + w2 + w3 (each the
// bf16 rounding of what is left), so x.w1 + x.w2 + x.w3 with fp32 accumulation gives
// fp32-level logits (the dropped remainder is below 2^-24 |w|).  mma.sync m16n8k16,
// CTA tile 128 tokens x 64 experts x 32 K, 8 warps of 32 x 32, double-buffered smem.
constexpr int RBM = 128, RBN = 64, RBK = 32, RPAD = 40;   // smem row: 32 bf16 + 8 pad

__device__ inline uint32_t pack_bf16x2(float lo, float hi) {
    return (uint32_t)f32_to_bf16_bits(lo) | ((uint32_t)f32_to_bf16_bits(hi) << 16);
}

__device__ inline void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

constexpr size_t kRouteMmaSmem = (size_t)2 * RBM * RPAD * 2 + (size_t)2 * 3 * RBN * RPAD * 2;   // 51,200 B

__global__ void __launch_bounds__(256) route_logits_mma_kernel(RouteArgs p) {
    extern __shared__ __align__(16) uint8_t rsm[];
    auto xs = reinterpret_cast<uint16_t(*)[RBM][RPAD]>(rsm);
    auto ws = reinterpret_cast<uint16_t(*)[3][RBN][RPAD]>(rsm + (size_t)2 * RBM * RPAD * 2);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = blockIdx.x * RBM, e0 = blockIdx.y * RBN;
    const int wm = warp >> 1, wn = warp & 1;            // warp tile: tokens 32wm.., experts 32wn..
    // K-tile partials added with Kahan's compensated summation (hi, and lo = minus the
    // running compensation): four fp32 operations a partial instead of the eight of a
    // full two-sum, with an error ~2^-48 of the sum of the partials' magnitudes
    Df acc[2][4][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[a][b][c] = Df{0.f, 0.f};

    // loaders: x tile 128 x 32 bf16 = 512 x 16 B (2 per thread); w tile 64 x 32 fp32 (8 floats per thread)
    uint4 xr[2];
    float4 wr[2];
    auto load = [&](int h0) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int idx = tid + 256 * u, row = idx >> 2, c = (idx & 3) * 8;
            const int t = t0 + row;
            xr[u] = t < p.T ? __ldg(reinterpret_cast<const uint4*>(p.x + (size_t)t * p.H + h0 + c))
                            : make_uint4(0, 0, 0, 0);
        }
        const int row = tid >> 2, c = (tid & 3) * 8, e = e0 + row;
        if (e < p.E) {
            const float4* src = reinterpret_cast<const float4*>(p.Wr + (size_t)e * p.H + h0 + c);
            wr[0] = __ldg(src);
            wr[1] = __ldg(src + 1);
        } else {
            wr[0] = wr[1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    auto store = [&](int buf) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int idx = tid + 256 * u, row = idx >> 2, c = (idx & 3) * 8;
            *reinterpret_cast<uint4*>(&xs[buf][row][c]) = xr[u];
        }
        const int row = tid >> 2, c = (tid & 3) * 8;
        const float w[8] = {wr[0].x, wr[0].y, wr[0].z, wr[0].w, wr[1].x, wr[1].y, wr[1].z, wr[1].w};
        float r1[8], r2[8], r3[8];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            r1[v] = __uint_as_float((uint32_t)f32_to_bf16_bits(w[v]) << 16);
            const float rem = w[v] - r1[v];
            r2[v] = __uint_as_float((uint32_t)f32_to_bf16_bits(rem) << 16);
            r3[v] = rem - r2[v];
        }
        *reinterpret_cast<uint4*>(&ws[buf][0][row][c]) =
            make_uint4(pack_bf16x2(r1[0], r1[1]), pack_bf16x2(r1[2], r1[3]), pack_bf16x2(r1[4], r1[5]),
                       pack_bf16x2(r1[6], r1[7]));
        *reinterpret_cast<uint4*>(&ws[buf][1][row][c]) =
            make_uint4(pack_bf16x2(r2[0], r2[1]), pack_bf16x2(r2[2], r2[3]), pack_bf16x2(r2[4], r2[5]),
                       pack_bf16x2(r2[6], r2[7]));
        *reinterpret_cast<uint4*>(&ws[buf][2][row][c]) =
            make_uint4(pack_bf16x2(r3[0], r3[1]), pack_bf16x2(r3[2], r3[3]), pack_bf16x2(r3[4], r3[5]),
                       pack_bf16x2(r3[6], r3[7]));
    };

    const int nk = p.H / RBK;
    load(0);
    store(0);
    __syncthreads();
    for (int kt = 0; kt < nk; ++kt) {
        const int buf = kt & 1;
        if (kt + 1 < nk) load((kt + 1) * RBK);
        // The MMA rounds its fp32 accumulator towards zero; chaining all of K through it
        // would let that bias grow with H.  Each 32-wide K tile is therefore summed in a
        // fresh accumulator and added to the total with round-to-nearest adds.
        float part[2][4][4];
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) part[a][b][0] = part[a][b][1] = part[a][b][2] = part[a][b][3] = 0.f;
#pragma unroll
        for (int k16 = 0; k16 < RBK; k16 += 16) {
            uint32_t af[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                // A 16x16 (tokens x k): lanes 0-15 rows 0-15 at k, lanes 16-31 rows 0-15 at k+8
                const int r = 32 * wm + 16 * mt + (lane & 15), cc = k16 + 8 * (lane >> 4);
                ldsm_x4(smem_u32(&xs[buf][r][cc]), af[mt][0], af[mt][1], af[mt][2], af[mt][3]);
            }
#pragma unroll
            for (int pl = 0; pl < 3; ++pl) {
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    // two n8 tiles of B (experts x k): matrices (n 0-7, k), (n 0-7, k+8), (n 8-15, k), (n 8-15, k+8)
                    const int r = 32 * wn + 16 * np + (lane & 7) + 8 * (lane >> 4), cc = k16 + 8 * ((lane >> 3) & 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(smem_u32(&ws[buf][pl][r][cc]), b0, b1, b2, b3);
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt) {
                        mma_bf16_16816(part[mt][2 * np][0], part[mt][2 * np][1], part[mt][2 * np][2],
                                       part[mt][2 * np][3], af[mt][0], af[mt][1], af[mt][2], af[mt][3], b0, b1);
                        mma_bf16_16816(part[mt][2 * np + 1][0], part[mt][2 * np + 1][1], part[mt][2 * np + 1][2],
                                       part[mt][2 * np + 1][3], af[mt][0], af[mt][1], af[mt][2], af[mt][3], b2, b3);
                    }
                }
            }
        }
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b)
#pragma unroll
                for (int c = 0; c < 4; ++c) kahan_add(acc[a][b][c], part[a][b][c]);
        if (kt + 1 < nk) store(buf ^ 1);
        __syncthreads();
    }
    const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int t = t0 + 32 * wm + 16 * mt + g + 8 * h;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int e = e0 + 32 * wn + 8 * nt + 2 * t4 + c;
                    if (t < p.T && e < p.E)
                        p.logits[(size_t)t * p.E + e] =
                            (float)((double)acc[mt][nt][2 * h + c].hi + (double)acc[mt][nt][2 * h + c].lo +
                                    (p.bias ? (double)p.bias[e] : 0.0));
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
        if (p.fixed_ids) {
            // caller-given routing: copied; an id outside [0, E), or one an earlier slot of
            // the token holds already, is reported and counted nowhere (its pair is left out
            // of the permutation's expert ranges), so no expert has more than T rows
            const size_t i = (size_t)t * p.k + lane;
            const int id = lane < p.k ? __ldg(p.fixed_ids + i) : -1 - lane;
            const unsigned same = __match_any_sync(0xffffffffu, id);
            if (lane < p.k) {
                p.r.topk_ids[i] = id;
                p.r.topk_w[i] = __ldg(p.fixed_w + i);
                if (id < 0 || id >= p.E) report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetRange | 2);
                else if (same & ((1u << lane) - 1u)) report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetRange | 5);
                else atomicAdd(&s_cnt[id], 1);
            }
            continue;
        }
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
    // last CTA: per-expert totals over the chunks, the exclusive scan over experts, then
    // each chunk's base in each expert's range (offset + the expert's rows in earlier
    // chunks).  A thread reads its expert's column 16 chunks at a time (independent
    // loads, one L2 round trip per 16 chunks).
    const int nchunks = gridDim.x;
    __shared__ int s_off[257];
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
        int run = 0;
        for (int q0 = 0; q0 < nchunks; q0 += 16) {
            int v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) v[u] = q0 + u < nchunks ? __ldcg(p.hist + (size_t)(q0 + u) * p.E + e) : 0;
#pragma unroll
            for (int u = 0; u < 16; ++u) run += v[u];
        }
        s_cnt[e] = run;
    }
    __syncthreads();
    if (warp == 0) warp_scan_counts(s_cnt, s_off, p.E, lane);
    __syncthreads();
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
        p.r.counts[e] = s_cnt[e];
        p.r.offsets[e] = s_off[e];
        int run = s_off[e];
        for (int q0 = 0; q0 < nchunks; q0 += 16) {
            int v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) v[u] = q0 + u < nchunks ? __ldcg(p.hist + (size_t)(q0 + u) * p.E + e) : 0;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                if (q0 + u < nchunks) p.hist[(size_t)(q0 + u) * p.E + e] = run;
                run += v[u];
            }
        }
    }
    if (threadIdx.x == 0) p.r.offsets[p.E] = s_off[p.E];
    if (warp == 0) {
        warp_active(s_cnt, p.E, p.S, p.active, p.ctrl, p.T, lane);
        if (lane == 0) p.ctrl->topk_ticket = 0;
    }
}

__global__ void __launch_bounds__(32) route_scatter_kernel(RouteArgs p) {
    griddep_launch_dependents();        // one wave of CTAs: the expert pass may start launching
    __shared__ int s_run[256];
    const int c = blockIdx.x, lane = threadIdx.x;
    for (int e = lane; e < p.E; e += 32) s_run[e] = p.hist[(size_t)c * p.E + e];
    __syncwarp();
    const int t0 = c * kChunk, t1 = min(p.T, t0 + kChunk);
    warp_scatter(p.r.topk_ids + (size_t)t0 * p.k, t0 * p.k, (t1 - t0) * p.k, s_run, p.r.perm, p.r.inv_perm, lane,
                 p.E, p.fixed_ids ? p.k : 0);
}

}  // namespace

cudaError_t launch_decode_operands(const RouteArgs& a, cudaStream_t s) {
    const int zwarps = a.T * 8 * ((a.H / 64 + 7) / 8);
    route_xz_kernel<<<(zwarps + 7) / 8, 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_route_fixed(const RouteArgs& a, cudaStream_t s) {
    if (a.ops) {
        const int zwarps = a.T * 8 * ((a.H / 64 + 7) / 8);
        route_xz_kernel<<<(zwarps + 7) / 8, 256, 0, s>>>(a);
    }
    const int nchunks = (a.T + kChunk - 1) / kChunk;
    route_topk_kernel<<<nchunks, 256, 0, s>>>(a);
    route_scatter_kernel<<<nchunks, 32, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t s) {
    if (a.T <= kSmallT) {
        const cudaError_t err = set_smem_limit(route_small_kernel, kRouteSmem);
        if (err != cudaSuccess) return err;
        route_small_kernel<<<a.E, 256, kRouteSmem, s>>>(a);
        return cudaGetLastError();
    }
    if (a.ops) {
        const int zwarps = a.T * 8 * ((a.H / 64 + 7) / 8);
        route_xz_kernel<<<(zwarps + 7) / 8, 256, 0, s>>>(a);
    }
    cudaError_t err = set_smem_limit(route_logits_mma_kernel, kRouteMmaSmem);
    if (err != cudaSuccess) return err;
    dim3 g1((a.T + RBM - 1) / RBM, (a.E + RBN - 1) / RBN);
    route_logits_mma_kernel<<<g1, 256, kRouteMmaSmem, s>>>(a);
    const int nchunks = (a.T + kChunk - 1) / kChunk;
    route_topk_kernel<<<nchunks, 256, 0, s>>>(a);
    route_scatter_kernel<<<nchunks, 32, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
