// Internal launcher interface between the C ABI (api.cu) and the kernels.
#pragma once
#include <utility>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace moe {

constexpr int kSmallT = 64;        // decode router / decode path threshold
constexpr int kChunk = 64;         // tokens per chunk of the large-T router (one CTA each)

struct RouteArgs {
    int T, H, E, k, S;
    const uint16_t* x;
    const float* Wr;
    const float* bias;
    float* logits;      // ws [T][E]
    int32_t* hist;      // ws [ceil(T/kChunk)][E]
    int32_t* active;    // ws [E+S]
    float* zx;          // ws fp16 planes [2][3][T][G8] of -Z/16, hi and lo (see route.cu)
    uint8_t* iq;        // ws integer operands of the tokens (T <= kFusedMaxT), else null
    int ops;            // form the decode operands (Z tables, integer operands) here
    const int32_t* fixed_ids;   // moe_route_fixed: the caller's expert ids [T][k] (else null)
    const float* fixed_w;       // moe_route_fixed: the caller's gates [T][k]
    Ctrl* ctrl;
    moe_routing r;
};

// K parts of the fused decode kernel (fused_kparts below)
struct FusedParts {
    int pg, pr, pd;
    int gsh_row0, gsh_rows;      // first row and number of rows with gate/up part sums
};

struct FfnArgs {
    int T, H, I, E, k, S;
    const uint8_t* packed;
    const uint16_t* x;       // bf16 [T][H]
    const int32_t* perm;
    const int32_t* inv_perm;
    const int32_t* counts;
    const int32_t* offsets;
    const float* topk_w;
    const int32_t* active;   // ws
    const float* zx;         // ws fp16 planes [2][3][T][G8] of -Z/16, hi and lo
    const uint8_t* iq;       // ws integer operands of the tokens (T <= kFusedMaxT), else null
    int iq_on;               // gate/up of ternary / 2-bit experts on the integer path
    Ctrl* ctrl;
    uint16_t* h;             // ws fp16 [T*(k+S)][I]
    float* ypart;            // ws f32 [nkp_dn][T*(k+S)][H]
    float* gpart;            // ws f32 [nkp_gu][T*(k+S)][2I] (aliases ypart; decode, nkp_gu > 1)
    int nkp_gu, nkp_dn;      // K parts of the decode gate/up and down passes (1 on the prefill path)
    uint32_t* tile_ctr;      // ws [H/16]
    uint16_t* y;             // bf16 [T][H], or fp32 [T][H] when y_f32
    int y_f32;               // the combine stores fp32 (MOE_OUT_F32)
    int num_ctas;
    FusedCtl* fc;            // ws: counters of the fused decode kernel
    uint32_t* dn_done;       // ws [H/16]: down tiles finished per 16-row slice of y (fused kernel)
    float* hf;               // ws fp32 [R16][I]: h of ternary / 2-bit experts (fused kernel)
    uint8_t* hq;             // ws integer operands of those h rows (iq_size(R16, I)); also the
                             // separate down launch's up to kIqMaxT tokens (the K-part reduction's)
    int R16;                 // rows those two regions hold: min(T, kFusedMaxT) (k + S)
    float* gsh;              // ws fp32 pairs [max(pg, pr)][gsh_rows][I] x {gate, up}: gate/up
                             // K-part sums (fused kernel; in the ypart region)
    uint32_t* gp_done;       // ws [fused_gp_counters]: K parts finished per split gate/up tile
    FusedParts fk;           // fused kernel K parts
};

// Workspace layout for T tokens (api.cu).  The control block, tile counters and the
// active-expert list sit at fixed offsets (independent of T).
struct Ws {
    size_t ctrl, tile_ctr, active, logits, hist, zx, iq, hf, hq, h, ypart, total;
};

// Integer-path operands of the fused decode kernel (operands.cuh, decode_fused.cu): per
// row (a token, or an h row of the down pass) and 64-group g (G groups, G8 = G padded to
// whole chunks), a 128-byte digit record [2 digits][4 lanes] x 16 bytes of the row's
// values on a 12-bit grid, then per (row, group) the pair {p = 2^-e / 4 (fp32),
// sum of q (int32)}:
//   digit records  [R][G] x 128 bytes         (offset 0)
//   pairs          [R][G8] x 8 bytes          (iq_pair_off)
// The fused decode kernel (decode_fused.cu) serves up to kFusedMaxT tokens.
constexpr int kFusedMaxT = 16;
// token counts for which MOE_PATH_AUTO / MOE_PATH_DECODE take the fused decode kernel,
// from the per-step times on the full-size layer, separate launches against the fused
// kernel: one token 90.3 against 101.7 us, two 121.0 against 147.2, three 144.2 against
// 152.4, four 182.4 against 184.3, eight 331.9 against 308.9, sixteen 525 against 535
// (451 against 562 with mixed formats and skewed routing)
constexpr int kFusedAutoMinT = 5, kFusedAutoMaxT = 8;
// token counts up to which the separate gate/up launch runs ternary and 2-bit experts on
// integer MMAs (two signed-byte digit columns per token fill one n8 tile at four tokens)
constexpr int kIqMaxT = 4;
__host__ __device__ inline size_t iq_pair_off(int64_t R, int64_t K) { return (size_t)R * (K / 64) * 128; }
__host__ __device__ inline size_t iq_size(int64_t R, int64_t K) {
    return iq_pair_off(R, K) + (size_t)8 * R * (8 * ((K / 64 + 7) / 8));
}
// Token operands, reserved for min(T, kFusedMaxT) tokens at every T >= 1 so that the
// workspace size never shrinks as T grows; used only when T <= kFusedMaxT.
inline size_t iq_bytes(int64_t T, int64_t H) {
    const int64_t t = T < kFusedMaxT ? T : kFusedMaxT;
    return t >= 1 ? iq_size(t, H) : 0;
}
Ws ws_layout(const moe_shape* s, int64_t T);

// Host-side argument checks of moe_route and moe_forward (api.cu); they enqueue nothing,
// so an entry point can run all of them before its first launch.
bool shape_ok(const moe_shape* s);
moe_status check_route_args(const moe_shape* shape, int32_t T, const uint16_t* d_x, const float* d_router_w,
                            const moe_routing* out, const void* d_ws, size_t ws_bytes);
struct ForwardPlan {
    bool prefill, fused;     // the tcgen05 kernels; the fused decode kernel; else the decode launches
    int nkp_gu, nkp_dn;      // K parts of the separate decode passes (1 otherwise)
    int launches;            // kernels of moe_route + moe_forward
};
moe_status plan_forward(const moe_shape* shape, int64_t T, moe_path path, ForwardPlan* fp);
moe_status check_forward_args(const moe_shape* shape, int32_t T, const void* d_packed, const uint16_t* d_x,
                              const moe_routing* r, const uint16_t* d_y, moe_path path, const void* d_ws,
                              size_t ws_bytes);

// K parts of the decode-path expert passes for T tokens.  With few tokens only a few
// experts are active and their 32-row blocks are fewer than the warps of the GPU, so
// K is split (into whole 8-group chunks) until there are about three units per warp
// of a reference 148-SM part; the warps take units at run time, which balances the
// SMs.  At one token on the full-size layer that is gate/up in 7 parts: 89.8 us per
// step, against 93.0 with 5 parts (two units per warp) and 90.5 with 14 (four).  Only
// for T <= kSmallT; 1 otherwise.
inline void decode_kparts(const moe_shape* s, int64_t T, int* nkp_gu, int* nkp_dn) {
    *nkp_gu = *nkp_dn = 1;
    if (T < 1 || T > kSmallT) return;
    const int64_t active = (T * s->top_k < s->n_experts ? T * s->top_k : s->n_experts) + s->n_shared;
    const int64_t target = 3 * 148 * 16;
    auto pick = [&](int K, int rows) {
        const int nc = (K / 64 + 7) / 8;
        const int64_t base = active * (rows / 32);
        for (int n = 1; n <= nc; ++n) {
            const int cpk = (nc + n - 1) / n, eff = (nc + cpk - 1) / cpk;
            if (base * eff >= target || n == nc) return eff;
        }
        return 1;
    };
    *nkp_gu = pick(s->hidden, 2 * s->inter);
    *nkp_dn = pick(s->inter, s->hidden);
}

// K parts of the fused decode kernel (T <= kFusedMaxT).  A gate/up tile of a shared
// expert has all T tokens against a routed tile's one or two, so the shared expert's
// chain (which every token goes through) is split into pg K parts, unless the gate/up
// tiles of all experts fit in one wave of warps (148 SMs x 16); at one or two tokens
// the routed gate/up tiles (pr parts) and every down tile (pd parts) are split too, so
// that the work comes in shorter units that fill the GPU in several waves.  The last
// part of a split gate/up tile sums the parts in part order (gp_done counts them);
// the down parts are summed in part order by the combine.  The sums live in the ypart
// region: the down parts [pd][T (k + S)][H] fp32, then the gate/up parts
// [max(pg, pr)][gsh rows][I] x {gate, up} fp32, whose rows are every expert row when
// routed tiles are split and the shared rows only otherwise.
// gate/up part counters kept in the workspace: every expert slot's tiles at two tokens
// if that stays small, else the shared experts' only
inline int64_t fused_gp_counters(const moe_shape* s) {
    const int64_t tg = 2 * s->inter / 16, all = (2 * s->top_k + s->n_shared) * tg;
    return all <= 8192 ? all : s->n_shared * tg;
}
inline FusedParts fused_kparts(const moe_shape* s, int64_t T) {
    FusedParts f = {1, 1, 1, 0, 0};
    const int nch = (int)((s->hidden / 64 + 7) / 8), nci = (int)((s->inter / 64 + 7) / 8);
    const int64_t tg = 2 * s->inter / 16, gu_tiles = (T * s->top_k + s->n_shared) * tg;
    if (T <= 2 && gu_tiles <= fused_gp_counters(s)) f.pr = nch < 2 ? nch : 2;
    if (s->n_shared && (gu_tiles > 148 * 16 || f.pr > 1)) f.pg = nch < 4 ? nch : 4;
    if (T <= 2 && nci >= 2) f.pd = 2;
    f.gsh_row0 = f.pr > 1 ? 0 : (int)(T * s->top_k);
    f.gsh_rows = (int)(f.pr > 1 ? T * (s->top_k + s->n_shared) : T * s->n_shared);
    return f;
}
inline size_t fused_ypart_floats(const moe_shape* s, int64_t T) {
    const FusedParts f = fused_kparts(s, T);
    const size_t dn = (size_t)f.pd * T * (s->top_k + s->n_shared) * s->hidden;
    const int pmax = f.pg > f.pr ? f.pg : f.pr;
    return dn + (pmax > 1 ? (size_t)pmax * f.gsh_rows * 2 * s->inter : 0);
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t s);
// the decode operands (Z tables) of a.T tokens, for the decode path above kSmallT tokens
cudaError_t launch_decode_operands(const RouteArgs& a, cudaStream_t s);
// the routing of caller-given expert ids and gates (a.fixed_ids): histogram, scan,
// permutation, active list and (if a.ops) the decode operands
cudaError_t launch_route_fixed(const RouteArgs& a, cudaStream_t s);
// decode-path expert kernels + combine; ev_gateup / ev_down (may be null) are recorded
// after the gate/up and the down kernel
cudaError_t launch_ffn_decode(const FfnArgs& a, cudaStream_t s, cudaEvent_t ev_gateup, cudaEvent_t ev_down);
// the whole decode forward (operands, gate/up, down, combine) as one persistent kernel,
// for 1 <= T <= kFusedMaxT
cudaError_t launch_ffn_fused(const FfnArgs& a, cudaStream_t s);
// prefill-path expert kernels (tcgen05) + combine; x16: fp16 scratch of T*(k+S)*H
cudaError_t launch_ffn_prefill(const FfnArgs& a, uint16_t* x16, cudaStream_t s, cudaEvent_t ev_gateup,
                               cudaEvent_t ev_down);
// expert-parallel row kernels (ep.cu): dst[i] = src[index[i] / div] (bf16 rows); y[t] =
// sum_j g[t][j] rows[inv_perm[t k + j]] + shared[t] (fp32 rows, bf16 y); bad indices are
// reported in ctrl
cudaError_t launch_gather_rows(int n, int H, const uint16_t* src, const int32_t* index, int div, int n_src,
                               uint16_t* dst, Ctrl* ctrl, cudaStream_t s);
cudaError_t launch_combine_pairs(int T, int k, int H, int n_rows, const float* rows, const int32_t* inv_perm,
                                 const float* gates, const float* shared, uint16_t* y, Ctrl* ctrl, cudaStream_t s);
// gate-weighted unpermute-combine of the partial rows into y
cudaError_t launch_combine(const FfnArgs& a, cudaStream_t s);

// Raises a kernel's dynamic shared memory limit on the current device.  The attribute
// belongs to the device's context, so it is set before every launch rather than once
// per process: a host-side call that enqueues nothing, cheap, and correct whichever
// device is current and from any number of host threads.
template <typename... KArgs>
inline cudaError_t set_smem_limit(void (*kern)(KArgs...), size_t bytes) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// Launches kern<<<grid, block, smem, s>>>(args...) with programmatic stream
// serialization: the kernel may begin while its predecessor in s is still running and
// synchronises with it through griddep_wait().
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Records event e on stream s.  While s is being captured into a CUDA graph the record
// becomes an event node of the graph (cudaEventRecordExternal), so that every replay
// records the event as an eager launch would; otherwise a plain record.
inline cudaError_t record_event(cudaEvent_t e, cudaStream_t s) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    const cudaError_t err = cudaStreamIsCapturing(s, &cs);
    if (err != cudaSuccess) return err;
    return cudaEventRecordWithFlags(e, s, cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal
                                                                              : cudaEventRecordDefault);
}

}  // namespace moe
