// Internal launcher interface between the C ABI (api.cu) and the kernels.
#pragma once
#include <utility>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace moe {

constexpr int kSmallT = 64;        // decode router / decode path threshold
constexpr int kChunk = 128;        // tokens per chunk of the large-T router

struct RouteArgs {
    int T, H, E, k, S;
    const uint16_t* x;
    const float* Wr;
    const float* bias;
    float* logits;      // ws [T][E]
    int32_t* hist;      // ws [ceil(T/kChunk)][E]
    int32_t* active;    // ws [E+S]
    float* zx;          // ws fp16 planes [2][3][T][G8] of -Z/16, hi and lo (see route.cu)
    uint8_t* iq;        // ws integer gate/up operands for T <= kIqMaxT (see route.cu), else null
    Ctrl* ctrl;
    moe_routing r;
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
    const uint8_t* iq;       // ws integer gate/up operands (T <= kIqMaxT), else null
    int iq_on;               // gate/up of ternary / 2-bit experts on the integer path
    Ctrl* ctrl;
    uint16_t* h;             // ws fp16 [T*(k+S)][I]
    float* ypart;            // ws f32 [nkp_dn][T*(k+S)][H]
    float* gpart;            // ws f32 [nkp_gu][T*(k+S)][2I] (aliases ypart; decode, nkp_gu > 1)
    int nkp_gu, nkp_dn;      // K parts of the decode gate/up and down passes (1 on the prefill path)
    uint32_t* tile_ctr;      // ws [H/16]
    uint16_t* y;             // bf16 [T][H]
    int num_ctas;
};

// Workspace layout for T tokens (api.cu).  The control block, tile counters and the
// active-expert list sit at fixed offsets (independent of T).
struct Ws {
    size_t ctrl, tile_ctr, active, logits, hist, zx, iq, h, ypart, total;
};

// Few-token gate/up on the integer tensor path (decode_ffn.cu, route.cu): up to
// kIqMaxT tokens, each as two signed-byte digit columns of one n8 MMA tile.  The
// region holds, per token t and 64-group g (G groups, G8 = G padded to whole chunks):
//   digit records  [T][G][2 digits][4 lanes] x 16 bytes          (offset 0)
//   factors p      fp32 [T][G8]                                   (iq_pq_off)
//   offset planes  fp16 [2 hi/lo][2 formats][T][G8] of -o sum x / 16  (iq_zq_off)
constexpr int kIqMaxT = 4;
__host__ __device__ inline size_t iq_pq_off(int64_t T, int64_t H) { return (size_t)T * (H / 64) * 128; }
__host__ __device__ inline size_t iq_zq_off(int64_t T, int64_t H) {
    return iq_pq_off(T, H) + (size_t)4 * T * (8 * ((H / 64 + 7) / 8));
}
// Reserved for min(T, kIqMaxT) tokens at every T >= 1, so that the workspace size
// never shrinks as T grows; used only when T <= kIqMaxT.
inline size_t iq_bytes(int64_t T, int64_t H) {
    const int64_t t = T < kIqMaxT ? T : kIqMaxT;
    return t >= 1 ? iq_zq_off(t, H) + (size_t)2 * 2 * 2 * t * (8 * ((H / 64 + 7) / 8)) : 0;
}
Ws ws_layout(const moe_shape* s, int64_t T);

// K parts of the decode-path expert passes for T tokens.  With few tokens only a few
// experts are active and their 32-row blocks are fewer than the warps of the GPU, so
// K is split (into whole 8-group chunks) until there are about three units per warp
// of a reference 148-SM part; the warps take units at run time, which balances the
// SMs (finer splits measured no faster).  Only for T <= kSmallT; 1 otherwise.
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

cudaError_t launch_route(const RouteArgs& a, cudaStream_t s);
// decode-path expert kernels + combine; ev_gateup / ev_down (may be null) are recorded
// after the gate/up and the down kernel
cudaError_t launch_ffn_decode(const FfnArgs& a, cudaStream_t s, cudaEvent_t ev_gateup, cudaEvent_t ev_down);
// prefill-path expert kernels (tcgen05) + combine; x16: fp16 scratch of T*(k+S)*H
cudaError_t launch_ffn_prefill(const FfnArgs& a, uint16_t* x16, cudaStream_t s, cudaEvent_t ev_gateup,
                               cudaEvent_t ev_down);
// gate-weighted unpermute-combine of the partial rows into y
cudaError_t launch_combine(const FfnArgs& a, cudaStream_t s);

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
