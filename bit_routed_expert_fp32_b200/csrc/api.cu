// C ABI of the routed-MoE layer (include/moe.h): argument checks, workspace
// layout and kernel launches.  Nothing here allocates memory or synchronises,
// except moe_get_error, which is documented to.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>

#include "kernels.h"
#include "moe.h"

namespace moe {

namespace {
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
}  // namespace

// Workspace layout.  The control block, tile counters and the active-expert list
// sit at fixed offsets (independent of T) so that their cleared state survives
// calls with different token counts; the token-sized arrays follow.
Ws ws_layout(const moe_shape* s, int64_t T) {
    Ws w;
    const int64_t E = s->n_experts, S = s->n_shared, k = s->top_k, H = s->hidden, I = s->inter;
    size_t off = 0;
    w.ctrl = off;
    off += 4096;
    w.tile_ctr = off;                         // [H/16] down, then the gate/up part counters
    off = align256(off + 4 * (size_t)(H / 16 + fused_gp_counters(s)));
    w.active = off;
    off = align256(off + 4 * (size_t)(E + S));
    w.logits = off;
    off = align256(off + 4 * (size_t)(T * E));
    w.hist = off;
    off = align256(off + 4 * (size_t)(((T + kChunk - 1) / kChunk) * E));
    w.zx = off;
    off = align256(off + 4 * (size_t)(3 * (8 * ((H / 64 + 7) / 8)) * T));   // two fp16 planes
    w.iq = off;
    off = align256(off + iq_bytes(T, H));
    // the fused decode kernel's fp32 h and its integer operands, for min(T, kFusedMaxT) tokens
    const int64_t r16 = (T < kFusedMaxT ? T : kFusedMaxT) * (k + S);
    w.hf = off;
    off = align256(off + 4 * (size_t)(r16 * I));
    w.hq = off;
    off = align256(off + (r16 > 0 ? iq_size(r16, I) : 0));
    // the fused kernel's need of the ypart region (its K-part sums) for every token
    // count up to min(T, kFusedMaxT)
    size_t yfused = 0;
    for (int64_t t = 1; t <= T && t <= kFusedMaxT; ++t) {
        const size_t y = fused_ypart_floats(s, t);
        yfused = yfused > y ? yfused : y;
    }
    w.h = off;
    off = align256(off + 2 * (size_t)(T * (k + S) * I));
    // ypart, and the decode gate/up partial sums that alias it: the largest need of any
    // token count up to T (the split into K parts shrinks as T grows), so a workspace
    // sized for T tokens serves every smaller T.
    size_t yfl = (size_t)(T * (k + S) * H);
    yfl = yfl > yfused ? yfl : yfused;
    for (int64_t t = 1; t <= T && t <= kSmallT; ++t) {
        int ngu = 1, ndn = 1;
        decode_kparts(s, t, &ngu, &ndn);
        const size_t rows = (size_t)(t * (k + S));
        const size_t need_dn = (size_t)ndn * rows * H, need_gu = ngu > 1 ? (size_t)ngu * rows * 2 * I : 0;
        yfl = yfl > need_dn ? yfl : need_dn;
        yfl = yfl > need_gu ? yfl : need_gu;
    }
    w.ypart = off;
    off = align256(off + 4 * yfl);
    w.total = off;
    return w;
}

}  // namespace moe

namespace moe {

bool shape_ok(const moe_shape* s) {
    return s && s->hidden > 0 && s->inter > 0 && s->hidden % 64 == 0 && s->inter % 64 == 0 &&
           s->n_experts >= 1 && s->n_experts <= 256 && s->top_k >= 1 && s->top_k <= 16 &&
           s->top_k <= s->n_experts && (s->n_shared == 0 || s->n_shared == 1);
}

namespace {

size_t ws_fixed_prefix(const moe_shape* s) { return ws_layout(s, 0).active; }

int sm_count() {
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// The kernels load tokens, router rows, weights and workspace regions in 16-byte
// pieces (vector loads, bulk copies): every such base pointer must be 16-byte aligned.
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

bool routing_ok(const moe_routing* r) {
    return r && r->topk_ids && r->topk_w && r->counts && r->offsets && r->perm && r->inv_perm;
}

moe_status check_path(moe_path path, int32_t T) {
    const int base = (int)path & ~MOE_OUT_F32;
    if (base != MOE_PATH_AUTO && base != MOE_PATH_DECODE && base != MOE_PATH_PREFILL && base != MOE_PATH_DECODE_FUSED)
        return MOE_ERR_INVALID_ARG;
    if (base == MOE_PATH_DECODE_FUSED && T > kFusedMaxT) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

moe_status check_common(const moe_shape* shape, int32_t T, const void* d_ws, size_t ws_bytes) {
    if (!shape_ok(shape) || T < 0) return MOE_ERR_INVALID_ARG;
    if ((int64_t)T * shape->top_k > (int64_t)INT32_MAX / 2) return MOE_ERR_UNSUPPORTED;
    if (!d_ws) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < ws_layout(shape, T).total) return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

}  // namespace

moe_status check_route_args(const moe_shape* shape, int32_t T, const uint16_t* d_x, const float* d_router_w,
                            const moe_routing* out, const void* d_ws, size_t ws_bytes) {
    const moe_status st = check_common(shape, T, d_ws, ws_bytes);
    if (st != MOE_OK) return st;
    if (!d_x || !d_router_w || !routing_ok(out)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(d_x) || !aligned16(d_router_w) || !aligned16(d_ws)) return MOE_ERR_INVALID_ARG;
    if (ws_fixed_prefix(shape) > 4096 + 65536) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

moe_status check_forward_args(const moe_shape* shape, int32_t T, const void* d_packed, const uint16_t* d_x,
                              const moe_routing* r, const uint16_t* d_y, moe_path path, const void* d_ws,
                              size_t ws_bytes) {
    const moe_status st = check_common(shape, T, d_ws, ws_bytes);
    if (st != MOE_OK) return st;
    if (!d_packed || !d_x || !d_y || !routing_ok(r)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(d_packed) || !aligned16(d_x) || !aligned16(d_y) || !aligned16(d_ws)) return MOE_ERR_INVALID_ARG;
    return check_path(path, T);
}

// Which kernels moe_forward runs for T tokens on `path` (its base value, without
// MOE_OUT_F32): the tcgen05 prefill kernels, the fused decode kernel (from
// kFusedAutoMinT to kFusedAutoMaxT tokens, where it measured faster on the full-size
// layer, or when asked for), or the separate decode launches with their K parts.
moe_status plan_forward(const moe_shape* shape, int64_t T, moe_path path, ForwardPlan* fp) {
    // The prefill kernels tile the gate/up rows and the hidden rows by 128.
    const bool tc_ok = shape->hidden % 128 == 0 && (2 * shape->inter) % 128 == 0;
    if (path == MOE_PATH_PREFILL && !tc_ok) return MOE_ERR_UNSUPPORTED;
    fp->prefill = path == MOE_PATH_PREFILL || (path == MOE_PATH_AUTO && T > kSmallT && tc_ok);
    fp->fused = !fp->prefill && T <= kFusedMaxT && shape->n_experts + shape->n_shared <= kMaxSlots &&
                (path == MOE_PATH_DECODE_FUSED || (T >= kFusedAutoMinT && T <= kFusedAutoMaxT));
    fp->nkp_gu = fp->nkp_dn = 1;
    if (!fp->prefill && !fp->fused) decode_kparts(shape, T, &fp->nkp_gu, &fp->nkp_dn);
    // moe_route: one kernel up to kSmallT tokens, else logits, top-k, scatter; moe_forward:
    // the fused kernel; or gather, gate/up, down, combine; or (decode operands above
    // kSmallT tokens,) gate/up, (K-part reduction,) down, combine
    const int route = T <= kSmallT ? 1 : 3;
    const int fwd = fp->fused ? 1 : fp->prefill ? 4 : (T > kSmallT ? 1 : 0) + 3 + (fp->nkp_gu > 1 ? 1 : 0);
    fp->launches = T > 0 ? route + fwd : 0;
    return MOE_OK;
}

// Writes the test-stall word of a workspace's control block (one thread).
__global__ void set_test_stall_kernel(Ctrl* c, uint32_t cycles) { c->test_stall = cycles; }

}  // namespace moe

namespace {
using namespace moe;
}  // namespace

extern "C" {

int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }

moe_status moe_event_record(void* event, void* stream) {
    if (!event) return MOE_ERR_INVALID_ARG;
    return moe::record_event(static_cast<cudaEvent_t>(event), static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
        case MOE_ERR_WORKSPACE: return "workspace or destination buffer too small";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_TIMEOUT: return "device-side wait timed out";
        case MOE_ERR_DEVICE_CHECK: return "device-side data check failed";
    }
    return "unknown status";
}

moe_status moe_workspace_size(const moe_shape* shape, int32_t max_tokens, size_t* bytes) {
    if (!shape_ok(shape) || max_tokens < 0 || !bytes) return MOE_ERR_INVALID_ARG;
    *bytes = ws_layout(shape, max_tokens).total;
    return MOE_OK;
}

moe_status moe_workspace_init(void* d_ws, size_t ws_bytes, void* stream) {
    if (!d_ws || ws_bytes < 4096) return MOE_ERR_INVALID_ARG;
    // Clears the control block and every counter that can follow it (up to H = 256K).
    const size_t n = ws_bytes < 4096 + 65536 ? ws_bytes : 4096 + 65536;
    if (cudaMemsetAsync(d_ws, 0, n, static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

moe_status moe_workspace_set_test_stall(void* d_ws, size_t ws_bytes, uint32_t cycles, void* stream) {
    if (!d_ws || ws_bytes < 4096) return MOE_ERR_INVALID_ARG;
    set_test_stall_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<Ctrl*>(d_ws), cycles);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_route(const moe_shape* shape, int32_t T, const uint16_t* d_x, const float* d_router_w,
                     const float* d_router_b, const moe_routing* out, void* d_ws, size_t ws_bytes, void* stream) {
    const moe_status st = check_route_args(shape, T, d_x, d_router_w, out, d_ws, ws_bytes);
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    const Ws w = ws_layout(shape, T);
    uint8_t* ws = static_cast<uint8_t*>(d_ws);
    RouteArgs a = {};     // every field not set below is zero (no fixed routing)
    a.T = T;
    a.H = shape->hidden;
    a.E = shape->n_experts;
    a.k = shape->top_k;
    a.S = shape->n_shared;
    a.x = d_x;
    a.Wr = d_router_w;
    a.bias = d_router_b;
    a.logits = reinterpret_cast<float*>(ws + w.logits);
    a.hist = reinterpret_cast<int32_t*>(ws + w.hist);
    a.active = reinterpret_cast<int32_t*>(ws + w.active);
    a.zx = reinterpret_cast<float*>(ws + w.zx);
    // The decode operands are formed by the router only for the decode kernels that do
    // not form them themselves (more than kFusedMaxT tokens).
    a.ops = T <= kSmallT;                                 // the decode operands (the decode
                                                          // path forms them itself above)
    a.iq = T <= kFusedMaxT ? ws + w.iq : nullptr;         // and the integer records
    a.ctrl = reinterpret_cast<Ctrl*>(ws + w.ctrl);
    a.r = *out;
    if (launch_route(a, static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

moe_status moe_route_fixed(const moe_shape* shape, int32_t T, const uint16_t* d_x, const int32_t* d_ids,
                           const float* d_gates, const moe_routing* out, void* d_ws, size_t ws_bytes, void* stream) {
    // the same checks as moe_route, with the caller's ids and gates in place of the router
    const float* present = reinterpret_cast<const float*>(d_ids);
    const moe_status st = check_route_args(shape, T, d_x, present, out, d_ws, ws_bytes);
    if (st != MOE_OK) return st;
    if (!d_ids || !d_gates) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    const Ws w = ws_layout(shape, T);
    uint8_t* ws = static_cast<uint8_t*>(d_ws);
    RouteArgs a = {};
    a.T = T;
    a.H = shape->hidden;
    a.E = shape->n_experts;
    a.k = shape->top_k;
    a.S = shape->n_shared;
    a.x = d_x;
    a.hist = reinterpret_cast<int32_t*>(ws + w.hist);
    a.active = reinterpret_cast<int32_t*>(ws + w.active);
    a.zx = reinterpret_cast<float*>(ws + w.zx);
    a.ops = T <= kSmallT;                                 // the decode operands (the decode
                                                          // path forms them itself above)
    a.iq = T <= kFusedMaxT ? ws + w.iq : nullptr;         // and the integer records
    a.fixed_ids = d_ids;
    a.fixed_w = d_gates;
    a.ctrl = reinterpret_cast<Ctrl*>(ws + w.ctrl);
    a.r = *out;
    return launch_route_fixed(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_gather_rows(int32_t n, int32_t hidden, const uint16_t* d_src, int32_t n_src, const int32_t* d_index,
                           int32_t divisor, uint16_t* d_dst, void* d_ws, size_t ws_bytes, void* stream) {
    if (n < 0 || hidden <= 0 || hidden % 64 != 0 || n_src < 0 || divisor < 1) return MOE_ERR_INVALID_ARG;
    if (n == 0) return MOE_OK;
    if (!d_src || !d_index || !d_dst || !d_ws || ws_bytes < 4096) return MOE_ERR_INVALID_ARG;
    return launch_gather_rows(n, hidden, d_src, d_index, divisor, n_src, d_dst, static_cast<Ctrl*>(d_ws),
                              static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

moe_status moe_combine_pairs(int32_t T, int32_t top_k, int32_t hidden, const float* d_rows, int32_t n_rows,
                             const int32_t* d_inv_perm, const float* d_gates, const float* d_shared, uint16_t* d_y,
                             void* d_ws, size_t ws_bytes, void* stream) {
    if (T < 0 || top_k < 1 || top_k > 16 || hidden <= 0 || hidden % 64 != 0 || n_rows < 0) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!d_rows || !d_inv_perm || !d_gates || !d_y || !d_ws || ws_bytes < 4096) return MOE_ERR_INVALID_ARG;
    return launch_combine_pairs(T, top_k, hidden, n_rows, d_rows, d_inv_perm, d_gates, d_shared, d_y,
                                static_cast<Ctrl*>(d_ws), static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

moe_status moe_forward_timed(const moe_shape* shape, int32_t T, const void* d_packed, const uint16_t* d_x,
                             const moe_routing* r, uint16_t* d_y, moe_path path, void* d_ws, size_t ws_bytes,
                             void* stream, void* const* events, int32_t n_events) {
    const moe_status st = check_forward_args(shape, T, d_packed, d_x, r, d_y, path, d_ws, ws_bytes);
    if (st != MOE_OK) return st;
    if (events && n_events < 4) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const Ws w = ws_layout(shape, T);
    uint8_t* ws = static_cast<uint8_t*>(d_ws);
    FfnArgs a = {};
    a.T = T;
    a.H = shape->hidden;
    a.I = shape->inter;
    a.E = shape->n_experts;
    a.k = shape->top_k;
    a.S = shape->n_shared;
    a.packed = static_cast<const uint8_t*>(d_packed);
    a.x = d_x;
    a.perm = r->perm;
    a.inv_perm = r->inv_perm;
    a.counts = r->counts;
    a.offsets = r->offsets;
    a.topk_w = r->topk_w;
    a.active = reinterpret_cast<const int32_t*>(ws + w.active);
    a.zx = reinterpret_cast<const float*>(ws + w.zx);
    a.iq = T <= kFusedMaxT ? ws + w.iq : nullptr;
    a.iq_on = T <= kIqMaxT && T <= kFusedMaxT;          // the router wrote the records
    a.fc = reinterpret_cast<FusedCtl*>(ws + w.ctrl + sizeof(Ctrl));
    a.dn_done = reinterpret_cast<uint32_t*>(ws + w.tile_ctr);
    a.hf = reinterpret_cast<float*>(ws + w.hf);
    a.hq = ws + w.hq;
    a.R16 = (T < kFusedMaxT ? T : kFusedMaxT) * (a.k + a.S);
    a.gp_done = a.dn_done + a.H / 16;
    a.fk = fused_kparts(shape, T >= 1 && T <= kFusedMaxT ? T : 1);
    a.ctrl = reinterpret_cast<Ctrl*>(ws + w.ctrl);
    a.h = reinterpret_cast<uint16_t*>(ws + w.h);
    a.ypart = reinterpret_cast<float*>(ws + w.ypart);
    a.gsh = a.ypart + (size_t)a.fk.pd * T * (a.k + a.S) * a.H;
    a.gpart = a.ypart;
    a.nkp_gu = a.nkp_dn = 1;
    a.tile_ctr = reinterpret_cast<uint32_t*>(ws + w.tile_ctr);
    a.y = d_y;
    a.y_f32 = ((int)path & MOE_OUT_F32) != 0;
    path = (moe_path)((int)path & ~MOE_OUT_F32);
    ForwardPlan fp;
    const moe_status pst = plan_forward(shape, T, path, &fp);
    if (pst != MOE_OK) return pst;
    a.num_ctas = sm_count();
    cudaEvent_t ev[4] = {nullptr, nullptr, nullptr, nullptr};
    if (events)
        for (int i = 0; i < 4; ++i) ev[i] = static_cast<cudaEvent_t>(events[i]);
    if (ev[0] && record_event(ev[0], s) != cudaSuccess) return MOE_ERR_CUDA;
    const bool prefill = fp.prefill, fused = fp.fused;
    cudaError_t err;
    if (fused) {
        // one kernel: the per-kernel events all follow it
        err = launch_ffn_fused(a, s);
        for (int i = 1; i < 3 && err == cudaSuccess; ++i)
            if (ev[i]) err = record_event(ev[i], s);
    } else {
        if (!prefill && T > kSmallT) {
            // the decode kernels' token operands (the router forms them up to kSmallT tokens)
            RouteArgs ra = {};
            ra.T = T;
            ra.H = a.H;
            ra.x = d_x;
            ra.zx = reinterpret_cast<float*>(ws + w.zx);
            ra.ctrl = a.ctrl;
            ra.ops = 1;
            if (launch_decode_operands(ra, s) != cudaSuccess) return MOE_ERR_CUDA;
        }
        a.nkp_gu = fp.nkp_gu;
        a.nkp_dn = fp.nkp_dn;
        err = prefill ? launch_ffn_prefill(a, reinterpret_cast<uint16_t*>(ws + w.ypart), s, ev[1], ev[2])
                      : launch_ffn_decode(a, s, ev[1], ev[2]);
    }
    if (err != cudaSuccess) return err == cudaErrorInvalidConfiguration ? MOE_ERR_UNSUPPORTED : MOE_ERR_CUDA;
    if (ev[3] && record_event(ev[3], s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

moe_status moe_forward_plan(const moe_shape* shape, int32_t T, moe_path path, int32_t* plan) {
    if (!shape_ok(shape) || T < 0 || !plan) return MOE_ERR_INVALID_ARG;
    if ((int64_t)T * shape->top_k > (int64_t)INT32_MAX / 2) return MOE_ERR_UNSUPPORTED;
    const moe_status st = check_path(path, T);
    if (st != MOE_OK) return st;
    ForwardPlan fp;
    const moe_status pst = plan_forward(shape, T, (moe_path)((int)path & ~MOE_OUT_F32), &fp);
    if (pst != MOE_OK) return pst;
    plan[0] = fp.prefill ? MOE_PATH_PREFILL : fp.fused ? MOE_PATH_DECODE_FUSED : MOE_PATH_DECODE;
    plan[1] = fp.launches;
    plan[2] = fp.nkp_gu;
    plan[3] = fp.nkp_dn;
    return MOE_OK;
}

moe_status moe_forward(const moe_shape* shape, int32_t T, const void* d_packed, const uint16_t* d_x,
                       const moe_routing* r, uint16_t* d_y, moe_path path, void* d_ws, size_t ws_bytes,
                       void* stream) {
    return moe_forward_timed(shape, T, d_packed, d_x, r, d_y, path, d_ws, ws_bytes, stream, nullptr, 0);
}

moe_status moe_get_error(void* d_ws, size_t ws_bytes, void* stream, uint32_t* detail) {
    if (!d_ws || ws_bytes < sizeof(Ctrl)) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    uint32_t word[2] = {0, 0};
    if (cudaMemcpy(word, d_ws, sizeof word, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemset(d_ws, 0, sizeof word) != cudaSuccess) return MOE_ERR_CUDA;
    if (detail) *detail = word[1];
    if (word[0] == MOE_ERR_TIMEOUT) return MOE_ERR_TIMEOUT;
    if (word[0] != 0) return MOE_ERR_DEVICE_CHECK;
    return MOE_OK;
}

}  // extern "C"
