/*
 * moe.h - C ABI of a routed mixture-of-experts FFN layer for NVIDIA B200 (sm_100a)
 * whose expert weights are stored as ternary, 2-bit or 3-bit codes with one fp16
 * scale per 64 weights along K.
 *
 * What the layer computes.  The engine the source pages describe runs a
 * DeepSeek-class MoE model by sending each token to a few experts and reading
 * only those experts' weights (ossradar.top, Xolotl README, "How it works, in one
 * paragraph"; yoney.dev news item, third paragraph).  Its expert weights are a
 * calibrated mix of ternary, 2-bit and 3-bit codes (ossradar.top README, "Get a
 * model"; shadowgraph.io README, "Get a model"), and its decode speed is set by the
 * expert bytes moved per token (ossradar.top README, "Fast mode (DeepSeek-V4.1)").
 * The pages give no formula, layout or interface; this header fixes them:
 *
 *   logits  L[t,e] = sum_h x[t,h] * Wr[e,h] + b[e]           (fp32 router)
 *   p       = softmax_e(L[t,:])
 *   ids     = the k experts with the largest p, largest first (equal -> lower id)
 *   g[t,j]  = p[ids[t,j]] / sum_j' p[ids[t,j']]               (top-k renormalised)
 *   expert  y_e(x) = Wd_e ( silu(Wg_e x) * (Wu_e x) ),  silu(a) = a / (1 + e^-a)
 *   output  y[t] = sum_j g[t,j] * y_{ids[t,j]}(x[t]) + sum_s y_shared_s(x[t])
 *
 * Conventions for every call below
 *   - The caller owns all memory; the library allocates nothing, host or device.
 *   - moe_route and moe_forward only enqueue work on the given CUDA stream
 *     (a cudaStream_t passed as void*; NULL = legacy default stream).  They never
 *     synchronise and never read device memory back to the host.
 *   - Argument errors are reported synchronously, before anything is enqueued.
 *     Launch failures return MOE_ERR_CUDA.  Problems seen on the device
 *     (a bounded wait that ran out, a corrupt packed header) are recorded in the
 *     workspace and read back with moe_get_error.
 *   - "d_" pointers are device pointers, "h_" pointers are host pointers.
 *   - All functions are reentrant; concurrent calls must use distinct workspaces.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 1

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,   /* null pointer, bad size, bad code value, ...         */
    MOE_ERR_UNSUPPORTED = 2,   /* valid but outside what the kernels handle           */
    MOE_ERR_WORKSPACE = 3,     /* workspace or destination buffer too small           */
    MOE_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed         */
    MOE_ERR_TIMEOUT = 5,       /* a device-side bounded wait ran out (moe_get_error)   */
    MOE_ERR_DEVICE_CHECK = 6   /* the device found bad data, e.g. a packed header     */
} moe_status;

typedef enum { MOE_FMT_TERNARY = 0, MOE_FMT_Q2 = 1, MOE_FMT_Q3 = 2 } moe_format;

/* MOE_PATH_AUTO picks DECODE for T <= 64 and PREFILL otherwise.  Both paths compute
 * the same function; they differ only in kernels and rounding of intermediates. */
typedef enum { MOE_PATH_AUTO = 0, MOE_PATH_DECODE = 1, MOE_PATH_PREFILL = 2 } moe_path;

/* Layer shape.  hidden and inter must be positive multiples of 64; 1 <= top_k <= 16;
 * top_k <= n_experts <= 256; n_shared in {0, 1}. */
typedef struct {
    int32_t hidden;     /* H */
    int32_t inter;      /* I, expert FFN width */
    int32_t n_experts;  /* E, routed experts */
    int32_t top_k;      /* k */
    int32_t n_shared;   /* S */
} moe_shape;

/* Routing result, written by moe_route (all device pointers, caller-allocated).
 *   topk_ids [T][k] int32   selected experts per token, largest gate first
 *   topk_w   [T][k] float   renormalised gates (sum to 1 per token)
 *   counts   [E]    int32   number of tokens routed to each expert
 *   offsets  [E+1]  int32   exclusive prefix sum of counts (offsets[E] = T*k)
 *   perm     [T*k]  int32   permuted row r -> source pair t*k + j; rows are ordered
 *                           by expert ascending, then token ascending
 *   inv_perm [T*k]  int32   source pair t*k + j -> permuted row r                */
typedef struct {
    int32_t* topk_ids;
    float* topk_w;
    int32_t* counts;
    int32_t* offsets;
    int32_t* perm;
    int32_t* inv_perm;
} moe_routing;

/* ---------------------------------------------------------------------------
 * Packed expert format, version 2 (defined by this library; the pages name the
 * ternary / 2-bit / 3-bit mix but give no layout).  Little-endian throughout;
 * offsets are from the start of the buffer; every array starts on 256 bytes.
 *
 * Header, 256 bytes:
 *    0 u32 magic 0x50454F4D ('M','O','E','P' in memory)   4 u32 version = 2
 *    8 i32 H   12 i32 I   16 i32 E   20 i32 S   24 i32 group = 64
 *   28 i32 interleave R = 8   32 u64 total bytes   40..255 zero
 * Expert table at byte 256: E+S entries (routed experts, then shared) of 64 bytes:
 *    0 u32 format (moe_format)   4 u32 zero
 *    8 u64 gu_scales  16 u64 gu_codes  24 u64 gu_hi   (gate/up matrix, K = H)
 *   32 u64 dn_scales  40 u64 dn_codes  48 u64 dn_hi   (down matrix,    K = I)
 *   56 u64 zero;  *_hi is 0 unless the format is MOE_FMT_Q3
 * Data follows the table, expert by expert, arrays in the order listed.
 *
 * Codes.  Element k of a row has a code c; the 2-bit field lo = c & 3 of elements
 * 16w .. 16w+15 forms "code word" w of the row (element 16w + 2p + h, p = 0..7,
 * h = 0/1, at bits 16h + 2p .. 16h + 2p + 1); for 3-bit codes the third bit hi = c >> 2
 * of elements 32v .. 32v+31 forms "third-bit word" v (element 32v + 16q + 2p + h at
 * bit 16h + 8q + p).  The value of element (n, k) with code c and scale s is
 *   ternary  (c - 1)   * s,  c in {0,1,2} (c = 3 is rejected by the packer)
 *   q2       (c - 1.5) * s,  c in 0..3
 *   q3       (c - 3.5) * s,  c = lo + 4*hi in 0..7
 * with s the fp16 scale of the element's group (64 consecutive k).
 *
 * Blocking.  A matrix W[N][K] (N a multiple of 16, K of 64) has G = K/64 groups per
 * row, cut into NC = ceil(G/8) chunks; chunk c holds groups 8c .. 8c+ng-1 with
 * ng = min(8, G - 8c).  Rows are cut into tiles of 16 (tile j = rows 16j..16j+15,
 * r = row within the tile).  Every array stores one contiguous block per
 * (tile, chunk), blocks in tile-major order:
 *   codes  block (j,c) at byte 4*K*j + 2048*c, 256*ng bytes: the 4*ng code words
 *          wl = 4*gl + q (gl = group in chunk, q = 16-element quarter) of each row,
 *          word (r, wl) at u32 index  r*32 + (wl ^ 4*(r%8))  if ng = 8,
 *                                     r*4*ng + wl            otherwise;
 *   hi     (3-bit only) block (j,c) at byte 128*G*j + 1024*c, 128*ng bytes: third-bit
 *          words vl = 2*gl + half of each row at u32 index
 *                                     r*16 + (vl ^ 2*((r%8)/2))  if ng = 8,
 *                                     r*2*ng + vl                 otherwise;
 *   scales block (j,c) at byte 256*NC*j + 256*c, 256 bytes: fp16 scale of group
 *          8c + gl of row r at half index r*8 + gl (zero where 8c + gl >= G).
 * (The XOR swizzles make the fragment reads of a 16-row chunk in shared memory free
 * of bank conflicts.)  Gate and up are fused into one matrix GU[2I][H]: row r lies in
 * block b = r/16; r%16 < 8 is gate row 8b + r%16, otherwise up row 8b + r%16 - 8.
 * Down is D[H][I].
 * ------------------------------------------------------------------------- */

/* One source matrix in the interchange layout the packer reads (host memory):
 *   codes  [rows][K/4]   2-bit field (low bits of the code) of element k at bits
 *                        2*(k%4) of byte k/4
 *   hi     [rows][K/8]   3-bit formats only (else NULL): third bit of the code of
 *                        element k at bit k%8 of byte k/8
 *   scales [rows][K/64]  fp16 bit patterns                                      */
typedef struct {
    const uint8_t* codes;
    const uint8_t* hi;
    const uint16_t* scales;
} moe_matrix_src;

/* Bytes needed for the packed buffer of this shape and these formats
 * (h_fmt: host array of E+S moe_format values). */
moe_status moe_packed_size(const moe_shape* shape, const uint8_t* h_fmt, size_t* bytes);

/* Pack experts [first, first+count) into the HOST buffer h_dst (h_dst_bytes >=
 * moe_packed_size); also (re)writes the header and the whole expert table, so the
 * buffer is complete once every expert has been packed by some call.  src is a host
 * array of count*3 matrices in the order gate [I][H], up [I][H], down [H][I] for
 * each expert.  The caller copies h_dst to the device (e.g. cudaMemcpy).
 * Errors: MOE_ERR_INVALID_ARG for null pointers, a bad format, first/count out of
 * range or a ternary code 3 (h_dst is then partly written); MOE_ERR_WORKSPACE if
 * h_dst_bytes is too small. */
moe_status moe_pack_experts(const moe_shape* shape, const uint8_t* h_fmt, int32_t first,
                            int32_t count, const moe_matrix_src* h_src, void* h_dst,
                            size_t h_dst_bytes);

/* The 2-bit copy of one 3-bit matrix, for the fast mode: a second packed buffer in
 * which the 3-bit experts are 2-bit, read instead of the model's own buffer on the
 * calls that ask for it (Indras-Mirror/Xolotl README, "Fast mode (DeepSeek-V4.1)":
 * decode speed follows the expert bytes read per token, so a lossy 2-bit copy of the
 * biggest expert format is kept beside the model and read instead; the model buffer
 * itself is unchanged).  The pages give no requantisation rule; this one keeps the
 * 64-weight groups and their layout: the code c = field + 4 hi (0..7) becomes
 * c' = c >> 1 (0..3) and the group scale s becomes s' = 2 s (exact in fp16), so each
 * weight (c' - 1.5) s' differs from (c - 3.5) s by exactly s / 2, the nearest of the
 * four 2-bit levels to each of the eight 3-bit ones.  Pack the result with
 * MOE_FMT_Q2 for that expert.  Host memory only, no CUDA calls.
 *   src       the 3-bit matrix in the interchange form (hi required), [rows][K]
 *   h_codes   out [rows][K/4]: 2-bit fields in the interchange form
 *   h_scales  out [rows][K/64]: fp16 bit patterns of 2 s
 * MOE_ERR_INVALID_ARG (nothing written): a null pointer, rows < 1, K < 64 or not a
 * multiple of 64, a scale that is not finite or whose double is not finite in fp16. */
moe_status moe_requantize_q3_to_q2(int32_t rows, int32_t K, const moe_matrix_src* src,
                                   uint8_t* h_codes, uint16_t* h_scales);

/* Device workspace needed for up to max_tokens tokens per call (both paths). */
moe_status moe_workspace_size(const moe_shape* shape, int32_t max_tokens, size_t* bytes);

/* Clears the workspace's counters and error word (enqueued on stream).  Call once
 * after allocating a workspace, and again after moe_get_error reported a problem.
 * Every later call leaves the counters cleared again. */
moe_status moe_workspace_init(void* d_ws, size_t ws_bytes, void* stream);

/* Route T tokens: fp32 router logits, softmax + top-k + renormalised gates,
 * per-expert histogram, prefix sum and permutation.
 *   d_x        bf16 bit patterns [T][H], row-major
 *   d_router_w fp32 [E][H], row-major
 *   d_router_b fp32 [E] added to the logits before the softmax, or NULL
 *   out        caller-allocated device arrays (see moe_routing)
 * Also leaves in d_ws the expert schedule that moe_forward reads, so moe_forward
 * must be given the same d_ws and T.  T = 0 is a no-op returning MOE_OK.
 * Tokens, router weights and bias must be finite: a NaN or infinity gives
 * unspecified routing and outputs (the few-token integer path does not carry a NaN
 * token through to y); nothing checks this on the device. */
moe_status moe_route(const moe_shape* shape, int32_t T, const uint16_t* d_x,
                     const float* d_router_w, const float* d_router_b, const moe_routing* out,
                     void* d_ws, size_t ws_bytes, void* stream);

/* Expert FFNs of the routed and shared experts and the gate-weighted combine,
 * using the routing of the preceding moe_route on the same d_ws.
 *   d_packed  packed experts (format above), device memory
 *   d_x       bf16 [T][H] (the same tokens as routed)
 *   r         the routing moe_route wrote
 *   d_y       bf16 [T][H] output, written in full
 * T = 0 is a no-op.  T > 64 with MOE_PATH_DECODE is allowed (slower). */
moe_status moe_forward(const moe_shape* shape, int32_t T, const void* d_packed,
                       const uint16_t* d_x, const moe_routing* r, uint16_t* d_y, moe_path path,
                       void* d_ws, size_t ws_bytes, void* stream);

/* Same as moe_forward; if events is not NULL it must hold n_events >= 4 cudaEvent_t
 * (passed as void*) that are recorded on the stream around the kernels: events[0]
 * before the first kernel, events[1] after the gate/up kernel, events[2] after the
 * down kernel, events[3] after the last kernel. */
moe_status moe_forward_timed(const moe_shape* shape, int32_t T, const void* d_packed,
                             const uint16_t* d_x, const moe_routing* r, uint16_t* d_y,
                             moe_path path, void* d_ws, size_t ws_bytes, void* stream,
                             void* const* events, int32_t n_events);

/* Synchronises the stream, reads the device error word from d_ws and clears it.
 * Returns MOE_OK, MOE_ERR_TIMEOUT or MOE_ERR_DEVICE_CHECK; *detail (if not NULL)
 * receives a kernel-specific code. For tests and diagnostics; not for hot loops. */
moe_status moe_get_error(void* d_ws, size_t ws_bytes, void* stream, uint32_t* detail);

/* No-allocation decode entry point.  The source pages have no counterpart to this
 * call: it exists for callers of this library that cannot allocate device memory,
 * such as a plugin inside a framework whose pool allocator owns all GPU memory, a
 * serving loop that cannot afford cudaMalloc / cudaFree (they may synchronise the
 * device), or code recording a CUDA graph, during which no allocation may happen.
 * It does what moe_route followed by moe_forward(MOE_PATH_DECODE) do, with the same
 * arguments and outputs (out: caller-allocated routing arrays; d_y: bf16 [T][H]), but
 * instead of a caller-given workspace it uses a scratch array that the library holds
 * in device memory: MOE_STATIC_WS_BYTES (8 MiB), held by every GPU that loads the
 * library until the process exits.  It allocates nothing itself.
 *   - If the workspace T tokens need (moe_workspace_size) exceeds MOE_STATIC_WS_BYTES
 *     it returns MOE_ERR_WORKSPACE and enqueues nothing; with the full-size layer
 *     (H 7168, I 2048, E 256, k 8, S 1) that allows up to 27 tokens per call.
 *   - The first call on each device looks up the scratch array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call before
 *     any stream capture.  Later calls only enqueue work.
 *   - All calls share the one array, and each call first clears its control block.
 *     Calls that overlap on the GPU (other streams, other host threads, other
 *     devices' calls do not overlap) race on the array: serialise them. */
#define MOE_STATIC_WS_BYTES ((size_t)8 << 20)
moe_status moe_decode_static(const moe_shape* shape, int32_t T, const uint16_t* d_x,
                             const float* d_router_w, const float* d_router_b, const void* d_packed,
                             const moe_routing* out, uint16_t* d_y, void* stream);

/* Records a caller-created CUDA event (cudaEvent_t, passed as void*) on a stream.
 * While the stream is being captured into a CUDA graph the record is captured as an
 * event node of the graph (cudaEventRecordExternal), so every replay of the graph
 * records the event; otherwise it is a plain cudaEventRecord.  moe_forward_timed
 * records its events the same way.  The pages have no counterpart: this exists so
 * that callers can time graph-replayed layer steps.
 * Errors: MOE_ERR_INVALID_ARG for a null event, MOE_ERR_CUDA if the record fails. */
moe_status moe_event_record(void* event, void* stream);

const char* moe_status_string(moe_status s);
int32_t moe_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */
