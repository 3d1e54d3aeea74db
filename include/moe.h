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

/* MOE_FMT_TERNARY_DENSE is a storage form of ternary experts (five codes per byte,
 * 1.6 bits per weight against 2): the packer writes it, the expert cache
 * (moe_cache_load) copies it from host memory and expands it on the GPU into
 * MOE_FMT_TERNARY, and no expert kernel reads it (moe_forward on a buffer that holds
 * it records MOE_ERR_DEVICE_CHECK with detail MOE_DETAIL_FORMAT and computes nothing). */
typedef enum { MOE_FMT_TERNARY = 0, MOE_FMT_Q2 = 1, MOE_FMT_Q3 = 2, MOE_FMT_TERNARY_DENSE = 3 } moe_format;

/* MOE_PATH_AUTO picks DECODE for T <= 64 and PREFILL otherwise.  DECODE runs the decode
 * kernels: for 5 <= T <= 8 the whole forward as one persistent kernel (the fused
 * decode kernel), otherwise separate gate/up, down and combine launches (the faster
 * choice at each T on the full-size layer).  MOE_PATH_DECODE_FUSED asks for the fused
 * decode kernel at any T <= 16 (MOE_ERR_UNSUPPORTED above).  All paths compute the
 * same function; they differ only in kernels and rounding of intermediates. */
typedef enum { MOE_PATH_AUTO = 0, MOE_PATH_DECODE = 1, MOE_PATH_PREFILL = 2, MOE_PATH_DECODE_FUSED = 3 } moe_path;

/* OR-ed into moe_forward's path: d_y is fp32 [T][H] instead of bf16 (the sums are not
 * rounded to bf16; the expert-parallel layer returns expert outputs this way, so that
 * its gate-weighted combine rounds once, as the single-GPU layer does). */
#define MOE_OUT_F32 0x10

/* Device pointers.  The token, output, router-weight, packed-expert and workspace
 * pointers given to moe_route and moe_forward must be 16-byte aligned (allocations from
 * cudaMalloc and the CUDA caching allocators are); others are MOE_ERR_INVALID_ARG. */

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
 * MOE_FMT_TERNARY_DENSE (a storage form): the ternary values as above, but the codes
 * array of a matrix holds ceil(K/5) bytes per packed row (rows in the same order as
 * the blocked arrays: packed row pr from byte pr*ceil(K/5)), element k in byte k/5 as
 * base-3 digit k%5 (byte i = sum over j < 5 of c(5i + j) 3^j, codes past K zero, at
 * most 242); the scales blocked as below; no third bits.
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

/* For tests of the failure path only (the pages have no counterpart).  cycles > 0
 * makes every expert kernel of the following moe_forward calls on this workspace first
 * wait, for at most `cycles` SM clock cycles, on a barrier that nothing completes.  The
 * wait runs out; the kernel records MOE_ERR_TIMEOUT with detail MOE_DETAIL_TEST_STALL
 * (low byte: which kernel), then takes the path every kernel takes when one of its
 * bounded waits runs out: it issues no further copies, waits (bounded) for the copies
 * it has in flight, releases its tensor memory and returns; d_y is then unspecified.
 * cycles = 0 (or moe_workspace_init) switches the stall off.  Enqueued on stream. */
moe_status moe_workspace_set_test_stall(void* d_ws, size_t ws_bytes, uint32_t cycles, void* stream);

/* Detail codes that moe_get_error returns beside MOE_ERR_TIMEOUT or
 * MOE_ERR_DEVICE_CHECK: the high bits say what happened, the low byte in which
 * kernel or wait. */
#define MOE_DETAIL_WAIT_FULL 0x100u   /* a wait for data (a copy, a stage) ran out        */
#define MOE_DETAIL_WAIT_EMPTY 0x200u  /* a wait for a free stage ran out                  */
#define MOE_DETAIL_DRAIN 0x300u       /* the wait for in-flight copies after a give-up    */
#define MOE_DETAIL_HEADER 0x400u      /* the packed buffer's header does not match        */
#define MOE_DETAIL_ROUTED_T 0x500u    /* moe_forward's T differs from moe_route's T       */
#define MOE_DETAIL_RANGE 0x600u       /* a token or expert activation outside fp16 range  */
#define MOE_DETAIL_TEST_STALL 0x700u  /* moe_workspace_set_test_stall's wait ran out      */
#define MOE_DETAIL_LOOP_CAP 0x800u    /* a work loop reached its iteration cap            */
#define MOE_DETAIL_FORMAT 0x900u      /* an expert in a storage form (dense ternary)      */

/* Route T tokens: fp32 router logits, softmax + top-k + renormalised gates,
 * per-expert histogram, prefix sum and permutation.
 *   d_x        bf16 bit patterns [T][H], row-major
 *   d_router_w fp32 [E][H], row-major
 *   d_router_b fp32 [E] added to the logits before the softmax, or NULL
 *   out        caller-allocated device arrays (see moe_routing)
 * Also leaves in d_ws the expert schedule that moe_forward reads, so moe_forward
 * must be given the same d_ws and T.  T = 0 is a no-op returning MOE_OK.
 * Router weights and bias must be finite (a NaN or infinity there gives unspecified
 * routing; nothing checks this).  Tokens must be finite with every |x| <= 65504: the
 * router checks each element and records MOE_ERR_DEVICE_CHECK with
 * MOE_DETAIL_RANGE | 1 for moe_get_error otherwise (routing and outputs are then
 * unspecified). */
moe_status moe_route(const moe_shape* shape, int32_t T, const uint16_t* d_x,
                     const float* d_router_w, const float* d_router_b, const moe_routing* out,
                     void* d_ws, size_t ws_bytes, void* stream);

/* moe_route with the expert choice given instead of computed: for callers that route
 * elsewhere, such as the expert-parallel layer, whose GPUs each run only their own
 * experts on the token rows sent to them (every row with one expert, gate 1).  Writes
 * the routing arrays (ids and gates copied from d_ids / d_gates, [T][k] each; counts,
 * offsets, perm, inv_perm computed as moe_route does) and the schedule in d_ws that
 * moe_forward reads.  Same argument rules and errors as moe_route; d_ids and d_gates
 * are device pointers.  An id outside [0, E) is recorded as MOE_ERR_DEVICE_CHECK
 * (MOE_DETAIL_RANGE | 2) and its pair is left out of every expert's rows; so is an id
 * that an earlier slot of the same token holds (MOE_DETAIL_RANGE | 5): a token's k ids
 * must be distinct, as moe_route's top-k makes them.  Outputs of a call with such a
 * pair are unspecified. */
moe_status moe_route_fixed(const moe_shape* shape, int32_t T, const uint16_t* d_x, const int32_t* d_ids,
                           const float* d_gates, const moe_routing* out, void* d_ws, size_t ws_bytes,
                           void* stream);

/* Expert-parallel row helpers (the layer's experts split over several GPUs; the pages
 * run their engine on more than one consumer GPU: molayo1419.me, "Delta Inference
 * Engine", the multi-GPU paragraph).  Both only enqueue one kernel on `stream` and
 * record bad indices in the control block of d_ws (moe_get_error), never faulting.
 *   moe_gather_rows:   d_dst[i][:] = d_src[d_index[i] / divisor][:] for i < n; bf16 rows
 *                      of `hidden` elements; d_src has n_src rows.  With d_index = perm
 *                      and divisor = top_k it builds the dispatch buffer (token rows in
 *                      expert-major order).  An index past d_src: MOE_DETAIL_RANGE | 3,
 *                      the row is zeroed.
 *   moe_combine_pairs: d_y[t][:] = sum_j d_gates[t][j] * d_rows[d_inv_perm[t k + j]][:]
 *                      (j ascending) + d_shared[t][:] (if not NULL), fp32 rows and sums
 *                      (moe_forward's MOE_OUT_F32 output), stored as bf16, for t < T;
 *                      d_rows has n_rows rows.  A row index past d_rows:
 *                      MOE_DETAIL_RANGE | 4, left out of the sum.
 * MOE_ERR_INVALID_ARG: a null pointer, hidden not a positive multiple of 64, a negative
 * count, divisor < 1, top_k outside 1..16. */
moe_status moe_gather_rows(int32_t n, int32_t hidden, const uint16_t* d_src, int32_t n_src,
                           const int32_t* d_index, int32_t divisor, uint16_t* d_dst, void* d_ws,
                           size_t ws_bytes, void* stream);
moe_status moe_combine_pairs(int32_t T, int32_t top_k, int32_t hidden, const float* d_rows, int32_t n_rows,
                             const int32_t* d_inv_perm, const float* d_gates, const float* d_shared,
                             uint16_t* d_y, void* d_ws, size_t ws_bytes, void* stream);

/* Host-tiered experts.  The engine on the pages keeps the experts that do not fit its
 * GPU in a pinned host-RAM arena and brings the ones a layer needs into GPU memory ahead
 * of use (ossradar.top, Xolotl README, "How it works, in one paragraph").  These calls
 * let a layer run from a device cache of n_slots expert slots in front of a packed
 * buffer h_packed in host memory (page-locked, so that the copies are asynchronous).
 * The cache d_cache is itself a packed buffer: the layer's header and expert table,
 * then the slots; pass it to moe_forward as d_packed.  Every expert the routing selects,
 * and the shared expert, must have been loaded into some slot first; which expert goes
 * to which slot (and when) is the caller's choice.
 *   moe_cache_size: bytes of the cache for n_slots slots (each as large as the largest
 *                   expert's span of the host buffer).
 *   moe_cache_init: writes the header and table (every entry pointing into slot 0 until
 *                   its expert is loaded); enqueued on stream.
 *   moe_cache_load: for i < n copies expert h_experts[i]'s span (its gate/up and down
 *                   arrays, contiguous in the packer's layout) into slot h_slots[i] and
 *                   points its table entry there: one cudaMemcpyAsync per expert and a
 *                   one-thread kernel for the entry, enqueued on stream (a prefetch
 *                   stream, with an event before the forward, overlaps it with compute).
 * MOE_ERR_INVALID_ARG: a null pointer, n_slots < 1, an expert or slot index out of
 * range, or a host buffer whose header does not describe the shape; MOE_ERR_WORKSPACE:
 * cache_bytes too small; MOE_ERR_CUDA: a copy or launch failed. */
moe_status moe_cache_size(const moe_shape* shape, const uint8_t* h_packed, int32_t n_slots, size_t* bytes);
moe_status moe_cache_init(const moe_shape* shape, const uint8_t* h_packed, int32_t n_slots, void* d_cache,
                          size_t cache_bytes, void* stream);
moe_status moe_cache_load(const moe_shape* shape, const uint8_t* h_packed, int32_t n_slots, void* d_cache,
                          size_t cache_bytes, const int32_t* h_experts, const int32_t* h_slots, int32_t n,
                          void* stream);

/* Expert FFNs of the routed and shared experts and the gate-weighted combine,
 * using the routing of the preceding moe_route on the same d_ws.
 *   d_packed  packed experts (format above), device memory
 *   d_x       bf16 [T][H] (the same tokens as routed)
 *   r         the routing moe_route wrote
 *   d_y       bf16 [T][H] output, written in full (fp32 with path | MOE_OUT_F32)
 * T = 0 is a no-op.  T > 64 with MOE_PATH_DECODE is allowed (slower).
 * Checked on the device (recorded for moe_get_error; d_y is then unspecified):
 *   - T must be the T of the preceding moe_route on d_ws; otherwise the expert
 *     kernels return without reading the routing (MOE_ERR_DEVICE_CHECK,
 *     MOE_DETAIL_ROUTED_T).
 *   - Range: the kernels hold tokens (prefill) and the expert activations
 *     h = silu(Wg x) * (Wu x) (both paths) in fp16, so they compute the layer for
 *     tokens with every |x| <= 65504 whose activations have every |h| <= 65504.  A
 *     token or an activation outside that range is reported as MOE_ERR_DEVICE_CHECK
 *     with MOE_DETAIL_RANGE (the router reports tokens, low byte 1; the gate/up
 *     kernels activations). */
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

/* The kernels that moe_route followed by moe_forward(shape, T, path) launch; host-only
 * (no device work, no CUDA call).  plan is a caller array of 4 int32:
 *   plan[0]  the kernels moe_forward runs: MOE_PATH_DECODE (separate gate/up, down and
 *            combine launches), MOE_PATH_PREFILL (the tcgen05 kernels) or
 *            MOE_PATH_DECODE_FUSED (the fused decode kernel)
 *   plan[1]  kernels launched by the two calls together (0 for T = 0)
 *   plan[2], plan[3]  K parts of the separate decode gate/up and down passes (1 on the
 *            other paths); gate/up in more than one part adds its reduction launch
 * Errors: those of moe_forward's argument checks on shape, T and path
 * (MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED); a null plan is MOE_ERR_INVALID_ARG. */
moe_status moe_forward_plan(const moe_shape* shape, int32_t T, moe_path path, int32_t* plan);

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
 *   - Every argument check of moe_route and moe_forward runs before anything is
 *     enqueued; a rejected call leaves the scratch array and d_y untouched.
 *   - If the workspace T tokens need (moe_workspace_size) exceeds MOE_STATIC_WS_BYTES
 *     it returns MOE_ERR_WORKSPACE; with the full-size layer (H 7168, I 2048, E 256,
 *     k 8, S 1) that allows up to 21 tokens per call.
 *   - The first call on each device (and the first after a cudaDeviceReset) looks up
 *     the scratch array's device address (cudaGetSymbolAddress) with that device
 *     current; make that first call before any stream capture.  Later calls only
 *     enqueue work.
 *   - All calls share the one array, and each call first clears its counters.
 *     Calls that overlap on the GPU (other streams, other host threads; other
 *     devices' calls do not overlap) race on the array: serialise them.
 *   - Problems found on the device (a bounded wait that ran out, a corrupt packed
 *     header) are recorded in the array and kept across later calls until
 *     moe_decode_static_get_error reads and clears them. */
#define MOE_STATIC_WS_BYTES ((size_t)8 << 20)
moe_status moe_decode_static(const moe_shape* shape, int32_t T, const uint16_t* d_x,
                             const float* d_router_w, const float* d_router_b, const void* d_packed,
                             const moe_routing* out, uint16_t* d_y, void* stream);

/* moe_get_error for the scratch array of moe_decode_static on the current device:
 * synchronises the stream, returns the first problem recorded by any
 * moe_decode_static call since the last read (MOE_OK, MOE_ERR_TIMEOUT or
 * MOE_ERR_DEVICE_CHECK; *detail, if not NULL, the detail code) and clears it.
 * MOE_ERR_CUDA if the array's address cannot be looked up or the copy fails. */
moe_status moe_decode_static_get_error(void* stream, uint32_t* detail);

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
