// Expert FFN kernels of the decode path (steps a4, a5, a8) and the gate-weighted
// unpermute-combine (a9): grouped skinny GEMMs over the packed ternary / 2-bit /
// 3-bit experts, for few tokens per expert.
//
// Decode speed is set by the expert bytes moved per token (ossradar.top, Xolotl
// README, "Fast mode (DeepSeek-V4.1)"), and each selected expert is read once for
// all of its tokens (the same README, "Latest": the CPU kernels that decode an
// expert once for its 4-8 tokens).  So every selected expert's packed bytes are
// streamed exactly once and applied to all of its tokens:
//
//  * Work item = (active expert, 16-row tile of the packed matrix, token pass of up
//    to 8*NT tokens).  Every warp owns whole items (items w, w + P, w + 2P, ... for P
//    warps in the grid) and walks the full K of each; no two warps share an item, so
//    there is no cross-warp reduction and no CTA-wide barrier in the main loop.
//  * Each warp streams its items through its own ring of NS shared-memory stages with
//    1-D bulk copies (cp.async.bulk on the TMA engine, completion on a per-stage
//    mbarrier); a stage holds one 8-group (512-wide) chunk of K for the 16 rows:
//    codes, third bits and fp16 scales, each a contiguous block of the packed format
//    (three copies per chunk).  The format's XOR swizzle keeps the fragment reads
//    free of bank conflicts.  The ring runs NS-1 chunks ahead, across items.
//  * A 32-bit code word (16 codes of one row) becomes eight bf16 / fp16 pairs with
//    shifts and lop3 (magic-number exponent trick: the code lands in the mantissa of
//    a power-of-two base, exactly), the A operand of mma.sync m16n8k16; the tokens
//    are N (8 per n-tile) and the B fragments come straight from the token rows.
//      gate/up: pairs stay "base + c"; each 64-wide group's accumulator starts at
//        -Z[token, group] (Z = sum base(k) x_k + o sum x_k, plus the third-bit bases
//        for 3-bit experts; computed by the router), so the MMA yields
//        sum (c_k - o) x_k.  bf16 MMAs: the tokens are bf16.
//      down: pairs are (c - o) exactly (one fp16x2 subtract); fp16 MMAs, h is fp16.
//    Each group result is scaled by its fp16 scale into an fp32 accumulator.
//    3-bit experts add an MMA for 4 * (third bit).
//  * gate/up: the 16 rows of a tile are 8 gate rows and the matching 8 up rows, which
//    the MMA places in the same thread (rows g and g + 8), so h = silu(gate) * up is
//    formed in registers and stored as fp16.
//  * down: partial rows (fp32) per (token, slot); the combine kernel then sums each
//    token's k slots in slot order with the gates, adds the shared expert and writes
//    y in bf16: deterministic, no floating-point atomics.
// Every wait is bounded; a wait that runs out records an error in the workspace and
// the warp carries on without waiting, so the kernel always terminates.
#include "kernels.h"

namespace moe {
namespace {

constexpr int CG = 8;                                  // 64-wide groups per chunk
constexpr int OFF_HI = 2048;                           // codes block: 16 rows x 32 words
constexpr int OFF_SC = OFF_HI + 1024;                  // third-bit block: 16 rows x 16 words
constexpr int STAGE = OFF_SC + 256;                    // scales block: 16 rows x 8 halves
constexpr int NS = 4;                                  // stages per warp (power of two)
constexpr long long kWaitLimit = 4000000000LL;         // clock cycles (~2 s)

// bf16 magic bases (exponent-only bit patterns) of the gate/up dequantiser
constexpr uint32_t kMag64 = 0x42804280u, kMag32 = 0x42004200u, kMag16 = 0x41804180u, kMag8 = 0x41004100u,
                   kMag4 = 0x40804080u, kMag512 = 0x44004400u, kMag256 = 0x43804380u, kMag128 = 0x43004300u;
// fp16 magic bases of the down dequantiser
constexpr uint32_t kH512 = 0x60006000u, kH256 = 0x5C005C00u, kH64 = 0x54005400u, kH16 = 0x4C004C00u,
                   kH4 = 0x44004400u, kH4096 = 0x6C006C00u, kH2048 = 0x68006800u, kH1024 = 0x64006400u,
                   kH128 = 0x58005800u, kH32 = 0x50005000u;

// ---- dequantisers (code word: element 2p + h of its 16 at bits 16h + 2p .. +1) ----

// bf16 pairs "base_p + c"; base per pair p: 64, 32, 8, 16, 4, 64, 16, 4.
__device__ inline void raw_codes_bf16(uint32_t w, uint32_t (&pr)[8]) {
    const uint32_t w1 = w << 1, w3 = w >> 3, w9 = w >> 9;
    pr[0] = lop3_and_or(w1, 0x00060006u, kMag64);   // bits 0-1 -> 1-2
    pr[1] = lop3_and_or(w, 0x000C000Cu, kMag32);    // bits 2-3
    pr[2] = lop3_and_or(w, 0x00300030u, kMag8);     // bits 4-5
    pr[3] = lop3_and_or(w3, 0x00180018u, kMag16);   // bits 6-7 -> 3-4
    pr[4] = lop3_and_or(w3, 0x00600060u, kMag4);    // bits 8-9 -> 5-6
    pr[5] = lop3_and_or(w9, 0x00060006u, kMag64);   // bits 10-11 -> 1-2
    pr[6] = lop3_and_or(w9, 0x00180018u, kMag16);   // bits 12-13 -> 3-4
    pr[7] = lop3_and_or(w9, 0x00600060u, kMag4);    // bits 14-15 -> 5-6
}

// bf16 pairs "base_p + 4 * bit" of the third code bit (bits 0..7 of each half of u);
// base per pair p: 512, 256, 128, 64, 32, 16, 8, 8.
__device__ inline void raw_hi_bf16(uint32_t u, uint32_t (&pr)[8]) {
    pr[0] = lop3_and_or(u, 0x00010001u, kMag512);
    pr[1] = lop3_and_or(u, 0x00020002u, kMag256);
    pr[2] = lop3_and_or(u, 0x00040004u, kMag128);
    pr[3] = lop3_and_or(u, 0x00080008u, kMag64);
    pr[4] = lop3_and_or(u, 0x00100010u, kMag32);
    pr[5] = lop3_and_or(u, 0x00200020u, kMag16);
    pr[6] = lop3_and_or(u, 0x00400040u, kMag8);
    pr[7] = lop3_and_or(u >> 1, 0x00400040u, kMag8);
}

// fp16 pairs (c - o), exact: the bases 512, 256, 64, 16, 4 have an ulp <= 1/2.
__device__ inline void exact_codes_f16(uint32_t w, const uint32_t (&sub)[5], uint32_t (&pr)[8]) {
    const uint32_t w1 = w << 1, w8 = w >> 8;
    pr[0] = f16x2_sub(lop3_and_or(w1, 0x00060006u, kH512), sub[0]);    // bits 0-1 -> 1-2
    pr[1] = f16x2_sub(lop3_and_or(w, 0x000C000Cu, kH256), sub[1]);     // bits 2-3
    pr[2] = f16x2_sub(lop3_and_or(w, 0x00300030u, kH64), sub[2]);      // bits 4-5
    pr[3] = f16x2_sub(lop3_and_or(w, 0x00C000C0u, kH16), sub[3]);      // bits 6-7
    pr[4] = f16x2_sub(lop3_and_or(w, 0x03000300u, kH4), sub[4]);       // bits 8-9
    pr[5] = f16x2_sub(lop3_and_or(w8, 0x000C000Cu, kH256), sub[1]);    // bits 10-11 -> 2-3
    pr[6] = f16x2_sub(lop3_and_or(w8, 0x00300030u, kH64), sub[2]);     // bits 12-13 -> 4-5
    pr[7] = f16x2_sub(lop3_and_or(w8, 0x00C000C0u, kH16), sub[3]);     // bits 14-15 -> 6-7
}

// fp16 pairs 4 * (third bit), exact.
__device__ inline void exact_hi_f16(uint32_t u, uint32_t (&pr)[8]) {
    pr[0] = f16x2_sub(lop3_and_or(u, 0x00010001u, kH4096), kH4096);
    pr[1] = f16x2_sub(lop3_and_or(u, 0x00020002u, kH2048), kH2048);
    pr[2] = f16x2_sub(lop3_and_or(u, 0x00040004u, kH1024), kH1024);
    pr[3] = f16x2_sub(lop3_and_or(u, 0x00080008u, kH512), kH512);
    pr[4] = f16x2_sub(lop3_and_or(u, 0x00100010u, kH256), kH256);
    pr[5] = f16x2_sub(lop3_and_or(u, 0x00200020u, kH128), kH128);
    pr[6] = f16x2_sub(lop3_and_or(u, 0x00400040u, kH64), kH64);
    pr[7] = f16x2_sub(lop3_and_or(u, 0x00800080u, kH32), kH32);
}

// L1 prefetch of chunk c's token lines and Z values for this lane's columns: lane t of a
// row takes the 128-byte lines of groups t and t + 4 (the row's B operand for the
// chunk is 8 lines), so the loads of the chunk hit L1 instead of waiting on L2.
// Only groups inside the row are touched (a partial last chunk has fewer).
template <int MODE, int NT, typename View>
__device__ inline void prefetch_chunk(const View& v, int c, int t, int G) {
    const int ng = min(CG, G - c * CG);
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const uint16_t* line0 = v.b[n] - 16 * t + c * CG * 64;
        if (t < ng) prefetch_l1(line0 + 64 * t);
        if (t + 4 < ng) prefetch_l1(line0 + 64 * (t + 4));
        if (MODE == 0) {
            prefetch_l1(v.z[n][0] + c * CG);
            prefetch_l1(v.z[n][1] + c * CG);
        }
    }
}

// Gate/up with few tokens: every SM reads the same token rows and Z values, so each CTA
// pulls them into L1 at the start.  The token rows are the caller's input (ready before
// the router ran); the Z values are the router's output and are prefetched only after
// griddep_wait(), so no stale line can enter L1.  The zx region is padded to 256 bytes,
// so whole lines stay inside it.
__device__ inline bool warm_fits(const FfnArgs& p) {
    return (size_t)p.T * p.H * 2 + (size_t)3 * p.T * (p.H / 64) * 4 <= 48 * 1024;
}
__device__ inline void warm_rows(const FfnArgs& p) {
    if (!warm_fits(p)) return;
    const size_t xb = (size_t)p.T * p.H * 2;
    for (size_t i = threadIdx.x; i < xb / 128; i += blockDim.x)
        prefetch_l1(reinterpret_cast<const uint8_t*>(p.x) + i * 128);
}
__device__ inline void warm_z(const FfnArgs& p) {
    if (!warm_fits(p)) return;
    const size_t zb = (size_t)3 * p.T * (p.H / 64) * 4;
    for (size_t i = threadIdx.x; i < (zb + 127) / 128; i += blockDim.x)
        prefetch_l1(reinterpret_cast<const uint8_t*>(p.zx) + i * 128);
}

__device__ inline float half_bits_to_f32(uint16_t h) { return __half2float(__ushort_as_half(h)); }

template <int MODE>
__device__ inline void mma4(float& d0, float& d1, float& d2, float& d3, const uint32_t (&pa)[8],
                            const uint32_t (&pb)[8], const uint32_t (&xb)[8]) {
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        if (MODE == 0)
            mma_bf16_16816(d0, d1, d2, d3, pa[2 * s], pb[2 * s], pa[2 * s + 1], pb[2 * s + 1], xb[2 * s],
                           xb[2 * s + 1]);
        else
            mma_f16_16816(d0, d1, d2, d3, pa[2 * s], pb[2 * s], pa[2 * s + 1], pb[2 * s + 1], xb[2 * s],
                          xb[2 * s + 1]);
    }
}

__device__ inline const PackedEntry* entry(const uint8_t* packed, int e) {
    return reinterpret_cast<const PackedEntry*>(packed + kHeaderBytes + (size_t)e * kEntryBytes);
}

struct CtaSched {
    int ok;
    int n_active;
    int n_items;
    int e[260];
    int fmt[260];
    int cnt[260];
    int ipre[261];   // item prefix over active experts
};

__device__ inline int find_active(const CtaSched& S, int item) {
    int lo = 0, hi = S.n_active - 1;     // largest a with ipre[a] <= item
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (S.ipre[mid] <= item) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

template <int MODE>
__device__ inline void mma_acc(float& d0, float& d1, float& d2, float& d3, uint32_t a0, uint32_t a1, uint32_t a2,
                               uint32_t a3, uint32_t b0, uint32_t b1) {
    if (MODE == 0)
        asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d0), "+f"(d1), "+f"(d2), "+f"(d3)
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    else
        asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d0), "+f"(d1), "+f"(d2), "+f"(d3)
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Per-lane view of one work item (16-row tile x token pass).
template <int NT>
struct ItemView {
    const uint16_t* b[NT];     // B-operand row of token column g of n-tile n (+16t elements)
    const float* z[NT][2];     // -Z rows of output columns 2t, 2t+1 (gate/up only)
    int orow[NT][2];           // output rows of columns 2t, 2t+1 (-1: no token)
};

// Dequantise the code words of rows g (wa) and g + 8 (wb) straight into MMA
// A-fragment order: quad s = {pair 2s of wa, pair 2s of wb, pair 2s+1 of wa, pair 2s+1 of wb}.
template <int MODE>
__device__ __forceinline__ void dequant_quads(uint32_t wa, uint32_t wb, const uint32_t (&sub)[5], uint32_t (&q)[16]) {
    uint32_t pa[8], pb[8];
    if (MODE == 0) {
        raw_codes_bf16(wa, pa);
        raw_codes_bf16(wb, pb);
    } else {
        exact_codes_f16(wa, sub, pa);
        exact_codes_f16(wb, sub, pb);
    }
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        q[4 * s + 0] = pa[2 * s];
        q[4 * s + 1] = pb[2 * s];
        q[4 * s + 2] = pa[2 * s + 1];
        q[4 * s + 3] = pb[2 * s + 1];
    }
}

template <int MODE>
__device__ __forceinline__ void dequant_hi_quads(uint32_t ua, uint32_t ub, uint32_t (&q)[16]) {
    uint32_t pa[8], pb[8];
    if (MODE == 0) {
        raw_hi_bf16(ua, pa);
        raw_hi_bf16(ub, pb);
    } else {
        exact_hi_f16(ua, pa);
        exact_hi_f16(ub, pb);
    }
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        q[4 * s + 0] = pa[2 * s];
        q[4 * s + 1] = pb[2 * s];
        q[4 * s + 2] = pa[2 * s + 1];
        q[4 * s + 3] = pb[2 * s + 1];
    }
}

// One 64-wide group: dequantise rows g and g+8, MMA against every n-tile, fold the
// scaled group result into acc.  wa/wb: code words, ua/ub: third-bit words (already
// shifted), s0/s1: scales, bx[n]: B row pointers of this group, zc[n]: -Z rows at
// this group (gate/up).
template <int MODE, int NT, bool Q3>
__device__ __forceinline__ void group_step(uint32_t wa, uint32_t wb, uint32_t ua, uint32_t ub, float s0, float s1,
                                           const uint16_t* const (&bx)[NT], const float* const (&zc)[NT][2],
                                           const uint32_t (&sub)[5], float (&acc)[NT][4]) {
    uint32_t q[16], hq[16];
    dequant_quads<MODE>(wa, wb, sub, q);
    if (Q3) dequant_hi_quads<MODE>(ua, ub, hq);
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const uint4 b0 = __ldg(reinterpret_cast<const uint4*>(bx[n]));
        const uint4 b1 = __ldg(reinterpret_cast<const uint4*>(bx[n]) + 1);
        float d0, d1, d2, d3;
        if (MODE == 0) {
            d0 = __ldg(zc[n][0]);
            d1 = __ldg(zc[n][1]);
            d2 = d0;
            d3 = d1;
        } else {
            d0 = d1 = d2 = d3 = 0.f;
        }
        mma_acc<MODE>(d0, d1, d2, d3, q[0], q[1], q[2], q[3], b0.x, b0.y);
        mma_acc<MODE>(d0, d1, d2, d3, q[4], q[5], q[6], q[7], b0.z, b0.w);
        mma_acc<MODE>(d0, d1, d2, d3, q[8], q[9], q[10], q[11], b1.x, b1.y);
        mma_acc<MODE>(d0, d1, d2, d3, q[12], q[13], q[14], q[15], b1.z, b1.w);
        if (Q3) {
            mma_acc<MODE>(d0, d1, d2, d3, hq[0], hq[1], hq[2], hq[3], b0.x, b0.y);
            mma_acc<MODE>(d0, d1, d2, d3, hq[4], hq[5], hq[6], hq[7], b0.z, b0.w);
            mma_acc<MODE>(d0, d1, d2, d3, hq[8], hq[9], hq[10], hq[11], b1.x, b1.y);
            mma_acc<MODE>(d0, d1, d2, d3, hq[12], hq[13], hq[14], hq[15], b1.z, b1.w);
        }
        acc[n][0] = fmaf(s0, d0, acc[n][0]);
        acc[n][1] = fmaf(s0, d1, acc[n][1]);
        acc[n][2] = fmaf(s1, d2, acc[n][2]);
        acc[n][3] = fmaf(s1, d3, acc[n][3]);
    }
}

// Producer side of a warp's ring: issues the three bulk copies of the next chunk.
template <int MODE>
struct RingProducer {
    const uint8_t* codes;
    const uint8_t* hi;
    const uint8_t* sc;
    int item, c, issued, j, q3, cur_item;
    __device__ void load_item(const FfnArgs& p, const CtaSched& S, int tiles) {
        const int a = find_active(S, item);
        j = (item - S.ipre[a]) % tiles;
        const PackedEntry* en = entry(p.packed, S.e[a]);
        codes = p.packed + (MODE == 0 ? en->gu_codes : en->dn_codes);
        hi = p.packed + (MODE == 0 ? en->gu_hi : en->dn_hi);
        sc = p.packed + (MODE == 0 ? en->gu_scales : en->dn_scales);
        q3 = S.fmt[a] == MOE_FMT_Q3;
        cur_item = item;
    }
    __device__ void issue(const FfnArgs& p, const CtaSched& S, int n_items, int P, int tiles, int K, int G, int NC,
                          uint8_t* ring, uint64_t* bar, uint64_t pol, int lane) {
        if (item >= n_items) return;
        if (item != cur_item) load_item(p, S, tiles);
        const int st = issued & (NS - 1);
        const int ng = min(CG, G - c * CG);
        if (elect_one()) {                      // warp-uniform issue, one elected lane
            uint8_t* dst = ring + (size_t)st * STAGE;
            const uint32_t cb = 256 * ng, hb = q3 ? 128 * ng : 0;
            mbar_arrive_expect_tx(&bar[st], cb + hb + 256);
            bulk_g2s_evict_first(dst, codes + (size_t)4 * K * j + 2048 * (size_t)c, cb, &bar[st], pol);
            bulk_g2s_evict_first(dst + OFF_SC, sc + (size_t)256 * NC * j + 256 * (size_t)c, 256, &bar[st], pol);
            if (hb) bulk_g2s_evict_first(dst + OFF_HI, hi + (size_t)128 * G * j + 1024 * (size_t)c, hb, &bar[st], pol);
        }
        ++issued;
        if (++c == NC) {
            c = 0;
            item += P;
        }
    }
};

template <int MODE, int NT, bool Q3>
__device__ __forceinline__ void run_item(const FfnArgs& p, const CtaSched& S, RingProducer<MODE>& prod,
                                         int& consumed, bool& aborted, const ItemView<NT>& v, const uint32_t (&sub)[5],
                                         float (&acc)[NT][4], int n_items, int P, int tiles, int K, int G, int NC,
                                         uint8_t* ring, uint64_t* bar, uint64_t pol, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const int sh = 8 * (t & 1);
    // swizzle offsets of group gl inside a full chunk: codes 4*(gl^g), third bits 2*(gl^(g/2))
    int sw4[CG], sw2[CG];
#pragma unroll
    for (int gl = 0; gl < CG; ++gl) {
        sw4[gl] = 4 * (gl ^ g);
        sw2[gl] = 2 * (gl ^ (g >> 1));
    }
    prefetch_chunk<MODE, NT>(v, 0, t, G);
    for (int c = 0; c < NC; ++c) {
        prod.issue(p, S, n_items, P, tiles, K, G, NC, ring, bar, pol, lane);
        if (c + 1 < NC) prefetch_chunk<MODE, NT>(v, c + 1, t, G);
        const int st = consumed & (NS - 1);
        if (!aborted && !mbar_wait_bounded(&bar[st], (uint32_t)(consumed / NS) & 1, kWaitLimit)) {
            aborted = true;
            report_error(p.ctrl, MOE_ERR_TIMEOUT, kDetWaitFull | MODE);
        }
        const uint8_t* stg = ring + (size_t)st * STAGE;
        const uint32_t* cw = reinterpret_cast<const uint32_t*>(stg);
        const uint32_t* hw = reinterpret_cast<const uint32_t*>(stg + OFF_HI);
        const uint16_t* scs = reinterpret_cast<const uint16_t*>(stg + OFF_SC) + g * 8;
        // this chunk's B rows and -Z rows (constant offsets per group below)
        const uint16_t* bc[NT];
        const float* zcb[NT][2];
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            bc[n] = v.b[n] + c * CG * 64;
            zcb[n][0] = MODE == 0 ? v.z[n][0] + c * CG : nullptr;
            zcb[n][1] = MODE == 0 ? v.z[n][1] + c * CG : nullptr;
        }
        const int ng = min(CG, G - c * CG);
        if (ng == CG) {
            const uint32_t* cwa = cw + g * 32 + t;          // row g; row g + 8 is 256 words on
            const uint32_t* hwa = hw + g * 16 + (t >> 1);   // row g; row g + 8 is 128 words on
#pragma unroll
            for (int gl = 0; gl < CG; ++gl) {
                const uint32_t wa = cwa[sw4[gl]], wb = cwa[sw4[gl] + 256];
                uint32_t ua = 0, ub = 0;
                if (Q3) {
                    ua = hwa[sw2[gl]] >> sh;
                    ub = hwa[sw2[gl] + 128] >> sh;
                }
                const uint16_t* bx[NT];
                const float* zc[NT][2];
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    bx[n] = bc[n] + gl * 64;
                    zc[n][0] = zcb[n][0] + gl;
                    zc[n][1] = zcb[n][1] + gl;
                }
                group_step<MODE, NT, Q3>(wa, wb, ua, ub, half_bits_to_f32(scs[gl]), half_bits_to_f32(scs[64 + gl]),
                                         bx, zc, sub, acc);
            }
        } else {
            for (int gl = 0; gl < ng; ++gl) {
                const uint32_t wa = cw[g * 4 * ng + 4 * gl + t], wb = cw[(g + 8) * 4 * ng + 4 * gl + t];
                uint32_t ua = 0, ub = 0;
                if (Q3) {
                    ua = hw[g * 2 * ng + 2 * gl + (t >> 1)] >> sh;
                    ub = hw[(g + 8) * 2 * ng + 2 * gl + (t >> 1)] >> sh;
                }
                const uint16_t* bx[NT];
                const float* zc[NT][2];
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    bx[n] = bc[n] + gl * 64;
                    zc[n][0] = zcb[n][0] + gl;
                    zc[n][1] = zcb[n][1] + gl;
                }
                group_step<MODE, NT, Q3>(wa, wb, ua, ub, half_bits_to_f32(scs[gl]), half_bits_to_f32(scs[64 + gl]),
                                         bx, zc, sub, acc);
            }
        }
        __syncwarp();          // every lane is done with this stage before it is refilled
        ++consumed;
    }
}

template <int MODE, int NT, int NW>
__global__ void __launch_bounds__(NW * 32, 1) ffn_decode_kernel(FfnArgs p) {
    constexpr int TB = 8 * NT;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ CtaSched S;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int K = MODE == 0 ? p.H : p.I;
    const int tiles = MODE == 0 ? (2 * p.I) / 16 : p.H / 16;
    const int G = K / 64, NC = (G + CG - 1) / CG;
    uint8_t* ring = smem + (size_t)warp * NS * STAGE;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + (size_t)NW * NS * STAGE) + warp * NS;

    // ---- header check and the CTA's copy of the expert schedule --------------------
    // Work that does not depend on the router's (or the previous pass's) outputs runs
    // before griddep_wait() and overlaps the predecessor's tail: the header check and
    // the token rows; the schedule and everything after read the predecessor's data.
    griddep_launch_dependents();                        // all CTAs of this grid are resident
    if (threadIdx.x == 0) {
        const uint32_t* hd = reinterpret_cast<const uint32_t*>(p.packed);
        S.ok = hd[0] == kMagic && hd[1] == kVersion && (int)hd[2] == p.H && (int)hd[3] == p.I &&
               (int)hd[4] == p.E && (int)hd[5] == p.S && hd[6] == 64u && hd[7] == (uint32_t)kInterleave;
    }
    if (MODE == 0) warm_rows(p);
    griddep_wait();
    if (threadIdx.x == 0) {
        if (!S.ok) report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetHeader);
        S.n_active = p.ctrl->n_active;
    }
    __syncthreads();
    if (!S.ok) return;
    const int nA = S.n_active;
    for (int a = threadIdx.x; a < nA; a += blockDim.x) {
        const int e = p.active[a];
        S.e[a] = e;
        S.fmt[a] = (int)entry(p.packed, e)->fmt;
        S.cnt[a] = e < p.E ? p.counts[e] : p.T;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int a = 0; a < nA; ++a) {
            S.ipre[a] = run;
            run += tiles * ((S.cnt[a] + TB - 1) / TB);
        }
        S.ipre[nA] = run;
        S.n_items = run;
    }
    if (MODE == 0) warm_z(p);
    if (lane == 0)
        for (int s = 0; s < NS; ++s) mbar_init(&bar[s], 1);
    fence_mbar_init();
    __syncthreads();
    const int n_items = S.n_items;
    const int P = gridDim.x * NW;
    // items dealt round-robin over the CTAs first (spreads each expert over many SMs)
    const int gw = warp * gridDim.x + blockIdx.x;
    const uint64_t pol = l2_policy_evict_first();

    RingProducer<MODE> prod;
    prod.item = gw;
    prod.c = 0;
    prod.issued = 0;
    prod.cur_item = -1;
    for (int i = 0; i < NS - 1; ++i) prod.issue(p, S, n_items, P, tiles, K, G, NC, ring, bar, pol, lane);

    bool aborted = false;
    int consumed = 0;
    for (int item = gw; item < n_items; item += P) {
        const int a = find_active(S, item);
        const int r = item - S.ipre[a];
        const int pass = r / tiles, j = r - pass * tiles;
        const int e = S.e[a], f = S.fmt[a], cnt = S.cnt[a];
        const int tb = pass * TB, nb = min(TB, cnt - tb);
        // Token columns of this pass.  Columns without a token read a valid row (the
        // pass's first token): their MMA outputs are never stored.
        ItemView<NT> v;
        const uint16_t* bsrc = MODE == 0 ? p.x : p.h;
        const int bld = MODE == 0 ? p.H : p.I;
        const float* zf = MODE == 0 ? p.zx + (size_t)f * p.T * G : nullptr;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int cb = n * 8 + g;
            const int i = tb + (cb < nb ? cb : 0);
            int brow;
            if (e < p.E) {
                const int hr = p.offsets[e] + i;
                brow = MODE == 0 ? p.perm[hr] / p.k : hr;
            } else {
                brow = MODE == 0 ? i : p.T * p.k + (e - p.E) * p.T + i;
            }
            v.b[n] = bsrc + (size_t)brow * bld + 16 * t;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int col = n * 8 + 2 * t + cc;
                const int ii = tb + (col < nb ? col : 0);
                int orow, ztok;
                if (e < p.E) {
                    orow = p.offsets[e] + ii;
                    ztok = p.perm[orow] / p.k;
                } else {
                    orow = p.T * p.k + (e - p.E) * p.T + ii;
                    ztok = ii;
                }
                v.orow[n][cc] = col < nb ? orow : -1;
                v.z[n][cc] = MODE == 0 ? zf + (size_t)ztok * G : nullptr;
            }
        }
        uint32_t sub[5] = {0, 0, 0, 0, 0};
        if (MODE == 1) {
            const float o = f == MOE_FMT_TERNARY ? 1.f : (f == MOE_FMT_Q2 ? 1.5f : 3.5f);
            sub[0] = f16x2_bits_of(512.f + o);
            sub[1] = f16x2_bits_of(256.f + o);
            sub[2] = f16x2_bits_of(64.f + o);
            sub[3] = f16x2_bits_of(16.f + o);
            sub[4] = f16x2_bits_of(4.f + o);
        }
        float acc[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
        if (f == MOE_FMT_Q3)
            run_item<MODE, NT, true>(p, S, prod, consumed, aborted, v, sub, acc, n_items, P, tiles, K, G, NC, ring, bar,
                                     pol, lane);
        else
            run_item<MODE, NT, false>(p, S, prod, consumed, aborted, v, sub, acc, n_items, P, tiles, K, G, NC, ring,
                                      bar, pol, lane);
        // epilogue
#pragma unroll
        for (int n = 0; n < NT; ++n) {
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                if (v.orow[n][cc] < 0) continue;
                if (MODE == 0) {
                    p.h[(size_t)v.orow[n][cc] * p.I + j * 8 + g] =
                        f32_to_f16_bits(silu_f(acc[n][cc]) * acc[n][2 + cc]);
                } else {
                    p.ypart[(size_t)v.orow[n][cc] * p.H + j * 16 + g] = acc[n][cc];
                    p.ypart[(size_t)v.orow[n][cc] * p.H + j * 16 + g + 8] = acc[n][2 + cc];
                }
            }
        }
    }
    // after a timeout the ring may still hold copies in flight: wait for them (bounded)
    if (aborted) {
        for (int q = consumed; q < prod.issued; ++q)
            if (!mbar_wait_bounded(&bar[q & (NS - 1)], (uint32_t)(q / NS) & 1, kWaitLimit)) {
                report_error(p.ctrl, MOE_ERR_TIMEOUT, kDetDrain | MODE);
                break;
            }
    }
}

// y[t] = sum_j g[t,j] * ypart[inv_perm[t*k + j]] + sum_s ypart[T*k + s*T + t], in slot
// order, fp32, stored as bf16.  One thread per 8 consecutive outputs.
__global__ void __launch_bounds__(256) combine_kernel(FfnArgs p) {
    griddep_wait();                                     // ypart comes from the down pass
    const int per_tok = p.H / 8;
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= p.T * per_tok) return;
    const int tok = idx / per_tok, c8 = (idx - tok * per_tok) * 8;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int sl = 0; sl < p.k; ++sl) {
        const int row = p.inv_perm[(size_t)tok * p.k + sl];
        const float gw = p.topk_w[(size_t)tok * p.k + sl];
        const float4* src = reinterpret_cast<const float4*>(p.ypart + (size_t)row * p.H + c8);
        const float4 v0 = __ldg(src), v1 = __ldg(src + 1);
        acc[0] = fmaf(gw, v0.x, acc[0]);
        acc[1] = fmaf(gw, v0.y, acc[1]);
        acc[2] = fmaf(gw, v0.z, acc[2]);
        acc[3] = fmaf(gw, v0.w, acc[3]);
        acc[4] = fmaf(gw, v1.x, acc[4]);
        acc[5] = fmaf(gw, v1.y, acc[5]);
        acc[6] = fmaf(gw, v1.z, acc[6]);
        acc[7] = fmaf(gw, v1.w, acc[7]);
    }
    for (int s = 0; s < p.S; ++s) {
        const float4* src =
            reinterpret_cast<const float4*>(p.ypart + ((size_t)p.T * p.k + (size_t)s * p.T + tok) * p.H + c8);
        const float4 v0 = __ldg(src), v1 = __ldg(src + 1);
        acc[0] += v0.x;
        acc[1] += v0.y;
        acc[2] += v0.z;
        acc[3] += v0.w;
        acc[4] += v1.x;
        acc[5] += v1.y;
        acc[6] += v1.z;
        acc[7] += v1.w;
    }
    uint4 o;
    o.x = (uint32_t)f32_to_bf16_bits(acc[0]) | ((uint32_t)f32_to_bf16_bits(acc[1]) << 16);
    o.y = (uint32_t)f32_to_bf16_bits(acc[2]) | ((uint32_t)f32_to_bf16_bits(acc[3]) << 16);
    o.z = (uint32_t)f32_to_bf16_bits(acc[4]) | ((uint32_t)f32_to_bf16_bits(acc[5]) << 16);
    o.w = (uint32_t)f32_to_bf16_bits(acc[6]) | ((uint32_t)f32_to_bf16_bits(acc[7]) << 16);
    *reinterpret_cast<uint4*>(p.y + (size_t)tok * p.H + c8) = o;
}

// ---- warp-pair kernel for up to 16 tokens -------------------------------------------
// A work item is (active expert, 32-row block = two 16-row tiles, token pass).  The two
// warps of a pair (w and w + NW/2 of a CTA) stream the first and the second half of the
// item's K chunks; the second adds its accumulators into the first's through shared
// memory, and the first runs the epilogue.  Against one tile per warp this shares the
// token fragments, the Z values, the loop and the address arithmetic between two tiles
// and gives each warp two independent MMA chains, while the K split keeps as many
// warps busy as there were items before.
constexpr int NS2 = 2;                                  // stages per warp
constexpr int STAGE2 = 2 * STAGE;                       // one stage: both tiles' blocks

template <int MODE, int NT, bool Q3>
__device__ __forceinline__ void group_step2(const uint32_t (&w)[2][2], const uint32_t (&u)[2][2],
                                            const float (&sc)[2][2], const uint16_t* const (&bx)[NT],
                                            const float* const (&zc)[NT][2], const uint32_t (&sub)[5],
                                            float (&acc)[2][NT][4]) {
    uint4 b0[NT], b1[NT];
    float z0[NT], z1[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        b0[n] = __ldg(reinterpret_cast<const uint4*>(bx[n]));
        b1[n] = __ldg(reinterpret_cast<const uint4*>(bx[n]) + 1);
        z0[n] = MODE == 0 ? __ldg(zc[n][0]) : 0.f;
        z1[n] = MODE == 0 ? __ldg(zc[n][1]) : 0.f;
    }
#pragma unroll
    for (int tl = 0; tl < 2; ++tl) {
        uint32_t q[16], hq[16];
        dequant_quads<MODE>(w[tl][0], w[tl][1], sub, q);
        if (Q3) dequant_hi_quads<MODE>(u[tl][0], u[tl][1], hq);
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            float d0 = z0[n], d1 = z1[n], d2 = z0[n], d3 = z1[n];
            mma_acc<MODE>(d0, d1, d2, d3, q[0], q[1], q[2], q[3], b0[n].x, b0[n].y);
            mma_acc<MODE>(d0, d1, d2, d3, q[4], q[5], q[6], q[7], b0[n].z, b0[n].w);
            mma_acc<MODE>(d0, d1, d2, d3, q[8], q[9], q[10], q[11], b1[n].x, b1[n].y);
            mma_acc<MODE>(d0, d1, d2, d3, q[12], q[13], q[14], q[15], b1[n].z, b1[n].w);
            if (Q3) {
                mma_acc<MODE>(d0, d1, d2, d3, hq[0], hq[1], hq[2], hq[3], b0[n].x, b0[n].y);
                mma_acc<MODE>(d0, d1, d2, d3, hq[4], hq[5], hq[6], hq[7], b0[n].z, b0[n].w);
                mma_acc<MODE>(d0, d1, d2, d3, hq[8], hq[9], hq[10], hq[11], b1[n].x, b1[n].y);
                mma_acc<MODE>(d0, d1, d2, d3, hq[12], hq[13], hq[14], hq[15], b1[n].z, b1[n].w);
            }
            acc[tl][n][0] = fmaf(sc[tl][0], d0, acc[tl][n][0]);
            acc[tl][n][1] = fmaf(sc[tl][0], d1, acc[tl][n][1]);
            acc[tl][n][2] = fmaf(sc[tl][1], d2, acc[tl][n][2]);
            acc[tl][n][3] = fmaf(sc[tl][1], d3, acc[tl][n][3]);
        }
    }
}

// Producer side of a pair warp's ring: the next chunk of both tiles (six bulk copies at
// most), issued by one elected lane of the converged warp.
template <int MODE>
struct PairProducer {
    const uint8_t* codes;
    const uint8_t* hi;
    const uint8_t* sc;
    int item, c, issued, jb, q3, cur_item;
    __device__ void load_item(const FfnArgs& p, const CtaSched& S, int blocks) {
        const int a = find_active(S, item);
        jb = (item - S.ipre[a]) % blocks;
        const PackedEntry* en = entry(p.packed, S.e[a]);
        codes = p.packed + (MODE == 0 ? en->gu_codes : en->dn_codes);
        hi = p.packed + (MODE == 0 ? en->gu_hi : en->dn_hi);
        sc = p.packed + (MODE == 0 ? en->gu_scales : en->dn_scales);
        q3 = S.fmt[a] == MOE_FMT_Q3;
        cur_item = item;
    }
    __device__ void issue(const FfnArgs& p, const CtaSched& S, int n_items, int P, int blocks, int K, int G, int NC,
                          int c_lo, int c_hi, uint8_t* ring, uint64_t* bar, uint64_t pol) {
        if (item >= n_items || c_lo >= c_hi) return;
        if (item != cur_item) load_item(p, S, blocks);
        const int st = issued % NS2;
        const int ng = min(CG, G - c * CG);
        if (elect_one()) {
            uint8_t* dst = ring + (size_t)st * STAGE2;
            const uint32_t cb = 256 * ng, hb = q3 ? 128 * ng : 0;
            mbar_arrive_expect_tx(&bar[st], 2 * (cb + hb + 256));
#pragma unroll
            for (int tl = 0; tl < 2; ++tl) {
                const int j = 2 * jb + tl;
                uint8_t* d = dst + tl * STAGE;
                bulk_g2s_evict_first(d, codes + (size_t)4 * K * j + 2048 * (size_t)c, cb, &bar[st], pol);
                bulk_g2s_evict_first(d + OFF_SC, sc + (size_t)256 * NC * j + 256 * (size_t)c, 256, &bar[st], pol);
                if (hb) bulk_g2s_evict_first(d + OFF_HI, hi + (size_t)128 * G * j + 1024 * (size_t)c, hb, &bar[st], pol);
            }
        }
        __syncwarp();
        ++issued;
        if (++c == c_hi) {
            c = c_lo;
            item += P;
        }
    }
};

template <int MODE, int NT, bool Q3>
__device__ __forceinline__ void run_item2(const FfnArgs& p, const CtaSched& S, PairProducer<MODE>& prod,
                                          int& consumed, bool& aborted, const ItemView<NT>& v,
                                          const uint32_t (&sub)[5], float (&acc)[2][NT][4], int n_items, int P,
                                          int blocks, int K, int G, int NC, int c_lo, int c_hi, uint8_t* ring,
                                          uint64_t* bar, uint64_t pol, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const int sh = 8 * (t & 1);
    if (c_lo < c_hi) prefetch_chunk<MODE, NT>(v, c_lo, t, G);
    for (int c = c_lo; c < c_hi; ++c) {
        prod.issue(p, S, n_items, P, blocks, K, G, NC, c_lo, c_hi, ring, bar, pol);
        if (c + 1 < c_hi) prefetch_chunk<MODE, NT>(v, c + 1, t, G);
        const int st = consumed % NS2;
        if (!aborted && !mbar_wait_bounded(&bar[st], (uint32_t)(consumed / NS2) & 1, kWaitLimit)) {
            aborted = true;
            report_error(p.ctrl, MOE_ERR_TIMEOUT, kDetWaitFull | MODE);
        }
        const uint8_t* stg = ring + (size_t)st * STAGE2;
        const uint16_t* bc[NT];
        const float* zcb[NT][2];
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            bc[n] = v.b[n] + c * CG * 64;
            zcb[n][0] = MODE == 0 ? v.z[n][0] + c * CG : nullptr;
            zcb[n][1] = MODE == 0 ? v.z[n][1] + c * CG : nullptr;
        }
        const int ng = min(CG, G - c * CG);
        // word offsets of rows g (and g + 8: +256 codes words, +128 third-bit words)
        const int cw_row = ng == CG ? g * 32 + t : g * 4 * ng + t;
        const int cw_row8 = ng == CG ? 256 : 8 * 4 * ng;
        const int hw_row = ng == CG ? g * 16 + (t >> 1) : g * 2 * ng + (t >> 1);
        const int hw_row8 = ng == CG ? 128 : 8 * 2 * ng;
        for (int gl = 0; gl < ng; ++gl) {
            const int cpos = cw_row + (ng == CG ? 4 * (gl ^ g) : 4 * gl);
            const int hpos = hw_row + (ng == CG ? 2 * (gl ^ (g >> 1)) : 2 * gl);
            uint32_t w[2][2], u[2][2] = {{0, 0}, {0, 0}};
            float scv[2][2];
#pragma unroll
            for (int tl = 0; tl < 2; ++tl) {
                const uint8_t* tb = stg + tl * STAGE;
                const uint32_t* cw = reinterpret_cast<const uint32_t*>(tb);
                w[tl][0] = cw[cpos];
                w[tl][1] = cw[cpos + cw_row8];
                if (Q3) {
                    const uint32_t* hw = reinterpret_cast<const uint32_t*>(tb + OFF_HI);
                    u[tl][0] = hw[hpos] >> sh;
                    u[tl][1] = hw[hpos + hw_row8] >> sh;
                }
                const uint16_t* scs = reinterpret_cast<const uint16_t*>(tb + OFF_SC) + g * 8;
                scv[tl][0] = half_bits_to_f32(scs[gl]);
                scv[tl][1] = half_bits_to_f32(scs[64 + gl]);
            }
            const uint16_t* bx[NT];
            const float* zc[NT][2];
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                bx[n] = bc[n] + gl * 64;
                zc[n][0] = zcb[n][0] + gl;
                zc[n][1] = zcb[n][1] + gl;
            }
            group_step2<MODE, NT, Q3>(w, u, scv, bx, zc, sub, acc);
        }
        __syncwarp();          // every lane is done with this stage before it is refilled
        ++consumed;
    }
}

template <int MODE, int NT, int NW>
__global__ void __launch_bounds__(NW * 32, 1) ffn_decode_pair_kernel(FfnArgs p) {
    constexpr int TB = 8 * NT, NPAIR = NW / 2;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ CtaSched S;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pair = warp % NPAIR, kh = warp / NPAIR;
    const int g = lane >> 2, t = lane & 3;
    const int K = MODE == 0 ? p.H : p.I;
    const int blocks = MODE == 0 ? (2 * p.I) / 32 : p.H / 32;
    const int G = K / 64, NC = (G + CG - 1) / CG;
    const int c_mid = (NC + 1) / 2;
    const int c_lo = kh == 0 ? 0 : c_mid, c_hi = kh == 0 ? c_mid : NC;
    uint8_t* ring = smem + (size_t)warp * NS2 * STAGE2;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + (size_t)NW * NS2 * STAGE2) + warp * NS2;
    float* red = reinterpret_cast<float*>(smem + (size_t)NW * NS2 * STAGE2 + (size_t)NW * NS2 * 8) +
                 (size_t)pair * (2 * NT * 4 * 32);

    // Work that does not depend on the router's (or the previous pass's) outputs runs
    // before griddep_wait() and overlaps the predecessor's tail: the header check and
    // the token rows; the schedule and everything after read the predecessor's data.
    griddep_launch_dependents();                        // all CTAs of this grid are resident
    if (threadIdx.x == 0) {
        const uint32_t* hd = reinterpret_cast<const uint32_t*>(p.packed);
        S.ok = hd[0] == kMagic && hd[1] == kVersion && (int)hd[2] == p.H && (int)hd[3] == p.I &&
               (int)hd[4] == p.E && (int)hd[5] == p.S && hd[6] == 64u && hd[7] == (uint32_t)kInterleave;
    }
    if (MODE == 0) warm_rows(p);
    griddep_wait();
    if (threadIdx.x == 0) {
        if (!S.ok) report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetHeader);
        S.n_active = p.ctrl->n_active;
    }
    __syncthreads();
    if (!S.ok) return;
    const int nA = S.n_active;
    for (int a = threadIdx.x; a < nA; a += blockDim.x) {
        const int e = p.active[a];
        S.e[a] = e;
        S.fmt[a] = (int)entry(p.packed, e)->fmt;
        S.cnt[a] = e < p.E ? p.counts[e] : p.T;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int a = 0; a < nA; ++a) {
            S.ipre[a] = run;
            run += blocks * ((S.cnt[a] + TB - 1) / TB);
        }
        S.ipre[nA] = run;
        S.n_items = run;
    }
    if (MODE == 0) warm_z(p);
    if (lane == 0)
        for (int s = 0; s < NS2; ++s) mbar_init(&bar[s], 1);
    fence_mbar_init();
    __syncthreads();
    const int n_items = S.n_items;
    const int P = gridDim.x * NPAIR;
    // items are dealt round-robin over the CTAs first, so that one expert's items (the
    // heavier 3-bit ones in particular) spread over many SMs instead of filling a few
    const int gp = pair * gridDim.x + blockIdx.x;
    const uint64_t pol = l2_policy_evict_first();

    PairProducer<MODE> prod;
    prod.item = gp;
    prod.c = c_lo;
    prod.issued = 0;
    prod.cur_item = -1;
    for (int i = 0; i < NS2 - 1; ++i) prod.issue(p, S, n_items, P, blocks, K, G, NC, c_lo, c_hi, ring, bar, pol);

    bool aborted = false;
    int consumed = 0;
    for (int item = gp; item < n_items; item += P) {
        const int a = find_active(S, item);
        const int r = item - S.ipre[a];
        const int pass = r / blocks, jb = r - pass * blocks;
        const int e = S.e[a], f = S.fmt[a], cnt = S.cnt[a];
        const int tb = pass * TB, nb = min(TB, cnt - tb);
        // Token columns of this pass.  Columns without a token read a valid row (the
        // pass's first token): their MMA outputs are never stored.
        ItemView<NT> v;
        const uint16_t* bsrc = MODE == 0 ? p.x : p.h;
        const int bld = MODE == 0 ? p.H : p.I;
        const float* zf = MODE == 0 ? p.zx + (size_t)f * p.T * G : nullptr;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int cb = n * 8 + g;
            const int i = tb + (cb < nb ? cb : 0);
            int brow;
            if (e < p.E) {
                const int hr = p.offsets[e] + i;
                brow = MODE == 0 ? p.perm[hr] / p.k : hr;
            } else {
                brow = MODE == 0 ? i : p.T * p.k + (e - p.E) * p.T + i;
            }
            v.b[n] = bsrc + (size_t)brow * bld + 16 * t;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int col = n * 8 + 2 * t + cc;
                const int ii = tb + (col < nb ? col : 0);
                int orow, ztok;
                if (e < p.E) {
                    orow = p.offsets[e] + ii;
                    ztok = p.perm[orow] / p.k;
                } else {
                    orow = p.T * p.k + (e - p.E) * p.T + ii;
                    ztok = ii;
                }
                v.orow[n][cc] = col < nb ? orow : -1;
                v.z[n][cc] = MODE == 0 ? zf + (size_t)ztok * G : nullptr;
            }
        }
        uint32_t sub[5] = {0, 0, 0, 0, 0};
        if (MODE == 1) {
            const float o = f == MOE_FMT_TERNARY ? 1.f : (f == MOE_FMT_Q2 ? 1.5f : 3.5f);
            sub[0] = f16x2_bits_of(512.f + o);
            sub[1] = f16x2_bits_of(256.f + o);
            sub[2] = f16x2_bits_of(64.f + o);
            sub[3] = f16x2_bits_of(16.f + o);
            sub[4] = f16x2_bits_of(4.f + o);
        }
        float acc[2][NT][4];
#pragma unroll
        for (int tl = 0; tl < 2; ++tl)
#pragma unroll
            for (int n = 0; n < NT; ++n) acc[tl][n][0] = acc[tl][n][1] = acc[tl][n][2] = acc[tl][n][3] = 0.f;
        if (f == MOE_FMT_Q3)
            run_item2<MODE, NT, true>(p, S, prod, consumed, aborted, v, sub, acc, n_items, P, blocks, K, G, NC, c_lo,
                                      c_hi, ring, bar, pol, lane);
        else
            run_item2<MODE, NT, false>(p, S, prod, consumed, aborted, v, sub, acc, n_items, P, blocks, K, G, NC, c_lo,
                                       c_hi, ring, bar, pol, lane);
        // the second K half hands its sums to the first through shared memory
        if (kh == 1) {
#pragma unroll
            for (int tl = 0; tl < 2; ++tl)
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int i = 0; i < 4; ++i) red[((tl * NT + n) * 4 + i) * 32 + lane] = acc[tl][n][i];
        }
        named_bar_sync(1 + pair, 64);
        if (kh == 0) {
#pragma unroll
            for (int tl = 0; tl < 2; ++tl)
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[tl][n][i] += red[((tl * NT + n) * 4 + i) * 32 + lane];
            // epilogue: tile j = 2 jb + tl
#pragma unroll
            for (int tl = 0; tl < 2; ++tl) {
                const int j = 2 * jb + tl;
#pragma unroll
                for (int n = 0; n < NT; ++n) {
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        if (v.orow[n][cc] < 0) continue;
                        if (MODE == 0) {
                            p.h[(size_t)v.orow[n][cc] * p.I + j * 8 + g] =
                                f32_to_f16_bits(silu_f(acc[tl][n][cc]) * acc[tl][n][2 + cc]);
                        } else {
                            p.ypart[(size_t)v.orow[n][cc] * p.H + j * 16 + g] = acc[tl][n][cc];
                            p.ypart[(size_t)v.orow[n][cc] * p.H + j * 16 + g + 8] = acc[tl][n][2 + cc];
                        }
                    }
                }
            }
        }
        named_bar_sync(1 + pair, 64);          // the first half has read the shared sums
    }
    // after a timeout the ring may still hold copies in flight: wait for them (bounded)
    if (aborted && lane == 0) {
        for (int q = consumed; q < prod.issued; ++q)
            if (!mbar_wait_bounded(&bar[q % NS2], (uint32_t)(q / NS2) & 1, kWaitLimit)) {
                report_error(p.ctrl, MOE_ERR_TIMEOUT, kDetDrain | MODE);
                break;
            }
    }
}

template <int NT, int NW>
constexpr size_t dyn_smem_pair() {
    return (size_t)NW * NS2 * STAGE2 + (size_t)NW * NS2 * 8 + (size_t)(NW / 2) * 2 * NT * 4 * 32 * 4;
}

template <int MODE, int NT, int NW>
cudaError_t launch_pair(const FfnArgs& a, cudaStream_t s) {
    static bool attr = false;
    if (!attr) {
        cudaError_t err = cudaFuncSetAttribute(ffn_decode_pair_kernel<MODE, NT, NW>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)dyn_smem_pair<NT, NW>());
        if (err != cudaSuccess) return err;
        attr = true;
    }
    return launch_pdl(ffn_decode_pair_kernel<MODE, NT, NW>, dim3(a.num_ctas), dim3(NW * 32), dyn_smem_pair<NT, NW>(),
                      s, a);
}

template <int NW>
constexpr size_t dyn_smem() { return (size_t)NW * NS * STAGE + (size_t)NW * NS * 8; }

template <int MODE, int NT, int NW>
cudaError_t launch_one(const FfnArgs& a, cudaStream_t s) {
    static bool attr = false;
    if (!attr) {
        cudaError_t err = cudaFuncSetAttribute(ffn_decode_kernel<MODE, NT, NW>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn_smem<NW>());
        if (err != cudaSuccess) return err;
        attr = true;
    }
    return launch_pdl(ffn_decode_kernel<MODE, NT, NW>, dim3(a.num_ctas), dim3(NW * 32), dyn_smem<NW>(), s, a);
}

// warps per CTA shrink as the token tile grows, to leave room for the accumulators
template <int MODE>
cudaError_t launch_mode(const FfnArgs& a, cudaStream_t s) {
    if (a.T <= 8) return launch_pair<MODE, 1, 16>(a, s);
    if (a.T <= 16) return launch_pair<MODE, 2, 12>(a, s);
    if (a.T <= 32) return launch_one<MODE, 4, 8>(a, s);
    return launch_one<MODE, 8, 8>(a, s);
}

}  // namespace

cudaError_t launch_ffn_decode(const FfnArgs& a, cudaStream_t s, cudaEvent_t ev_gateup, cudaEvent_t ev_down) {
    cudaError_t err = launch_mode<0>(a, s);
    if (err != cudaSuccess) return err;
    if (ev_gateup && (err = record_event(ev_gateup, s)) != cudaSuccess) return err;
    err = launch_mode<1>(a, s);
    if (err != cudaSuccess) return err;
    if (ev_down && (err = record_event(ev_down, s)) != cudaSuccess) return err;
    return launch_combine(a, s);
}

cudaError_t launch_combine(const FfnArgs& a, cudaStream_t s) {
    const long long n = (long long)a.T * (a.H / 8);
    return launch_pdl(combine_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, a);
}

}  // namespace moe
