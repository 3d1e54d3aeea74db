// Expert FFN kernels of the decode path (gate/up + SwiGLU and down, routed and shared
// experts; at 1 to 4 and 9 to 64 tokens, while from 5 to 8 tokens the fused kernel of
// decode_fused.cu runs instead) and the gate-weighted unpermute-combine used by the
// decode and prefill paths: grouped skinny GEMMs over the packed ternary / 2-bit / 3-bit
// experts, for few tokens per expert.
//
// Decode speed is set by the expert bytes moved per token (ossradar.top, Xolotl
// README, "Fast mode (DeepSeek-V4.1)"), and each selected expert is read once for
// all of its tokens (the same README, "Latest": the CPU kernels that decode an
// expert once for its 4-8 tokens).  So every selected expert's packed bytes are
// streamed exactly once and applied to all of its tokens:
//
//  * Work unit = (active expert, 32-row block = two 16-row tiles of the packed
//    matrix, K part, token pass of up to 8 tokens).  With one or two tokens there are
//    fewer 32-row blocks than warps on the GPU, so K is cut into parts (whole 8-group
//    chunks) and every part writes its own fp32 partial sums; the parts are added in
//    a fixed order afterwards (finalize_gateup_kernel, combine_kernel), so the result
//    does not depend on which warp ran what.  The warps of a persistent grid (one CTA
//    of 16 warps per SM) take units at run time from a per-launch counter, one unit
//    ahead of need, which balances SMs and SM sub-partitions whatever the expert mix.
//    An expert with more than 8 tokens has one unit per pass; the passes of a block
//    are consecutive units, taken at about the same time, so the block's bytes come
//    from HBM once and from L2 for the other passes.
//  * Each warp streams its units through its own ring of NS shared-memory stages with
//    1-D bulk copies (cp.async.bulk on the TMA engine, completion on a per-stage
//    mbarrier); a stage holds one 8-group (512-wide) chunk of K for both tiles:
//    codes, third bits and fp16 scales, each a contiguous block of the packed format.
//    The format's XOR swizzle keeps the fragment reads free of bank conflicts.  The
//    ring runs ahead across units; there is no CTA-wide barrier in the main loop.
//  * A full chunk is processed in four steps of two groups (a rolled loop keeps the
//    code inside the instruction cache): per 64-wide group and tile, two code
//    words become sixteen bf16 / fp16 pairs with shifts and lop3 (magic-number
//    exponent trick: the code lands in the mantissa of a power-of-two base, exactly),
//    the A operand of mma.sync m16n8k16; the tokens are N (8 per n-tile) and the B
//    fragments come straight from the token rows (L1-resident).
//      gate/up: pairs stay "base + c", so a group's MMAs yield sum (base_k + c_k) x_k;
//        once per chunk a small fp16 MMA of the scales against the router's table of
//        -Z (Z = sum base(k) x_k + o sum x_k, plus the third-bit bases for 3-bit
//        experts) removes the offsets, leaving sum (c_k - o) x_k.  bf16 MMAs: the
//        tokens are bf16.
//      down: pairs are (c - o) exactly (one fp16x2 subtract); fp16 MMAs, h is fp16.
//    Each group result is scaled by its fp16 scale into an fp32 accumulator.
//    3-bit experts add an MMA per k-step for 4 * (third bit).
//  * gate/up with at most 4 tokens, ternary and 2-bit experts: integer MMAs instead
//    (u8 codes masked out of the code words against signed-byte digits of the tokens
//    on a 12-bit grid per group, the code offset removed exactly in the integer sums;
//    "few-token gate/up on the integer tensor path" below), which halves the
//    dequantiser's ALU work and the MMA chain per group.
//  * gate/up: the 16 rows of a tile are 8 gate rows and the matching 8 up rows, which
//    the MMA places in the same thread (rows g and g + 8), so with a single K part
//    h = silu(gate) * up is formed in registers and stored as fp16; with several K
//    parts the raw sums go to gpart and finalize_gateup_kernel forms h.
//  * down: partial rows (fp32) per (K part, token, slot); the combine kernel then
//    sums the parts, each token's k slots in slot order with the gates, adds the
//    shared expert and writes y in bf16: deterministic, no floating-point atomics.
// Every wait is bounded; a wait that runs out records an error in the workspace and the
// warp gives up: it issues no more copies, waits (bounded) for those in flight and
// leaves, so the kernel always terminates.
#include "kernels.h"
#include "dequant.cuh"
#include "iqmma.cuh"
#include "operands.cuh"      // iq_group: the K-part reduction forms h's integer operands

namespace moe {
namespace {

constexpr int CG = 8;                                  // 64-wide groups per chunk
constexpr int OFF_HI = 2048;                           // codes block: 16 rows x 32 words
constexpr int OFF_SC = OFF_HI + 1024;                  // third-bit block: 16 rows x 16 words
constexpr int TSTAGE = OFF_SC + 256;                   // scales block: 16 rows x 8 halves
constexpr int NTL = 2;                                 // 16-row tiles per block
constexpr int STAGE = NTL * TSTAGE;                    // one chunk of both tiles of a block
constexpr int NW = 16;                                 // warps per CTA
constexpr int NS = 2;                                  // stages per warp
constexpr int TP = 8;                                  // tokens per pass (one n-tile)
constexpr long long kWaitLimit = 4000000000LL;         // clock cycles (~2 s)
constexpr uint32_t kRangeDecode = 0x40;                // detail low byte: an activation of these kernels

using namespace dq;

// ---- the CTA's copy of the schedule -------------------------------------------------
constexpr int kMaxActive = 260;
constexpr int kPermSmem = 1024;                        // routed pairs staged in shared memory

struct CtaSched {
    int ok;
    uint32_t stall;            // failure-path tests: cycles of warp 0's wait on stall_bar (0 = off)
    int n_active;
    int n_units;
    int perm_in_smem;
    int e[kMaxActive];
    int fmt[kMaxActive];
    int cnt[kMaxActive];       // tokens of the expert
    int off[kMaxActive];       // first permuted row (routed experts)
    int upre[kMaxActive + 1];  // expert-pass prefix over active experts
    int one_pass;              // every active expert has at most 8 tokens
    int n_ep;                  // expert passes
    int tok[kPermSmem];        // source token of permuted row r (perm[r] / k)
};

struct UnitPos {
    int a, pass, jb, kp;
};

// Division by a divisor fixed for the launch, through a float reciprocal and one
// correction step (exact for dividends below 2^22).
struct FastDiv {
    int d;
    float inv;
    __device__ __forceinline__ void init(int dd) {
        d = dd;
        inv = 1.0f / (float)dd;
    }
    __device__ __forceinline__ int div(int n) const {
        int q = (int)((float)n * inv);
        if ((q + 1) * d <= n) ++q;
        else if (q * d > n) --q;
        return q;
    }
};

// Units are ordered (active expert, token pass, 32-row block, K part), K part fastest;
// unit u -> expert pass ep = u / (blocks * nkp), then block and K part.  ep is the
// active expert itself when every active expert has one pass (at most 8 tokens).
__device__ __forceinline__ UnitPos unit_pos(const CtaSched& S, int u, const FastDiv& per_ep, const FastDiv& nkp) {
    UnitPos q;
    const int ep = per_ep.div(u);
    const int r = u - ep * per_ep.d;
    q.jb = nkp.div(r);
    q.kp = r - q.jb * nkp.d;
    if (S.one_pass) {
        q.a = ep;
        q.pass = 0;
    } else {
        int lo = 0, hi = S.n_active - 1;               // largest a with upre[a] <= ep
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (S.upre[mid] <= ep) lo = mid;
            else hi = mid - 1;
        }
        q.a = lo;
        q.pass = ep - S.upre[lo];
    }
    return q;
}

__device__ __forceinline__ int src_token(const FfnArgs& p, const CtaSched& S, int row) {
    return S.perm_in_smem ? S.tok[row] : __ldg(p.perm + row) / p.k;
}

// Per-lane view of one unit: B row, -Z rows and output rows of this lane's columns.
struct UnitView {
    const uint16_t* b;         // B-operand row of token column g (+16t elements)
    const uint16_t* z;         // gate/up: -Z/16 (hi plane) of token column g, groups 2t, 2t+1
    const uint4* bq;           // integer path: digit record of column g, lane t, group 0
    const float2* pq;          // integer path: pairs {p, sum q} of token t, group 0
    int o4;                    // integer path: 4 o (4 ternary, 6 two-bit)
    int orow[2];               // output rows of columns 2t, 2t+1 (-1: no token); integer path: token t
};

// Columns without a token read a valid row (the pass's first token); their MMA
// outputs are never stored.
template <int MODE>
__device__ __forceinline__ void make_view(const FfnArgs& p, const CtaSched& S, int a, int pass, int g, int t,
                                          UnitView& v) {
    const int e = S.e[a], f = S.fmt[a], cnt = S.cnt[a];
    const int tb = pass * TP, nb = min(TP, cnt - tb);
    const bool routed = e < p.E;
    const int G = p.H / 64;
    const int srow0 = p.T * p.k + (e - p.E) * p.T;     // first row of a shared expert
    const int i = tb + (g < nb ? g : 0);
    int brow;
    if (routed) {
        const int hr = S.off[a] + i;
        brow = MODE == 0 ? src_token(p, S, hr) : hr;
    } else {
        brow = MODE == 0 ? i : srow0 + i;
    }
    v.b = (MODE == 0 ? p.x : p.h) + (size_t)brow * (MODE == 0 ? p.H : p.I) + 16 * t;
    const int G8 = 8 * ((G + 7) / 8);
    v.z = MODE == 0 ? reinterpret_cast<const uint16_t*>(p.zx) + ((size_t)f * p.T + brow) * G8 + 2 * t : nullptr;
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
        const int col = 2 * t + cc;
        const int ii = tb + (col < nb ? col : 0);
        const int orow = routed ? S.off[a] + ii : srow0 + ii;
        v.orow[cc] = col < nb ? orow : -1;
    }
}

// Lane constants for reading a stage: cw_lane = 32g + t and g4 = 4g locate the code
// words (row g; row g + 8 is 256 words on), hw_lane = 16g + t/2 and g2 = 2(g/2) the
// third-bit words (row g + 8: 128 words on), sh the third-bit half of this lane.
struct LaneGeo {
    int g, t, cw_lane, g4, hw_lane, g2, sh;
    int zplane;                // elements from the hi to the lo plane of the Z table
};

__device__ __forceinline__ uint32_t f16x2_mul16(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Gate/up: the group MMAs sum (base + c) x from zero; this subtracts the offsets of a
// whole 8-group chunk at once, acc[row][col] += sum_gl 16 s[row][gl] * (-Z[col][gl] / 16),
// as two m16n8k8 fp16 MMAs per tile (the hi and lo halves of -Z / 16).  A: this lane's
// scale words of rows g and g + 8 (groups 2t, 2t+1), times 16 (exact); B: the two
// fp16 halves of -Z / 16 for token column g at groups 2t, 2t+1.  Groups past K in a
// partial chunk have zero scales and zero Z.
__device__ __forceinline__ void z_correction(const uint8_t* stg, int c, const UnitView& v, const LaneGeo& L,
                                             float (&acc)[NTL][4]) {
    constexpr uint32_t kSixteen = 0x4C004C00u;         // fp16 16.0 in both halves
    const uint32_t bhi = __ldg(reinterpret_cast<const uint32_t*>(v.z + 8 * c));
    const uint32_t blo = __ldg(reinterpret_cast<const uint32_t*>(v.z + L.zplane + 8 * c));
#pragma unroll
    for (int tl = 0; tl < NTL; ++tl) {
        const uint32_t* scw = reinterpret_cast<const uint32_t*>(stg + tl * TSTAGE + OFF_SC);
        const uint32_t a0 = f16x2_mul16(scw[4 * L.g + L.t], kSixteen);
        const uint32_t a1 = f16x2_mul16(scw[4 * (L.g + 8) + L.t], kSixteen);
        mma_f16_1688(acc[tl], a0, a1, bhi);
        mma_f16_1688(acc[tl], a0, a1, blo);
    }
}

// Group gl of a full chunk, every tile of the block: code words from the swizzled
// stage, the B fragments of the group, the MMAs and the scaled fold into acc.  s2:
// per tile, the scale words of rows g and g + 8 that hold groups gl & ~1 and gl | 1;
// HI selects the half of group gl.
template <int MODE, bool Q3, int HI>
__device__ __forceinline__ void group_full(const uint8_t* stg, int gl, const uint16_t* bx, const LaneGeo& L,
                                           const uint32_t (&s2)[NTL][2], const uint32_t (&sub)[5],
                                           float (&acc)[NTL][4]) {
    const uint32_t* cw = reinterpret_cast<const uint32_t*>(stg);
    const int cpos = L.cw_lane + ((4 * gl) ^ L.g4);
    uint32_t w[NTL][2], u[NTL][2];
#pragma unroll
    for (int tl = 0; tl < NTL; ++tl) {
        w[tl][0] = cw[cpos + tl * (TSTAGE / 4)];
        w[tl][1] = cw[cpos + tl * (TSTAGE / 4) + 256];
        u[tl][0] = u[tl][1] = 0;
    }
    if (Q3) {
        const uint32_t* hw = reinterpret_cast<const uint32_t*>(stg + OFF_HI);
        const int hpos = L.hw_lane + ((2 * gl) ^ L.g2);
#pragma unroll
        for (int tl = 0; tl < NTL; ++tl) {
            u[tl][0] = hw[hpos + tl * (TSTAGE / 4)] >> L.sh;
            u[tl][1] = hw[hpos + tl * (TSTAGE / 4) + 128] >> L.sh;
        }
    }
    const uint4 x0 = __ldg(reinterpret_cast<const uint4*>(bx + 64 * gl));
    const uint4 x1 = __ldg(reinterpret_cast<const uint4*>(bx + 64 * gl) + 1);
#pragma unroll
    for (int tl = 0; tl < NTL; ++tl) {
        uint32_t pa[8], pb[8];
        dequant_rows<MODE>(w[tl][0], w[tl][1], sub, pa, pb);
        float d[4];
        mma_group_first<MODE>(d, pa, pb, x0, x1);
        if (Q3) {
            dequant_hi_rows<MODE>(u[tl][0], u[tl][1], pa, pb);
            mma_group<MODE>(d, pa, pb, x0, x1);
        }
        const float s0 = HI ? half_hi(s2[tl][0]) : half_lo(s2[tl][0]);
        const float s1 = HI ? half_hi(s2[tl][1]) : half_lo(s2[tl][1]);
        acc[tl][0] = fmaf(s0, d[0], acc[tl][0]);
        acc[tl][1] = fmaf(s0, d[1], acc[tl][1]);
        acc[tl][2] = fmaf(s1, d[2], acc[tl][2]);
        acc[tl][3] = fmaf(s1, d[3], acc[tl][3]);
    }
}

// One full 8-group chunk of every tile of a block against this lane's token column,
// as four steps of two groups (a rolled loop keeps the code inside the instruction
// cache).  stg: the stage; c: chunk index (selects the B columns and the Z entries).
template <int MODE, bool Q3>
__device__ __forceinline__ void chunk_full(const uint8_t* stg, int c, const UnitView& v, const LaneGeo& L,
                                           const uint32_t (&sub)[5], float (&acc)[NTL][4]) {
    const uint32_t* scw = reinterpret_cast<const uint32_t*>(stg + OFF_SC);   // row r: words 4r .. 4r+3
    const uint16_t* bx = v.b + c * (CG * 64);
    if (MODE == 0) z_correction(stg, c, v, L, acc);
#pragma unroll 1
    for (int gp = 0; gp < CG / 2; ++gp) {
        uint32_t s2[NTL][2];
#pragma unroll
        for (int tl = 0; tl < NTL; ++tl) {
            s2[tl][0] = scw[tl * (TSTAGE / 4) + 4 * L.g + gp];
            s2[tl][1] = scw[tl * (TSTAGE / 4) + 4 * (L.g + 8) + gp];
        }
        group_full<MODE, Q3, 0>(stg, 2 * gp, bx, L, s2, sub, acc);
        group_full<MODE, Q3, 1>(stg, 2 * gp + 1, bx, L, s2, sub, acc);
    }
}

// A chunk with ng < 8 groups (the last one when K / 64 is not a multiple of 8):
// unswizzled rows of 4 ng code words and 2 ng third-bit words.
template <int MODE, bool Q3>
__device__ __forceinline__ void chunk_partial(const uint8_t* stg, int c, int ng, const UnitView& v,
                                              const LaneGeo& L, const uint32_t (&sub)[5], float (&acc)[NTL][4]) {
    const int g = L.g, t = L.t;
    if (MODE == 0) z_correction(stg, c, v, L, acc);
    for (int gl = 0; gl < ng; ++gl) {
        const uint16_t* bp = v.b + c * (CG * 64) + 64 * gl;
        const uint4 x0 = __ldg(reinterpret_cast<const uint4*>(bp));
        const uint4 x1 = __ldg(reinterpret_cast<const uint4*>(bp) + 1);
#pragma unroll
        for (int tl = 0; tl < NTL; ++tl) {
            const uint8_t* tb = stg + tl * TSTAGE;
            const uint32_t* cw = reinterpret_cast<const uint32_t*>(tb);
            const uint32_t* hw = reinterpret_cast<const uint32_t*>(tb + OFF_HI);
            const uint16_t* scs = reinterpret_cast<const uint16_t*>(tb + OFF_SC);
            uint32_t pa[8], pb[8];
            dequant_rows<MODE>(cw[g * 4 * ng + 4 * gl + t], cw[(g + 8) * 4 * ng + 4 * gl + t], sub, pa, pb);
            float d[4];
            mma_group_first<MODE>(d, pa, pb, x0, x1);
            if (Q3) {
                dequant_hi_rows<MODE>(hw[g * 2 * ng + 2 * gl + (t >> 1)] >> L.sh,
                                      hw[(g + 8) * 2 * ng + 2 * gl + (t >> 1)] >> L.sh, pa, pb);
                mma_group<MODE>(d, pa, pb, x0, x1);
            }
            const float s0 = __half2float(__ushort_as_half(scs[g * 8 + gl]));
            const float s1 = __half2float(__ushort_as_half(scs[(g + 8) * 8 + gl]));
            acc[tl][0] = fmaf(s0, d[0], acc[tl][0]);
            acc[tl][1] = fmaf(s0, d[1], acc[tl][1]);
            acc[tl][2] = fmaf(s1, d[2], acc[tl][2]);
            acc[tl][3] = fmaf(s1, d[3], acc[tl][3]);
        }
    }
}

// Per-launch geometry of one expert pass (gate/up: K = H, rows 2I; down: K = I, rows H).
struct Geo {
    int K, G, NC, blocks, nkp, cpk;
};

// Producer side of a warp's ring.  Units are handed out at run time: the elected lane
// takes the next unit index from the launch's work counter one unit ahead of need, so
// the atomic's latency hides behind a chunk of work and every warp keeps busy until
// the counter runs out.  The producer issues the bulk copies of one chunk (both tiles
// of the block) per call and remembers which unit and chunk each of the last NS
// issues carried, which is what the consumer reads back NS - 1 calls later.
template <int MODE>
struct Producer {
    const uint8_t* codes;
    const uint8_t* hi;
    const uint8_t* sc;
    int cur, jb, c, c_end, q3, cur_a, issued;
    int pend;                                         // lane 0: the unit grabbed for after cur
    int hu[NS], hc[NS];                               // unit / chunk of the last NS issues (0 = latest)
    __device__ __forceinline__ int grab(uint32_t* ctr, int lane) {
        int g = 0;
        if (lane == 0) g = (int)atomicAdd(ctr, 1u);
        return g;
    }
    __device__ void start(const FfnArgs& p, const CtaSched& S, const Geo& geo, const FastDiv& per_ep,
                          const FastDiv& nkp, uint32_t* ctr, int lane, int unit) {
        cur = unit;
        if (cur >= S.n_units) {
            cur = -1;
            return;
        }
        const UnitPos q = unit_pos(S, cur, per_ep, nkp);
        jb = q.jb;
        c = q.kp * geo.cpk;
        c_end = min(geo.NC, c + geo.cpk);
        if (q.a != cur_a) {
            cur_a = q.a;
            const PackedEntry* en = entry(p.packed, S.e[q.a]);
            codes = p.packed + (MODE == 0 ? en->gu_codes : en->dn_codes);
            hi = p.packed + (MODE == 0 ? en->gu_hi : en->dn_hi);
            sc = p.packed + (MODE == 0 ? en->gu_scales : en->dn_scales);
            q3 = S.fmt[q.a] == MOE_FMT_Q3;
        }
        pend = grab(ctr, lane);                       // the unit after this one
    }
    __device__ void issue(const FfnArgs& p, const CtaSched& S, const Geo& geo, const FastDiv& per_ep,
                          const FastDiv& nkp, uint32_t* ctr, int lane, uint8_t* ring, uint64_t* bar,
                          uint64_t pol) {
#pragma unroll
        for (int i = NS - 1; i > 0; --i) {
            hu[i] = hu[i - 1];
            hc[i] = hc[i - 1];
        }
        hu[0] = cur;
        hc[0] = c;
        if (cur < 0) return;
        const int st = issued % NS;
        const int ng = min(CG, geo.G - c * CG);
        if (elect_one()) {
            uint8_t* dst = ring + (size_t)st * STAGE;
            const uint32_t cb = 256 * ng, hb = q3 ? 128 * ng : 0;
            mbar_arrive_expect_tx(&bar[st], NTL * (cb + hb + 256));
#pragma unroll
            for (int tl = 0; tl < NTL; ++tl) {
                const int j = NTL * jb + tl;
                uint8_t* d = dst + tl * TSTAGE;
                bulk_g2s_evict_first(d, codes + (size_t)4 * geo.K * j + 2048 * (size_t)c, cb, &bar[st], pol);
                bulk_g2s_evict_first(d + OFF_SC, sc + (size_t)256 * geo.NC * j + 256 * (size_t)c, 256, &bar[st],
                                     pol);
                if (hb)
                    bulk_g2s_evict_first(d + OFF_HI, hi + (size_t)128 * geo.G * j + 1024 * (size_t)c, hb, &bar[st],
                                         pol);
            }
        }
        __syncwarp();
        ++issued;
        if (++c == c_end) start(p, S, geo, per_ep, nkp, ctr, lane, __shfl_sync(0xffffffffu, pend, 0));
    }
};

// ---- few-token gate/up on the integer tensor path (ternary and 2-bit experts) ----
// With at most kIqMaxT tokens a pass uses one n8 tile as two signed-byte digit columns
// per token (column 2j + d: digit d of token j; the router writes the digit records and
// pairs, operands.cuh).  The four u8 A registers of a code word need no add (iqmma.cuh),
// the accumulator of the low digit starts at 1.5 x 2^23 - 4 o sum q, so the joined int32
// sum read as fp32 is 1.5 x 2^23 + the offset-corrected dot product exactly; per group
// acc += s p (that sum) with p = 2^-e / 4 of this lane's token.  The record and the pair
// of a group are loaded once and serve both tiles of the block.  Lane (g, t) ends with
// rows g (gate) and g + 8 (up) of token t, packed as one fp32 pair per tile.
__device__ __forceinline__ void iq_tile(uint32_t w0, uint32_t w1, const uint4& b, int c0, unsigned long long spf,
                                        unsigned long long& acc) {
    const uint32_t w0s = w0 >> 4, w1s = w1 >> 4;
    int d[4];
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%10,%11};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(w0 & 0x03030303u), "r"(w1 & 0x03030303u), "r"(w0 & 0x0C0C0C0Cu), "r"(w1 & 0x0C0C0C0Cu), "r"(b.x),
          "r"(b.y), "r"(c0), "r"(0));
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(w0s & 0x03030303u), "r"(w1s & 0x03030303u), "r"(w0s & 0x0C0C0C0Cu), "r"(w1s & 0x0C0C0C0Cu),
          "r"(b.z), "r"(b.w));
    const unsigned long long D = iq::add2(iq::pk2(__int_as_float(d[0] + 256 * d[1]), __int_as_float(d[2] + 256 * d[3])),
                                          iq::pk2(-iq::kIqMagicF, -iq::kIqMagicF));
    acc = iq::fma2(spf, D, acc);
}

__device__ __forceinline__ unsigned long long scale_pair(uint32_t wg, uint32_t wu, bool hi) {
    const uint16_t hg = (uint16_t)(hi ? wg >> 16 : wg), hu = (uint16_t)(hi ? wu >> 16 : wu);
    return iq::pk2(__half2float(__ushort_as_half(hg)), __half2float(__ushort_as_half(hu)));
}

// A full chunk (8 groups, swizzled code words: this lane's word of group gl is at byte
// sw ^ 16 gl of the tile's stage, row g + 8 1024 bytes on), in group pairs so that the
// scale words stay in registers with static indices.
__device__ __forceinline__ void chunk_full_iq(const uint8_t* stg, int c, const UnitView& v, const LaneGeo& L,
                                              unsigned long long (&ia)[NTL]) {
    const uint4* rec = v.bq + 64 * c;
    const float4* prs = reinterpret_cast<const float4*>(v.pq + CG * c);     // two pairs per load
    const int sw = 128 * L.g + 16 * (L.g & 7) + 4 * L.t;
#pragma unroll 1
    for (int gp = 0; gp < CG / 2; ++gp) {
        uint32_t sg[NTL], su[NTL];
#pragma unroll
        for (int tl = 0; tl < NTL; ++tl) {
            const uint32_t* scw = reinterpret_cast<const uint32_t*>(stg + tl * TSTAGE + OFF_SC);
            sg[tl] = scw[4 * L.g + gp];
            su[tl] = scw[4 * (L.g + 8) + gp];
        }
        const float4 pr = __ldg(prs + gp);
        const uint4 b0 = __ldg(rec + 16 * gp), b1 = __ldg(rec + 16 * gp + 8);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int gl = 2 * gp + h;
            const float pf = h ? pr.z : pr.x;
            const int c0 = (int)iq::kIqMagic - v.o4 * __float_as_int(h ? pr.w : pr.y);
#pragma unroll
            for (int tl = 0; tl < NTL; ++tl) {
                const uint32_t* wp = reinterpret_cast<const uint32_t*>(stg + tl * TSTAGE + (sw ^ (16 * gl)));
                iq_tile(wp[0], wp[256], h ? b1 : b0, c0, iq::mul2(scale_pair(sg[tl], su[tl], h), iq::pk2(pf, pf)),
                        ia[tl]);
            }
        }
    }
}

// A partial chunk (ng < 8 groups, code words unswizzled: 4 ng words per row).
__device__ __forceinline__ void chunk_partial_iq(const uint8_t* stg, int c, int ng, const UnitView& v,
                                                 const LaneGeo& L, unsigned long long (&ia)[NTL]) {
    for (int gl = 0; gl < ng; ++gl) {
        const uint4 b = __ldg(v.bq + 64 * c + 8 * gl);
        const float2 pr = __ldg(v.pq + CG * c + gl);
        const int c0 = (int)iq::kIqMagic - v.o4 * __float_as_int(pr.y);
#pragma unroll
        for (int tl = 0; tl < NTL; ++tl) {
            const uint8_t* tb = stg + tl * TSTAGE;
            const uint32_t* cw = reinterpret_cast<const uint32_t*>(tb);
            const unsigned long long sv = iq::pk2(iq::iq_scale_of(tb, L.g, gl), iq::iq_scale_of(tb, L.g + 8, gl));
            iq_tile(cw[L.g * 4 * ng + 4 * gl + L.t], cw[(L.g + 8) * 4 * ng + 4 * gl + L.t], b, c0,
                    iq::mul2(sv, iq::pk2(pr.x, pr.x)), ia[tl]);
        }
    }
}

// View of an integer-path unit (T <= kIqMaxT: one pass of at most four tokens).  B
// column g is digit g & 1 of the pass's token g >> 1 (gate/up: the router's records of
// the token; down: the K-part reduction's records of the token's h row); the outputs of
// this lane are token t's.  Columns and outputs without a token read the pass's first
// token and are never stored.
template <int MODE>
__device__ __forceinline__ void make_view_iq(const FfnArgs& p, const CtaSched& S, int a, int g, int t, UnitView& v) {
    const int e = S.e[a], nb = min(kIqMaxT, S.cnt[a]);
    const bool routed = e < p.E;
    const int G = (MODE == 0 ? p.H : p.I) / 64, G8 = 8 * ((G + 7) / 8);
    const int ib = (g >> 1) < nb ? (g >> 1) : 0, it = t < nb ? t : 0;
    const int srow0 = p.T * p.k + (e - p.E) * p.T;     // first row of a shared expert
    int rb, rt;                                         // record row of column g, pair row of token t
    if (MODE == 0) {
        rb = routed ? src_token(p, S, S.off[a] + ib) : ib;
        rt = routed ? src_token(p, S, S.off[a] + it) : it;
    } else {
        rb = routed ? S.off[a] + ib : srow0 + ib;
        rt = routed ? S.off[a] + it : srow0 + it;
    }
    const uint8_t* base = MODE == 0 ? p.iq : p.hq;
    const size_t poff = MODE == 0 ? iq_pair_off(p.T, p.H) : iq_pair_off(p.R16, p.I);
    // records [rows][G][2 digits][4 lanes] of 16 bytes; pairs [rows][G8]
    v.bq = reinterpret_cast<const uint4*>(base) + ((size_t)rb * G * 8 + 4 * (g & 1) + t);
    v.pq = reinterpret_cast<const float2*>(base + poff) + (size_t)rt * G8;
    v.o4 = S.fmt[a] == MOE_FMT_TERNARY ? 4 : 6;
    v.b = nullptr;
    v.z = nullptr;
    v.orow[0] = t < nb ? (routed ? S.off[a] + t : srow0 + t) : -1;
    v.orow[1] = -1;
}

// Integer-path unit end: gate/up: h directly, or this K part's gate and up sums; down:
// this K part's output rows.  Activations outside the fp16 range are reported.
template <int MODE>
__device__ __forceinline__ void unit_epilogue_iq(const FfnArgs& p, const Geo& geo, const UnitPos& q,
                                                 const UnitView& v, const LaneGeo& L,
                                                 const unsigned long long (&ia)[NTL]) {
    const int orow = v.orow[0];
    if (orow < 0) return;
    const size_t R = (size_t)p.T * (p.k + p.S);
#pragma unroll
    for (int tl = 0; tl < NTL; ++tl) {
        const int j = NTL * q.jb + tl;
        const float2 r = iq::up2(ia[tl]);
        if (MODE == 0 && geo.nkp == 1) {
            const float hv = silu_f(r.x) * r.y;
            if (!in_f16_range(hv)) report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetRange | kRangeDecode);
            p.h[(size_t)orow * p.I + j * 8 + L.g] = f32_to_f16_bits(hv);
        } else {
            float* dst = MODE == 0 ? p.gpart + ((size_t)q.kp * R + orow) * (2 * p.I) + j * 16 + L.g
                                   : p.ypart + ((size_t)q.kp * R + orow) * p.H + j * 16 + L.g;
            dst[0] = r.x;
            dst[8] = r.y;
        }
    }
}

// The output of one finished unit: tile j = NTL jb + tl, rows g (gate / first half) and
// g + 8 (up / second half) of this lane's token columns.
template <int MODE>
__device__ __forceinline__ void unit_epilogue(const FfnArgs& p, const Geo& geo, const UnitPos& q, const UnitView& v,
                                              const LaneGeo& L, const float (&acc)[NTL][4]) {
    const size_t R = (size_t)p.T * (p.k + p.S);
#pragma unroll
    for (int tl = 0; tl < NTL; ++tl) {
        const int j = NTL * q.jb + tl;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int orow = v.orow[cc];
            if (orow < 0) continue;
            if (MODE == 0 && geo.nkp == 1) {
                const float hv = silu_f(acc[tl][cc]) * acc[tl][2 + cc];
                if (!in_f16_range(hv)) report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetRange | kRangeDecode);
                p.h[(size_t)orow * p.I + j * 8 + L.g] = f32_to_f16_bits(hv);
            } else if (MODE == 0) {
                float* dst = p.gpart + ((size_t)q.kp * R + orow) * (2 * p.I) + j * 16 + L.g;
                dst[0] = acc[tl][cc];
                dst[8] = acc[tl][2 + cc];
            } else {
                float* dst = p.ypart + ((size_t)q.kp * R + orow) * p.H + j * 16 + L.g;
                dst[0] = acc[tl][cc];
                dst[8] = acc[tl][2 + cc];
            }
        }
    }
}

// Gate/up with few tokens: every SM reads the same token rows and Z values, so each CTA
// pulls them into L1 at the start.  The token rows are the caller's input (ready before
// the router ran); the Z values are the router's output and are prefetched only after
// griddep_wait(), so no stale line can enter L1.  The zx region is padded to 256 bytes,
// so whole lines stay inside it.
__device__ inline size_t z_bytes(const FfnArgs& p) { return (size_t)3 * p.T * (8 * ((p.H / 64 + 7) / 8)) * 4; }
__device__ inline bool warm_fits(const FfnArgs& p) { return (size_t)p.T * p.H * 2 + z_bytes(p) <= 48 * 1024; }
__device__ inline void warm_rows(const FfnArgs& p) {
    if (!warm_fits(p)) return;
    const size_t xb = (size_t)p.T * p.H * 2;
    for (size_t i = threadIdx.x; i < xb / 128; i += blockDim.x)
        prefetch_l1(reinterpret_cast<const uint8_t*>(p.x) + i * 128);
}
__device__ inline void warm_z(const FfnArgs& p) {
    if (!warm_fits(p)) return;
    const size_t zb = z_bytes(p);
    for (size_t i = threadIdx.x; i < (zb + 127) / 128; i += blockDim.x)
        prefetch_l1(reinterpret_cast<const uint8_t*>(p.zx) + i * 128);
}

// IQ: ternary and 2-bit experts take the integer path (T <= kIqMaxT; down: when the K-part
// reduction formed h's records).
template <int MODE, bool IQ>
__global__ void __launch_bounds__(NW * 32, 1) ffn_decode_kernel(FfnArgs p) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ CtaSched S;
    __shared__ uint64_t stall_bar;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    Geo geo;
    geo.K = MODE == 0 ? p.H : p.I;
    geo.G = geo.K / 64;
    geo.NC = (geo.G + CG - 1) / CG;
    geo.blocks = MODE == 0 ? (2 * p.I) / (16 * NTL) : p.H / (16 * NTL);
    geo.nkp = MODE == 0 ? p.nkp_gu : p.nkp_dn;
    geo.cpk = (geo.NC + geo.nkp - 1) / geo.nkp;
    uint8_t* ring = smem + (size_t)warp * NS * STAGE;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + (size_t)NW * NS * STAGE) + warp * NS;

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
        if (!S.ok) {
            report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetHeader);
        } else if (__ldcg(&p.ctrl->routed_T) != p.T) {
            // the schedule in the workspace was routed for another T: do not read it
            report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetRoutedT | MODE);
            S.ok = 0;
        }
        S.n_active = __ldcg(&p.ctrl->n_active);
        S.perm_in_smem = p.T * p.k <= kPermSmem;
        S.stall = p.ctrl->test_stall;
    }
    __syncthreads();
    if (!S.ok) return;
    const int nA = S.n_active;
    for (int a = threadIdx.x; a < nA; a += blockDim.x) {
        const int e = p.active[a];
        S.e[a] = e;
        S.fmt[a] = (int)entry(p.packed, e)->fmt;
        S.cnt[a] = e < p.E ? p.counts[e] : p.T;
        S.off[a] = e < p.E ? p.offsets[e] : 0;
        if (S.fmt[a] > MOE_FMT_Q3) {            // a storage form (dense ternary): not read here
            if (blockIdx.x == 0) report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetFormat | MODE);
            S.ok = 0;
        }
    }
    if (S.perm_in_smem)
        for (int r = threadIdx.x; r < p.T * p.k; r += blockDim.x) S.tok[r] = p.perm[r] / p.k;
    __syncthreads();
    if (!S.ok) return;
    if (threadIdx.x == 0) {
        int run = 0, one = 1;
        for (int a = 0; a < nA; ++a) {
            S.upre[a] = run;
            const int np = (S.cnt[a] + TP - 1) / TP;
            run += np;
            one &= np == 1;
        }
        S.upre[nA] = run;
        S.n_ep = run;
        S.one_pass = one;
        S.n_units = run * geo.blocks * geo.nkp;
    }
    if (MODE == 0) warm_z(p);
    if (lane == 0)
        for (int s = 0; s < NS; ++s) mbar_init(&bar[s], 1);
    if (threadIdx.x == 0) mbar_init(&stall_bar, 1);            // nothing ever arrives on it
    fence_mbar_init();
    __syncthreads();
    // Units come from the launch's work counter (zeroed by the router and by the
    // combine, so every forward starts from 0); a warp grabs its first unit here and
    // each following one a unit ahead of need (Producer).
    uint32_t* ctr = &p.ctrl->work[MODE];
    FastDiv per_ep, fkp;
    per_ep.init(geo.blocks * geo.nkp);
    fkp.init(geo.nkp);
    const uint64_t pol = l2_policy_evict_first();

    Producer<MODE> prod;
    prod.issued = 0;
    prod.cur_a = -1;
#pragma unroll
    for (int i = 0; i < NS; ++i) prod.hu[i] = -1;
    prod.start(p, S, geo, per_ep, fkp, ctr, lane, __shfl_sync(0xffffffffu, prod.grab(ctr, lane), 0));
    for (int i = 0; i < NS - 1; ++i) prod.issue(p, S, geo, per_ep, fkp, ctr, lane, ring, bar, pol);

    LaneGeo L;
    L.g = lane >> 2;
    L.t = lane & 3;
    L.cw_lane = 32 * L.g + L.t;
    L.g4 = 4 * L.g;
    L.hw_lane = 16 * L.g + (L.t >> 1);
    L.g2 = 2 * (L.g >> 1);
    L.sh = 8 * (L.t & 1);
    L.zplane = 3 * p.T * (8 * ((p.H / 64 + 7) / 8));
    bool aborted = false;
    int consumed = 0;
    // The chunk to consume is the one issued NS - 1 issues ago (hu / hc[NS - 1] after
    // the next issue).  A unit ends when the next chunk belongs to another unit.
    int unit = -1, view_a = -1, view_pass = -1;
    bool q3 = false;
    UnitPos q;
    q.a = q.pass = q.jb = q.kp = 0;
    UnitView v;
    uint32_t sub[5] = {0, 0, 0, 0, 0};
    float acc[NTL][4];
    unsigned long long ia[NTL];                        // integer path: (gate, up) of token t per tile
    bool iqu = false;                                  // the current unit is on the integer path
    // failure-path tests: warp 0 waits on a barrier nothing completes; the wait runs out
    // and the warp takes the give-up path below
    if (warp == 0 && S.stall) {
        int done = 0;
        if (lane == 0) done = mbar_wait_bounded(&stall_bar, 0, S.stall);
        if (!__shfl_sync(0xffffffffu, done, 0)) {
            aborted = true;
            if (lane == 0) report_error(p.ctrl, MOE_ERR_TIMEOUT, kDetTestStall | MODE);
        }
    }
    // A warp consumes at most every chunk of every unit once, plus the empty issues at
    // the end: a cap that consistent counters never reach.
    const long long max_iters = (long long)S.n_units * geo.cpk + NS + 2;
    long long iters = 0;
    while (!aborted) {
        if (++iters > max_iters) {
            aborted = true;
            if (lane == 0) report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetLoopCap | MODE);
            break;
        }
        prod.issue(p, S, geo, per_ep, fkp, ctr, lane, ring, bar, pol);
        const int hu = prod.hu[NS - 1], c = prod.hc[NS - 1];
        if (hu < 0) {                                   // nothing left (or nothing at all)
            if (unit >= 0) {
                if (IQ && iqu) unit_epilogue_iq<MODE>(p, geo, q, v, L, ia);
                else unit_epilogue<MODE>(p, geo, q, v, L, acc);
            }
            break;
        }
        if (hu != unit) {
            if (unit >= 0) {
                if (IQ && iqu) unit_epilogue_iq<MODE>(p, geo, q, v, L, ia);
                else unit_epilogue<MODE>(p, geo, q, v, L, acc);
            }
            unit = hu;
            q = unit_pos(S, unit, per_ep, fkp);
            if (q.a != view_a || q.pass != view_pass) {
                view_a = q.a;
                view_pass = q.pass;
                q3 = S.fmt[q.a] == MOE_FMT_Q3;
                iqu = IQ && !q3;
                if (IQ && iqu) make_view_iq<MODE>(p, S, q.a, L.g, L.t, v);
                else make_view<MODE>(p, S, q.a, q.pass, L.g, L.t, v);
                if (MODE == 1) {
                    const int f = S.fmt[q.a];
                    const float o = f == MOE_FMT_TERNARY ? 1.f : (f == MOE_FMT_Q2 ? 1.5f : 3.5f);
                    sub[0] = f16x2_bits_of(512.f + o);
                    sub[1] = f16x2_bits_of(256.f + o);
                    sub[2] = f16x2_bits_of(64.f + o);
                    sub[3] = f16x2_bits_of(16.f + o);
                    sub[4] = f16x2_bits_of(4.f + o);
                }
            }
#pragma unroll
            for (int tl = 0; tl < NTL; ++tl) {
                acc[tl][0] = acc[tl][1] = acc[tl][2] = acc[tl][3] = 0.f;
                ia[tl] = 0ull;                          // the fp32 pair (0, 0)
            }
        }
        const int st = consumed % NS;
        int ok = 1;
        if (lane == 0 && !mbar_wait_bounded(&bar[st], (uint32_t)(consumed / NS) & 1, kWaitLimit)) {
            ok = 0;
            report_error(p.ctrl, MOE_ERR_TIMEOUT, kDetWaitFull | MODE);
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
            // give up: issue nothing more; the copies in flight are waited for below
            aborted = true;
            break;
        }
        const uint8_t* stg = ring + (size_t)st * STAGE;
        const int ng = min(CG, geo.G - c * CG);
        if (IQ && iqu) {
            if (ng == CG) chunk_full_iq(stg, c, v, L, ia);
            else chunk_partial_iq(stg, c, ng, v, L, ia);
        } else if (ng == CG) {
            if (q3) chunk_full<MODE, true>(stg, c, v, L, sub, acc);
            else chunk_full<MODE, false>(stg, c, v, L, sub, acc);
        } else {
            if (q3) chunk_partial<MODE, true>(stg, c, ng, v, L, sub, acc);
            else chunk_partial<MODE, false>(stg, c, ng, v, L, sub, acc);
        }
        __syncwarp();          // every lane is done with this stage before it is refilled
        ++consumed;
    }
    // after a timeout the ring may still hold copies in flight: wait for them (bounded)
    if (aborted) {
        for (int qd = consumed; qd < prod.issued; ++qd)
            if (!mbar_wait_bounded(&bar[qd % NS], (uint32_t)(qd / NS) & 1, kWaitLimit)) {
                report_error(p.ctrl, MOE_ERR_TIMEOUT, kDetDrain | MODE);
                break;
            }
    }
}

// h[row][i] = silu(sum_kp gate) * (sum_kp up) for every (token, slot) row, the K parts
// added in order.  One thread per 4 consecutive h columns (4 gate and 4 up sums per
// part); every part's loads are issued before the first add, so the kernel costs one
// L2 round trip.
constexpr int kMaxParts = 16;                           // K parts: at most ceil(K / 512)

__global__ void __launch_bounds__(128) finalize_gateup_kernel(FfnArgs p) {
    griddep_launch_dependents();                        // a single small wave
    griddep_wait();                                     // gpart comes from the gate/up pass
    const int per_row = p.I / 4;
    const size_t R = (size_t)p.T * (p.k + p.S);
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= R * per_row) return;
    const size_t row = idx / per_row;
    const int q = (int)(idx - row * per_row);           // columns 4q .. 4q+3
    const int j = q >> 1, half = q & 1;                 // tile j: gate sums at 16j + 4half, up at +8
    const float* base = p.gpart + row * (2 * p.I) + j * 16 + 4 * half;
    const size_t pstride = R * (2 * p.I);
    float4 gv[kMaxParts], uv[kMaxParts];
#pragma unroll
    for (int kp = 0; kp < kMaxParts; ++kp) {
        if (kp < p.nkp_gu) {
            gv[kp] = __ldcg(reinterpret_cast<const float4*>(base + kp * pstride));
            uv[kp] = __ldcg(reinterpret_cast<const float4*>(base + kp * pstride + 8));
        }
    }
    float4 gs = make_float4(0.f, 0.f, 0.f, 0.f), us = gs;
#pragma unroll
    for (int kp = 0; kp < kMaxParts; ++kp) {
        if (kp < p.nkp_gu) {
            gs.x += gv[kp].x; gs.y += gv[kp].y; gs.z += gv[kp].z; gs.w += gv[kp].w;
            us.x += uv[kp].x; us.y += uv[kp].y; us.z += uv[kp].z; us.w += uv[kp].w;
        }
    }
    const float h0 = silu_f(gs.x) * us.x, h1 = silu_f(gs.y) * us.y, h2 = silu_f(gs.z) * us.z,
                h3 = silu_f(gs.w) * us.w;
    if (!(in_f16_range(h0) && in_f16_range(h1) && in_f16_range(h2) && in_f16_range(h3)))
        report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetRange | kRangeDecode);
    uint2 o;
    o.x = (uint32_t)f32_to_f16_bits(h0) | ((uint32_t)f32_to_f16_bits(h1) << 16);
    o.y = (uint32_t)f32_to_f16_bits(h2) | ((uint32_t)f32_to_f16_bits(h3) << 16);
    *reinterpret_cast<uint2*>(p.h + row * p.I + 4 * q) = o;
}

// The same reduction when the down pass runs ternary and 2-bit experts on integer MMAs
// (up to kIqMaxT tokens): one warp per (row, 64-column group of h), two columns per
// lane; besides fp16 h it forms the row's integer operands from the fp32 h on a 12-bit
// grid per group (iq_group: digit records and pairs in the hq region, pairs of the
// padding groups zero).
__global__ void __launch_bounds__(128) finalize_gateup_iq_kernel(FfnArgs p) {
    griddep_launch_dependents();                        // a single small wave
    griddep_wait();                                     // gpart comes from the gate/up pass
    const int GI = p.I / 64, GI8 = 8 * ((GI + 7) / 8);
    const size_t R = (size_t)p.T * (p.k + p.S);
    const size_t w = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= R * GI8) return;                           // whole warps
    const size_t row = w / GI8;
    const int gq = (int)(w - row * GI8);
    float2* pairs = reinterpret_cast<float2*>(p.hq + iq_pair_off(p.R16, p.I)) + row * GI8;
    if (gq >= GI) {
        if (lane == 0) pairs[gq] = make_float2(0.f, 0.f);
        return;
    }
    const int c = gq * 64 + 2 * lane;                   // h columns c, c + 1 (tile c / 8, rows c % 8)
    const float* base = p.gpart + row * (2 * p.I) + (c >> 3) * 16 + (c & 7);
    const size_t pstride = R * (2 * p.I);
    float2 gv[kMaxParts], uv[kMaxParts];
#pragma unroll
    for (int kp = 0; kp < kMaxParts; ++kp) {
        if (kp < p.nkp_gu) {
            gv[kp] = __ldcg(reinterpret_cast<const float2*>(base + kp * pstride));
            uv[kp] = __ldcg(reinterpret_cast<const float2*>(base + kp * pstride + 8));
        }
    }
    float2 gs = make_float2(0.f, 0.f), us = gs;
#pragma unroll
    for (int kp = 0; kp < kMaxParts; ++kp) {
        if (kp < p.nkp_gu) {
            gs.x += gv[kp].x; gs.y += gv[kp].y;
            us.x += uv[kp].x; us.y += uv[kp].y;
        }
    }
    const float h0 = silu_f(gs.x) * us.x, h1 = silu_f(gs.y) * us.y;
    if (!(in_f16_range(h0) && in_f16_range(h1))) report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetRange | kRangeDecode);
    *reinterpret_cast<uint32_t*>(p.h + row * p.I + c) =
        (uint32_t)f32_to_f16_bits(h0) | ((uint32_t)f32_to_f16_bits(h1) << 16);
    iq_group(h0, h1, lane, p.hq + (row * GI + gq) * 128, pairs + gq);
}

// y[t] = sum_j g[t,j] * ypart[inv_perm[t*k + j]] + sum_s ypart[T*k + s*T + t], in slot
// order, each row first summed over its K parts in order; fp32, stored as bf16.  For few
// tokens: one thread per 4 consecutive outputs, the slot rows and gates loaded first,
// then every partial row, so the pass costs two L2 round trips.
constexpr int kMaxRows = 12;                            // k + S rows per token ...
constexpr int kMaxKp = 4;                               // ... and K parts held in registers

__device__ __forceinline__ void add4(float4& a, const float4& b) {
    a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
}

__global__ void __launch_bounds__(128) combine_kernel(FfnArgs p) {
    griddep_wait();                                     // ypart comes from the down pass
    if (__ldcg(&p.ctrl->routed_T) != p.T) return;       // inv_perm is another T's (reported by the FFN kernels)
    if (blockIdx.x == 0 && threadIdx.x == 0) {          // both expert passes are complete
        p.ctrl->work[0] = 0;
        p.ctrl->work[1] = 0;
    }
    const int per_tok = p.H / 4;
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (size_t)p.T * per_tok) return;
    const int tok = (int)(idx / per_tok), c4 = (int)(idx - (size_t)tok * per_tok) * 4;
    const size_t R = (size_t)p.T * (p.k + p.S);
    const size_t pstride = R * p.H;
    const int nrows = p.k + p.S;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (nrows <= kMaxRows && p.nkp_dn <= kMaxKp) {
        int rows[kMaxRows];
        float gw[kMaxRows];
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r) {
            if (r < p.k) {
                rows[r] = __ldg(p.inv_perm + (size_t)tok * p.k + r);
                gw[r] = __ldg(p.topk_w + (size_t)tok * p.k + r);
            } else if (r < nrows) {
                rows[r] = p.T * p.k + (r - p.k) * p.T + tok;
                gw[r] = 1.f;
            }
        }
        float4 v[kMaxKp][kMaxRows];
#pragma unroll
        for (int kp = 0; kp < kMaxKp; ++kp)
#pragma unroll
            for (int r = 0; r < kMaxRows; ++r)
                if (r < nrows && kp < p.nkp_dn)
                    v[kp][r] = __ldcg(reinterpret_cast<const float4*>(p.ypart + kp * pstride + (size_t)rows[r] * p.H + c4));
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r) {
            if (r >= nrows) continue;
            float4 s = v[0][r];
#pragma unroll
            for (int kp = 1; kp < kMaxKp; ++kp)
                if (kp < p.nkp_dn) add4(s, v[kp][r]);
            if (r < p.k) {
                acc.x = fmaf(gw[r], s.x, acc.x);
                acc.y = fmaf(gw[r], s.y, acc.y);
                acc.z = fmaf(gw[r], s.z, acc.z);
                acc.w = fmaf(gw[r], s.w, acc.w);
            } else {
                add4(acc, s);
            }
        }
    } else {
        // many parts: the same sums, one row at a time
        for (int r = 0; r < nrows; ++r) {
            const int row = r < p.k ? p.inv_perm[(size_t)tok * p.k + r] : p.T * p.k + (r - p.k) * p.T + tok;
            const float* src = p.ypart + (size_t)row * p.H + c4;
            float4 s = __ldcg(reinterpret_cast<const float4*>(src));
            for (int kp = 1; kp < p.nkp_dn; ++kp) add4(s, __ldcg(reinterpret_cast<const float4*>(src + kp * pstride)));
            if (r < p.k) {
                const float g = p.topk_w[(size_t)tok * p.k + r];
                acc.x = fmaf(g, s.x, acc.x);
                acc.y = fmaf(g, s.y, acc.y);
                acc.z = fmaf(g, s.z, acc.z);
                acc.w = fmaf(g, s.w, acc.w);
            } else {
                add4(acc, s);
            }
        }
    }
    if (p.y_f32) {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.y) + (size_t)tok * p.H + c4) = acc;
        return;
    }
    uint2 o;
    o.x = (uint32_t)f32_to_bf16_bits(acc.x) | ((uint32_t)f32_to_bf16_bits(acc.y) << 16);
    o.y = (uint32_t)f32_to_bf16_bits(acc.z) | ((uint32_t)f32_to_bf16_bits(acc.w) << 16);
    *reinterpret_cast<uint2*>(p.y + (size_t)tok * p.H + c4) = o;
}

// The same combine for many tokens: one thread per 8 consecutive outputs of a token
// (two 16-byte loads per row and part), rows one after another.
__global__ void __launch_bounds__(256) combine_rows_kernel(FfnArgs p) {
    griddep_wait();                                     // ypart comes from the down pass
    if (__ldcg(&p.ctrl->routed_T) != p.T) return;       // inv_perm is another T's (reported by the FFN kernels)
    if (blockIdx.x == 0 && threadIdx.x == 0) {          // both expert passes are complete
        p.ctrl->work[0] = 0;
        p.ctrl->work[1] = 0;
    }
    const int per_tok = p.H / 8;
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (size_t)p.T * per_tok) return;
    const int tok = (int)(idx / per_tok), c8 = (int)(idx - (size_t)tok * per_tok) * 8;
    const size_t pstride = (size_t)p.T * (p.k + p.S) * p.H;
    float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
    for (int r = 0; r < p.k + p.S; ++r) {
        const int row = r < p.k ? p.inv_perm[(size_t)tok * p.k + r] : p.T * p.k + (r - p.k) * p.T + tok;
        const float4* src = reinterpret_cast<const float4*>(p.ypart + (size_t)row * p.H + c8);
        float4 s0 = __ldcg(src), s1 = __ldcg(src + 1);
        for (int kp = 1; kp < p.nkp_dn; ++kp) {
            add4(s0, __ldcg(src + kp * (pstride / 4)));
            add4(s1, __ldcg(src + kp * (pstride / 4) + 1));
        }
        if (r < p.k) {
            const float g = p.topk_w[(size_t)tok * p.k + r];
            a0.x = fmaf(g, s0.x, a0.x);
            a0.y = fmaf(g, s0.y, a0.y);
            a0.z = fmaf(g, s0.z, a0.z);
            a0.w = fmaf(g, s0.w, a0.w);
            a1.x = fmaf(g, s1.x, a1.x);
            a1.y = fmaf(g, s1.y, a1.y);
            a1.z = fmaf(g, s1.z, a1.z);
            a1.w = fmaf(g, s1.w, a1.w);
        } else {
            add4(a0, s0);
            add4(a1, s1);
        }
    }
    if (p.y_f32) {
        float4* d = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.y) + (size_t)tok * p.H + c8);
        d[0] = a0;
        d[1] = a1;
        return;
    }
    uint4 o;
    o.x = (uint32_t)f32_to_bf16_bits(a0.x) | ((uint32_t)f32_to_bf16_bits(a0.y) << 16);
    o.y = (uint32_t)f32_to_bf16_bits(a0.z) | ((uint32_t)f32_to_bf16_bits(a0.w) << 16);
    o.z = (uint32_t)f32_to_bf16_bits(a1.x) | ((uint32_t)f32_to_bf16_bits(a1.y) << 16);
    o.w = (uint32_t)f32_to_bf16_bits(a1.z) | ((uint32_t)f32_to_bf16_bits(a1.w) << 16);
    *reinterpret_cast<uint4*>(p.y + (size_t)tok * p.H + c8) = o;
}

constexpr size_t kDynSmem = (size_t)NW * NS * STAGE + (size_t)NW * NS * 8;

template <int MODE, bool IQ>
cudaError_t launch_mode(const FfnArgs& a, cudaStream_t s) {
    const cudaError_t err = set_smem_limit(ffn_decode_kernel<MODE, IQ>, kDynSmem);
    if (err != cudaSuccess) return err;
    return launch_pdl(ffn_decode_kernel<MODE, IQ>, dim3(a.num_ctas), dim3(NW * 32), kDynSmem, s, a);
}

}  // namespace

cudaError_t launch_ffn_decode(const FfnArgs& a, cudaStream_t s, cudaEvent_t ev_gateup, cudaEvent_t ev_down) {
    const bool iq_gu = a.iq_on && a.iq;
    // the down pass on the integer path when the K-part reduction can form h's records
    const bool iq_dn = iq_gu && a.nkp_gu > 1 && a.hq && (long long)a.T * (a.k + a.S) <= a.R16;
    cudaError_t err = iq_gu ? launch_mode<0, true>(a, s) : launch_mode<0, false>(a, s);
    if (err != cudaSuccess) return err;
    if (iq_dn) {
        const long long n = (long long)a.T * (a.k + a.S) * (8 * ((a.I / 64 + 7) / 8)) * 32;   // threads
        err = launch_pdl(finalize_gateup_iq_kernel, dim3((unsigned)((n + 127) / 128)), dim3(128), 0, s, a);
        if (err != cudaSuccess) return err;
    } else if (a.nkp_gu > 1) {
        const long long n = (long long)a.T * (a.k + a.S) * (a.I / 4);
        err = launch_pdl(finalize_gateup_kernel, dim3((unsigned)((n + 127) / 128)), dim3(128), 0, s, a);
        if (err != cudaSuccess) return err;
    }
    if (ev_gateup && (err = record_event(ev_gateup, s)) != cudaSuccess) return err;
    err = iq_dn ? launch_mode<1, true>(a, s) : launch_mode<1, false>(a, s);
    if (err != cudaSuccess) return err;
    if (ev_down && (err = record_event(ev_down, s)) != cudaSuccess) return err;
    return launch_combine(a, s);
}

cudaError_t launch_combine(const FfnArgs& a, cudaStream_t s) {
    // few tokens: a latency-bound pass, every load issued up front; many tokens: rows
    if (a.T <= kSmallT) {
        const long long n = (long long)a.T * (a.H / 4);
        return launch_pdl(combine_kernel, dim3((unsigned)((n + 127) / 128)), dim3(128), 0, s, a);
    }
    const long long n = (long long)a.T * (a.H / 8);
    return launch_pdl(combine_rows_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, a);
}

}  // namespace moe
