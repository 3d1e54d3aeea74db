// The decode forward for few tokens (1 <= T <= 16) as ONE persistent kernel: the
// gate/up + SwiGLU pass and the down pass of every selected expert and of the shared
// expert, and the gate-weighted combine into y.
//
// Decode speed is set by the expert bytes moved per token (ossradar.top, Xolotl README,
// "Fast mode (DeepSeek-V4.1)"), and each selected expert is read once for all of its
// tokens (the same README, "Latest").  With one token, a step reads about 117 MB in
// ~18 us at the HBM roofline, so the step cannot afford kernel boundaries (a launch,
// a ramp and a tail each) between its phases; instead the phases are units of work in
// one queue and wait on each other through counters in the workspace:
//
//   gate/up   (expert, 16-row tile of the fused gate/up matrix, all of K or one of
//             its K parts): h = silu(gate) * up (fp16 for the bf16 down path, fp32
//             for the integer one); a split tile's last part sums the parts in order
//   down      (expert, 16-row tile of the down matrix, all of K or one K part): needs
//             every gate/up tile of its expert (and, on the integer path, the expert's
//             h operands, formed by its first down units); fp32 rows of y_e
//   combine   the down unit that finishes a 16-row slice of y last for all experts
//             and parts sums the slice's rows, the routed ones weighted by their gates
//             in slot order, plus the shared expert's, and stores bf16 (deterministic)
//
// Units are handed out in that order from one counter (one unit ahead of need), so
// every wait is for a unit some running warp already holds: the queue cannot deadlock,
// whatever the number of resident CTAs.  The shared expert's gate/up tiles come
// first (every token's chain runs through them), split into K parts when the gate/up
// tiles of all experts do not fit in one wave of warps.  The token operands (the integer path's digit records, the Z tables) are formed by the
// router launch this kernel follows (programmatic dependent launch: the prologue
// overlaps the router's tail, griddepcontrol.wait comes before the first unit).
//
// Inside a unit a warp streams its tile's 8-group chunks (codes, third bits, fp16
// scales: contiguous blocks of the packed format) through its own ring of NS
// shared-memory stages with 1-D bulk copies, and the ring runs ahead into the next
// unit.  Gate/up of ternary and 2-bit experts runs on the integer tensor path (u8 codes
// masked out of the code words against signed-byte token digits on a 12-bit grid per
// token and group; passes of 4 tokens per n8 MMA tile); 3-bit experts use the bf16
// dequantiser ("base + c" in the mantissa of a power of two, the offsets removed once
// per chunk by a small MMA against the token's Z table; passes of 8 tokens); down
// dequantises exact fp16 (c - o) against fp16 h.
//
// Every wait is bounded (mbarriers and counters); a wait that runs out records
// MOE_ERR_TIMEOUT and raises an abort flag that makes every warp stop working, wait
// (bounded) for its own copies in flight and leave.  The last warp to leave resets the
// counters, so the next launch starts from zero.
#include "kernels.h"
#include "dequant.cuh"
#include "operands.cuh"      // iq_group: the down pass forms its h operands
#include "iqmma.cuh"

namespace moe {
namespace {

using namespace dq;
using namespace iq;

constexpr int NW = 16;                           // warps per CTA (one CTA per SM)
constexpr int NS = 3;                            // ring stages per warp
constexpr int CG = 8;                            // 64-wide groups per chunk
constexpr int OFF_HI = 2048;                     // stage: codes 16 rows x 32 words
constexpr int OFF_SC = OFF_HI + 1024;            //        third bits 16 rows x 16 words
constexpr int STAGE = OFF_SC + 256;              //        scales 16 rows x 8 halves
constexpr int MAXP = 4;                          // integer passes per unit (4 tokens each)
constexpr int MAXPB = 2;                         // bf16 / fp16 passes per unit (8 tokens each)
constexpr long long kWaitLimit = 4000000000LL;   // clock cycles (~2 s)
constexpr size_t kFusedSmem = (size_t)NW * NS * STAGE + (size_t)NW * NS * 8;
// At up to kStageMaxT tokens the tokens' integer records and pairs (iq_size(T, H): 15 KB
// a token at H = 7168) are copied once per CTA into shared memory behind the rings:
// every routed gate/up tile of the launch reads the same few tokens, and shared-memory
// loads have a short, fixed latency where L1 hits do not (and an acquire load clears L1).
#ifndef MOE_STAGE_TOKENS
#define MOE_STAGE_TOKENS 1
#endif
constexpr int kStageMaxT = MOE_STAGE_TOKENS ? 2 : 0;
inline size_t fused_smem_bytes(int T, int H) { return kFusedSmem + (T <= kStageMaxT ? iq_size(T, H) : 0); }

static_assert(MAXP * 4 >= kFusedMaxT && MAXPB * 8 >= kFusedMaxT, "passes cover kFusedMaxT tokens");

// ---- global-memory synchronisation ---------------------------------------------------
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Lane 0 waits until *ctr >= target (or the launch aborts), bounded.  It polls with
// relaxed loads and a growing sleep (an acquire load also drops the SM's L1 contents,
// which the other warps on the SM are using), then makes one acquire load; the warp
// barrier orders the other lanes' later loads after it.  Returns false if the wait ran
// out or the launch aborted.
__device__ __forceinline__ bool wait_counter(const uint32_t* ctr, uint32_t target, FusedCtl* fc, Ctrl* ctrl,
                                             uint32_t detail, int lane) {
    int ok = 1;
    if (lane == 0) {
        if (ld_relaxed(ctr) < target) {
            const long long t0 = clock64();
            uint32_t ns = 128;
            while (true) {
                __nanosleep(ns);
                if (ns < 1024) ns *= 2;
                if (ld_relaxed(ctr) >= target) break;
                if (ld_relaxed(&fc->abort)) {
                    ok = 0;
                    break;
                }
                if (clock64() - t0 > kWaitLimit) {
                    report_error(ctrl, MOE_ERR_TIMEOUT, detail);
                    atomicExch(&fc->abort, 1u);
                    ok = 0;
                    break;
                }
            }
        }
        if (ok) (void)ld_acquire(ctr);
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// All lanes' stores of this unit happen-before the counter increment: the warp barrier
// orders them before lane 0's increment, which is a release at GPU scope (cumulative
// over what lane 0 has observed).  signal_counter returns the old value; post_counter
// does not wait for it.
__device__ __forceinline__ uint32_t signal_counter(uint32_t* ctr, int lane) {
    __syncwarp();
    uint32_t old = 0;
    if (lane == 0) asm volatile("atom.add.release.gpu.global.u32 %0, [%1], 1;" : "=r"(old) : "l"(ctr) : "memory");
    return __shfl_sync(0xffffffffu, old, 0);
}
__device__ __forceinline__ void post_counter(uint32_t* ctr, int lane) {
    __syncwarp();
    if (lane == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
}

__device__ __forceinline__ const PackedEntry* pentry(const uint8_t* packed, int e) {
    return reinterpret_cast<const PackedEntry*>(packed + kHeaderBytes + (size_t)e * kEntryBytes);
}

// ---- the work queue --------------------------------------------------------------------
enum : int { U_NONE = 0, U_GU = 2, U_DN = 3, U_PENDING = 4 };   // PENDING: not taken yet

struct Layout {        // unit index ranges (resolve)
    int nsgu;                   // shared gate/up units (tiles x K parts)
    int tg, td;                 // 16-row tiles per expert: gate/up (2I/16), down (H/16)
    int nch, nci;               // 8-group chunks per row: gate/up (K = H), down (K = I)
    int S;                      // shared experts (their slots come first)
    int pg, pr, pd;             // K parts: shared gate/up tiles, routed gate/up tiles, down tiles
    int cpg, cpr, cpd;          // chunks per part
    int shares;                 // down tiles per expert that form the h operands (integer path)
    int nr;                     // routed experts with tokens
    int total;                  // all units
    bool t_ok;                  // the routing is for this call's T
};

// A unit is four integers; everything else about its expert comes from the CTA's slot
// table in shared memory (a few registers per warp instead of a copy of it).
struct Unit {
    int kind, idx, slot, tile, part;
};

// Per expert slot (shared experts first, then the routed experts with tokens, in the
// router's active order): table index, format, tokens, first row, and the packed
// blocks of tile 0 of its gate/up and down matrices.
struct SlotInfo {
    const uint8_t* base[6];     // gate/up codes, third bits, scales; down codes, third bits, scales
    int e, fmt, cnt, row0;
};
struct CtaState {
    SlotInfo slot[kMaxSlots];
    int routed;                 // 0: not read, 1: being read by one warp, 2: ready
    int nr, t_ok;
};

__device__ __forceinline__ void fill_slot(SlotInfo& si, const FfnArgs& p, int e, int cnt, int row0) {
    const PackedEntry* en = pentry(p.packed, e);
    si.e = e;
    si.fmt = (int)en->fmt;
    if (si.fmt > MOE_FMT_Q3) {
        // a storage form (dense ternary) the kernels do not read: the launch aborts
        // before any unit is taken (every warp reads the routing first)
        report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetFormat | 0x20);
        atomicExch(&p.fc->abort, 1u);
        si.fmt = MOE_FMT_Q2;
    }
    si.cnt = cnt;
    si.row0 = row0;
    si.base[0] = p.packed + en->gu_codes;
    si.base[1] = p.packed + en->gu_hi;
    si.base[2] = p.packed + en->gu_scales;
    si.base[3] = p.packed + en->dn_codes;
    si.base[4] = p.packed + en->dn_hi;
    si.base[5] = p.packed + en->dn_scales;
}

// The routing, once per CTA: every warp waits for the router grid (griddepcontrol.wait,
// before it reads any router output); the first warp of the CTA to get here fills the
// routed slots of the table, the others wait for it (bounded).  Returns the routed
// expert count (-1 if that wait ran out; then the launch aborts) and whether the
// routing is for this call's T.
__device__ __noinline__ int read_routing(CtaState& cs, const FfnArgs& p, int lane, int* t_ok) {
    griddep_wait();
    int mine = 0;
    if (lane == 0) mine = atomicCAS(&cs.routed, 0, 1) == 0;
    mine = __shfl_sync(0xffffffffu, mine, 0);
    int ok = 1;
    if (mine) {
        int nr = 0, tok = 1;
        if (lane == 0) {
            // from L2: this SM's L1 may hold the control block's line from before the
            // router wrote it (the test-stall word shares the line)
            tok = __ldcg(&p.ctrl->routed_T) == p.T;
            nr = tok ? __ldcg(&p.ctrl->n_active) - p.S : 0;
            if (!tok) report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetRoutedT | 0x20);
        }
        nr = __shfl_sync(0xffffffffu, nr, 0);
        tok = __shfl_sync(0xffffffffu, tok, 0);
        for (int a = lane; a < nr; a += 32) {
            const int e = __ldcg(p.active + a);
            fill_slot(cs.slot[p.S + a], p, e, __ldcg(p.counts + e), __ldcg(p.offsets + e));
        }
        if (lane == 0) {
            cs.nr = nr;
            cs.t_ok = tok;
        }
        __syncwarp();
        __threadfence_block();
        if (lane == 0) *reinterpret_cast<volatile int*>(&cs.routed) = 2;
        __syncwarp();
    } else if (lane == 0) {
        const long long t0 = clock64();
        while (*reinterpret_cast<volatile int*>(&cs.routed) != 2) {
            if (clock64() - t0 > kWaitLimit) {
                report_error(p.ctrl, MOE_ERR_TIMEOUT, kDetWaitFull | 0x24);
                atomicExch(&p.fc->abort, 1u);
                ok = 0;
                break;
            }
            __nanosleep(100);
        }
        __threadfence_block();
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    *t_ok = ok && *reinterpret_cast<volatile int*>(&cs.t_ok) != 0;
    return ok ? *reinterpret_cast<volatile int*>(&cs.nr) : -1;
}

// Unit u -> its kind, slot, tile and K part (U_NONE past the last unit).  The order:
// the shared experts' gate/up tiles (K parts fastest; every token goes through them,
// so they are the longest chain), the routed experts' gate/up tiles (slot order),
// then the down tiles: every slot's first `shares` tiles (they form the integer
// path's h operands) before the rest, slots in order (the shared ones first), tiles
// ascending, K parts fastest.
__device__ __forceinline__ Unit resolve(const FfnArgs& p, const Layout& L, int u) {
    Unit U;
    U.kind = U_NONE;
    U.idx = u;
    U.slot = 0;
    U.tile = 0;
    U.part = 0;
    if (u < 0 || u >= L.total) return U;
    int v = u;
    if (v < L.nsgu) {
        const int per = L.tg * L.pg;
        U.kind = U_GU;
        U.slot = v / per;
        const int r = v - U.slot * per;
        U.tile = r / L.pg;
        U.part = r - U.tile * L.pg;
        return U;
    }
    v -= L.nsgu;
    if (v < L.nr * L.tg * L.pr) {
        const int per = L.tg * L.pr, a = v / per;
        const int r = v - a * per;
        U.kind = U_GU;
        U.slot = p.S + a;
        U.tile = r / L.pr;
        U.part = r - U.tile * L.pr;
        return U;
    }
    v -= L.nr * L.tg * L.pr;
    U.kind = U_DN;
    const int n_slots = p.S + L.nr;
    const int b1 = L.shares * L.pd, rest = (L.td - L.shares) * L.pd;
    int d, r;
    if (v < n_slots * b1) {
        d = v / b1;
        r = v - d * b1;
    } else {
        v -= n_slots * b1;
        d = v / rest;
        r = v - d * rest + b1;
    }
    U.slot = d;
    U.tile = r / L.pd;
    U.part = r - U.tile * L.pd;
    return U;
}

__device__ __forceinline__ bool streams(const Unit& U) { return U.kind == U_GU || U.kind == U_DN; }
// The unit's chunks: [c0, c0 + n) of its matrix's K (one K part of it, if split).
__device__ __forceinline__ int unit_cpp(const Unit& U, const Layout& L) {      // chunks per part
    return U.kind == U_DN ? L.cpd : (U.slot < L.S ? L.cpg : L.cpr);
}
__device__ __forceinline__ int unit_c0(const Unit& U, const Layout& L) { return U.part * unit_cpp(U, L); }
__device__ __forceinline__ int unit_nc(const Unit& U, const Layout& L) {
    const int c0 = unit_c0(U, L);
    return min(U.kind == U_DN ? L.nci : L.nch, c0 + unit_cpp(U, L)) - c0;
}
// K parts of a gate/up tile of this unit's slot
__device__ __forceinline__ int gu_parts(const Unit& U, const Layout& L) { return U.slot < L.S ? L.pg : L.pr; }
// A gate/up tile split into K parts: the parts' sums go to gsh, the last part forms h.
__device__ __forceinline__ bool gu_split(const Unit& U, const Layout& L) {
    return U.kind == U_GU && gu_parts(U, L) > 1;
}

// The warp's next unit, taken from the launch's counter only when the ring is about to
// need it (when the current unit's last chunks are being issued): a unit held early by a
// warp that is still busy would hold back every unit that waits for it.
struct Queue {
    Unit nxt;
};

__device__ __forceinline__ void take_next(Queue& Q, const FfnArgs& p, const Layout& L, int lane) {
    if (Q.nxt.kind != U_PENDING) return;
    int u = 0;
    if (lane == 0) u = (int)atomicAdd(&p.fc->work, 1u);
    Q.nxt = resolve(p, L, __shfl_sync(0xffffffffu, u, 0));
}

// Source token of permuted row r of a slot's expert (routed: perm / k; shared: r - row0).
__device__ __forceinline__ int row_token(const FfnArgs& p, int slot, int row0, int r) {
    return slot < p.S ? r - row0 : __ldcg(p.perm + r) / p.k;
}

// ---- per-warp ring -------------------------------------------------------------------
struct Ring {
    uint8_t* base;
    uint64_t* bar;
    int issued, consumed;
    int iw, ic;                // issue cursor: unit (0 = current, 1 = next) and chunk
};

// Issues the bulk copies of chunk c of unit U into the next stage (whole warp,
// converged; one elected lane issues).
__device__ __forceinline__ void issue_chunk(Ring& R, const CtaState& cs, const FfnArgs& p, const Unit& U, int c,
                                            uint64_t pol) {
    const int st = R.issued % NS;
    const bool dn = U.kind == U_DN;
    const SlotInfo& si = cs.slot[U.slot];
    const int K = dn ? p.I : p.H, G = K / 64, NC = (G + CG - 1) / CG;
    const int ng = min(CG, G - c * CG);
    if (elect_one()) {
        uint8_t* dst = R.base + (size_t)st * STAGE;
        const uint32_t cb = 256 * ng, hb = si.fmt == MOE_FMT_Q3 ? 128 * ng : 0;
        const int b = dn ? 3 : 0;
        mbar_arrive_expect_tx(&R.bar[st], cb + hb + 256);
        bulk_g2s_evict_first(dst, si.base[b] + (size_t)4 * K * U.tile + 2048 * (size_t)c, cb, &R.bar[st], pol);
        bulk_g2s_evict_first(dst + OFF_SC, si.base[b + 2] + (size_t)256 * NC * U.tile + 256 * (size_t)c, 256,
                             &R.bar[st], pol);
        if (hb)
            bulk_g2s_evict_first(dst + OFF_HI, si.base[b + 1] + (size_t)128 * G * U.tile + 1024 * (size_t)c, hb,
                                 &R.bar[st], pol);
    }
    __syncwarp();
    ++R.issued;
}

// Keeps up to NS chunks in flight: the current unit's, then the next unit's (if it is
// known and streams).  The next unit is taken only once the current one has passed its
// waits (allow_next): a warp waiting on a dependency holds one unit, not two.  Stops
// issuing after an abort.
__device__ __forceinline__ void top_up(Ring& R, const CtaState& cs, const Unit& cur, Queue& Q, bool stop,
                                       uint64_t pol, int lane, const FfnArgs& p, const Layout& L,
                                       bool allow_next = true) {
    if (stop) return;
    while (R.issued - R.consumed < NS) {
        if (R.iw == 0) {
            if (streams(cur) && R.ic < unit_nc(cur, L)) {
                issue_chunk(R, cs, p, cur, unit_c0(cur, L) + R.ic++, pol);
                continue;
            }
            if (!allow_next) break;
            R.iw = 1;
            R.ic = 0;
            take_next(Q, p, L, lane);
        }
        if (streams(Q.nxt) && R.ic < unit_nc(Q.nxt, L)) {
            issue_chunk(R, cs, p, Q.nxt, unit_c0(Q.nxt, L) + R.ic++, pol);
            continue;
        }
        break;
    }
}

// Waits for the stage of the next chunk to consume; false if the wait ran out (then
// the abort flag is raised).
__device__ __forceinline__ bool wait_stage(Ring& R, FusedCtl* fc, Ctrl* ctrl, int lane) {
    const int st = R.consumed % NS;
    int ok = 1;
    if (lane == 0 && !mbar_wait_bounded(&R.bar[st], (uint32_t)(R.consumed / NS) & 1, kWaitLimit)) {
        report_error(ctrl, MOE_ERR_TIMEOUT, kDetWaitFull | 0x20);
        atomicExch(&fc->abort, 1u);
        ok = 0;
    }
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// ---- stage readers ---------------------------------------------------------------------
// code word (r, wl) and third-bit word (r, vl) of a stage (swizzled when the chunk is full)
__device__ __forceinline__ int cw_idx(int r, int wl, bool full, int ng) {
    return full ? r * 32 + (wl ^ (4 * (r & 7))) : r * 4 * ng + wl;
}
__device__ __forceinline__ int hw_idx(int r, int vl, bool full, int ng) {
    return full ? r * 16 + (vl ^ (2 * ((r & 7) >> 1))) : r * 2 * ng + vl;
}
__device__ __forceinline__ float scale_of(const uint8_t* stg, int r, int gl) {
    return __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(stg + OFF_SC)[r * 8 + gl]));
}

__device__ __forceinline__ uint32_t f16x2_mul16(uint32_t a) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(0x4C004C00u));
    return r;
}

// The chunk's offset correction, C += sum_gl 16 s[row][gl] * (-Z[col][gl] / 16) as two
// m16n8k8 fp16 MMAs (hi and lo halves of -Z / 16): A = this lane's scale words of rows
// g, g + 8 for groups 2t, 2t + 1 (x 16, exact), B = the halves of column g at groups
// 2t, 2t + 1 (zero pointer: a column without correction).
__device__ __forceinline__ void zcorr(const uint8_t* stg, const uint16_t* zhi, int zplane, int c, int g, int t,
                                      float (&d)[4]) {
    const uint32_t* scw = reinterpret_cast<const uint32_t*>(stg + OFF_SC);
    const uint32_t a0 = f16x2_mul16(scw[4 * g + t]), a1 = f16x2_mul16(scw[4 * (g + 8) + t]);
    const uint32_t bhi = zhi ? *reinterpret_cast<const uint32_t*>(zhi + 8 * c) : 0u;
    const uint32_t blo = zhi ? *reinterpret_cast<const uint32_t*>(zhi + zplane + 8 * c) : 0u;
    mma_f16_1688(d, a0, a1, bhi);
    mma_f16_1688(d, a0, a1, blo);
}

// ---- gate/up on the bf16 path (3-bit) and down on the exact fp16 path ---------------------
// Pass q holds tokens (gate/up) or rows (down) 8q .. 8q + 7 of the expert: B column g is
// 8q + g; lane (g, t) ends with rows g, g + 8 of columns 8q + 2t, 8q + 2t + 1.
template <int NP>
struct BfView {
    uint32_t b[NP];      // B row of column g (+ 16 t elements), elements from x (gate/up) or h (down)
    int z[NP];           // gate/up: -Z/16 (hi plane, 3-bit) of column g, group 2t, in halves
    int orow[NP][2];     // output rows of columns 2t, 2t + 1 (-1: none)
};

template <int MODE, bool Q3, bool FULL, int NP>
__device__ __forceinline__ void chunk_bf(const uint8_t* stg, int c, int ng, const BfView<NP>& v, const uint16_t* bbase,
                                         const uint16_t* zbase, int zplane, int np, const uint32_t (&sub)[5], int g,
                                         int t, float (&acc)[NP][4]) {
    if (MODE == 0) {
#pragma unroll
        for (int q = 0; q < NP; ++q)
            if (q < np) zcorr(stg, zbase + v.z[q], zplane, c, g, t, acc[q]);
    }
    const uint32_t* cw = reinterpret_cast<const uint32_t*>(stg);
    const uint32_t* hw = reinterpret_cast<const uint32_t*>(stg + OFF_HI);
    const int sh = 8 * (t & 1);
#pragma unroll 1
    for (int gl = 0; gl < (FULL ? CG : ng); ++gl) {
        uint32_t pa[8], pb[8], ha[8], hb[8];
        dequant_rows<MODE>(cw[cw_idx(g, 4 * gl + t, FULL, ng)], cw[cw_idx(g + 8, 4 * gl + t, FULL, ng)], sub, pa, pb);
        if (Q3)
            dequant_hi_rows<MODE>(hw[hw_idx(g, 2 * gl + (t >> 1), FULL, ng)] >> sh,
                                  hw[hw_idx(g + 8, 2 * gl + (t >> 1), FULL, ng)] >> sh, ha, hb);
        const float s0 = scale_of(stg, g, gl), s1 = scale_of(stg, g + 8, gl);
        const int grp = c * CG + gl;
#pragma unroll
        for (int q = 0; q < NP; ++q) {
            if (q < np) {
                const uint4* bp = reinterpret_cast<const uint4*>(bbase + v.b[q] + 64 * grp);
                const uint4 x0 = bp[0], x1 = bp[1];
                float d[4];
                mma_group_first<MODE>(d, pa, pb, x0, x1);
                if (Q3) mma_group<MODE>(d, ha, hb, x0, x1);
                acc[q][0] = fmaf(s0, d[0], acc[q][0]);
                acc[q][1] = fmaf(s0, d[1], acc[q][1]);
                acc[q][2] = fmaf(s1, d[2], acc[q][2]);
                acc[q][3] = fmaf(s1, d[3], acc[q][3]);
            }
        }
    }
}

// chunk_bf for a full chunk, with the addressing hoisted as in chunk_iq_full: code word
// of group gl at cw_sw ^ (16 gl) (row g + 8: 1024 bytes on), third-bit word at
// hw_sw ^ (8 gl) (row g + 8: 512 bytes on; hw_sw = 64 g + 8 ((g mod 8) / 2) + 4 (t / 2)),
// the chunk's scales in one 16-byte load per row, the B rows from one pointer per pass.
template <int MODE, bool Q3, int NP>
__device__ __forceinline__ void chunk_bf_full(const uint8_t* stg, int c, const BfView<NP>& v, const uint16_t* bbase,
                                              const uint16_t* zbase, int zplane, int np, const uint32_t (&sub)[5],
                                              int cw_sw, int hw_sw, int g, int t, float (&acc)[NP][4]) {
    if (MODE == 0) {
#pragma unroll
        for (int q = 0; q < NP; ++q)
            if (NP == 1 || q < np) zcorr(stg, zbase + v.z[q], zplane, c, g, t, acc[q]);
    }
    const uint4 sg4 = *reinterpret_cast<const uint4*>(stg + OFF_SC + 16 * g);
    const uint4 su4 = *reinterpret_cast<const uint4*>(stg + OFF_SC + 16 * (g + 8));
    const uint32_t sg[4] = {sg4.x, sg4.y, sg4.z, sg4.w}, su[4] = {su4.x, su4.y, su4.z, su4.w};
    const int sh = 8 * (t & 1);
    const uint4* bp[NP];
#pragma unroll
    for (int q = 0; q < NP; ++q) bp[q] = reinterpret_cast<const uint4*>(bbase + v.b[q] + 64 * CG * c);
#pragma unroll 2
    for (int gl = 0; gl < CG; ++gl) {
        const uint32_t* wp = reinterpret_cast<const uint32_t*>(stg + (cw_sw ^ (16 * gl)));
        uint32_t pa[8], pb[8], ha[8], hb[8];
        dequant_rows<MODE>(wp[0], wp[256], sub, pa, pb);
        if (Q3) {
            const uint32_t* hp = reinterpret_cast<const uint32_t*>(stg + OFF_HI + (hw_sw ^ (8 * gl)));
            dequant_hi_rows<MODE>(hp[0] >> sh, hp[128] >> sh, ha, hb);
        }
        const uint32_t hg = (gl & 1) ? sg[gl >> 1] >> 16 : sg[gl >> 1] & 0xFFFFu;
        const uint32_t hu = (gl & 1) ? su[gl >> 1] >> 16 : su[gl >> 1] & 0xFFFFu;
        const float s0 = __half2float(__ushort_as_half((uint16_t)hg)), s1 = __half2float(__ushort_as_half((uint16_t)hu));
#pragma unroll
        for (int q = 0; q < NP; ++q) {
            if (NP == 1 || q < np) {
                const uint4 x0 = bp[q][8 * gl], x1 = bp[q][8 * gl + 1];
                float d[4];
                mma_group_first<MODE>(d, pa, pb, x0, x1);
                if (Q3) mma_group<MODE>(d, ha, hb, x0, x1);
                acc[q][0] = fmaf(s0, d[0], acc[q][0]);
                acc[q][1] = fmaf(s0, d[1], acc[q][1]);
                acc[q][2] = fmaf(s1, d[2], acc[q][2]);
                acc[q][3] = fmaf(s1, d[3], acc[q][3]);
            }
        }
    }
}

// The next chunk's stage of the current unit (the ring topped up first, into the next
// unit if the current one is all issued), once its copies have landed; nullptr if
// nothing is in flight (after an abort).  A wait that runs out raises stop.
__device__ __forceinline__ const uint8_t* next_stage(Ring& R, const CtaState& cs, const Unit& cur, Queue& Q,
                                                     bool& stop, FusedCtl* fc, Ctrl* ctrl, int lane, uint64_t pol,
                                                     const FfnArgs& p, const Layout& L) {
    top_up(R, cs, cur, Q, stop, pol, lane, p, L);
    if (R.consumed >= R.issued) return nullptr;
    if (!wait_stage(R, fc, ctrl, lane)) stop = true;
    return R.base + (size_t)(R.consumed % NS) * STAGE;
}

// Every lane is done with the stage: it may be refilled.
__device__ __forceinline__ void release_stage(Ring& R) {
    __syncwarp();
    ++R.consumed;
}

// Where a unit's fp32 results go: a split shared gate/up tile's {gate, up} sums of K part
// U.part (gsh, rows of the shared experts only), and a down tile's rows of y_e for K part
// U.part (ypart [part][T (k + S)][H]).
__device__ __forceinline__ float2* gsh_at(const FfnArgs& p, int part, int orow, int hcol) {
    return reinterpret_cast<float2*>(p.gsh) + ((size_t)part * p.fk.gsh_rows + (orow - p.fk.gsh_row0)) * p.I + hcol;
}
__device__ __forceinline__ float* ypart_at(const FfnArgs& p, const Unit& U, int orow, int col) {
    return p.ypart + ((size_t)U.part * p.T * (p.k + p.S) + orow) * p.H + col;
}

// A tile of a ternary or 2-bit expert on the integer path, with NP passes of 4 rows.
// MODE 0 (gate/up): B = the tokens' digit records, output h = silu(gate) * up in fp32
// (hf, quantised later for the down pass); MODE 1 (down): B = the expert's h rows'
// digit records, output fp32 rows of y_e (ypart).
template <int MODE, int NP, bool STG = false>
__device__ __forceinline__ void unit_iq(const FfnArgs& p, const Layout& L, const CtaState& cs, const Unit& cur,
                                        Queue& Q, Ring& R, bool& stop, bool ready, const IqBase& B, int G, int G8,
                                        FusedCtl* fc, uint64_t pol, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const int cnt = cs.slot[cur.slot].cnt, row0 = cs.slot[cur.slot].row0;
    const int np = (cnt + 3) / 4;
    IqView<NP> v;
#pragma unroll
    for (int q = 0; q < NP; ++q) {
        const int ib = 4 * q + (g >> 1), it = 4 * q + t;
        const int rb = row0 + (ib < cnt ? ib : 0), rt = row0 + (it < cnt ? it : 0);
        const int tb = MODE == 0 ? row_token(p, cur.slot, row0, rb) : rb;   // record row: token, or h row
        const int tk = MODE == 0 ? row_token(p, cur.slot, row0, rt) : rt;
        v.bq[q] = (uint32_t)(((size_t)tb * G * 2 + (g & 1)) * 4 + t);
        v.pq[q] = (uint32_t)((size_t)tk * G8);
        v.orow[q] = it < cnt ? row0 + it : -1;
    }
    const int o4 = cs.slot[cur.slot].fmt == MOE_FMT_TERNARY ? 4 : 6;
    const int K = MODE == 0 ? p.H : p.I, GK = K / 64;
    const int sw = 128 * g + 16 * (g & 7) + 4 * t;       // this lane's word of group 0, swizzled
    unsigned long long acc[NP];
#pragma unroll
    for (int q = 0; q < NP; ++q) acc[q] = 0ull;
    const int c0 = unit_c0(cur, L), c1 = c0 + unit_nc(cur, L);
    for (int c = c0; c < c1; ++c) {
        const uint8_t* stg = next_stage(R, cs, cur, Q, stop, fc, p.ctrl, lane, pol, p, L);
        if (!stg) break;
        const int ng = min(CG, GK - c * CG);
        if (ready && !stop) {
            if (ng == CG) chunk_iq_full<NP, STG>(stg, c, v, B, np, o4, sw, g, acc);
            else chunk_gu_iq<NP, false>(stg, c, ng, v, B, np, o4, g, t, acc);
        }
        release_stage(R);
    }
    if (MODE == 0) {
        // h = silu(gate) * up in fp32 for the down pass's quantisation; a value outside
        // the fp16 range is reported (the range the layer is defined for)
        bool range_ok = true;
        if (ready && !stop) {
            const int hcol = cur.tile * 8 + g;
            const bool split = gu_split(cur, L);
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                if (q < np && v.orow[q] >= 0) {
                    const float2 a = up2(acc[q]);
                    if (split) {
                        *gsh_at(p, cur.part, v.orow[q], hcol) = a;
                    } else {
                        const float hv = silu_f(a.x) * a.y;
                        range_ok &= in_f16_range(hv);
                        p.hf[(size_t)v.orow[q] * p.I + hcol] = hv;
                    }
                }
            }
        }
        if (!__all_sync(0xffffffffu, range_ok) && lane == 0)
            report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetRange | 0x20);
    } else if (ready && !stop) {
        // rows 16 tile + g and 16 tile + g + 8 of y_e for token 4q + t, fp32
#pragma unroll
        for (int q = 0; q < NP; ++q) {
            if (q < np && v.orow[q] >= 0) {
                const float2 a = up2(acc[q]);
                float* dst = ypart_at(p, cur, v.orow[q], cur.tile * 16 + g);
                dst[0] = a.x;
                dst[8] = a.y;
            }
        }
    }
}

// The down pass's integer operands of expert slot `cur.slot`: groups gq = tile,
// tile + td, ... of every h row of the expert (its cnt tokens), each on its own 12-bit
// grid (iq_group).  Groups past I (padding to whole chunks) get a zero pair.
__device__ __forceinline__ void quantise_h_share(const FfnArgs& p, const CtaState& cs, const Unit& cur, int td,
                                                 int lane) {
    const int GI = p.I / 64, GI8 = 8 * ((GI + 7) / 8);
    const int cnt = cs.slot[cur.slot].cnt, row0 = cs.slot[cur.slot].row0;
    float2* pairs = reinterpret_cast<float2*>(p.hq + iq_pair_off(p.R16, p.I));
    for (int gq = cur.tile; gq < GI8; gq += td) {
        for (int r = 0; r < cnt; ++r) {
            const int row = row0 + r;
            if (gq >= GI) {
                if (lane == 0) pairs[(size_t)row * GI8 + gq] = make_float2(0.f, 0.f);
                continue;
            }
            const float2 hv = *reinterpret_cast<const float2*>(p.hf + (size_t)row * p.I + gq * 64 + 2 * lane);
            iq_group(hv.x, hv.y, lane, p.hq + ((size_t)row * GI + gq) * 128, pairs + (size_t)row * GI8 + gq);
        }
    }
}

// A gate/up tile of a 3-bit expert (MODE 0: bf16 path, B = tokens) or a down tile of any
// expert (MODE 1: exact fp16 path, B = h), with NP passes of 8 columns.
template <int MODE, bool Q3, int NP>
__device__ __forceinline__ void unit_bf(const FfnArgs& p, const Layout& L, const CtaState& cs, const Unit& cur,
                                        Queue& Q, Ring& R, bool& stop, bool ready, const uint16_t* zq3,
                                        int zplane_q3, int G8, FusedCtl* fc, uint64_t pol, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const int cnt = cs.slot[cur.slot].cnt, row0 = cs.slot[cur.slot].row0, fmt = cs.slot[cur.slot].fmt;
    const int np = (cnt + 7) / 8;
    const int K = MODE == 0 ? p.H : p.I, GK = K / 64;
    BfView<NP> v;
#pragma unroll
    for (int q = 0; q < NP; ++q) {
        const int ib = 8 * q + g;
        const int rb = row0 + (ib < cnt ? ib : 0);
        if (MODE == 0) {
            const int tb = row_token(p, cur.slot, row0, rb);
            v.b[q] = (uint32_t)((size_t)tb * p.H + 16 * t);
            v.z[q] = (int)((size_t)tb * G8 + 2 * t);
        } else {
            v.b[q] = (uint32_t)((size_t)rb * p.I + 16 * t);
            v.z[q] = 0;
        }
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int col = 8 * q + 2 * t + cc;
            v.orow[q][cc] = col < cnt ? row0 + col : -1;
        }
    }
    uint32_t sub[5] = {0, 0, 0, 0, 0};
    if (MODE == 1) {
        const float o = fmt == MOE_FMT_TERNARY ? 1.f : (fmt == MOE_FMT_Q2 ? 1.5f : 3.5f);
        sub[0] = f16x2_bits_of(512.f + o);
        sub[1] = f16x2_bits_of(256.f + o);
        sub[2] = f16x2_bits_of(64.f + o);
        sub[3] = f16x2_bits_of(16.f + o);
        sub[4] = f16x2_bits_of(4.f + o);
    }
    const uint16_t* bbase = MODE == 0 ? p.x : p.h;
    const int cw_sw = 128 * g + 16 * (g & 7) + 4 * t;                 // swizzled word offsets of group 0
    const int hw_sw = 64 * g + 8 * ((g & 7) >> 1) + 4 * (t >> 1);
    float acc[NP][4];
#pragma unroll
    for (int q = 0; q < NP; ++q) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0.f;
    const int c0 = unit_c0(cur, L), c1 = c0 + unit_nc(cur, L);
    for (int c = c0; c < c1; ++c) {
        const uint8_t* stg = next_stage(R, cs, cur, Q, stop, fc, p.ctrl, lane, pol, p, L);
        if (!stg) break;
        const int ng = min(CG, GK - c * CG);
        if (ready && !stop) {
            if (ng == CG)
                chunk_bf_full<MODE, Q3, NP>(stg, c, v, bbase, zq3, zplane_q3, np, sub, cw_sw, hw_sw, g, t, acc);
            else chunk_bf<MODE, Q3, false, NP>(stg, c, ng, v, bbase, zq3, zplane_q3, np, sub, g, t, acc);
        }
        release_stage(R);
    }
    if (!ready || stop) return;
    if (MODE == 0) {
        bool range_ok = true;
        const int hcol = cur.tile * 8 + g;
        const bool split = gu_split(cur, L);
#pragma unroll
        for (int q = 0; q < NP; ++q)
#pragma unroll
            for (int cc = 0; cc < 2; ++cc)
                if (q < np && v.orow[q][cc] >= 0) {
                    if (split) {
                        *gsh_at(p, cur.part, v.orow[q][cc], hcol) = make_float2(acc[q][cc], acc[q][2 + cc]);
                    } else {
                        const float hv = silu_f(acc[q][cc]) * acc[q][2 + cc];
                        range_ok &= in_f16_range(hv);
                        p.h[(size_t)v.orow[q][cc] * p.I + hcol] = f32_to_f16_bits(hv);
                    }
                }
        if (!__all_sync(0xffffffffu, range_ok) && lane == 0)
            report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetRange | 0x20);
    } else {
        // rows 16 tile + g and 16 tile + g + 8 of y_e for this lane's columns, fp32
#pragma unroll
        for (int q = 0; q < NP; ++q)
#pragma unroll
            for (int cc = 0; cc < 2; ++cc)
                if (q < np && v.orow[q][cc] >= 0) {
                    float* dst = ypart_at(p, cur, v.orow[q][cc], cur.tile * 16 + g);
                    dst[0] = acc[q][cc];
                    dst[8] = acc[q][2 + cc];
                }
    }
}

// The last K part of a split gate/up tile: h = silu(gate) * up of its 8 columns for
// the expert's rows, from the parts' sums added in part order; fp16 h for a 3-bit
// expert (the bf16 path's down operand), fp32 hf for the integer path.
__device__ __forceinline__ void finish_gu(const FfnArgs& p, const Layout& L, const CtaState& cs, const Unit& cur,
                                          int lane) {
    const int cnt = cs.slot[cur.slot].cnt, row0 = cs.slot[cur.slot].row0;
    const bool q3 = cs.slot[cur.slot].fmt == MOE_FMT_Q3;
    const size_t part_stride = (size_t)p.fk.gsh_rows * p.I;
    const int parts = gu_parts(cur, L);
    bool range_ok = true;
    for (int i = lane; i < cnt * 8; i += 32) {
        const int orow = row0 + (i >> 3), hcol = cur.tile * 8 + (i & 7);
        const float2* src = gsh_at(p, 0, orow, hcol);
        float gs = 0.f, us = 0.f;
        for (int part = 0; part < parts; ++part) {
            const float2 v = __ldcg(src + part * part_stride);
            gs += v.x;
            us += v.y;
        }
        const float hv = silu_f(gs) * us;
        range_ok &= in_f16_range(hv);
        if (q3) p.h[(size_t)orow * p.I + hcol] = f32_to_f16_bits(hv);
        else p.hf[(size_t)orow * p.I + hcol] = hv;
    }
    if (!__all_sync(0xffffffffu, range_ok) && lane == 0) report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetRange | 0x20);
}

// y[t][16 tile + r] for every token t and r < 16: the routed rows weighted by their gates
// in slot order, then the shared rows, summed in fp32 and stored as bf16.  A row's value
// is the sum of its pd K parts, in part order.  The loads of an output go out in two
// rounds: the row indices and gates of eight slots (and the shared rows' values), then
// those slots' values.
__device__ __forceinline__ float ypart_row(const FfnArgs& p, int row, int col, int pd, size_t part_stride) {
    const float* src = p.ypart + (size_t)row * p.H + col;
    float v = __ldcg(src);
    for (int part = 1; part < pd; ++part) v += __ldcg(src + part * part_stride);
    return v;
}

__device__ __forceinline__ void combine_slice(const FfnArgs& p, int tile, int pd, int lane) {
    const size_t part_stride = (size_t)p.T * (p.k + p.S) * p.H;
    for (int i = lane; i < p.T * 16; i += 32) {
        const int tok = i >> 4, col = tile * 16 + (i & 15);
        const float ysh = p.S ? ypart_row(p, p.T * p.k + tok, col, pd, part_stride) : 0.f;   // S <= 1
        float y = 0.f;
        for (int r0 = 0; r0 < p.k; r0 += 8) {
            int row[8];
            float gw[8], v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const bool on = r0 + u < p.k;
                row[u] = on ? __ldcg(p.inv_perm + (size_t)tok * p.k + r0 + u) : -1;
                gw[u] = on ? __ldcg(p.topk_w + (size_t)tok * p.k + r0 + u) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = row[u] >= 0 ? ypart_row(p, row[u], col, pd, part_stride) : 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (r0 + u < p.k) y = fmaf(gw[u], v[u], y);
        }
        y += ysh;
        if (p.y_f32) reinterpret_cast<float*>(p.y)[(size_t)tok * p.H + col] = y;
        else p.y[(size_t)tok * p.H + col] = f32_to_bf16_bits(y);
    }
}

// ---- the kernel ---------------------------------------------------------------------
__global__ void __launch_bounds__(NW * 32, 1) ffn_fused_kernel(const __grid_constant__ FfnArgs p) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t stall_bar;
    __shared__ CtaState cs;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    FusedCtl* fc = p.fc;
    Ctrl* ctrl = p.ctrl;
    // No griddepcontrol.launch_dependents here: a following forward on the same
    // workspace must not start before this launch has reset the counters it shares.

    Ring R;
    R.base = smem + (size_t)warp * NS * STAGE;
    R.bar = reinterpret_cast<uint64_t*>(smem + (size_t)NW * NS * STAGE) + warp * NS;
    R.issued = R.consumed = 0;
    R.iw = 0;
    R.ic = 0;
    if (lane == 0)
        for (int s = 0; s < NS; ++s) mbar_init(&R.bar[s], 1);
    __shared__ int hdr_ok;
    if (threadIdx.x == 0) {
        mbar_init(&stall_bar, 1);                               // nothing ever arrives on it
        cs.routed = 0;
        // every CTA checks the packed buffer's header before it reads the expert table
        const uint32_t* hd = reinterpret_cast<const uint32_t*>(p.packed);
        hdr_ok = hd[0] == kMagic && hd[1] == kVersion && (int)hd[2] == p.H && (int)hd[3] == p.I &&
                 (int)hd[4] == p.E && (int)hd[5] == p.S && hd[6] == 64u && hd[7] == (uint32_t)kInterleave;
        if (!hdr_ok) {
            report_error(ctrl, MOE_ERR_DEVICE_CHECK, kDetHeader);
            atomicExch(&fc->abort, 1u);
        }
    }
    __syncthreads();
    if (hdr_ok && warp == 0 && lane < p.S)                      // the shared experts' slots
        fill_slot(cs.slot[lane], p, p.E + lane, p.T, p.T * p.k + lane * p.T);
    fence_mbar_init();
    __syncthreads();

    // failure-path tests: one warp per CTA waits on a barrier nothing completes; the
    // wait runs out and the launch takes its abort path
    if (warp == 0 && ctrl->test_stall) {
        int done = 0;
        if (lane == 0) done = mbar_wait_bounded(&stall_bar, 0, ctrl->test_stall);
        if (!__shfl_sync(0xffffffffu, done, 0) && lane == 0) {
            report_error(ctrl, MOE_ERR_TIMEOUT, kDetTestStall | 0x20);
            atomicExch(&fc->abort, 1u);
        }
        __syncwarp();
    }

    const int G = p.H / 64, G8 = 8 * ((G + 7) / 8);
    Layout L;
    L.tg = 2 * p.I / 16;
    L.td = p.H / 16;
    L.nch = (p.H / 64 + CG - 1) / CG;
    L.nci = (p.I / 64 + CG - 1) / CG;
    L.S = p.S;
    // K parts (no empty part: the part count is re-derived from the chunks per part)
    L.cpg = (L.nch + max(1, p.fk.pg) - 1) / max(1, p.fk.pg);
    L.pg = (L.nch + L.cpg - 1) / L.cpg;
    L.cpr = (L.nch + max(1, p.fk.pr) - 1) / max(1, p.fk.pr);
    L.pr = (L.nch + L.cpr - 1) / L.cpr;
    L.cpd = (L.nci + max(1, p.fk.pd) - 1) / max(1, p.fk.pd);
    L.pd = (L.nci + L.cpd - 1) / L.cpd;
    L.nsgu = p.S * L.tg * L.pg;
    const int zplane_q3 = 3 * p.T * G8;          // hi -> lo plane of the Z tables (elements)
    const uint16_t* zq3 = reinterpret_cast<const uint16_t*>(p.zx) + (size_t)2 * p.T * G8;   // format 2 plane
    IqBase IB;                                    // the tokens' integer operands (gate/up)
    IB.bq = reinterpret_cast<const uint4*>(p.iq);
    IB.pq = reinterpret_cast<const float2*>(p.iq + iq_pair_off(p.T, p.H));
    const int GI = p.I / 64, GI8 = 8 * ((GI + 7) / 8);
    L.shares = min(L.td, GI8);
    IqBase HB;                                    // the h rows' integer operands (down)
    HB.bq = reinterpret_cast<const uint4*>(p.hq);
    HB.pq = reinterpret_cast<const float2*>(p.hq + iq_pair_off(p.R16, p.I));
    const uint64_t pol = l2_policy_evict_first();

    // The routing and the token operands (Z tables, integer records) come from the
    // router launch this one follows: wait for it, then every unit is known.
    bool stop = !hdr_ok;
    {
        int tok = 0;
        const int nr = read_routing(cs, p, lane, &tok);
        stop = stop || nr < 0 || ld_relaxed(&fc->abort) != 0;
        L.nr = nr < 0 ? 0 : nr;
        L.t_ok = tok != 0;
        L.total = L.nsgu + L.nr * L.tg * L.pr + (p.S + L.nr) * L.td * L.pd;
    }
    const bool staged = p.T <= kStageMaxT;
    IqBase IBs = IB;
    if (staged) {                                 // every warp of the CTA is here
        uint4* dst = reinterpret_cast<uint4*>(smem + kFusedSmem);
        const uint4* src = reinterpret_cast<const uint4*>(p.iq);
        const int n16 = (int)(iq_size(p.T, p.H) / 16);
        for (int i = threadIdx.x; i < n16; i += blockDim.x) dst[i] = __ldcg(src + i);
        IBs.bq = dst;
        IBs.pq = reinterpret_cast<const float2*>(smem + kFusedSmem + iq_pair_off(p.T, p.H));
        __syncthreads();
    }
    Queue Q;
    Q.nxt.kind = U_PENDING;
    take_next(Q, p, L, lane);
    Unit cur = Q.nxt;
    Q.nxt.kind = U_PENDING;
    int iters = 0;
    while (true) {
        if (cur.kind == U_NONE) break;            // the queue is empty
        if (++iters > L.total + 2) {              // cannot happen with consistent counters
            if (lane == 0) {
                report_error(ctrl, MOE_ERR_DEVICE_CHECK, kDetLoopCap | 0x20);
                atomicExch(&fc->abort, 1u);
            }
            break;
        }
        stop = stop || ld_relaxed(&fc->abort) != 0;
        top_up(R, cs, cur, Q, stop, pol, lane, p, L, false);
        {
            // ---------------- a gate/up or down tile ----------------------------------
            const bool dn = cur.kind == U_DN;
            const int cnt = cs.slot[cur.slot].cnt;
            const bool q3 = cs.slot[cur.slot].fmt == MOE_FMT_Q3;
            bool ready = !stop;
            if (ready && dn) ready = wait_counter(&fc->gu_done[cur.slot], (uint32_t)L.tg, fc, ctrl, kDetWaitFull | 0x22, lane);
            if (dn && !q3) {
                // integer down pass: h of this expert on a 12-bit grid per 64-group, formed
                // by K part 0 of the expert's first down tiles (a share each), waited for by all
                if (cur.tile < L.shares && cur.part == 0) {
                    if (ready) quantise_h_share(p, cs, cur, L.td, lane);
                    post_counter(&fc->hq_done[cur.slot], lane);
                }
                if (ready)
                    ready = wait_counter(&fc->hq_done[cur.slot], (uint32_t)L.shares, fc, ctrl, kDetWaitFull | 0x23, lane);
            }
            if (!dn && !q3) {
                if (staged) unit_iq<0, 1, true>(p, L, cs, cur, Q, R, stop, ready, IBs, G, G8, fc, pol, lane);
                else if (cnt <= 4) unit_iq<0, 1>(p, L, cs, cur, Q, R, stop, ready, IB, G, G8, fc, pol, lane);
                else if (cnt <= 8) unit_iq<0, 2>(p, L, cs, cur, Q, R, stop, ready, IB, G, G8, fc, pol, lane);
                else unit_iq<0, 4>(p, L, cs, cur, Q, R, stop, ready, IB, G, G8, fc, pol, lane);
            } else if (dn && !q3) {
                if (cnt <= 4) unit_iq<1, 1>(p, L, cs, cur, Q, R, stop, ready, HB, GI, GI8, fc, pol, lane);
                else if (cnt <= 8) unit_iq<1, 2>(p, L, cs, cur, Q, R, stop, ready, HB, GI, GI8, fc, pol, lane);
                else unit_iq<1, 4>(p, L, cs, cur, Q, R, stop, ready, HB, GI, GI8, fc, pol, lane);
            } else if (!dn) {
                if (cnt <= 8) unit_bf<0, true, 1>(p, L, cs, cur, Q, R, stop, ready, zq3, zplane_q3, G8, fc, pol, lane);
                else unit_bf<0, true, 2>(p, L, cs, cur, Q, R, stop, ready, zq3, zplane_q3, G8, fc, pol, lane);
            } else {
                if (cnt <= 8) unit_bf<1, true, 1>(p, L, cs, cur, Q, R, stop, ready, zq3, 0, G8, fc, pol, lane);
                else unit_bf<1, true, 2>(p, L, cs, cur, Q, R, stop, ready, zq3, 0, G8, fc, pol, lane);
            }
            stop = stop || !ready;
            if (!dn && gu_split(cur, L)) {
                // the last K part of a gate/up tile forms its h
                uint32_t* ctr = &p.gp_done[cur.slot * L.tg + cur.tile];
                if (signal_counter(ctr, lane) == (uint32_t)gu_parts(cur, L) - 1) {
                    (void)ld_acquire(ctr);
                    if (!stop) finish_gu(p, L, cs, cur, lane);
                    post_counter(&fc->gu_done[cur.slot], lane);
                }
            } else if (!dn) {
                post_counter(&fc->gu_done[cur.slot], lane);
            } else {
                const uint32_t n_parts = (uint32_t)((L.nr + p.S) * L.pd);
                const uint32_t old = signal_counter(&p.dn_done[cur.tile], lane);
                if (old == n_parts - 1 && !stop && L.t_ok) {
                    // the last expert part of this 16-row slice: combine it (fixed order)
                    (void)ld_acquire(&p.dn_done[cur.tile]);
                    combine_slice(p, cur.tile, L.pd, lane);
                }
            }
        }
        // next unit: the issue cursor moves from "next" to "current"
        if (R.iw == 1) R.iw = 0;
        else R.ic = 0;
        take_next(Q, p, L, lane);
        cur = Q.nxt;
        Q.nxt.kind = U_PENDING;
    }

    // copies still in flight (only after an abort): wait for them, bounded
    if (lane == 0)
        for (int qd = R.consumed; qd < R.issued; ++qd)
            if (!mbar_wait_bounded(&R.bar[qd % NS], (uint32_t)(qd / NS) & 1, kWaitLimit)) {
                report_error(ctrl, MOE_ERR_TIMEOUT, kDetDrain | 0x20);
                break;
            }
    __syncwarp();
    // the last warp of the launch resets the counters for the next one
    const uint32_t n_warps = gridDim.x * NW;
    if (signal_counter(&fc->warps_done, lane) == n_warps - 1) {
        (void)ld_acquire(&fc->warps_done);
        for (int i = lane; i < kMaxSlots; i += 32) {
            fc->gu_done[i] = 0;
            fc->hq_done[i] = 0;
        }
        for (int i = lane; i < p.H / 16; i += 32) p.dn_done[i] = 0;
        const int n_ctr = (L.pr > 1 ? p.S + L.nr : p.S) * L.tg;
        for (int i = lane; i < n_ctr; i += 32) p.gp_done[i] = 0;
        __syncwarp();
        if (lane == 0) {
            fc->work = 0;
            fc->abort = 0;
            __threadfence();
            fc->warps_done = 0;
        }
    }
}

}  // namespace

cudaError_t launch_ffn_fused(const FfnArgs& a, cudaStream_t s) {
    if (a.T < 1 || a.T > kFusedMaxT || a.E + a.S > kMaxSlots) return cudaErrorInvalidConfiguration;
    const size_t smem = fused_smem_bytes(a.T, a.H);
    const cudaError_t err = set_smem_limit(ffn_fused_kernel, smem);
    if (err != cudaSuccess) return err;
    return launch_pdl(ffn_fused_kernel, dim3(a.num_ctas), dim3(NW * 32), smem, s, a);
}

}  // namespace moe
