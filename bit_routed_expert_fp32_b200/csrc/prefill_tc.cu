// Prefill path (routed and shared experts): grouped GEMMs over the packed experts on the
// 5th-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// With thousands of tokens each selected expert meets hundreds of tokens, so its
// FFN is a dense contraction and belongs on the tensor cores.  The engine on the
// pages sweeps a long prompt in batches of 6-9K tokens (shadowgraph.io README,
// paragraph under the model table); here one call takes all T tokens.
//
// Orientation ("swap-AB"): D[M = 128 weight rows][N <= 192 tokens] = W_tile x X^T.
// Weights are the A operand, so every tile has a full M of 128 whatever the token
// count, and a tile's N is the expert's token count rounded up to 16 (experts with
// more than 192 tokens are split evenly into several N-tiles).
//
// The dequantised A tile lives in tensor memory, not shared memory: shared memory then
// carries only the B tiles and the packed weights, which halves its traffic per stage
// (with A in shared memory the tile was written and read back every stage).
//
//  * Dequantisation producers (warps 0-7; warp w owns TMEM lane quarter w % 4, i.e.
//    tile rows 32q .. 32q+31 one per lane, and K half w / 4 of every 64-wide stage).
//    Lane 0 of each warp brings its two 16-row packed blocks in by bulk copies, one
//    512-wide K chunk per slot of a two-slot ring of its own (eight issuing threads
//    keep enough bytes in flight).  A lane reads its row's code words (plus third bits
//    and the fp16 scale) from the ring, turns them into fp16 (c - o) * s (exact codes,
//    one rounding) and stores the 16 pairs with one tcgen05.st into the stage's A
//    columns; tcgen05.wait::st + fence, one arrive per warp.
//  * TMA producer (warp 12): one 2-D tensor-map load per stage for the B tile (K-major,
//    SWIZZLE_128B) from the gathered fp16 token rows (gate/up) or from h (down),
//    completion counted in bytes on the stage's mbarrier.
//  * MMA issuer (warp 13, one elected lane): per stage four tcgen05.mma.kind::f16
//    (K = 16 each) with A from tensor memory and B from shared memory, fp32
//    accumulation in TMEM; tcgen05.commit releases the stage to the producers and,
//    after the last stage, hands the accumulator to the epilogue (gate/up: two
//    accumulators of 192 columns alternate between tiles, so the epilogue of one tile
//    overlaps the main loop of the next; down: one of 256 columns, see TcCfg).
//  * Epilogue (warps 8-11, TMEM lanes 32q..32q+31): tcgen05.ld 16 columns at a time.
//    gate/up: rows 16b..16b+7 are gate rows and 16b+8..16b+15 the matching up rows,
//    i.e. TMEM lanes l and l+8 of the same warp: h = silu(gate) * up is formed with
//    one shuffle and stored as fp16.  down: fp32 partial rows per (token, slot) for
//    the deterministic combine kernel.
// Every wait is bounded (an error is recorded and the kernel carries on), and TMEM is
// released on every exit path.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kernels.h"

namespace moe {
namespace {

constexpr int BM = 128;                       // weight rows per tile (UMMA M)
constexpr int BK = 64;                        // K per stage (one scale group)
constexpr int kDqWarps = 8, kEpiWarp0 = 8, kTmaWarp = 12, kMmaWarp = 13;   // warps 8-11: epilogue
constexpr int kPkwBytes = 2 * 3328;          // a dequantiser warp's packed ring (below)
// Per pass: the token tile (UMMA N, at most BN tokens; an expert with more tokens is split
// into equal N tiles), the fp32 accumulators in tensor memory that the tiles use in
// turn, and the pipeline stages.  Gate/up keeps two accumulators of 192 columns, so the
// epilogue of one tile overlaps the main loop of the next.  Down has a quarter of the
// gate/up FLOPs per weight byte, so the weight re-reads of a second N tile cost it more
// than its epilogue: one accumulator of 256 columns (an expert of up to 256 tokens is one
// tile) and three stages, the same shared memory in all.
template <int MODE>
struct TcCfg {
    static constexpr int BN = MODE == 0 ? 192 : 256;
    static constexpr int NACC = MODE == 0 ? 2 : 1;
    static constexpr int NSTG = MODE == 0 ? 4 : 3;
    static constexpr int STG_BYTES = BN * BK * 2;          // a stage's shared memory is its B tile
    // Tensor memory (512 columns x 128 lanes x 32 bit): NACC fp32 accumulators of BN
    // columns, then NSTG A stages of 32 columns (128 rows x 64 fp16, two per column).
    static constexpr uint32_t kACol0 = NACC * BN;
    static constexpr size_t SMEM = (size_t)NSTG * STG_BYTES + (size_t)kDqWarps * 2 * kPkwBytes + 4 * 512 + 1024;
};
static_assert(TcCfg<0>::kACol0 + 32 * TcCfg<0>::NSTG <= 512 && TcCfg<1>::kACol0 + 32 * TcCfg<1>::NSTG <= 512,
              "TMEM columns");
static_assert(TcCfg<0>::BN % 16 == 0 && TcCfg<1>::BN % 16 == 0 && TcCfg<1>::BN <= 256, "UMMA N");
// Per-warp packed ring: each dequantiser warp streams the two 16-row blocks of its TMEM
// lane quarter, one 8-group chunk (codes, third bits, scales of the packed format) of
// both per slot.
constexpr int NP = 2;
constexpr int PK_CODES = 0, PK_HI = 2048, PK_SC = 3072, PK_BYTES = 3328, PKW_BYTES = 2 * PK_BYTES;
static_assert(PKW_BYTES == kPkwBytes, "packed ring size");
constexpr int kThreads = 448;                 // 14 warps

// B tiles: one tensor-map load per stage, from the map whose box (64, 128 or 256 token
// rows) is the smallest that covers the tile's tokens.  A single thread issues bulk
// loads at a limited rate, so one large box beats several small ones.
struct BMaps {
    CUtensorMap m[3];   // box rows 64, 128, BN of the pass
};
__device__ inline int box_index(int n) { return n <= 64 ? 0 : (n <= 128 ? 1 : 2); }
__host__ __device__ constexpr int box_rows(int i, int bn) { return i == 0 ? 64 : (i == 1 ? 128 : bn); }
constexpr long long kWaitLimit = 4000000000LL;

constexpr uint32_t kH512 = 0x60006000u, kH256 = 0x5C005C00u, kH64 = 0x54005400u, kH16 = 0x4C004C00u,
                   kH4 = 0x44004400u, kH4096 = 0x6C006C00u, kH2048 = 0x68006800u, kH1024 = 0x64006400u,
                   kH128 = 0x58005800u, kH32 = 0x50005000u;

// fp16 pairs (c - o), exact (bases 512, 256, 64, 16, 4 have an ulp <= 1/2).
__device__ inline void codes_f16(uint32_t w, const uint32_t (&sub)[5], uint32_t (&pr)[8]) {
    const uint32_t w1 = w << 1, w8 = w >> 8;
    pr[0] = f16x2_sub(lop3_and_or(w1, 0x00060006u, kH512), sub[0]);
    pr[1] = f16x2_sub(lop3_and_or(w, 0x000C000Cu, kH256), sub[1]);
    pr[2] = f16x2_sub(lop3_and_or(w, 0x00300030u, kH64), sub[2]);
    pr[3] = f16x2_sub(lop3_and_or(w, 0x00C000C0u, kH16), sub[3]);
    pr[4] = f16x2_sub(lop3_and_or(w, 0x03000300u, kH4), sub[4]);
    pr[5] = f16x2_sub(lop3_and_or(w8, 0x000C000Cu, kH256), sub[1]);
    pr[6] = f16x2_sub(lop3_and_or(w8, 0x00300030u, kH64), sub[2]);
    pr[7] = f16x2_sub(lop3_and_or(w8, 0x00C000C0u, kH16), sub[3]);
}

// fp16 pairs 4 * (third bit), exact, for bits 0..7 of each half of u.
__device__ inline void hi_f16(uint32_t u, uint32_t (&pr)[8]) {
    pr[0] = f16x2_sub(lop3_and_or(u, 0x00010001u, kH4096), kH4096);
    pr[1] = f16x2_sub(lop3_and_or(u, 0x00020002u, kH2048), kH2048);
    pr[2] = f16x2_sub(lop3_and_or(u, 0x00040004u, kH1024), kH1024);
    pr[3] = f16x2_sub(lop3_and_or(u, 0x00080008u, kH512), kH512);
    pr[4] = f16x2_sub(lop3_and_or(u, 0x00100010u, kH256), kH256);
    pr[5] = f16x2_sub(lop3_and_or(u, 0x00200020u, kH128), kH128);
    pr[6] = f16x2_sub(lop3_and_or(u, 0x00400040u, kH64), kH64);
    pr[7] = f16x2_sub(lop3_and_or(u, 0x00800080u, kH32), kH32);
}

// silu(a) = a / (1 + e^-a) with the fast exponential and division (relative error
// ~1e-6, far below the fp16 rounding of h); for a -> -inf the quotient goes to 0.
__device__ inline float silu_fast(float a) { return __fdividef(a, 1.0f + __expf(-a)); }

__device__ inline uint32_t f16x2_add(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ inline uint32_t f16x2_mul(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// ---- tcgen05 / TMA wrappers ---------------------------------------------------------
__device__ inline void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ inline void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ inline void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ inline void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// SWIZZLE_128B K-major shared-memory matrix descriptor: 8-row groups 1024 bytes apart.
__device__ inline uint64_t smem_desc(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// kind::f16 instruction descriptor: fp16 A and B (K-major), fp32 D, M = 128, N.
__device__ inline uint32_t instr_desc(int n) {
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

// D[M = 128][N] (+)= A[M][K = 16] B[N][K]^T with A read from tensor memory (128 lanes =
// rows, 8 columns = 16 fp16 along K) and B from shared memory (descriptor).
__device__ inline void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(acc)
        : "memory");
}

// Each thread writes 16 consecutive 32-bit columns of its own TMEM lane.
__device__ inline void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ inline void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ inline void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ inline void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ inline void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}


__device__ inline const PackedEntry* entry(const uint8_t* packed, int e) {
    return reinterpret_cast<const PackedEntry*>(packed + kHeaderBytes + (size_t)e * kEntryBytes);
}

struct TcSched {
    int ok, n_active, n_tiles, abort_flag;
    uint32_t tmem;
    uint32_t stall;  // failure-path tests: cycles of the MMA issuer's wait on stall_bar (0 = off)
    int pad[2];
    int e[260];
    int fmt[260];
    int cnt[260];
    int nt[260];     // N-tiles per active expert
    int nb[260];     // tokens per N-tile (multiple of 16, <= 256)
    int tpre[261];   // tile prefix over active experts
};

struct TileInfo {
    int a, e, f, mt, n0, N, row0;   // N: tokens in this tile; row0: first permuted row
};

__device__ inline int ld_volatile(const int& v) { return *reinterpret_cast<const volatile int*>(&v); }
__device__ inline void st_volatile(int& v, int x) { *reinterpret_cast<volatile int*>(&v) = x; }

__device__ inline TileInfo tile_info(const TcSched& S, const FfnArgs& p, int tile, int mtiles) {
    int lo = 0, hi = S.n_active - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (S.tpre[mid] <= tile) lo = mid;
        else hi = mid - 1;
    }
    TileInfo ti;
    ti.a = lo;
    ti.e = S.e[lo];
    ti.f = S.fmt[lo];
    const int r = tile - S.tpre[lo];
    const int ntile = r / mtiles;
    ti.mt = r - ntile * mtiles;
    ti.n0 = ntile * S.nb[lo];
    ti.N = min(S.nb[lo], S.cnt[lo] - ti.n0);
    ti.row0 = (ti.e < p.E ? p.offsets[ti.e] : p.T * p.k + (ti.e - p.E) * p.T) + ti.n0;
    return ti;
}

__device__ bool wait_or_flag(TcSched& S, uint64_t* bar, uint32_t parity, const FfnArgs& p, uint32_t detail) {
    if (ld_volatile(S.abort_flag)) return false;
    if (mbar_wait_bounded_suspend(bar, parity, kWaitLimit)) return true;
    st_volatile(S.abort_flag, 1);
    report_error(p.ctrl, MOE_ERR_TIMEOUT, detail);
    return false;
}

template <int MODE>   // 0: gate/up (B = gathered tokens, K = H); 1: down (B = h, K = I)
__global__ void __launch_bounds__(kThreads, 1) tc_gemm_kernel(FfnArgs p, const __grid_constant__ BMaps bmaps) {
    constexpr int BN = TcCfg<MODE>::BN, NACC = TcCfg<MODE>::NACC, NSTG = TcCfg<MODE>::NSTG;
    constexpr int STG_BYTES = TcCfg<MODE>::STG_BYTES;
    constexpr uint32_t kACol0 = TcCfg<MODE>::kACol0;
    extern __shared__ uint8_t smem_raw[];
    __shared__ TcSched S;
    __shared__ __align__(8) uint64_t full_a[NSTG], full_b[NSTG], empty_[NSTG], acc_full[NACC], acc_empty[NACC], mma_done,
        pk_full[kDqWarps][NP], stall_bar;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int K = MODE == 0 ? p.H : p.I;
    const int M_total = MODE == 0 ? 2 * p.I : p.H;
    const int mtiles = M_total / BM;
    const int KS = K / BK;                 // K stages per tile
    const int G = K / 64, NC = (G + 7) / 8;

    // launched with programmatic serialization: the launch overlaps the predecessor's
    // tail; nothing is read before the predecessor has finished
    griddep_launch_dependents();        // one CTA per SM: every CTA of this grid is resident
    griddep_wait();
    if (threadIdx.x == 0) {
        const uint32_t* hd = reinterpret_cast<const uint32_t*>(p.packed);
        const bool hdr_ok = hd[0] == kMagic && hd[1] == kVersion && (int)hd[2] == p.H && (int)hd[3] == p.I &&
                            (int)hd[4] == p.E && (int)hd[5] == p.S && hd[6] == 64u &&
                            hd[7] == (uint32_t)kInterleave;
        // the schedule in the workspace must be the one routed for these T tokens
        const bool t_ok = p.ctrl->routed_T == p.T;
        S.ok = hdr_ok && t_ok;
        S.abort_flag = 0;
        if (!hdr_ok) report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetHeader);
        else if (!t_ok) report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetRoutedT | 0x10 | MODE);
        S.n_active = p.ctrl->n_active;
        S.stall = p.ctrl->test_stall;
    }
    __syncthreads();
    if (!S.ok) return;
    const int nA = S.n_active;
    for (int a = threadIdx.x; a < nA; a += blockDim.x) {
        const int e = p.active[a];
        const int c = e < p.E ? p.counts[e] : p.T;
        const int nt = (c + BN - 1) / BN;
        int nb = (c + nt - 1) / nt;
        nb = (nb + 15) & ~15;
        S.e[a] = e;
        S.fmt[a] = (int)entry(p.packed, e)->fmt;
        S.cnt[a] = c;
        S.nt[a] = nt;
        S.nb[a] = nb;
        if (S.fmt[a] > MOE_FMT_Q3) {            // a storage form (dense ternary): not read here
            if (blockIdx.x == 0) report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetFormat | 0x10 | MODE);
            S.ok = 0;
        }
    }
    __syncthreads();
    if (!S.ok) return;
    if (threadIdx.x == 0) {
        int run = 0;
        for (int a = 0; a < nA; ++a) {
            S.tpre[a] = run;
            run += S.nt[a] * mtiles;
        }
        S.tpre[nA] = run;
        S.n_tiles = run;
        for (int i = 0; i < NSTG; ++i) {
            mbar_init(&full_a[i], kDqWarps);                 // one arrive per dequantiser warp
            mbar_init(&full_b[i], 1);
            mbar_init(&empty_[i], 1);
        }
        for (int w = 0; w < kDqWarps; ++w)
            for (int i = 0; i < NP; ++i) mbar_init(&pk_full[w][i], 1);
        for (int i = 0; i < NACC; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 4 * 32);
        }
        mbar_init(&mma_done, 1);
        mbar_init(&stall_bar, 1);                       // nothing ever arrives on it
        fence_mbar_init();
    }
    if (warp == kMmaWarp) tmem_alloc(&S.tmem, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem;
    const int n_tiles = S.n_tiles;

    if (warp < kDqWarps) {
        // ======================= dequantisation producers (A) =======================
        // Warp w writes TMEM lane quarter q = w % 4 (tile rows 32q .. 32q+31, one per
        // lane) and K half kh = w / 4 of every stage (columns 16 kh .. 16 kh + 15 of the
        // stage's 32); a lane's row is row r16 of packed block 2q + blk.
        const int q = warp & 3, kh = warp >> 2;
        const int blk = lane >> 4, r16 = lane & 15, rs = r16 & 7;
        uint8_t* const ring = smem + (size_t)NSTG * STG_BYTES + (size_t)warp * NP * PKW_BYTES;
        uint64_t* const pfull = pk_full[warp];
        const uint32_t a_lane = tmem + ((uint32_t)(32 * q) << 16) + kACol0 + 16 * kh;
        // Issue cursor: the next (tile, chunk) of this warp's two blocks to bring in.
        struct Cursor {
            int tile, c;
            const uint8_t *cb, *hb, *sb;
            bool q3;
        } cur{n_tiles, 0, nullptr, nullptr, nullptr, false};
        auto load_tile = [&](Cursor& u) {
            if (u.tile >= n_tiles) return;
            const TileInfo ti = tile_info(S, p, u.tile, mtiles);
            const PackedEntry* en = entry(p.packed, ti.e);
            const int j = ti.mt * (BM / 16) + 2 * q;
            u.cb = p.packed + (MODE == 0 ? en->gu_codes : en->dn_codes) + (size_t)4 * K * j;
            u.hb = p.packed + (MODE == 0 ? en->gu_hi : en->dn_hi) + (size_t)128 * G * j;
            u.sb = p.packed + (MODE == 0 ? en->gu_scales : en->dn_scales) + (size_t)256 * NC * j;
            u.q3 = ti.f == MOE_FMT_Q3;
        };
        int issued = 0, consumed = 0;
        // (whole warp, converged) bring the cursor's chunk of both blocks into slot
        // issued % NP and advance the cursor; one elected lane issues the copies
        auto issue = [&]() {
            if (cur.tile >= n_tiles) return;
            const int ps = issued % NP;
            const int ng = min(8, G - 8 * cur.c);
            const uint32_t cbytes = 256 * ng, hbytes = cur.q3 ? 128 * ng : 0;
            uint8_t* dst = ring + (size_t)ps * PKW_BYTES;
            if (elect_one()) {
                mbar_arrive_expect_tx(&pfull[ps], 2 * (cbytes + hbytes + 256));
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    uint8_t* d = dst + b * PK_BYTES;
                    bulk_g2s(d + PK_CODES, cur.cb + (size_t)4 * K * b + 2048 * (size_t)cur.c, cbytes, &pfull[ps]);
                    bulk_g2s(d + PK_SC, cur.sb + (size_t)256 * NC * b + 256 * (size_t)cur.c, 256, &pfull[ps]);
                    if (hbytes)
                        bulk_g2s(d + PK_HI, cur.hb + (size_t)128 * G * b + 1024 * (size_t)cur.c, hbytes, &pfull[ps]);
                }
            }
            __syncwarp();
            ++issued;
            if (++cur.c == NC) {
                cur.c = 0;
                cur.tile += gridDim.x;
                load_tile(cur);
            }
        };
        cur.tile = blockIdx.x;
        cur.c = 0;
        load_tile(cur);
        for (int d = 0; d < NP; ++d) issue();
        int slot = 0;
        uint32_t eph = 1;                              // parity of the empty phase awaited
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
            const TileInfo ti = tile_info(S, p, tile, mtiles);
            const bool q3 = ti.f == MOE_FMT_Q3;
            const float o = ti.f == MOE_FMT_TERNARY ? 1.f : (ti.f == MOE_FMT_Q2 ? 1.5f : 3.5f);
            uint32_t sub[5];
            sub[0] = f16x2_bits_of(512.f + o);
            sub[1] = f16x2_bits_of(256.f + o);
            sub[2] = f16x2_bits_of(64.f + o);
            sub[3] = f16x2_bits_of(16.f + o);
            sub[4] = f16x2_bits_of(4.f + o);
            for (int c = 0; c < NC; ++c) {
                const int ps = consumed % NP;
                const int ng = min(8, G - 8 * c);
                if (lane == 0 && !mbar_try_wait(&pfull[ps], (consumed / NP) & 1))
                    wait_or_flag(S, &pfull[ps], (consumed / NP) & 1, p, kDetWaitFull | 0x40 | MODE);
                __syncwarp();
                const uint8_t* pk = ring + (size_t)ps * PKW_BYTES + blk * PK_BYTES;
                // this lane's 2 code words, third-bit word and the row's scales of the chunk
                const uint8_t* cw_base = pk + PK_CODES + (ng == 8 ? r16 * 128 : r16 * 16 * ng) + 8 * kh;
                const uint8_t* hw_base = pk + PK_HI + (ng == 8 ? r16 * 64 : r16 * 8 * ng) + 4 * kh;
                const uint16_t* sc_base = reinterpret_cast<const uint16_t*>(pk + PK_SC + r16 * 16);
                auto load = [&](int gl, uint2& cw, uint32_t& hw, uint32_t& s2) {
                    const int cpos = ng == 8 ? gl ^ rs : gl;
                    const int hpos = ng == 8 ? gl ^ (rs >> 1) : gl;
                    cw = *reinterpret_cast<const uint2*>(cw_base + 16 * cpos);
                    hw = q3 ? *reinterpret_cast<const uint32_t*>(hw_base + 8 * hpos) : 0u;
                    s2 = (uint32_t)sc_base[gl] * 0x10001u;
                };
                uint2 cw;
                uint32_t hw, s2;
                load(0, cw, hw, s2);
                for (int gl = 0; gl < ng; ++gl) {
                    // the next group's words are read while this one is converted
                    uint2 cw_n = cw;
                    uint32_t hw_n = hw, s2_n = s2;
                    if (gl + 1 < ng) load(gl + 1, cw_n, hw_n, s2_n);
                    // fp16 (c - o) * s of K elements 32 kh .. 32 kh + 31 of this group, as
                    // 16 pairs in K order (quarter qq of the half -> columns 8 qq .. 8 qq + 7)
                    uint32_t r[16];
                    const uint32_t words[2] = {cw.x, cw.y};
#pragma unroll
                    for (int qq = 0; qq < 2; ++qq) {
                        uint32_t pr[8];
                        codes_f16(words[qq], sub, pr);
                        if (q3) {
                            uint32_t hp[8];
                            hi_f16(hw >> (8 * qq), hp);
#pragma unroll
                            for (int v = 0; v < 8; ++v) pr[v] = f16x2_add(pr[v], hp[v]);
                        }
#pragma unroll
                        for (int v = 0; v < 8; ++v) r[8 * qq + v] = f16x2_mul(pr[v], s2);
                    }
                    // only now wait for the stage's slot
                    if (lane == 0 && !mbar_try_wait(&empty_[slot], eph))
                        wait_or_flag(S, &empty_[slot], eph, p, kDetWaitEmpty | 0x10 | MODE);
                    __syncwarp();
                    tmem_st16(a_lane + 32 * slot, r);
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&full_a[slot]);
                    if (++slot == NSTG) {
                        slot = 0;
                        eph ^= 1;
                    }
                    cw = cw_n;
                    hw = hw_n;
                    s2 = s2_n;
                }
                // every lane has read the slot: refill it with the chunk NP ahead
                __syncwarp();
                ++consumed;
                if (!ld_volatile(S.abort_flag)) issue();
            }
        }
        // after an abort, no bulk copy may still target shared memory at exit: wait
        // (bounded) for the most recent phase issued on each slot
        if (lane == 0 && ld_volatile(S.abort_flag))
            for (int d = 0; d < NP && d < issued; ++d) {
                const int q2 = issued - 1 - d;
                if (!mbar_wait_bounded(&pfull[q2 % NP], (q2 / NP) & 1, kWaitLimit)) {
                    report_error(p.ctrl, MOE_ERR_TIMEOUT, kDetDrain | 0x50 | MODE);
                    break;
                }
            }
    } else if (warp == kTmaWarp) {
        // ============================ TMA producer (B) ===============================
        // whole warp, converged; one elected lane issues
        int it = 0, issued = 0, slot = 0;
        uint32_t eph = 1;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
            const TileInfo ti = tile_info(S, p, tile, mtiles);
            const int bx = box_index(ti.N);
            const uint32_t bbytes = (uint32_t)box_rows(bx, BN) * BK * 2;
            for (int ks = 0; ks < KS; ++ks, ++it) {
                if (!mbar_try_wait(&empty_[slot], eph))
                    wait_or_flag(S, &empty_[slot], eph, p, kDetWaitEmpty | 0x20 | MODE);
                __syncwarp();
                if (!ld_volatile(S.abort_flag)) {
                    if (elect_one()) {
                        mbar_arrive_expect_tx(&full_b[slot], bbytes);
                        tma_load_2d(smem + (size_t)slot * STG_BYTES, &bmaps.m[bx], ks * BK, ti.row0, &full_b[slot]);
                    }
                    __syncwarp();
                    issued = it + 1;
                }
                if (++slot == NSTG) {
                    slot = 0;
                    eph ^= 1;
                }
            }
        }
        // no TMA write may still target shared memory at exit (matters only after an
        // abort: normally the MMA issuer has consumed every stage)
        if (lane == 0 && ld_volatile(S.abort_flag))
            for (int d = 0; d < NSTG && d < issued; ++d) {
                const int q2 = issued - 1 - d;
                if (!mbar_wait_bounded(&full_b[q2 % NSTG], (q2 / NSTG) & 1, kWaitLimit)) {
                    report_error(p.ctrl, MOE_ERR_TIMEOUT, kDetDrain | MODE);
                    break;
                }
            }
    } else if (warp == kMmaWarp) {
        // ============================== MMA issuer ===================================
        // The whole warp runs the loop (its control flow and the descriptors stay
        // warp-uniform) and one elected lane issues tcgen05.mma / commit.  The per-stage
        // path is short, since it bounds the stage rate: slot and phase advance
        // incrementally, descriptors are precomputed, and the bounded wait is entered
        // only when the barrier is not already complete.
        const uint64_t b_desc0 = smem_desc(smem_u32(smem));
        constexpr uint32_t kSlotStep = STG_BYTES >> 4;
        int slot = 0, tc = 0;
        uint32_t phase = 0;
        bool ok = true;
        if (S.stall) {
            // failure-path tests: a bounded wait on a barrier that nothing completes; it
            // runs out and the CTA takes the give-up path below (as for any wait)
            bool done = false;
            if (lane == 0) done = mbar_wait_bounded(&stall_bar, 0, S.stall);
            if (!__shfl_sync(0xffffffffu, done, 0)) {
                if (lane == 0) {
                    st_volatile(S.abort_flag, 1);
                    report_error(p.ctrl, MOE_ERR_TIMEOUT, kDetTestStall | 0x10 | MODE);
                }
                ok = false;
            }
            __syncwarp();
        }
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tc) {
            const TileInfo ti = tile_info(S, p, tile, mtiles);
            const int buf = tc % NACC;
            const uint32_t acc_par = (uint32_t)(tc / NACC) & 1;
            const int n16 = (ti.N + 15) & ~15;
            const uint32_t idesc = instr_desc(n16);
            if (!mbar_try_wait(&acc_empty[buf], acc_par ^ 1))
                ok &= wait_or_flag(S, &acc_empty[buf], acc_par ^ 1, p, kDetWaitEmpty | 0x30 | MODE);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            const uint32_t d_tmem = tmem + buf * BN;
            for (int ks = 0; ks < KS; ++ks) {
                if (!mbar_try_wait(&full_a[slot], phase))
                    ok &= wait_or_flag(S, &full_a[slot], phase, p, kDetWaitFull | 0x10 | MODE);
                if (!mbar_try_wait(&full_b[slot], phase))
                    ok &= wait_or_flag(S, &full_b[slot], phase, p, kDetWaitFull | 0x20 | MODE);
                ok = __all_sync(0xffffffffu, ok);
                tc_fence_after();                       // A was written by tcgen05.st of other warps
                const uint32_t a_tm = tmem + kACol0 + 32 * slot;
                const uint64_t bd = b_desc0 + (uint64_t)(slot * kSlotStep);
                if (elect_one()) {
                    if (ok) {
#pragma unroll
                        for (int k16 = 0; k16 < BK / 16; ++k16)
                            umma_f16_ts(d_tmem, a_tm + 8 * k16, bd + 2 * k16, idesc, (ks | k16) != 0 ? 1u : 0u);
                    }
                    umma_commit(&empty_[slot]);
                }
                __syncwarp();
                if (++slot == NSTG) {
                    slot = 0;
                    phase ^= 1;
                }
            }
            if (elect_one()) umma_commit(&acc_full[buf]);
            __syncwarp();
        }
        // every MMA this warp issued has completed once this commit arrives
        if (elect_one()) umma_commit(&mma_done);
        __syncwarp();
        if (lane == 0 && !mbar_wait_bounded(&mma_done, 0, kWaitLimit)) report_error(p.ctrl, MOE_ERR_TIMEOUT, kDetDrain | 0x40);
    } else if (warp >= kEpiWarp0) {
        // =============================== epilogue ====================================
        const int q = warp & 3;                       // TMEM lanes 32q .. 32q+31 (warps 8-11)
        uint16_t* const stg = reinterpret_cast<uint16_t*>(smem + (size_t)NSTG * STG_BYTES +
                                                           (size_t)kDqWarps * NP * PKW_BYTES) + q * 256;
        int tc = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tc) {
            const TileInfo ti = tile_info(S, p, tile, mtiles);
            const int buf = tc % NACC;
            const uint32_t acc_par = (uint32_t)(tc / NACC) & 1;
            // a long wait (a whole tile's main loop): poll slowly to leave the issue slots
            // to the dequantisers on this sub-partition
            if (!mbar_try_wait(&acc_full[buf], acc_par) && !ld_volatile(S.abort_flag) &&
                !mbar_wait_bounded_backoff(&acc_full[buf], acc_par, kWaitLimit, 256)) {
                st_volatile(S.abort_flag, 1);
                report_error(p.ctrl, MOE_ERR_TIMEOUT, kDetWaitFull | 0x30 | MODE);
            }
            tc_fence_after();
            const uint32_t tbase = tmem + buf * BN + ((uint32_t)(32 * q) << 16);
            const int mrow = ti.mt * BM + 32 * q + lane;    // row of the packed matrix
            const int hcol0 = (ti.mt * BM + 32 * q) / 2;         // first h column of this warp (gate/up)
            for (int c0 = 0; c0 < ti.N; c0 += 16) {
                uint32_t v[16];
                tmem_ld16(tbase + c0, v);
                if (MODE == 0) {
                    // lanes l < 8 and 16 <= l < 24 hold gate rows, l + 8 the matching up
                    // rows: h for 16 tokens x this warp's 16 h columns, transposed through
                    // shared memory into one 16-byte store per lane
                    const bool gate_lane = (lane & 15) < 8;
                    const int lc = ((lane >> 4) << 3) | (lane & 7);    // h column within the warp
                    bool range_ok = true;
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        const float a = __uint_as_float(v[u]);
                        const float b = __shfl_down_sync(0xffffffffu, a, 8);
                        const float hv = silu_fast(a) * b;
                        range_ok &= !gate_lane || c0 + u >= ti.N || in_f16_range(hv);
                        if (gate_lane) stg[u * 16 + lc] = f32_to_f16_bits(hv);
                    }
                    // h outside the fp16 range: reported, not carried on (see moe_forward)
                    if (!__all_sync(0xffffffffu, range_ok) && lane == 0)
                        report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetRange | 0x10);
                    __syncwarp();
                    const int u = lane >> 1, half = lane & 1;
                    if (c0 + u < ti.N)
                        *reinterpret_cast<uint4*>(p.h + (size_t)(ti.row0 + c0 + u) * p.I + hcol0 + 8 * half) =
                            *reinterpret_cast<const uint4*>(stg + u * 16 + 8 * half);
                    __syncwarp();
                } else {
#pragma unroll
                    for (int u = 0; u < 16; ++u)
                        if (c0 + u < ti.N) p.ypart[(size_t)(ti.row0 + c0 + u) * p.H + mrow] = __uint_as_float(v[u]);
                }
            }
            tc_fence_before();
            mbar_arrive(&acc_empty[buf]);
        }
    }
    // all roles are done (waits are bounded): make sure no MMA is still writing, then
    // release the tensor memory
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

// X16[r][:] = fp16(x[token of permuted row r][:]); rows T*k .. are the shared expert's.
// One block per row, threads over 8-element column chunks.
__global__ void __launch_bounds__(256) gather_x16_kernel(FfnArgs p, uint16_t* x16) {
    griddep_wait();                     // perm comes from the router
    if (p.ctrl->routed_T != p.T) return;   // another T was routed: perm may point past x (reported by the GEMM)
    const int r = blockIdx.x;
    const int tk = p.T * p.k;
    const int tok = r < tk ? __ldg(p.perm + r) / p.k : (r - tk) % p.T;
    const uint4* src = reinterpret_cast<const uint4*>(p.x + (size_t)tok * p.H);
    uint4* dst = reinterpret_cast<uint4*>(x16 + (size_t)r * p.H);
    for (int c = threadIdx.x; c < p.H / 8; c += blockDim.x) {
        const uint4 v = __ldg(src + c);
        const uint32_t in[4] = {v.x, v.y, v.z, v.w};
        uint32_t out[4];
        bool ok = true;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float lo = __uint_as_float(in[u] << 16), hi = __uint_as_float(in[u] & 0xFFFF0000u);
            ok &= in_f16_range(lo) && in_f16_range(hi);
            out[u] = (uint32_t)f32_to_f16_bits(lo) | ((uint32_t)f32_to_f16_bits(hi) << 16);
        }
        // a token outside the fp16 range is reported, not carried on (see moe_forward)
        if (!ok) report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetRange | 1);
        dst[c] = make_uint4(out[0], out[1], out[2], out[3]);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

// 2-D fp16 tensor map over rows x K (K-major), boxes of 64 K x box_rows, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, long long rows, int K, int box_rows) {
    auto enc = get_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {BK, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_maps(BMaps* b, const void* base, long long rows, int K, int bn) {
    return make_map(&b->m[0], base, rows, K, box_rows(0, bn)) && make_map(&b->m[1], base, rows, K, box_rows(1, bn)) &&
           make_map(&b->m[2], base, rows, K, box_rows(2, bn));
}

template <int MODE>
cudaError_t launch_tc(const FfnArgs& a, const BMaps& maps, cudaStream_t s) {
    constexpr size_t smem = TcCfg<MODE>::SMEM;
    const cudaError_t err = set_smem_limit(tc_gemm_kernel<MODE>, smem);
    if (err != cudaSuccess) return err;
    return launch_pdl(tc_gemm_kernel<MODE>, dim3(a.num_ctas), dim3(kThreads), smem, s, a, maps);
}

}  // namespace

cudaError_t launch_ffn_prefill(const FfnArgs& a, uint16_t* x16, cudaStream_t s, cudaEvent_t ev_gateup,
                               cudaEvent_t ev_down) {
    if ((2 * a.I) % BM != 0 || a.H % BM != 0) return cudaErrorInvalidConfiguration;
    const long long rows = (long long)a.T * (a.k + a.S);
    if (rows > 2147483647LL) return cudaErrorInvalidConfiguration;
    cudaError_t err = launch_pdl(gather_x16_kernel, dim3((unsigned)rows), dim3(256), 0, s, a, x16);
    if (err != cudaSuccess) return err;
    BMaps mx, mh;
    if (!make_maps(&mx, x16, rows, a.H, TcCfg<0>::BN) || !make_maps(&mh, a.h, rows, a.I, TcCfg<1>::BN))
        return cudaErrorInvalidConfiguration;
    err = launch_tc<0>(a, mx, s);
    if (err != cudaSuccess) return err;
    if (ev_gateup && (err = record_event(ev_gateup, s)) != cudaSuccess) return err;
    err = launch_tc<1>(a, mh, s);
    if (err != cudaSuccess) return err;
    if (ev_down && (err = record_event(ev_down, s)) != cudaSuccess) return err;
    return launch_combine(a, s);
}

}  // namespace moe
