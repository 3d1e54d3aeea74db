// Expert FFN kernels of the decode path (steps a4, a5, a8 and the combine):
// grouped skinny GEMMs over the packed ternary / 2-bit / 3-bit experts.
//
// Decode speed is set by the expert bytes moved per token (ossradar.top, Xolotl
// README, "Fast mode (DeepSeek-V4.1)"), and each selected expert is read once for
// all of its tokens (the same README, "Latest", the CPU kernels that decode an
// expert once for its 4-8 tokens).  So the kernels stream every selected expert's
// packed bytes exactly once through shared memory and apply them to all of its
// tokens:
//
//  * Work unit = (active expert, 16-row tile of the packed matrix).  A persistent
//    grid of one CTA per SM takes a contiguous range of units whose cumulative
//    packed bytes (times the number of 64-token passes) is an equal share.
//  * One producer warp stages each unit with 1-D bulk copies (cp.async.bulk, TMA
//    engine) into a ring of shared-memory stages, completion on mbarriers.  Code
//    rows land at a padded stride so the fragment reads below are conflict-free.
//  * Eight consumer warps split K.  Each 32-bit code word (16 codes of one row) is
//    turned into bf16 pairs (c - o) with shift / lop3 / bf16x2-subtract (magic-number
//    exponent trick, exact), fed to mma.sync m16n8k16 as the A operand with the
//    tokens as N (8 per n-tile); B fragments come straight from the token rows.
//    Each 64-wide group is accumulated from zero and folded into fp32 with its fp16
//    scale.  3-bit experts add a second MMA for 4 * (third bit).
//  * gate/up: rows are interleaved 8 gate / 8 up, so one tile yields 8 outputs of
//    h = silu(gate) * up for each token, kept in fp16 (the down projection then runs
//    fp16 MMAs with an fp16 dequantiser: the tokens are bf16, h is not).
//  * down: each unit writes its partial rows (fp32) for each (token, slot); the
//    last CTA to finish a 16-row output tile (atomic ticket over all active experts)
//    sums the tile in fixed slot order with the gates, adds the shared expert and
//    writes y (bf16).  Deterministic and free of floating-point atomics.
// Every wait is bounded; a wait that runs out records an error in the workspace and
// the kernel carries on without waiting, so it always terminates.
#include "kernels.h"

namespace moe {
namespace {

constexpr int kCWarps = 8;                       // consumer warps
constexpr int kThreads = (kCWarps + 1) * 32;     // + 1 producer warp
constexpr int kMaxTok = 64;                      // tokens per pass
constexpr long long kWaitLimit = 4000000000LL;   // clock cycles (~2 s) before giving up

// bf16 magic bases used by the gate/up dequantiser (exponent-only patterns, mantissa 0)
constexpr uint32_t kMag64 = 0x42804280u, kMag32 = 0x42004200u, kMag16 = 0x41804180u, kMag8 = 0x41004100u,
                   kMag4 = 0x40804080u, kMag512 = 0x44004400u, kMag256 = 0x43804380u, kMag128 = 0x43004300u;
// fp16 magic bases used by the down dequantiser
constexpr uint32_t kH512 = 0x60006000u, kH256 = 0x5C005C00u, kH64 = 0x54005400u, kH16 = 0x4C004C00u,
                   kH4 = 0x44004400u, kH4096 = 0x6C006C00u, kH2048 = 0x68006800u, kH1024 = 0x64006400u,
                   kH128 = 0x58005800u, kH32 = 0x50005000u;

struct Geom {
    int K, G, rs0, rs1, off_hi, off_sc, bytes;
};

__host__ __device__ inline Geom make_geom(int K) {
    Geom g;
    g.K = K;
    g.G = K / 64;
    g.rs0 = K / 16 + ((g.G % 2 == 0) ? 4 : 0);       // words; rs0 = 4 (mod 8) -> no bank conflicts
    const int w1 = hi_words(K);
    g.rs1 = w1 + ((w1 % 8 == 0) ? 4 : 0);
    g.off_hi = 16 * g.rs0 * 4;
    g.off_sc = g.off_hi + 16 * g.rs1 * 4;
    g.bytes = g.off_sc + 16 * g.G * 2;
    g.bytes = (g.bytes + 127) & ~127;
    return g;
}

__host__ __device__ inline long long unit_bytes(int fmt, int K) {
    return 16LL * (K / 4 + K / 32 + (fmt == MOE_FMT_Q3 ? hi_words(K) * 4 : 0));
}

// Shared-memory bookkeeping placed at the start of the dynamic buffer.
struct Sched {
    int n_active;
    int start_a, start_j, end_a, end_j;
    int abort_flag;
    int last_flag;
    int pad;
    int e[260];
    int fmt[260];
    int cnt[260];
    long long w[260];     // cost of one unit of active expert a
    long long pre[261];   // cost prefix over active experts
    int tok[kMaxTok];     // B-operand row of each token of the current pass
    int hrow[kMaxTok];    // output row of each token of the current pass
};

__device__ inline int ld_volatile(const int& v) { return *reinterpret_cast<const volatile int*>(&v); }
__device__ inline void st_volatile(int& v, int x) { *reinterpret_cast<volatile int*>(&v) = x; }

__device__ inline const PackedEntry* entry(const uint8_t* packed, int e) {
    return reinterpret_cast<const PackedEntry*>(packed + kHeaderBytes + (size_t)e * kEntryBytes);
}

// First unit (a, j) whose doubled cost midpoint times G reaches 2 * c * total.
__device__ void first_unit(const Sched& s, int tiles, long long total, int G, int c, int* oa, int* oj) {
    const long long target = 2LL * c * total;
    for (int a = 0; a < s.n_active; ++a) {
        const long long w = s.w[a], P = s.pre[a];
        if ((2 * P + (2LL * tiles - 1) * w) * G < target) continue;
        long long num = target - (2 * P + w) * G;
        long long j = num <= 0 ? 0 : (num + 2 * w * G - 1) / (2 * w * G);
        *oa = a;
        *oj = (int)j;
        return;
    }
    *oa = s.n_active;
    *oj = 0;
}

__device__ inline void dequant_codes(uint32_t w, const uint32_t (&sub)[5], uint32_t (&pr)[8]) {
    const uint32_t w1 = w << 1, w3 = w >> 3, w9 = w >> 9;
    pr[0] = bf16x2_sub(lop3_and_or(w1, 0x00060006u, kMag64), sub[0]);   // pair 0, bits 0-1 -> 1-2
    pr[1] = bf16x2_sub(lop3_and_or(w, 0x000C000Cu, kMag32), sub[1]);    // pair 1, bits 2-3
    pr[2] = bf16x2_sub(lop3_and_or(w, 0x00300030u, kMag8), sub[2]);     // pair 2, bits 4-5
    pr[3] = bf16x2_sub(lop3_and_or(w3, 0x00180018u, kMag16), sub[3]);   // pair 3, bits 6-7 -> 3-4
    pr[4] = bf16x2_sub(lop3_and_or(w3, 0x00600060u, kMag4), sub[4]);    // pair 4, bits 8-9 -> 5-6
    pr[5] = bf16x2_sub(lop3_and_or(w9, 0x00060006u, kMag64), sub[0]);   // pair 5, bits 10-11 -> 1-2
    pr[6] = bf16x2_sub(lop3_and_or(w9, 0x00180018u, kMag16), sub[3]);   // pair 6, bits 12-13 -> 3-4
    pr[7] = bf16x2_sub(lop3_and_or(w9, 0x00600060u, kMag4), sub[4]);    // pair 7, bits 14-15 -> 5-6
}

// 4 * (third code bit) for the 8 pairs of one thread (bits 0..7 of each half of u).
__device__ inline void dequant_hi(uint32_t u, uint32_t (&pr)[8]) {
    const uint32_t u1 = u >> 1;
    pr[0] = bf16x2_sub(lop3_and_or(u, 0x00010001u, kMag512), kMag512);
    pr[1] = bf16x2_sub(lop3_and_or(u, 0x00020002u, kMag256), kMag256);
    pr[2] = bf16x2_sub(lop3_and_or(u, 0x00040004u, kMag128), kMag128);
    pr[3] = bf16x2_sub(lop3_and_or(u, 0x00080008u, kMag64), kMag64);
    pr[4] = bf16x2_sub(lop3_and_or(u, 0x00100010u, kMag32), kMag32);
    pr[5] = bf16x2_sub(lop3_and_or(u, 0x00200020u, kMag16), kMag16);
    pr[6] = bf16x2_sub(lop3_and_or(u, 0x00400040u, kMag8), kMag8);
    pr[7] = bf16x2_sub(lop3_and_or(u1, 0x00400040u, kMag8), kMag8);
}

// binary16 variant: pairs land at mantissa bits 1-2 (base 512), 2-3 (256), 4-5 (64),
// 6-7 (16), 8-9 (4); base + o stays exactly representable because every base has a
// unit in the last place of at most 1/2.
__device__ inline void dequant_codes_f16(uint32_t w, const uint32_t (&sub)[5], uint32_t (&pr)[8]) {
    const uint32_t w1 = w << 1, w8 = w >> 8;
    pr[0] = f16x2_sub(lop3_and_or(w1, 0x00060006u, kH512), sub[0]);    // pair 0, bits 0-1 -> 1-2
    pr[1] = f16x2_sub(lop3_and_or(w, 0x000C000Cu, kH256), sub[1]);     // pair 1, bits 2-3
    pr[2] = f16x2_sub(lop3_and_or(w, 0x00300030u, kH64), sub[2]);      // pair 2, bits 4-5
    pr[3] = f16x2_sub(lop3_and_or(w, 0x00C000C0u, kH16), sub[3]);      // pair 3, bits 6-7
    pr[4] = f16x2_sub(lop3_and_or(w, 0x03000300u, kH4), sub[4]);       // pair 4, bits 8-9
    pr[5] = f16x2_sub(lop3_and_or(w8, 0x000C000Cu, kH256), sub[1]);    // pair 5, bits 10-11 -> 2-3
    pr[6] = f16x2_sub(lop3_and_or(w8, 0x00300030u, kH64), sub[2]);     // pair 6, bits 12-13 -> 4-5
    pr[7] = f16x2_sub(lop3_and_or(w8, 0x00C000C0u, kH16), sub[3]);     // pair 7, bits 14-15 -> 6-7
}

__device__ inline void dequant_hi_f16(uint32_t u, uint32_t (&pr)[8]) {
    pr[0] = f16x2_sub(lop3_and_or(u, 0x00010001u, kH4096), kH4096);
    pr[1] = f16x2_sub(lop3_and_or(u, 0x00020002u, kH2048), kH2048);
    pr[2] = f16x2_sub(lop3_and_or(u, 0x00040004u, kH1024), kH1024);
    pr[3] = f16x2_sub(lop3_and_or(u, 0x00080008u, kH512), kH512);
    pr[4] = f16x2_sub(lop3_and_or(u, 0x00100010u, kH256), kH256);
    pr[5] = f16x2_sub(lop3_and_or(u, 0x00200020u, kH128), kH128);
    pr[6] = f16x2_sub(lop3_and_or(u, 0x00400040u, kH64), kH64);
    pr[7] = f16x2_sub(lop3_and_or(u, 0x00800080u, kH32), kH32);
}

__device__ inline float half_bits_to_f32(uint16_t h) { return __half2float(__ushort_as_half(h)); }

template <int MODE>  // 0: gate/up + SwiGLU -> h ; 1: down -> partial rows + combine -> y
__global__ void __launch_bounds__(kThreads, 1) ffn_mma_kernel(FfnArgs p, int nstage, int tokblk) {
    extern __shared__ __align__(1024) uint8_t smem[];
    Sched& S = *reinterpret_cast<Sched*>(smem);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + sizeof(Sched));
    uint64_t* empty = full + nstage;
    const int red_stride = tokblk + 4;
    float* red = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(empty + nstage));
    const size_t red_bytes = (size_t)kCWarps * 16 * red_stride * 4;
    uint8_t* stages = smem + ((sizeof(Sched) + 16 * nstage + red_bytes + 1023) & ~size_t(1023));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int K = MODE == 0 ? p.H : p.I;
    const int tiles = MODE == 0 ? (2 * p.I) / 16 : p.H / 16;
    const Geom geo = make_geom(K);

    // ---- header check and per-CTA schedule ---------------------------------------
    if (tid == 0) {
        const uint32_t* hd = reinterpret_cast<const uint32_t*>(p.packed);
        bool ok = hd[0] == kMagic && hd[1] == 1u && (int)hd[2] == p.H && (int)hd[3] == p.I &&
                  (int)hd[4] == p.E && (int)hd[5] == p.S && hd[6] == 64u && hd[7] == (uint32_t)kInterleave;
        S.abort_flag = ok ? 0 : 1;
        if (!ok) report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetHeader);
        S.n_active = p.ctrl->n_active;
        S.last_flag = 0;
    }
    __syncthreads();
    if (S.abort_flag) return;
    const int nA = S.n_active;
    for (int a = tid; a < nA; a += blockDim.x) {
        const int e = p.active[a];
        const int f = (int)entry(p.packed, e)->fmt;
        const int c = e < p.E ? p.counts[e] : p.T;
        const int passes = (c + kMaxTok - 1) / kMaxTok;
        S.e[a] = e;
        S.fmt[a] = f;
        S.cnt[a] = c;
        S.w[a] = unit_bytes(f, K) * (passes > 0 ? passes : 1);
    }
    __syncthreads();
    if (tid == 0) {
        long long run = 0;
        for (int a = 0; a < nA; ++a) {
            S.pre[a] = run;
            run += S.w[a] * tiles;
        }
        S.pre[nA] = run;
        first_unit(S, tiles, run, gridDim.x, blockIdx.x, &S.start_a, &S.start_j);
        first_unit(S, tiles, run, gridDim.x, blockIdx.x + 1, &S.end_a, &S.end_j);
        for (int i = 0; i < nstage; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kCWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();

    const int end_a = S.end_a, end_j = S.end_j;

    if (warp == kCWarps) {
        // ================================ producer ================================
        const uint64_t pol = l2_policy_evict_first();
        int it = 0;
        for (int a = S.start_a, j = S.start_j; a < end_a || (a == end_a && j < end_j);) {
            const int st = it % nstage;
            const uint32_t round = (uint32_t)(it / nstage);
            if (it >= nstage && !ld_volatile(S.abort_flag)) {
                bool ok = mbar_wait_bounded(&empty[st], (round - 1) & 1, kWaitLimit);
                if (!ok) {
                    st_volatile(S.abort_flag, 1);
                    report_error(p.ctrl, MOE_ERR_TIMEOUT, kDetWaitEmpty | MODE);
                }
            }
            if (ld_volatile(S.abort_flag)) break;
            const PackedEntry* en = entry(p.packed, S.e[a]);
            const int f = S.fmt[a];
            const uint8_t* codes = p.packed + (MODE == 0 ? en->gu_codes : en->dn_codes);
            const uint8_t* hi = p.packed + (MODE == 0 ? en->gu_hi : en->dn_hi);
            const uint8_t* sc = p.packed + (MODE == 0 ? en->gu_scales : en->dn_scales);
            uint8_t* dst = stages + (size_t)st * geo.bytes;
            const uint32_t row_bytes = K / 4, hi_bytes = hi_words(K) * 4, sc_bytes = 16 * geo.G * 2;
            const uint32_t tx = 16 * row_bytes + sc_bytes + (f == MOE_FMT_Q3 ? 16 * hi_bytes : 0);
            if (lane == 0) mbar_arrive_expect_tx(&full[st], tx);
            __syncwarp();
            if (lane < 16) {
                const size_t r = (size_t)j * 16 + lane;
                bulk_g2s_evict_first(dst + lane * geo.rs0 * 4, codes + r * row_bytes, row_bytes, &full[st], pol);
            } else if (f == MOE_FMT_Q3) {
                const size_t r = (size_t)j * 16 + (lane - 16);
                bulk_g2s_evict_first(dst + geo.off_hi + (lane - 16) * geo.rs1 * 4, hi + r * hi_bytes, hi_bytes,
                                     &full[st], pol);
            }
            if (lane == 0)
                bulk_g2s_evict_first(dst + geo.off_sc, sc + (size_t)j * sc_bytes, sc_bytes, &full[st], pol);
            ++it;
            if (++j == tiles) {
                j = 0;
                ++a;
            }
        }
        // drain: make sure no copy still targets this CTA's shared memory at exit
        for (int i = 0; i < nstage && i < it; ++i) {
            const int idx = it - 1 - i;
            const int st = idx % nstage;
            if (!mbar_wait_bounded(&full[st], (uint32_t)(idx / nstage) & 1, kWaitLimit)) {
                report_error(p.ctrl, MOE_ERR_TIMEOUT, kDetDrain | MODE);
                break;
            }
        }
        return;
    }

    // ================================ consumers ===================================
    const int g = lane >> 2, t = lane & 3;
    int it = 0;
    for (int a = S.start_a, j = S.start_j; a < end_a || (a == end_a && j < end_j);) {
        const int st = it % nstage;
        const uint32_t par = (uint32_t)(it / nstage) & 1;
        if (!ld_volatile(S.abort_flag)) {
            if (!mbar_wait_bounded(&full[st], par, kWaitLimit)) {
                st_volatile(S.abort_flag, 1);
                report_error(p.ctrl, MOE_ERR_TIMEOUT, kDetWaitFull | MODE);
            }
        }
        const int e = S.e[a], f = S.fmt[a], cnt = S.cnt[a];
        const float o = f == MOE_FMT_TERNARY ? 1.f : (f == MOE_FMT_Q2 ? 1.5f : 3.5f);
        uint32_t sub[5];
        if (MODE == 0) {
            sub[0] = bf16x2_bits_of(64.f + o);
            sub[1] = bf16x2_bits_of(32.f + o);
            sub[2] = bf16x2_bits_of(8.f + o);
            sub[3] = bf16x2_bits_of(16.f + o);
            sub[4] = bf16x2_bits_of(4.f + o);
        } else {
            sub[0] = f16x2_bits_of(512.f + o);
            sub[1] = f16x2_bits_of(256.f + o);
            sub[2] = f16x2_bits_of(64.f + o);
            sub[3] = f16x2_bits_of(16.f + o);
            sub[4] = f16x2_bits_of(4.f + o);
        }
        const uint8_t* stg = stages + (size_t)st * geo.bytes;
        const uint32_t* cw = reinterpret_cast<const uint32_t*>(stg);
        const uint32_t* hw = reinterpret_cast<const uint32_t*>(stg + geo.off_hi);
        const uint16_t* scs = reinterpret_cast<const uint16_t*>(stg + geo.off_sc);
        const uint16_t* bsrc = MODE == 0 ? p.x : p.h;
        const int bld = MODE == 0 ? p.H : p.I;   // leading dimension of the B rows

        for (int tb = 0; tb < cnt; tb += tokblk) {
            const int nb = min(tokblk, cnt - tb);
            if (tid < tokblk) {
                int trow = -1, hr = -1;
                if (tid < nb) {
                    const int i = tb + tid;
                    if (e < p.E) {
                        hr = p.offsets[e] + i;
                        trow = MODE == 0 ? p.perm[hr] / p.k : hr;
                    } else {
                        hr = p.T * p.k + (e - p.E) * p.T + i;
                        trow = MODE == 0 ? i : hr;
                    }
                }
                S.tok[tid] = trow;
                S.hrow[tid] = hr;
            }
            named_bar_sync(1, kCWarps * 32);
            const int nt = (nb + 7) >> 3;
            float acc[8][4];
#pragma unroll
            for (int n = 0; n < 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
            int brow[8];
#pragma unroll
            for (int n = 0; n < 8; ++n) brow[n] = (n < nt) ? S.tok[n * 8 + g] : -1;

            for (int G = warp; G < geo.G; G += kCWarps) {
                uint32_t pa[8], pb[8], ha[8], hb[8];
                if (MODE == 0) {
                    dequant_codes(cw[g * geo.rs0 + G * 4 + t], sub, pa);
                    dequant_codes(cw[(g + 8) * geo.rs0 + G * 4 + t], sub, pb);
                } else {
                    dequant_codes_f16(cw[g * geo.rs0 + G * 4 + t], sub, pa);
                    dequant_codes_f16(cw[(g + 8) * geo.rs0 + G * 4 + t], sub, pb);
                }
                if (f == MOE_FMT_Q3) {
                    const int wi = 2 * G + (t >> 1), sh = 8 * (t & 1);
                    if (MODE == 0) {
                        dequant_hi(hw[g * geo.rs1 + wi] >> sh, ha);
                        dequant_hi(hw[(g + 8) * geo.rs1 + wi] >> sh, hb);
                    } else {
                        dequant_hi_f16(hw[g * geo.rs1 + wi] >> sh, ha);
                        dequant_hi_f16(hw[(g + 8) * geo.rs1 + wi] >> sh, hb);
                    }
                }
                const float s0 = half_bits_to_f32(scs[g * geo.G + G]);
                const float s1 = half_bits_to_f32(scs[(g + 8) * geo.G + G]);
#pragma unroll
                for (int n = 0; n < 8; ++n) {
                    if (n >= nt) break;
                    uint4 q0 = make_uint4(0, 0, 0, 0), q1 = q0;
                    if (brow[n] >= 0) {
                        const uint16_t* bp = bsrc + (size_t)brow[n] * bld + G * 64 + 16 * t;
                        q0 = ldg_nc_v4(bp);
                        q1 = ldg_nc_v4(bp + 8);
                    }
                    const uint32_t xb[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
                    float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
#pragma unroll
                    for (int s = 0; s < 4; ++s) {
                        if (MODE == 0)
                            mma_bf16_16816(d0, d1, d2, d3, pa[2 * s], pb[2 * s], pa[2 * s + 1], pb[2 * s + 1],
                                           xb[2 * s], xb[2 * s + 1]);
                        else
                            mma_f16_16816(d0, d1, d2, d3, pa[2 * s], pb[2 * s], pa[2 * s + 1], pb[2 * s + 1],
                                          xb[2 * s], xb[2 * s + 1]);
                    }
                    if (f == MOE_FMT_Q3) {
#pragma unroll
                        for (int s = 0; s < 4; ++s) {
                            if (MODE == 0)
                                mma_bf16_16816(d0, d1, d2, d3, ha[2 * s], hb[2 * s], ha[2 * s + 1], hb[2 * s + 1],
                                               xb[2 * s], xb[2 * s + 1]);
                            else
                                mma_f16_16816(d0, d1, d2, d3, ha[2 * s], hb[2 * s], ha[2 * s + 1], hb[2 * s + 1],
                                              xb[2 * s], xb[2 * s + 1]);
                        }
                    }
                    acc[n][0] = fmaf(s0, d0, acc[n][0]);
                    acc[n][1] = fmaf(s0, d1, acc[n][1]);
                    acc[n][2] = fmaf(s1, d2, acc[n][2]);
                    acc[n][3] = fmaf(s1, d3, acc[n][3]);
                }
            }
            // per-warp partial sums -> shared memory
            float* rw = red + (size_t)warp * 16 * red_stride;
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                if (n >= nt) break;
                const int c0 = n * 8 + 2 * t;
                rw[g * red_stride + c0] = acc[n][0];
                rw[g * red_stride + c0 + 1] = acc[n][1];
                rw[(g + 8) * red_stride + c0] = acc[n][2];
                rw[(g + 8) * red_stride + c0 + 1] = acc[n][3];
            }
            named_bar_sync(1, kCWarps * 32);
            if (MODE == 0) {
                for (int item = tid; item < 8 * nb; item += kCWarps * 32) {
                    const int jj = item & 7, tok = item >> 3;
                    float av = 0.f, bv = 0.f;
#pragma unroll
                    for (int w = 0; w < kCWarps; ++w) {
                        av += red[(size_t)w * 16 * red_stride + jj * red_stride + tok];
                        bv += red[(size_t)w * 16 * red_stride + (jj + 8) * red_stride + tok];
                    }
                    p.h[(size_t)S.hrow[tok] * p.I + j * 8 + jj] = f32_to_f16_bits(silu_f(av) * bv);
                }
            } else {
                for (int item = tid; item < 16 * nb; item += kCWarps * 32) {
                    const int r = item & 15, tok = item >> 4;
                    float v = 0.f;
#pragma unroll
                    for (int w = 0; w < kCWarps; ++w) v += red[(size_t)w * 16 * red_stride + r * red_stride + tok];
                    p.ypart[(size_t)S.hrow[tok] * p.H + j * 16 + r] = v;
                }
            }
            named_bar_sync(1, kCWarps * 32);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);

        if (MODE == 1) {
            // last-arriver combine of output tile j over all active experts
            __threadfence();
            named_bar_sync(1, kCWarps * 32);
            if (tid == 0) S.last_flag = atomicAdd(&p.tile_ctr[j], 1u) == (uint32_t)(nA - 1);
            named_bar_sync(1, kCWarps * 32);
            if (S.last_flag) {
                __threadfence();
                for (int item = tid; item < p.T * 16; item += kCWarps * 32) {
                    const int tok = item >> 4, r = item & 15;
                    const size_t col = (size_t)j * 16 + r;
                    float v = 0.f;
                    for (int sl = 0; sl < p.k; ++sl) {
                        const int row = p.inv_perm[(size_t)tok * p.k + sl];
                        v = fmaf(p.topk_w[(size_t)tok * p.k + sl], ldcg_f32(p.ypart + (size_t)row * p.H + col), v);
                    }
                    for (int s = 0; s < p.S; ++s)
                        v += ldcg_f32(p.ypart + ((size_t)p.T * p.k + (size_t)s * p.T + tok) * p.H + col);
                    p.y[(size_t)tok * p.H + col] = f32_to_bf16_bits(v);
                }
                named_bar_sync(1, kCWarps * 32);
                if (tid == 0) {
                    p.tile_ctr[j] = 0u;
                    S.last_flag = 0;
                }
                named_bar_sync(1, kCWarps * 32);
            }
        }
        ++it;
        if (++j == tiles) {
            j = 0;
            ++a;
        }
    }
}

size_t fixed_smem(int nstage, int tokblk) {
    const size_t red_bytes = (size_t)kCWarps * 16 * (tokblk + 4) * 4;
    return (sizeof(Sched) + 16 * nstage + red_bytes + 1023) & ~size_t(1023);
}

template <int MODE>
cudaError_t launch_mode(const FfnArgs& a, cudaStream_t s) {
    static int max_smem = 0;
    if (!max_smem) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    }
    const int K = MODE == 0 ? a.H : a.I;
    const Geom geo = make_geom(K);
    const int tokblk = min(kMaxTok, ((a.T + 7) / 8) * 8);
    int nstage = 16;
    while (nstage > 2 && fixed_smem(nstage, tokblk) + (size_t)nstage * geo.bytes > (size_t)max_smem) --nstage;
    const size_t smem = fixed_smem(nstage, tokblk) + (size_t)nstage * geo.bytes;
    if (smem > (size_t)max_smem) return cudaErrorInvalidConfiguration;
    static size_t attr_set = 0;   // largest dynamic size enabled so far for this kernel
    if (smem > attr_set) {
        cudaError_t err = cudaFuncSetAttribute(ffn_mma_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               max_smem);
        if (err != cudaSuccess) return err;
        attr_set = (size_t)max_smem;
    }
    ffn_mma_kernel<MODE><<<a.num_ctas, kThreads, smem, s>>>(a, nstage, tokblk);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ffn_mma(const FfnArgs& a, cudaStream_t s, cudaEvent_t mid_event) {
    cudaError_t err = launch_mode<0>(a, s);
    if (err != cudaSuccess) return err;
    if (mid_event) cudaEventRecord(mid_event, s);
    return launch_mode<1>(a, s);
}

}  // namespace moe
