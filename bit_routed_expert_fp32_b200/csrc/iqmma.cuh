// The integer tensor path of the decode kernels for ternary and 2-bit experts (the fused
// decode kernel, decode_fused.cu; the separate gate/up launch, decode_ffn.cu).
//
// A code word (16 codes of a row, 2 bits each) is masked into four byte classes c:
// classes 0 and 2 hold the code, 1 and 3 four times the code (w & 0x03030303,
// w & 0x0C0C0C0C, the same of w >> 4), the u8 A operands of two m16n8k32 MMAs.  B holds
// signed-byte digits of the token (or of h) on a 12-bit grid per 64-group, two digits
// d0 + 256 d1 per value, 4q for the plain classes and q for the x4 ones, so every
// product is 4 c q (the operand records and factors are formed in operands.cuh).  The
// accumulator starts at the bit pattern of 1.5 x 2^23 minus 4 o sum q, so that the int32
// sum read as fp32 is 1.5 x 2^23 + the exactly offset-corrected dot product; one
// subtract, the row's scale and the group's factor 2^-e / 4 then fold it into fp32.
#pragma once
#include "common.cuh"

namespace moe {
namespace iq {

constexpr uint32_t kIqMagic = 0x4B400000u;       // 1.5 * 2^23
constexpr float kIqMagicF = 12582912.0f;
constexpr int kCg = 8;                           // groups per chunk
constexpr int kOffSc = 3072;                     // a tile's chunk stage: codes 2 KB, third bits 1 KB, scales

// ---- packed fp32 pairs (Blackwell f32x2 arithmetic) ---------------------------------
__device__ __forceinline__ unsigned long long pk2(float a, float b) {
    unsigned long long r;
    asm("mov.b64 %0, {%1,%2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float2 up2(unsigned long long v) {
    float2 r;
    asm("mov.b64 {%0,%1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b,
                                                   unsigned long long c) {
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ unsigned long long add2(unsigned long long a, unsigned long long b) {
    unsigned long long d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b) {
    unsigned long long d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// scale of row r, group gl of a chunk stage (fp16 [16 rows][8 groups])
__device__ __forceinline__ float iq_scale_of(const uint8_t* stg, int r, int gl) {
    return __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(stg + kOffSc)[r * 8 + gl]));
}
// code word (r, wl) of a chunk stage (swizzled when the chunk is full)
__device__ __forceinline__ int iq_cw_idx(int r, int wl, bool full, int ng) {
    return full ? r * 32 + (wl ^ (4 * (r & 7))) : r * 4 * ng + wl;
}

// ---- gate/up on the integer path (ternary, 2-bit) ----------------------------------------
// Pass q holds tokens 4q .. 4q + 3 of the expert.  B column g = digit (g & 1) of token
// 4q + (g >> 1); lane (g, t) ends with rows g (gate) and g + 8 (up) of token 4q + t.
// Offsets (32-bit, to keep registers): bq in 16-byte units from the digit records, pq in
// floats from the factors, zq in halves from the offset planes (-1: no correction).
template <int NP>
struct IqView {
    uint32_t bq[NP];     // digit record of column g, lane t, group 0 (16-byte units)
    uint32_t pq[NP];     // pair {p, sum q} of token 4q + t, group 0
    int orow[NP];        // h row of token 4q + t (-1: none)
};

struct IqBase {
    const uint4* bq;     // digit records
    const float2* pq;    // pairs
};

__device__ __forceinline__ void imma2(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t a4,
                                      uint32_t a5, uint32_t a6, uint32_t a7, const uint4& b) {
    asm(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%10,%11};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b.x), "r"(b.y), "r"(kIqMagic), "r"(0));
    asm(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a4), "r"(a5), "r"(a6), "r"(a7), "r"(b.z), "r"(b.w));
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ float2 lds64f(uint32_t a) {
    float2 v;
    asm("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
    return v;
}

// o4 = 4 o: 4 for ternary codes, 6 for 2-bit codes (the offset removed exactly, in the
// integer sums: sum 4 (c - o) q = D - o4 sum q).
template <int NP, bool FULL>
__device__ __forceinline__ void chunk_gu_iq(const uint8_t* stg, int c, int ng, const IqView<NP>& v, const IqBase& B,
                                            int np, int o4, int g, int t, unsigned long long (&acc)[NP]) {
    const uint32_t* cw = reinterpret_cast<const uint32_t*>(stg);
#pragma unroll 2
    for (int gl = 0; gl < (FULL ? kCg : ng); ++gl) {
        const uint32_t w0 = cw[iq_cw_idx(g, 4 * gl + t, FULL, ng)], w1 = cw[iq_cw_idx(g + 8, 4 * gl + t, FULL, ng)];
        const uint32_t w0s = w0 >> 4, w1s = w1 >> 4;
        const uint32_t m0 = w0 & 0x03030303u, m1 = w1 & 0x03030303u, n0 = w0 & 0x0C0C0C0Cu, n1 = w1 & 0x0C0C0C0Cu;
        const uint32_t m0s = w0s & 0x03030303u, m1s = w1s & 0x03030303u, n0s = w0s & 0x0C0C0C0Cu,
                       n1s = w1s & 0x0C0C0C0Cu;
        const unsigned long long sv = pk2(iq_scale_of(stg, g, gl), iq_scale_of(stg, g + 8, gl));
        const int grp = c * kCg + gl;
#pragma unroll
        for (int q = 0; q < NP; ++q) {
            if (q < np) {
                const uint4 b = B.bq[v.bq[q] + grp * 8];
                const float2 pr = B.pq[v.pq[q] + grp];
                const float pf = pr.x;
                const int corr = o4 * __float_as_int(pr.y);
                int d[4];
                imma2(d, m0, m1, n0, n1, m0s, m1s, n0s, n1s, b);
                const unsigned long long D =
                    add2(pk2(__int_as_float(d[0] + 256 * d[1] - corr), __int_as_float(d[2] + 256 * d[3] - corr)),
                         pk2(-kIqMagicF, -kIqMagicF));
                acc[q] = fma2(mul2(sv, pk2(pf, pf)), D, acc[q]);
            }
        }
    }
}

// The same for a full chunk (8 groups), with the addressing hoisted: the swizzled
// position of this lane's code word for group gl is sw ^ (16 gl) bytes into the stage
// (sw = 128 g + 16 (g mod 8) + 4 t; the row's 128-byte block keeps bits 4-6 free for
// the XOR), row g + 8 is 1024 bytes further; the digit records and the pairs of the
// chunk are at fixed offsets from one pointer each; the scales of the chunk come in
// with one 16-byte load per row; and the code offset is folded into the accumulator's
// start value, M - o4 sum q, so the low digit's sum comes out already corrected.
// STG: the records and pairs are in shared memory (B points there; read with ld.shared,
// which never changes during the launch once staged).
template <int NP, bool STG>
__device__ __forceinline__ void chunk_iq_full(const uint8_t* stg, int c, const IqView<NP>& v, const IqBase& B, int np,
                                              int o4, int sw, int g, unsigned long long (&acc)[NP]) {
    const uint4 sg4 = *reinterpret_cast<const uint4*>(stg + kOffSc + 16 * g);
    const uint4 su4 = *reinterpret_cast<const uint4*>(stg + kOffSc + 16 * (g + 8));
    const uint32_t sg[4] = {sg4.x, sg4.y, sg4.z, sg4.w}, su[4] = {su4.x, su4.y, su4.z, su4.w};
    const uint4* rec[NP];
    const float2* prs[NP];
    uint32_t rec_s[NP], prs_s[NP];
#pragma unroll
    for (int q = 0; q < NP; ++q) {
        rec[q] = B.bq + v.bq[q] + 64 * c;
        prs[q] = B.pq + v.pq[q] + kCg * c;
        if (STG) {
            rec_s[q] = (uint32_t)__cvta_generic_to_shared(rec[q]);
            prs_s[q] = (uint32_t)__cvta_generic_to_shared(prs[q]);
        }
    }
#pragma unroll(NP == 1 ? 8 : 2)
    for (int gl = 0; gl < kCg; ++gl) {
        const uint32_t* wp = reinterpret_cast<const uint32_t*>(stg + (sw ^ (16 * gl)));
        const uint32_t w0 = wp[0], w1 = wp[256];
        const uint32_t w0s = w0 >> 4, w1s = w1 >> 4;
        const uint32_t m0 = w0 & 0x03030303u, m1 = w1 & 0x03030303u, n0 = w0 & 0x0C0C0C0Cu, n1 = w1 & 0x0C0C0C0Cu;
        const uint32_t m0s = w0s & 0x03030303u, m1s = w1s & 0x03030303u, n0s = w0s & 0x0C0C0C0Cu,
                       n1s = w1s & 0x0C0C0C0Cu;
        const uint32_t hg = (gl & 1) ? sg[gl >> 1] >> 16 : sg[gl >> 1] & 0xFFFFu;
        const uint32_t hu = (gl & 1) ? su[gl >> 1] >> 16 : su[gl >> 1] & 0xFFFFu;
        const unsigned long long sv = pk2(__half2float(__ushort_as_half((uint16_t)hg)),
                                          __half2float(__ushort_as_half((uint16_t)hu)));
#pragma unroll
        for (int q = 0; q < NP; ++q) {
            if (NP == 1 || q < np) {
                const uint4 b = STG ? lds128(rec_s[q] + 128 * gl) : rec[q][8 * gl];
                const float2 pr = STG ? lds64f(prs_s[q] + 8 * gl) : prs[q][gl];
                const int c0 = (int)kIqMagic - o4 * __float_as_int(pr.y);
                int d[4];
                asm(
                    "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                    "{%10,%11,%10,%11};"
                    : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
                    : "r"(m0), "r"(m1), "r"(n0), "r"(n1), "r"(b.x), "r"(b.y), "r"(c0), "r"(0));
                asm(
                    "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                    "{%0,%1,%2,%3};"
                    : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
                    : "r"(m0s), "r"(m1s), "r"(n0s), "r"(n1s), "r"(b.z), "r"(b.w));
                const unsigned long long D =
                    add2(pk2(__int_as_float(d[0] + 256 * d[1]), __int_as_float(d[2] + 256 * d[3])),
                         pk2(-kIqMagicF, -kIqMagicF));
                acc[q] = fma2(mul2(sv, pk2(pr.x, pr.x)), D, acc[q]);
            }
        }
    }
}

}  // namespace iq
}  // namespace moe
