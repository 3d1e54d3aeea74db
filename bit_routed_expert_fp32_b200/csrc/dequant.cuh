// Dequantisers of the packed code words into MMA operands, and the mma.sync wrappers
// the decode-path kernels share (decode_ffn.cu, decode_fused.cu).
//
// Code word: element 2p + h of its 16 elements at bits 16h + 2p .. 16h + 2p + 1 (the
// packed format in include/moe.h).  The "magic number" conversions OR a code into the
// mantissa of an exponent-only bf16 / fp16 constant, so that "base + c" (or, after
// one subtract, c - o) comes out exactly.
#pragma once
#include "common.cuh"

namespace moe {
namespace dq {

// bf16 magic bases (exponent-only bit patterns) of the gate/up dequantiser
constexpr uint32_t kMag128 = 0x43004300u, kMag32 = 0x42004200u, kMag8 = 0x41004100u, kMag64 = 0x42804280u,
                   kMag16 = 0x41804180u, kMag512 = 0x44004400u, kMag256 = 0x43804380u;
// fp16 magic bases of the down dequantiser
constexpr uint32_t kH512 = 0x60006000u, kH256 = 0x5C005C00u, kH64 = 0x54005400u, kH16 = 0x4C004C00u,
                   kH4 = 0x44004400u, kH4096 = 0x6C006C00u, kH2048 = 0x68006800u, kH1024 = 0x64006400u,
                   kH128 = 0x58005800u, kH32 = 0x50005000u;

// ---- dequantisers (code word: element 2p + h of its 16 at bits 16h + 2p .. +1) ----

// bf16 pairs "base_p + c"; base per pair p: 128, 32, 8, 128, 32, 8, 128, 32 (a code
// at mantissa bits 0-1 / 2-3 / 4-5 of 128 / 32 / 8 has weight exactly 1).
__device__ __forceinline__ void raw_codes_bf16(uint32_t w, uint32_t (&pr)[8]) {
    const uint32_t w6 = w >> 6, w12 = w >> 12;
    pr[0] = lop3_and_or(w, 0x00030003u, kMag128);     // bits 0-1
    pr[1] = lop3_and_or(w, 0x000C000Cu, kMag32);      // bits 2-3
    pr[2] = lop3_and_or(w, 0x00300030u, kMag8);       // bits 4-5
    pr[3] = lop3_and_or(w6, 0x00030003u, kMag128);    // bits 6-7 -> 0-1
    pr[4] = lop3_and_or(w6, 0x000C000Cu, kMag32);     // bits 8-9 -> 2-3
    pr[5] = lop3_and_or(w6, 0x00300030u, kMag8);      // bits 10-11 -> 4-5
    pr[6] = lop3_and_or(w12, 0x00030003u, kMag128);   // bits 12-13 -> 0-1
    pr[7] = lop3_and_or(w12, 0x000C000Cu, kMag32);    // bits 14-15 -> 2-3
}

// bf16 pairs "base_p + 4 * bit" of the third code bit (bits 0..7 of each half of u);
// base per pair p: 512, 256, 128, 64, 32, 16, 8, 8.
__device__ __forceinline__ void raw_hi_bf16(uint32_t u, uint32_t (&pr)[8]) {
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
__device__ __forceinline__ void exact_codes_f16(uint32_t w, const uint32_t (&sub)[5], uint32_t (&pr)[8]) {
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
__device__ __forceinline__ void exact_hi_f16(uint32_t u, uint32_t (&pr)[8]) {
    pr[0] = f16x2_sub(lop3_and_or(u, 0x00010001u, kH4096), kH4096);
    pr[1] = f16x2_sub(lop3_and_or(u, 0x00020002u, kH2048), kH2048);
    pr[2] = f16x2_sub(lop3_and_or(u, 0x00040004u, kH1024), kH1024);
    pr[3] = f16x2_sub(lop3_and_or(u, 0x00080008u, kH512), kH512);
    pr[4] = f16x2_sub(lop3_and_or(u, 0x00100010u, kH256), kH256);
    pr[5] = f16x2_sub(lop3_and_or(u, 0x00200020u, kH128), kH128);
    pr[6] = f16x2_sub(lop3_and_or(u, 0x00400040u, kH64), kH64);
    pr[7] = f16x2_sub(lop3_and_or(u, 0x00800080u, kH32), kH32);
}

// Rows g (wa) and g + 8 (wb) straight into MMA A-fragment order: k-step s uses
// {pair 2s of wa, pair 2s of wb, pair 2s+1 of wa, pair 2s+1 of wb}.
template <int MODE>
__device__ __forceinline__ void dequant_rows(uint32_t wa, uint32_t wb, const uint32_t (&sub)[5], uint32_t (&pa)[8],
                                             uint32_t (&pb)[8]) {
    if (MODE == 0) {
        raw_codes_bf16(wa, pa);
        raw_codes_bf16(wb, pb);
    } else {
        exact_codes_f16(wa, sub, pa);
        exact_codes_f16(wb, sub, pb);
    }
}

template <int MODE>
__device__ __forceinline__ void dequant_hi_rows(uint32_t ua, uint32_t ub, uint32_t (&pa)[8], uint32_t (&pb)[8]) {
    if (MODE == 0) {
        raw_hi_bf16(ua, pa);
        raw_hi_bf16(ub, pb);
    } else {
        exact_hi_f16(ua, pa);
        exact_hi_f16(ub, pb);
    }
}

template <int MODE>
__device__ __forceinline__ void mma_acc(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
    if (MODE == 0)
        asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    else
        asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The four k-steps of one 64-wide group of one tile against one n-tile (xb: the B
// fragments of the group, pairs 0..7 of this lane's 16 elements).
template <int MODE>
__device__ __forceinline__ void mma_group(float (&d)[4], const uint32_t (&pa)[8], const uint32_t (&pb)[8],
                                          const uint4& x0, const uint4& x1) {
    mma_acc<MODE>(d, pa[0], pb[0], pa[1], pb[1], x0.x, x0.y);
    mma_acc<MODE>(d, pa[2], pb[2], pa[3], pb[3], x0.z, x0.w);
    mma_acc<MODE>(d, pa[4], pb[4], pa[5], pb[5], x1.x, x1.y);
    mma_acc<MODE>(d, pa[6], pb[6], pa[7], pb[7], x1.z, x1.w);
}

// The same four k-steps with a zero accumulator input (the group's sum starts at 0).
template <int MODE>
__device__ __forceinline__ void mma_group_first(float (&d)[4], const uint32_t (&pa)[8], const uint32_t (&pb)[8],
                                                const uint4& x0, const uint4& x1) {
    const float zero = 0.f;
    if (MODE == 0)
        asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%10,%10,%10,%10};"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "r"(pa[0]), "r"(pb[0]), "r"(pa[1]), "r"(pb[1]), "r"(x0.x), "r"(x0.y), "f"(zero));
    else
        asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%10,%10,%10,%10};"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "r"(pa[0]), "r"(pb[0]), "r"(pa[1]), "r"(pb[1]), "r"(x0.x), "r"(x0.y), "f"(zero));
    mma_acc<MODE>(d, pa[2], pb[2], pa[3], pb[3], x0.z, x0.w);
    mma_acc<MODE>(d, pa[4], pb[4], pa[5], pb[5], x1.x, x1.y);
    mma_acc<MODE>(d, pa[6], pb[6], pa[7], pb[7], x1.z, x1.w);
}

// acc += A B with A 16 x 8 fp16 (row-major fragment: rows g and g + 8, k = 2t, 2t+1)
// and B 8 x 8 fp16 (k = 2t, 2t+1 of column g); fp32 accumulation.
__device__ __forceinline__ void mma_f16_1688(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
    asm("mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(b0));
}

__device__ __forceinline__ float half_lo(uint32_t w) { return __half2float(__ushort_as_half((uint16_t)(w & 0xFFFFu))); }
__device__ __forceinline__ float half_hi(uint32_t w) { return __half2float(__ushort_as_half((uint16_t)(w >> 16))); }
__device__ __forceinline__ const PackedEntry* entry(const uint8_t* packed, int e) {
    return reinterpret_cast<const PackedEntry*>(packed + kHeaderBytes + (size_t)e * kEntryBytes);
}

}  // namespace dq
}  // namespace moe
