// Per-token operands of the decode-path gate/up kernels, formed from the bf16 tokens:
// the Z tables of the bf16 dequantiser's offset correction and the integer path's
// token digits, factors and offset planes (used by route.cu, decode_fused.cu and, for the
// integer records of h, decode_ffn.cu).
#pragma once
#include "kernels.h"

namespace moe {

struct OperandArgs {
    int T, H;
    const uint16_t* x;   // bf16 [T][H]
    float* zx;           // fp16 planes [2][3][T][G8] of -Z/16 (hi, lo)
    uint8_t* iq;         // integer operands for T tokens (kernels.h), or null
    Ctrl* ctrl;
};

__device__ inline float op_bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ inline float op_bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ inline float op_warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// The gate/up expert kernel feeds the MMA with "base + c" values straight out of the
// code words (no per-pair subtraction), so each 64-wide group's MMA yields
// sum (base + c) x, and the kernel subtracts Z once per 8-group chunk with a small MMA
// of the scales against Z.  For token t and group G (elements x_e, e = 0..63):
//   Bx = sum_e lo_base(e) x_e,  Hx = sum_e hi_base(e) x_e,  Sx = sum_e x_e,
// with lo_base / hi_base the magic bases the expert kernel uses for the pair that
// holds element e (pair p = (e % 16) / 2):  lo 128,32,8,128,32,8,128,32 and
// hi 512,256,128,64,32,16,8,8.  Then for code offset o:
//   Z_ternary = Bx + Sx,  Z_q2 = Bx + 1.5 Sx,  Z_q3 = Bx + Hx + 3.5 Sx.
// Stored as -Z / 16 split exactly into two fp16 halves (hi = the rounding, lo = the
// rounding of what is left), in planes z16[hl][format][T][G8] with the group count
// padded to whole chunks (G8 = 8 ceil(G / 8); the padding is zero): the B fragments of
// the correction MMA.  The 1/16 keeps Z inside the fp16 range; the kernel scales the
// A side (the fp16 scales) by 16, exactly.
__device__ inline void compute_z(const OperandArgs& p, int t, int Gi, int lane) {
    const int G = p.H / 64, G8 = 8 * ((G + 7) / 8);
    float z[3] = {0.f, 0.f, 0.f};
    if (Gi < G) {
        const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(p.x + (size_t)t * p.H + Gi * 64) + lane);
        const float x0 = op_bf16lo(v), x1 = op_bf16hi(v);
        // tokens outside the fp16 range (or not finite) are outside what the expert
        // kernels compute: reported, not carried on (see moe_forward)
        if (!in_f16_range(x0) || !in_f16_range(x1)) report_error(p.ctrl, MOE_ERR_DEVICE_CHECK, kDetRange | 1);
        // the bases of pair p = lane % 8: lo 128, 32, 8, 128, 32, 8, 128, 32 = 2^(7 - 2 (p % 3));
        // hi 512, 256, 128, 64, 32, 16, 8, 8 = 2^(9 - min(p, 6)) (computed: no indexed table)
        const int pp = lane & 7;
        const float bl = __int_as_float((127 + 7 - 2 * (pp % 3)) << 23);
        const float bh = __int_as_float((127 + 9 - min(pp, 6)) << 23);
        float bx = fmaf(bl, x0, bl * x1), hx = fmaf(bh, x0, bh * x1), sx = x0 + x1;
        bx = op_warp_sum(bx);
        hx = op_warp_sum(hx);
        sx = op_warp_sum(sx);
        z[0] = bx + sx;
        z[1] = fmaf(1.5f, sx, bx);
        z[2] = fmaf(3.5f, sx, bx + hx);
    }
    if (lane < 3) {
        const float zs = -0.0625f * (lane == 0 ? z[0] : (lane == 1 ? z[1] : z[2]));
        const __half hi = __float2half_rn(zs);
        const __half lo = __float2half_rn(zs - __half2float(hi));
        uint16_t* z16 = reinterpret_cast<uint16_t*>(p.zx);
        const size_t i = ((size_t)lane * p.T + t) * G8 + Gi, plane = (size_t)3 * p.T * G8;
        z16[i] = __half_as_ushort(hi);
        z16[plane + i] = __half_as_ushort(lo);
    }
}

// Integer operands of one row and 64-group for the decode kernels' integer MMAs
// (ternary and 2-bit experts): the group's values v (two per lane: elements 2 lane and
// 2 lane + 1) go on a 12-bit grid, e = 11 - floor(log2 max |v|), q = rint(v 2^e) (exact
// for every v above 2^-4 of the group maximum).  The kernel masks each code word into
// four byte classes c (two per MMA): classes 0 and 2 hold the code, 1 and 3 four times
// the code, so B = 4q for even c and q for odd c makes every product 4 c q.  Element k
// of the group sits in lane k / 16 of the record, class c = (k mod 8) / 2, byte
// 2 (k mod 2) + (k mod 16) / 8 (the inverse of the code word's element order); B is
// split into signed bytes lo + 256 hi, one record half per digit.  The pair holds
// p = 2^-e / 4, which turns the integer sums into value units, and sum q, from which
// the kernel removes the code offset exactly: sum 4 (c - o) q = D - 4 o sum q.
__device__ inline void iq_group(float v0, float v1, int lane, uint8_t* rec, float2* pair) {
    const float v[2] = {v0, v1};
    const float m = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fmaxf(fabsf(v0), fabsf(v1)))));
    const int e = m > 0.f ? 11 - ilogbf(m) : 0;
    int qsum = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int q = (int)rintf(ldexpf(v[h], e));
        qsum += q;
        const int k = 2 * lane + h, lt = k >> 4, off = k & 15;
        const int c = (off & 7) >> 1, b = 2 * (off & 1) + (off >> 3);
        const int bv = (c & 1) ? q : 4 * q;
        const int lo = (int)(int8_t)(uint8_t)(bv & 0xFF), hi = (bv - lo) >> 8;
        const int pos = 16 * lt + 4 * c + b;
        rec[pos] = (uint8_t)lo;
        rec[64 + pos] = (uint8_t)hi;
    }
    qsum = (int)__reduce_add_sync(0xffffffffu, (uint32_t)qsum);
    if (lane == 0) *pair = make_float2(ldexpf(0.25f, -e), __int_as_float(qsum));
}

// The token operands for token t, group Gi (a whole warp); groups past K (the padding of
// the last chunk) get a zero pair.
__device__ inline void compute_iq(const OperandArgs& p, int t, int Gi, int lane) {
    const int G = p.H / 64, G8 = 8 * ((G + 7) / 8);
    float2* pairs = reinterpret_cast<float2*>(p.iq + iq_pair_off(p.T, p.H)) + (size_t)t * G8;
    if (Gi >= G) {
        if (lane == 0) pairs[Gi] = make_float2(0.f, 0.f);
        return;
    }
    const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(p.x + (size_t)t * p.H + Gi * 64) + lane);
    iq_group(op_bf16lo(v), op_bf16hi(v), lane, p.iq + ((size_t)t * G + Gi) * 128, pairs + Gi);
}

}  // namespace moe
