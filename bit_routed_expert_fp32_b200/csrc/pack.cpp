// Host-side packer: interchange-form codes and fp16 scales -> packed format v2
// (layout documented in include/moe.h), including the dense ternary storage form.
// Pure host code, no CUDA calls.
#include <stdint.h>
#include <string.h>

#include <vector>

#include "moe.h"

namespace {

constexpr uint32_t kMagic = 0x50454F4Du;
constexpr int kHeader = 256;
constexpr int kEntry = 64;

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
// chunks of up to 8 groups of 64 along K
inline int n_chunks(int K) { return (K / 64 + 7) / 8; }

bool shape_ok(const moe_shape* s) {
    return s && s->hidden > 0 && s->inter > 0 && s->hidden % 64 == 0 && s->inter % 64 == 0 &&
           s->n_experts >= 1 && s->n_experts <= 256 && s->top_k >= 1 && s->top_k <= 16 &&
           s->top_k <= s->n_experts && (s->n_shared == 0 || s->n_shared == 1);
}

struct MatLayout {
    size_t scales, codes, hi;  // byte offsets (hi = 0 when absent)
};
struct ExpertLayout {
    uint32_t fmt;
    MatLayout gu, dn;
};

// bytes of a dense ternary row: five codes per byte
inline size_t dense_row_bytes(int K) { return (size_t)(K + 4) / 5; }
size_t mat_bytes(int rows, int K, uint32_t fmt, MatLayout* m, size_t off) {
    off = align256(off);
    m->scales = off;
    off = align256(off + (size_t)(rows / 16) * 256 * n_chunks(K));
    m->codes = off;
    off += fmt == MOE_FMT_TERNARY_DENSE ? (size_t)rows * dense_row_bytes(K) : (size_t)rows * (K / 4);
    if (fmt == MOE_FMT_Q3) {
        off = align256(off);
        m->hi = off;
        off += (size_t)rows * (K / 8);
    } else {
        m->hi = 0;
    }
    return off;
}

// Computes every expert's offsets; returns the total size.
size_t layout(const moe_shape* s, const uint8_t* fmt, std::vector<ExpertLayout>* out) {
    const int H = s->hidden, I = s->inter, n = s->n_experts + s->n_shared;
    size_t off = align256(kHeader + (size_t)kEntry * n);
    if (out) out->resize(n);
    for (int e = 0; e < n; ++e) {
        ExpertLayout L;
        L.fmt = fmt[e];
        off = mat_bytes(2 * I, H, L.fmt, &L.gu, off);
        off = mat_bytes(H, I, L.fmt, &L.dn, off);
        if (out) (*out)[e] = L;
    }
    return align256(off);
}

// 16 natural-order 2-bit codes (code i at bits 2i) -> kernel word (even elements in
// the low half at bits 2p, odd elements in the high half at bits 16 + 2p).
inline uint32_t squeeze_pairs(uint32_t x) {  // keep fields at bits 4i..4i+1, compact
    x &= 0x33333333u;
    x = (x | (x >> 2)) & 0x0F0F0F0Fu;
    x = (x | (x >> 4)) & 0x00FF00FFu;
    x = (x | (x >> 8)) & 0x0000FFFFu;
    return x;
}
inline uint32_t code_word(uint32_t nat) { return squeeze_pairs(nat) | (squeeze_pairs(nat >> 2) << 16); }

// 32 natural-order third bits (element i at bit i) -> kernel word (element
// 16q + 2p + h at bit 16h + 8q + p).
inline uint32_t squeeze_bits(uint32_t x) {
    x &= 0x55555555u;
    x = (x | (x >> 1)) & 0x33333333u;
    x = (x | (x >> 2)) & 0x0F0F0F0Fu;
    x = (x | (x >> 4)) & 0x00FF00FFu;
    x = (x | (x >> 8)) & 0x0000FFFFu;
    return x;
}
inline uint32_t hi_word(uint32_t nat) { return squeeze_bits(nat) | (squeeze_bits(nat >> 1) << 16); }

inline uint32_t load_u32(const uint8_t* p) {
    return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}
inline void store_u32(uint8_t* p, uint32_t v) {
    p[0] = (uint8_t)v;
    p[1] = (uint8_t)(v >> 8);
    p[2] = (uint8_t)(v >> 16);
    p[3] = (uint8_t)(v >> 24);
}

// Packs one source row (K elements) into packed row `dr` (tile dr/16, row dr%16) of a
// matrix, in the tile/chunk-blocked, swizzled layout documented in moe.h.
bool pack_row(const moe_matrix_src& src, int sr, int K, uint32_t fmt, uint8_t* base, const MatLayout& m, int dr) {
    const uint8_t* codes = src.codes + (size_t)sr * (K / 4);
    if (fmt == MOE_FMT_TERNARY || fmt == MOE_FMT_TERNARY_DENSE) {
        for (int b = 0; b < K / 4; ++b)
            if (codes[b] & (codes[b] >> 1) & 0x55) return false;   // a field equal to 3
    }
    const int G = K / 64, NC = n_chunks(K), j = dr / 16, r = dr % 16;
    const uint16_t* ssrc = src.scales + (size_t)sr * G;
    const uint8_t* hi = fmt == MOE_FMT_Q3 ? src.hi + (size_t)sr * (K / 8) : nullptr;
    if (fmt == MOE_FMT_TERNARY_DENSE) {
        // packed row dr: byte i = sum over j < 5 of c(5i + j) 3^j (codes past K are 0)
        uint8_t* drow = base + m.codes + (size_t)dr * dense_row_bytes(K);
        for (size_t i = 0; i < dense_row_bytes(K); ++i) {
            uint32_t v = 0;
            for (int d = 4; d >= 0; --d) {
                const int k = 5 * (int)i + d;
                const uint32_t c = k < K ? (codes[k / 4] >> (2 * (k % 4))) & 3u : 0u;
                v = 3 * v + c;
            }
            drow[i] = (uint8_t)v;
        }
    }
    for (int c = 0; c < NC; ++c) {
        const int ng = G - 8 * c < 8 ? G - 8 * c : 8;
        uint8_t* cblk = base + m.codes + (size_t)4 * K * j + 2048 * (size_t)c;
        for (int wl = 0; wl < 4 * ng && fmt != MOE_FMT_TERNARY_DENSE; ++wl) {
            const int pos = ng == 8 ? r * 32 + (wl ^ (4 * (r % 8))) : r * 4 * ng + wl;
            store_u32(cblk + 4 * pos, code_word(load_u32(codes + 4 * (32 * c + wl))));
        }
        uint8_t* sblk = base + m.scales + (size_t)256 * NC * j + 256 * (size_t)c + 16 * r;
        for (int gl = 0; gl < 8; ++gl) {
            const uint16_t v = 8 * c + gl < G ? ssrc[8 * c + gl] : 0;
            sblk[2 * gl] = (uint8_t)v;
            sblk[2 * gl + 1] = (uint8_t)(v >> 8);
        }
        if (hi) {
            uint8_t* hblk = base + m.hi + (size_t)128 * G * j + 1024 * (size_t)c;
            for (int vl = 0; vl < 2 * ng; ++vl) {
                const int pos = ng == 8 ? r * 16 + (vl ^ (2 * ((r % 8) / 2))) : r * 2 * ng + vl;
                store_u32(hblk + 4 * pos, hi_word(load_u32(hi + 4 * (16 * c + vl))));
            }
        }
    }
    return true;
}

void write_header(const moe_shape* s, const std::vector<ExpertLayout>& L, size_t total, uint8_t* dst) {
    memset(dst, 0, kHeader);
    uint32_t h[8] = {kMagic, 2u, (uint32_t)s->hidden, (uint32_t)s->inter, (uint32_t)s->n_experts,
                     (uint32_t)s->n_shared, 64u, 8u};
    for (int i = 0; i < 8; ++i) store_u32(dst + 4 * i, h[i]);
    store_u32(dst + 32, (uint32_t)total);
    store_u32(dst + 36, (uint32_t)((uint64_t)total >> 32));
    for (size_t e = 0; e < L.size(); ++e) {
        uint8_t* ent = dst + kHeader + e * kEntry;
        memset(ent, 0, kEntry);
        uint64_t v[8] = {L[e].fmt, L[e].gu.scales, L[e].gu.codes, L[e].gu.hi,
                         L[e].dn.scales, L[e].dn.codes, L[e].dn.hi, 0};
        store_u32(ent, (uint32_t)v[0]);
        for (int i = 1; i < 8; ++i) {
            store_u32(ent + 8 * i, (uint32_t)v[i]);
            store_u32(ent + 8 * i + 4, (uint32_t)(v[i] >> 32));
        }
    }
}

}  // namespace

extern "C" moe_status moe_packed_size(const moe_shape* shape, const uint8_t* h_fmt, size_t* bytes) {
    if (!shape_ok(shape) || !h_fmt || !bytes) return MOE_ERR_INVALID_ARG;
    for (int e = 0; e < shape->n_experts + shape->n_shared; ++e)
        if (h_fmt[e] > MOE_FMT_TERNARY_DENSE) return MOE_ERR_INVALID_ARG;
    *bytes = layout(shape, h_fmt, nullptr);
    return MOE_OK;
}

extern "C" moe_status moe_pack_experts(const moe_shape* shape, const uint8_t* h_fmt, int32_t first, int32_t count,
                                       const moe_matrix_src* h_src, void* h_dst, size_t h_dst_bytes) {
    if (!shape_ok(shape) || !h_fmt || !h_dst || (count > 0 && !h_src)) return MOE_ERR_INVALID_ARG;
    const int n = shape->n_experts + shape->n_shared;
    if (first < 0 || count < 0 || first + count > n) return MOE_ERR_INVALID_ARG;
    for (int e = 0; e < n; ++e)
        if (h_fmt[e] > MOE_FMT_TERNARY_DENSE) return MOE_ERR_INVALID_ARG;
    std::vector<ExpertLayout> L;
    const size_t total = layout(shape, h_fmt, &L);
    if (h_dst_bytes < total) return MOE_ERR_WORKSPACE;
    uint8_t* dst = static_cast<uint8_t*>(h_dst);
    write_header(shape, L, total, dst);
    const int H = shape->hidden, I = shape->inter;
    for (int i = 0; i < count; ++i) {
        const int e = first + i;
        const uint32_t fmt = h_fmt[e];
        const moe_matrix_src* m = h_src + 3 * (size_t)i;   // gate, up, down
        for (int q = 0; q < 3; ++q) {
            if (!m[q].codes || !m[q].scales || (fmt == MOE_FMT_Q3 && !m[q].hi)) return MOE_ERR_INVALID_ARG;
        }
        for (int r = 0; r < 2 * I; ++r) {
            const int b = r / 16, j = r % 16;
            const bool gate = j < 8;
            const int sr = 8 * b + (gate ? j : j - 8);
            if (!pack_row(gate ? m[0] : m[1], sr, H, fmt, dst, L[e].gu, r)) return MOE_ERR_INVALID_ARG;
        }
        for (int r = 0; r < H; ++r)
            if (!pack_row(m[2], r, I, fmt, dst, L[e].dn, r)) return MOE_ERR_INVALID_ARG;
    }
    return MOE_OK;
}

extern "C" moe_status moe_requantize_q3_to_q2(int32_t rows, int32_t K, const moe_matrix_src* src,
                                              uint8_t* h_codes, uint16_t* h_scales) {
    if (rows < 1 || K < 64 || K % 64 != 0 || !src || !src->codes || !src->hi || !src->scales || !h_codes ||
        !h_scales)
        return MOE_ERR_INVALID_ARG;
    const size_t G = (size_t)K / 64, nsc = (size_t)rows * G;
    // fp16 doubling: one more in the exponent field, or a left shift of a subnormal's
    // mantissa (which carries into the exponent field exactly when the result is
    // normal); an exponent field of 30 or 31 (largest binade, inf, nan) is refused
    for (size_t i = 0; i < nsc; ++i)
        if (((src->scales[i] >> 10) & 0x1F) >= 30) return MOE_ERR_INVALID_ARG;
    for (size_t i = 0; i < nsc; ++i) {
        const uint16_t b = src->scales[i], sign = b & 0x8000, mag = b & 0x7FFF;
        h_scales[i] = (uint16_t)(sign | ((mag >> 10) ? mag + 0x0400 : mag << 1));
    }
    // element k: 2-bit field at bits 2(k%4) of byte k/4, third bit at bit k%8 of byte k/8;
    // c >> 1 has the field's high bit as its low bit and the third bit as its high bit
    const size_t cb = (size_t)K / 4, hb = (size_t)K / 8;
    for (int r = 0; r < rows; ++r) {
        const uint8_t* c = src->codes + r * cb;
        const uint8_t* h = src->hi + r * hb;
        uint8_t* o = h_codes + r * cb;
        for (size_t j = 0; j < cb; ++j) {
            uint8_t v = 0;
            for (int i = 0; i < 4; ++i) {
                const size_t k = 4 * j + i;
                const unsigned lo = (c[j] >> (2 * i)) & 3u, third = (h[k / 8] >> (k % 8)) & 1u;
                v |= (uint8_t)(((lo >> 1) | (third << 1)) << (2 * i));
            }
            o[j] = v;
        }
    }
    return MOE_OK;
}
