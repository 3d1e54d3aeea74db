// Host-tiered experts: a device-side cache of expert slots in front of a packed layer
// that lives in (page-locked) host memory.
//
// The engine on the pages keeps the experts that do not fit its GPU in a pinned host-RAM
// arena and on NVMe, and brings the experts a layer needs into GPU memory ahead of use
// (ossradar.top, Xolotl README, "How it works, in one paragraph").  On B200 a whole layer
// fits in HBM, so this tier only matters for models larger than HBM; it is built so
// that a caller can run the layer from a cache of n slots instead of from a resident
// buffer.  The cache buffer is itself a valid packed buffer (the layer's header and
// expert table, then n equal slots): loading expert e into slot s copies e's contiguous
// span of the host buffer (its gate/up and down arrays, in the packer's order) into the
// slot and rewrites e's table entry to point there, all enqueued on the caller's stream
// (cudaMemcpyAsync, one per expert, and a one-thread kernel for the entry).
// moe_forward then reads the cache buffer like any packed buffer; which experts must be
// resident (those the routing selected, and the shared expert) is the caller's choice.
//
// A ternary expert may be stored in the host buffer in the dense storage form (five
// codes per byte: 1.6 bits per weight against 2, i.e. ~18 % fewer bytes to move
// over PCIe for the expert with its scales).  Its span is copied into a staging area
// behind the slots and expanded there on the GPU into the kernels' 2-bit ternary
// layout (one thread per code word; the scales, blocked the same way in both forms,
// are copied as they are); its table entry then says MOE_FMT_TERNARY.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "kernels.h"
#include "moe.h"

namespace {

using moe::kEntryBytes;
using moe::kHeaderBytes;

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline uint64_t rd64(const uint8_t* p) {
    uint64_t v = 0;
    memcpy(&v, p, 8);
    return v;
}
inline uint32_t rd32(const uint8_t* p) {
    uint32_t v = 0;
    memcpy(&v, p, 4);
    return v;
}

struct HostLayer {
    int n;                                 // expert tables (E + S)
    size_t total;                          // bytes of the host buffer
    std::vector<uint64_t> start, end;      // each expert's contiguous span
    std::vector<uint32_t> fmt;
};

// Offsets, from the start of an expert's span, of its arrays in the kernels' layout
// (the packer's order: gate/up scales, codes, third bits; down scales, codes, third
// bits; each 256-byte aligned), and the span's size.
struct SpanLayout {
    uint64_t gs, gc, gh, ds, dc, dh, bytes;
};
SpanLayout span_layout(const moe_shape* s, uint32_t fmt) {
    const uint64_t H = s->hidden, I = s->inter, nch = (H / 64 + 7) / 8, nci = (I / 64 + 7) / 8;
    SpanLayout L = {};
    uint64_t off = 0;
    L.gs = off;
    off = align256(off + (2 * I / 16) * 256 * nch);
    L.gc = off;
    off += 2 * I * H / 4;
    if (fmt == MOE_FMT_Q3) {
        off = align256(off);
        L.gh = off;
        off += 2 * I * H / 8;
    }
    off = align256(off);
    L.ds = off;
    off = align256(off + (H / 16) * 256 * nci);
    L.dc = off;
    off += H * I / 4;
    if (fmt == MOE_FMT_Q3) {
        off = align256(off);
        L.dh = off;
        off += H * I / 8;
    }
    L.bytes = off;
    return L;
}

// Reads the header and expert table of a host packed buffer (format version 2) and
// finds each expert's span: from its first array to the next expert's first array (or
// the end of the buffer).  False if the header does not describe `shape`.
bool parse(const moe_shape* s, const uint8_t* h, HostLayer* L) {
    if (!s || !h) return false;
    const int n = s->n_experts + s->n_shared;
    if (rd32(h) != moe::kMagic || rd32(h + 4) != moe::kVersion || (int)rd32(h + 8) != s->hidden ||
        (int)rd32(h + 12) != s->inter || (int)rd32(h + 16) != s->n_experts || (int)rd32(h + 20) != s->n_shared)
        return false;
    L->n = n;
    L->total = rd64(h + 32);
    L->start.resize(n);
    L->end.resize(n);
    L->fmt.resize(n);
    std::vector<std::pair<uint64_t, int>> order(n);
    for (int e = 0; e < n; ++e) {
        const uint8_t* ent = h + kHeaderBytes + (size_t)e * kEntryBytes;
        L->fmt[e] = rd32(ent);
        if (L->fmt[e] > MOE_FMT_TERNARY_DENSE) return false;
        uint64_t lo = UINT64_MAX;
        for (int i = 1; i < 7; ++i) {
            const uint64_t v = rd64(ent + 8 * i);
            if (v) lo = std::min(lo, v);
        }
        if (lo == UINT64_MAX || lo >= L->total) return false;
        L->start[e] = lo;
        order[e] = {lo, e};
    }
    std::sort(order.begin(), order.end());
    for (int i = 0; i < n; ++i) L->end[order[i].second] = i + 1 < n ? order[i + 1].first : L->total;
    return true;
}

size_t table_bytes(int n) { return align256((size_t)kHeaderBytes + (size_t)kEntryBytes * n); }

// A slot holds any expert in the kernels' layout (a dense ternary one once expanded).
size_t slot_bytes(const moe_shape* s, const HostLayer& L) {
    uint64_t m = 0;
    for (int e = 0; e < L.n; ++e)
        m = std::max(m, L.fmt[e] == MOE_FMT_TERNARY_DENSE ? span_layout(s, MOE_FMT_TERNARY).bytes : L.end[e] - L.start[e]);
    return align256(m);
}

// The staging area for dense experts' spans (behind the slots; 0 if there are none).
size_t staging_bytes(const HostLayer& L) {
    uint64_t m = 0;
    for (int e = 0; e < L.n; ++e)
        if (L.fmt[e] == MOE_FMT_TERNARY_DENSE) m = std::max(m, L.end[e] - L.start[e]);
    return align256(m);
}

size_t cache_total(const moe_shape* s, const HostLayer& L, int n_slots) {
    return table_bytes(L.n) + (size_t)n_slots * slot_bytes(s, L) + staging_bytes(L);
}

// The 7 table words of expert e placed at byte `at` of the cache: as in the host
// buffer, rebased; a dense ternary expert in its expanded layout, as MOE_FMT_TERNARY.
void entry_words(const moe_shape* s, const uint8_t* h, const HostLayer& L, int e, uint64_t at, uint64_t w[7]) {
    if (L.fmt[e] == MOE_FMT_TERNARY_DENSE) {
        const SpanLayout X = span_layout(s, MOE_FMT_TERNARY);
        const uint64_t v[7] = {MOE_FMT_TERNARY, at + X.gs, at + X.gc, 0, at + X.ds, at + X.dc, 0};
        for (int i = 0; i < 7; ++i) w[i] = v[i];
        return;
    }
    const uint8_t* ent = h + kHeaderBytes + (size_t)e * kEntryBytes;
    w[0] = rd64(ent);
    for (int i = 1; i < 7; ++i) {
        const uint64_t v = rd64(ent + 8 * i);
        w[i] = v ? v - L.start[e] + at : 0;
    }
}

// One dense ternary expert -> the kernels' layout of its slot, in one launch: the code
// words of both matrices (one thread per 32-bit word: 16 codes of a packed row, read
// from the about four bytes that hold them through a table of each byte value's five
// base-3 digits, built in shared memory by every CTA), then the scales, copied in
// 16-byte pieces (the same blocked layout in both forms).
struct ExpandArgs {
    const uint8_t* gc_src;      // dense codes, packed rows of ceil(K/5) bytes
    const uint8_t* dc_src;
    const uint4* gs_src;        // blocked scales
    const uint4* ds_src;
    uint8_t* gc_dst;            // blocked 2-bit code words
    uint8_t* dc_dst;
    uint4* gs_dst;
    uint4* ds_dst;
    int H, I;
    unsigned long long n_gw, n_dw, n_gs, n_ds;   // words of each code array, 16-byte pieces of each scale array
};

__device__ __forceinline__ uint32_t expand_word(const uint8_t* __restrict__ src, int K, unsigned long long w,
                                                const uint16_t* tab) {
    const int wpr = K / 16;                                   // words per row
    const int pr = (int)(w / wpr), q16 = (int)(w % wpr);
    const uint8_t* row = src + (size_t)pr * ((K + 4) / 5);
    const int k0 = 16 * q16, b0 = k0 / 5;
    uint32_t d[4];                                            // digits of the (up to) four bytes
#pragma unroll
    for (int i = 0; i < 4; ++i) d[i] = b0 + i < (K + 4) / 5 ? tab[row[b0 + i]] : 0u;
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const int k = k0 + e, bi = k / 5 - b0, di = k % 5;
        word |= ((d[bi] >> (2 * di)) & 3u) << (16 * (e & 1) + 2 * (e >> 1));
    }
    return word;
}

__device__ __forceinline__ size_t word_pos(int K, unsigned long long w) {
    const int wpr = K / 16;
    const int pr = (int)(w / wpr), q16 = (int)(w % wpr);
    const int G = K / 64, g = q16 / 4, c = g / 8, gl = g % 8, wl = 4 * gl + q16 % 4;
    const int ng = G - 8 * c < 8 ? G - 8 * c : 8;
    const int j = pr / 16, r = pr % 16;
    const int pos = ng == 8 ? r * 32 + (wl ^ (4 * (r % 8))) : r * 4 * ng + wl;
    return (size_t)4 * K * j + 2048 * (size_t)c + 4 * (size_t)pos;
}

__global__ void __launch_bounds__(256) expand_ternary_kernel(const __grid_constant__ ExpandArgs a) {
    __shared__ uint16_t tab[256];                             // byte value -> digits at bits 2d
    for (int b = threadIdx.x; b < 256; b += blockDim.x) {
        uint32_t v = b, t = 0;
        for (int dd = 0; dd < 5; ++dd) {
            t |= (v % 3) << (2 * dd);
            v /= 3;
        }
        tab[b] = (uint16_t)t;
    }
    __syncthreads();
    unsigned long long i = (unsigned long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < a.n_gw) {
        *reinterpret_cast<uint32_t*>(a.gc_dst + word_pos(a.H, i)) = expand_word(a.gc_src, a.H, i, tab);
        return;
    }
    i -= a.n_gw;
    if (i < a.n_dw) {
        *reinterpret_cast<uint32_t*>(a.dc_dst + word_pos(a.I, i)) = expand_word(a.dc_src, a.I, i, tab);
        return;
    }
    i -= a.n_dw;
    if (i < a.n_gs) {
        a.gs_dst[i] = a.gs_src[i];
        return;
    }
    i -= a.n_gs;
    if (i < a.n_ds) a.ds_dst[i] = a.ds_src[i];
}

// The eight 64-bit words of an expert table entry (format; six array offsets; zero).
__global__ void write_entry_kernel(uint64_t* dst, uint64_t w0, uint64_t w1, uint64_t w2, uint64_t w3, uint64_t w4,
                                   uint64_t w5, uint64_t w6) {
    dst[0] = w0;
    dst[1] = w1;
    dst[2] = w2;
    dst[3] = w3;
    dst[4] = w4;
    dst[5] = w5;
    dst[6] = w6;
    dst[7] = 0;
}

}  // namespace

extern "C" moe_status moe_cache_size(const moe_shape* shape, const uint8_t* h_packed, int32_t n_slots,
                                     size_t* bytes) {
    HostLayer L;
    if (!moe::shape_ok(shape) || !h_packed || !bytes || n_slots < 1) return MOE_ERR_INVALID_ARG;
    if (!parse(shape, h_packed, &L)) return MOE_ERR_INVALID_ARG;
    *bytes = cache_total(shape, L, n_slots);
    return MOE_OK;
}

extern "C" moe_status moe_cache_init(const moe_shape* shape, const uint8_t* h_packed, int32_t n_slots,
                                     void* d_cache, size_t cache_bytes, void* stream) {
    HostLayer L;
    if (!moe::shape_ok(shape) || !h_packed || !d_cache || n_slots < 1) return MOE_ERR_INVALID_ARG;
    if (!parse(shape, h_packed, &L)) return MOE_ERR_INVALID_ARG;
    if (cache_bytes < cache_total(shape, L, n_slots)) return MOE_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // header and table as in the host buffer; every entry is rebased onto slot 0 so that
    // it points into the cache buffer even before its expert is loaded
    std::vector<uint8_t> head(h_packed, h_packed + kHeaderBytes);
    uint8_t* d = static_cast<uint8_t*>(d_cache);
    if (cudaMemcpyAsync(d, head.data(), kHeaderBytes, cudaMemcpyHostToDevice, s) != cudaSuccess) return MOE_ERR_CUDA;
    // the pageable header copy above is staged before cudaMemcpyAsync returns; the
    // entries go in by kernel arguments
    const size_t base = table_bytes(L.n);
    for (int e = 0; e < L.n; ++e) {
        uint64_t w[7];
        entry_words(shape, h_packed, L, e, base, w);
        write_entry_kernel<<<1, 1, 0, s>>>(reinterpret_cast<uint64_t*>(d + kHeaderBytes + (size_t)e * kEntryBytes),
                                           w[0], w[1], w[2], w[3], w[4], w[5], w[6]);
    }
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" moe_status moe_cache_load(const moe_shape* shape, const uint8_t* h_packed, int32_t n_slots,
                                     void* d_cache, size_t cache_bytes, const int32_t* h_experts,
                                     const int32_t* h_slots, int32_t n, void* stream) {
    HostLayer L;
    if (!moe::shape_ok(shape) || !h_packed || !d_cache || n_slots < 1 || n < 0) return MOE_ERR_INVALID_ARG;
    if (n > 0 && (!h_experts || !h_slots)) return MOE_ERR_INVALID_ARG;
    if (!parse(shape, h_packed, &L)) return MOE_ERR_INVALID_ARG;
    const size_t sb = slot_bytes(shape, L), base = table_bytes(L.n);
    if (cache_bytes < cache_total(shape, L, n_slots)) return MOE_ERR_WORKSPACE;
    for (int i = 0; i < n; ++i)
        if (h_experts[i] < 0 || h_experts[i] >= L.n || h_slots[i] < 0 || h_slots[i] >= n_slots)
            return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* d = static_cast<uint8_t*>(d_cache);
    uint8_t* staging = d + base + (size_t)n_slots * sb;
    const int H = shape->hidden, I = shape->inter;
    for (int i = 0; i < n; ++i) {
        const int e = h_experts[i];
        const size_t slot0 = base + (size_t)h_slots[i] * sb, span = L.end[e] - L.start[e];
        if (L.fmt[e] != MOE_FMT_TERNARY_DENSE) {
            if (cudaMemcpyAsync(d + slot0, h_packed + L.start[e], span, cudaMemcpyHostToDevice, s) != cudaSuccess)
                return MOE_ERR_CUDA;
        } else {
            // the dense span into the staging area (stream order serialises its reuse),
            // then scales copied and codes expanded into the slot's 2-bit layout
            if (cudaMemcpyAsync(staging, h_packed + L.start[e], span, cudaMemcpyHostToDevice, s) != cudaSuccess)
                return MOE_ERR_CUDA;
            const uint8_t* ent = h_packed + kHeaderBytes + (size_t)e * kEntryBytes;
            const uint64_t hs_gs = rd64(ent + 8) - L.start[e], hs_gc = rd64(ent + 16) - L.start[e];
            const uint64_t hs_ds = rd64(ent + 32) - L.start[e], hs_dc = rd64(ent + 40) - L.start[e];
            const SpanLayout X = span_layout(shape, MOE_FMT_TERNARY);
            const uint64_t nch = (H / 64 + 7) / 8, nci = (I / 64 + 7) / 8;
            ExpandArgs ea;
            ea.gc_src = staging + hs_gc;
            ea.dc_src = staging + hs_dc;
            ea.gs_src = reinterpret_cast<const uint4*>(staging + hs_gs);
            ea.ds_src = reinterpret_cast<const uint4*>(staging + hs_ds);
            ea.gc_dst = d + slot0 + X.gc;
            ea.dc_dst = d + slot0 + X.dc;
            ea.gs_dst = reinterpret_cast<uint4*>(d + slot0 + X.gs);
            ea.ds_dst = reinterpret_cast<uint4*>(d + slot0 + X.ds);
            ea.H = H;
            ea.I = I;
            ea.n_gw = (unsigned long long)(2 * I) * (H / 16);
            ea.n_dw = (unsigned long long)H * (I / 16);
            ea.n_gs = (unsigned long long)(2 * I / 16) * 256 * nch / 16;
            ea.n_ds = (unsigned long long)(H / 16) * 256 * nci / 16;
            const unsigned long long n = ea.n_gw + ea.n_dw + ea.n_gs + ea.n_ds;
            expand_ternary_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(ea);
            if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
        }
        uint64_t w[7];
        entry_words(shape, h_packed, L, e, slot0, w);
        write_entry_kernel<<<1, 1, 0, s>>>(reinterpret_cast<uint64_t*>(d + kHeaderBytes + (size_t)e * kEntryBytes),
                                           w[0], w[1], w[2], w[3], w[4], w[5], w[6]);
    }
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
