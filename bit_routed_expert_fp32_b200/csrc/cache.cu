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
};

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
    std::vector<std::pair<uint64_t, int>> order(n);
    for (int e = 0; e < n; ++e) {
        const uint8_t* ent = h + kHeaderBytes + (size_t)e * kEntryBytes;
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

size_t slot_bytes(const HostLayer& L) {
    uint64_t m = 0;
    for (int e = 0; e < L.n; ++e) m = std::max(m, L.end[e] - L.start[e]);
    return align256(m);
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
    *bytes = table_bytes(L.n) + (size_t)n_slots * slot_bytes(L);
    return MOE_OK;
}

extern "C" moe_status moe_cache_init(const moe_shape* shape, const uint8_t* h_packed, int32_t n_slots,
                                     void* d_cache, size_t cache_bytes, void* stream) {
    HostLayer L;
    if (!moe::shape_ok(shape) || !h_packed || !d_cache || n_slots < 1) return MOE_ERR_INVALID_ARG;
    if (!parse(shape, h_packed, &L)) return MOE_ERR_INVALID_ARG;
    if (cache_bytes < table_bytes(L.n) + (size_t)n_slots * slot_bytes(L)) return MOE_ERR_WORKSPACE;
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
        const uint8_t* ent = h_packed + kHeaderBytes + (size_t)e * kEntryBytes;
        uint64_t w[7];
        w[0] = rd64(ent);
        for (int i = 1; i < 7; ++i) {
            const uint64_t v = rd64(ent + 8 * i);
            w[i] = v ? v - L.start[e] + base : 0;
        }
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
    const size_t sb = slot_bytes(L), base = table_bytes(L.n);
    if (cache_bytes < base + (size_t)n_slots * sb) return MOE_ERR_WORKSPACE;
    for (int i = 0; i < n; ++i)
        if (h_experts[i] < 0 || h_experts[i] >= L.n || h_slots[i] < 0 || h_slots[i] >= n_slots)
            return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* d = static_cast<uint8_t*>(d_cache);
    for (int i = 0; i < n; ++i) {
        const int e = h_experts[i];
        const size_t slot0 = base + (size_t)h_slots[i] * sb;
        if (cudaMemcpyAsync(d + slot0, h_packed + L.start[e], L.end[e] - L.start[e], cudaMemcpyHostToDevice, s) !=
            cudaSuccess)
            return MOE_ERR_CUDA;
        const uint8_t* ent = h_packed + kHeaderBytes + (size_t)e * kEntryBytes;
        uint64_t w[7];
        w[0] = rd64(ent);
        for (int k = 1; k < 7; ++k) {
            const uint64_t v = rd64(ent + 8 * k);
            w[k] = v ? v - L.start[e] + slot0 : 0;
        }
        write_entry_kernel<<<1, 1, 0, s>>>(reinterpret_cast<uint64_t*>(d + kHeaderBytes + (size_t)e * kEntryBytes),
                                           w[0], w[1], w[2], w[3], w[4], w[5], w[6]);
    }
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
