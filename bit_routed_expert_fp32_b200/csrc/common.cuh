// Device helpers shared by the kernels: packed-table access, PTX wrappers for
// mbarriers and bulk (TMA) copies, bounded waits and the workspace error word.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// ---- packed format (see include/moe.h) ----------------------------------------
constexpr uint32_t kMagic = 0x50454F4Du;
constexpr uint32_t kVersion = 2u;
constexpr int kGroup = 64;
constexpr int kInterleave = 8;
constexpr int kHeaderBytes = 256;
constexpr int kEntryBytes = 64;

struct __align__(16) PackedEntry {
    uint32_t fmt;
    uint32_t zero;
    uint64_t gu_scales, gu_codes, gu_hi;
    uint64_t dn_scales, dn_codes, dn_hi;
    uint64_t zero2;
};
static_assert(sizeof(PackedEntry) == kEntryBytes, "entry layout");


// ---- workspace control block --------------------------------------------------
// The first 4 KiB of the workspace; zeroed by moe_workspace_init.
struct Ctrl {
    uint32_t err_code;      // 0 = ok, else moe_status
    uint32_t err_detail;    // kernel-specific detail (where a wait gave up, ...)
    uint32_t route_ticket;  // last-block counters (self-resetting)
    uint32_t topk_ticket;
    int32_t n_active;       // experts with tokens + shared experts, written by moe_route
    int32_t routed_T;       // T of the last moe_route
    uint32_t work[2];       // decode work counters (gate/up, down); zeroed by the router and the combine
    uint32_t test_stall;    // failure-path tests only: cycles of a wait nothing completes (0 = off)
    uint32_t pad[55];
};
static_assert(sizeof(Ctrl) == 256, "control block layout");

// Counters of the fused decode kernel, right after Ctrl in the control block.  Every
// launch leaves them at zero again (the last warp to finish resets them); the
// workspace initialisation zeroes them first.
constexpr int kMaxSlots = 272;              // expert slots: shared experts, then routed (>= E + S)
struct FusedCtl {
    uint32_t work;          // next work unit to hand out
    uint32_t spare;
    uint32_t warps_done;    // warps that have left the unit loop
    uint32_t abort;         // set when a wait ran out: every warp stops working
    uint32_t pad[12];
    uint32_t gu_done[kMaxSlots];   // gate/up tiles finished per expert slot
    uint32_t hq_done[kMaxSlots];   // shares of the down pass's h operands formed per slot
};
static_assert(256 + sizeof(FusedCtl) <= 4096, "control block size");

// error detail codes
enum : uint32_t {
    kDetWaitFull = 0x100,
    kDetWaitEmpty = 0x200,
    kDetDrain = 0x300,
    kDetHeader = 0x400,
    kDetRoutedT = 0x500,    // moe_forward's T differs from the preceding moe_route's
    kDetRange = 0x600,      // a token or an expert activation outside the fp16 range
    kDetTestStall = 0x700,  // the failure-path test's wait ran out
    kDetLoopCap = 0x800,    // a work loop reached its iteration cap
    kDetFormat = 0x900,     // an expert's format is not one the kernels read (a storage form)
};

__device__ inline void report_error(Ctrl* c, uint32_t code, uint32_t detail) {
    if (atomicCAS(&c->err_code, 0u, code) == 0u) atomicExch(&c->err_detail, detail);
}

// |v| <= 65504, the largest finite fp16 value (false for NaN and infinities).
__device__ inline bool in_f16_range(float v) { return fabsf(v) <= 65504.f; }

// ---- PTX wrappers -----------------------------------------------------------------
__device__ inline uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ inline void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ inline void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ inline void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ inline void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ inline bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait: gives up after `limit` clock cycles and returns false.  The clock is
// read once per 64 polls so that a waiting warp issues few instructions.
__device__ inline bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, long long limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > limit) return false;
    }
}

// One lane of a converged warp (elect.sync): issue single-thread async instructions
// (bulk copies, tensor-map loads, tcgen05.mma) from warp-uniform code under this
// predicate, so their operands stay warp-uniform.
__device__ inline bool elect_one() {
    uint32_t r;
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}" : "=r"(r));
    return r != 0;
}

// Bounded wait with a sleep of about `ns` nanoseconds between polls, for long waits
// where a little wake-up latency costs nothing.
__device__ inline bool mbar_wait_bounded_backoff(uint64_t* bar, uint32_t parity, long long limit, uint32_t ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        __nanosleep(ns);
        if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > limit) return false;
    }
}

// try_wait with a suspend-time hint: a thread whose phase has not completed is
// suspended (it issues nothing) until the phase completes or about `ns` nanoseconds
// have passed.
__device__ inline bool mbar_try_wait_suspend(uint64_t* bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, "
        "p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

// Bounded wait that leaves the issue slots to the working warps while it waits: the
// thread sleeps in the barrier between checks of the clock.
__device__ inline bool mbar_wait_bounded_suspend(uint64_t* bar, uint32_t parity, long long limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait_suspend(bar, parity, 20000u)) return true;
        if (clock64() - t0 > limit) return false;
    }
}

// 1-D bulk copy global -> shared, completion counted on `bar` (bytes % 16 == 0,
// both addresses 16-byte aligned).
__device__ inline void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start before its predecessor in the stream has finished: it must
// call griddep_wait() before it reads anything the predecessor writes (or overwrites
// anything the predecessor reads).  griddep_launch_dependents() lets the next kernel's
// launch begin; kernels call it only when all of their CTAs are resident at once, so
// the successor's CTAs never take an SM that one of their own still needs.  Both are
// no-ops for kernels launched without the attribute.
__device__ inline void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ inline void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// Prefetch the line holding p into L1 (no register result, never blocks).
__device__ inline void prefetch_l1(const void* p) { asm volatile("prefetch.global.L1 [%0];" ::"l"(p)); }

// Bulk prefetch of [src, src + bytes) into L2 (16-byte aligned address and size).
__device__ inline void bulk_prefetch_l2(const void* src_gmem, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src_gmem), "r"(bytes) : "memory");
}

__device__ inline void bulk_g2s_evict_first(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], "
        "%4;" ::"r"(smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ inline uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ inline void named_bar_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ inline uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t magic) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(mask), "r"(magic));
    return r;
}

__device__ inline uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ inline void mma_bf16_16816(float& d0, float& d1, float& d2, float& d3, uint32_t a0, uint32_t a1,
                                      uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d0), "+f"(d1), "+f"(d2), "+f"(d3)
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ inline uint32_t f16x2_sub(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ inline void mma_f16_16816(float& d0, float& d1, float& d2, float& d3, uint32_t a0, uint32_t a1,
                                     uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d0), "+f"(d1), "+f"(d2), "+f"(d3)
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ inline uint4 ldg_nc_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ inline float ldcg_f32(const float* p) {
    float v;
    asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

__device__ inline float silu_f(float a) { return a / (1.0f + expf(-a)); }

__device__ inline uint16_t f32_to_bf16_bits(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ inline uint16_t f32_to_f16_bits(float f) { return __half_as_ushort(__float2half_rn(f)); }

__host__ __device__ inline uint32_t f16x2_bits_of(float v) {
    // exact for the small dequantiser constants (all representable in binary16)
    return (uint32_t)__half_as_ushort(__float2half_rn(v)) * 0x10001u;
}

__host__ __device__ inline uint32_t bf16x2_bits_of(float lo_hi_same) {
    // exact conversion for the small constants used by the dequantiser
    union { float f; uint32_t u; } v;
    v.f = lo_hi_same;
    uint32_t b = v.u >> 16;   // all constants used are exact in bf16 (checked on the host)
    return b | (b << 16);
}

}  // namespace moe
