// moe_decode_static: route + decode-path forward with a scratch area the library
// holds itself, for callers that cannot allocate device memory.
//
// Why: some callers of this library cannot call cudaMalloc.  A plugin running
// inside a framework whose pool allocator owns all of the GPU's memory must not
// allocate behind its back; a serving loop cannot afford cudaMalloc / cudaFree,
// which may synchronise the whole device; and code that is recording a CUDA graph
// may not allocate while the capture is open.  This entry point needs only the
// caller's inputs and outputs: its scratch is the file-scope array below, which
// every GPU that loads the library holds (kStaticWsBytes) until the process exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "kernels.h"
#include "moe.h"

namespace {

constexpr size_t kStaticWsBytes = MOE_STATIC_WS_BYTES;   // 8 MiB
constexpr int kMaxDevices = 64;

// The scratch area.  Host code must not use this symbol as a device address (on the
// host it names a host-side stand-in); it takes the address from
// cudaGetSymbolAddress, once per device context.
static __device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

// Device address of g_static_ws per device, with the id of the context it was looked
// up in: after cudaDeviceReset the device gets a new primary context (a new id), the
// module is loaded again and the address is looked up again.
struct AddrSlot {
    unsigned long long ctx_id;
    void* addr;
};
AddrSlot g_addr[kMaxDevices] = {};
std::mutex g_addr_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context, 0 if there is none yet or the
// driver does not offer context ids.
unsigned long long current_ctx_id() {
    static CtxGetCurrentFn get_cur = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void* f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_cur = reinterpret_cast<CtxGetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(f);
    });
    if (!get_cur || !get_id) return 0;
    CUcontext c = nullptr;
    unsigned long long id = 0;
    if (get_cur(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Set-up, once per device context, with that device current: the device address of
// the scratch array.  Returns nullptr if the lookup fails.
void* static_ws_addr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_addr_mu);
    const unsigned long long id = current_ctx_id();
    if (g_addr[dev].addr && id != 0 && g_addr[dev].ctx_id == id) return g_addr[dev].addr;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || !p) return nullptr;
    g_addr[dev].addr = p;
    g_addr[dev].ctx_id = current_ctx_id();   // the lookup made the primary context current
    return p;
}

}  // namespace

extern "C" moe_status moe_decode_static(const moe_shape* shape, int32_t T, const uint16_t* d_x,
                                        const float* d_router_w, const float* d_router_b, const void* d_packed,
                                        const moe_routing* out, uint16_t* d_y, void* stream) {
    // Every argument check of both calls first: a rejected call enqueues nothing and
    // leaves the scratch array and the outputs as they were.  The workspace pointer
    // given to the checks only stands for "present"; the size is the array's, so a
    // call whose workspace does not fit returns MOE_ERR_WORKSPACE here.
    const void* present = &kStaticWsBytes;
    moe_status st = moe::check_route_args(shape, T, d_x, d_router_w, out, present, kStaticWsBytes);
    if (st != MOE_OK) return st;
    st = moe::check_forward_args(shape, T, d_packed, d_x, out, d_y, MOE_PATH_DECODE, present, kStaticWsBytes);
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    void* ws = static_ws_addr();
    if (!ws) return MOE_ERR_CUDA;
    // The array keeps the previous call's contents: clear the control block and the
    // counters after it (tickets and work counters must start at zero), but keep the
    // error word and its detail (the first 8 bytes) until moe_decode_static_get_error
    // reads them, so that a call that gave up on the device is not forgotten.
    const size_t n = (size_t)4096 + 65536;
    if (cudaMemsetAsync(static_cast<uint8_t*>(ws) + 8, 0, n - 8, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return MOE_ERR_CUDA;
    st = moe_route(shape, T, d_x, d_router_w, d_router_b, out, ws, kStaticWsBytes, stream);
    if (st != MOE_OK) return st;
    return moe_forward(shape, T, d_packed, d_x, out, d_y, MOE_PATH_DECODE, ws, kStaticWsBytes, stream);
}

extern "C" moe_status moe_decode_static_get_error(void* stream, uint32_t* detail) {
    void* ws = static_ws_addr();
    if (!ws) return MOE_ERR_CUDA;
    return moe_get_error(ws, kStaticWsBytes, stream, detail);
}
