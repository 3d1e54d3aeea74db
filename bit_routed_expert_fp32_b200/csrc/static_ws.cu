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
#include <cuda_runtime.h>

#include "kernels.h"
#include "moe.h"

namespace {

constexpr size_t kStaticWsBytes = MOE_STATIC_WS_BYTES;   // 8 MiB
constexpr int kMaxDevices = 64;

// The scratch area.  Host code must not use this symbol as a device address (on the
// host it names a host-side stand-in); it takes the address from
// cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

// Device address of g_static_ws per device, filled on the first call on that device.
void* g_ws_addr[kMaxDevices] = {nullptr};

}  // namespace

extern "C" moe_status moe_decode_static(const moe_shape* shape, int32_t T, const uint16_t* d_x,
                                        const float* d_router_w, const float* d_router_b, const void* d_packed,
                                        const moe_routing* out, uint16_t* d_y, void* stream) {
    if (!shape || T < 0) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (shape->hidden <= 0 || shape->inter <= 0 || shape->n_experts <= 0) return MOE_ERR_INVALID_ARG;
    // Everything the route and forward calls need must fit the fixed scratch area.
    if (moe::ws_layout(shape, T).total > kStaticWsBytes) return MOE_ERR_WORKSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    if (!g_ws_addr[dev]) {
        // Set-up, once per device, with that device current: the symbol's device address.
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || !p) return MOE_ERR_CUDA;
        g_ws_addr[dev] = p;
    }
    void* ws = g_ws_addr[dev];
    // The array keeps the previous call's contents: clear the control block and the
    // counters (the error word and the tickets must start at zero).
    moe_status st = moe_workspace_init(ws, kStaticWsBytes, stream);
    if (st != MOE_OK) return st;
    st = moe_route(shape, T, d_x, d_router_w, d_router_b, out, ws, kStaticWsBytes, stream);
    if (st != MOE_OK) return st;
    return moe_forward(shape, T, d_packed, d_x, out, d_y, MOE_PATH_DECODE, ws, kStaticWsBytes, stream);
}
