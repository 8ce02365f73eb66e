// moe_layer_static_ws: the whole layer without a caller-provided workspace.
//
// Some callers cannot allocate device memory: programs whose device memory is
// owned by another allocator (a serving framework's pool or an arena fixed at
// start-up, where an extra cudaMalloc would break the memory budget), latency-
// critical decode loops that must not pay for cudaMalloc / cudaFree (both can
// synchronise the device and stall other streams), and deployments that forbid
// any allocation after initialisation. For them this entry point takes its
// scratch from one array compiled into the library instead of from `ws`.
//
// The array is a file-scope __device__ object, so every GPU that loads the
// library holds MOE_STATIC_WS_BYTES of it until the process exits. Host code
// must not pass the array's symbol to a kernel (on the host it is only a
// stand-in, not a device address): its device address is looked up once per
// device with cudaGetSymbolAddress, with that device current, on the first
// call made on that device.
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace {

static __device__ __align__(256) unsigned char g_static_ws[MOE_STATIC_WS_BYTES];

constexpr int kMaxDevices = 64;
std::atomic<void *> g_static_ws_addr[kMaxDevices];

// Device address of g_static_ws on the current device (set-up on first use).
moe_status static_ws_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    void *p = g_static_ws_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        const cudaError_t e = cudaGetSymbolAddress(&p, g_static_ws);
        if (e != cudaSuccess || !p) return MOE_ERR_CUDA;
        g_static_ws_addr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_layer_static_ws(const moe_dims *dims, const moe_weights *weights, const uint16_t *x,
                                          const int32_t *token_ids, float *y, void *stream) {
    size_t need = 0;
    moe_status st = moe_workspace_size(dims, &need);
    if (st != MOE_OK) return st;
    if (need > (size_t)MOE_STATIC_WS_BYTES) return MOE_ERR_INVALID_ARG;  // too large for the built-in array
    void *ws = nullptr;
    if ((st = static_ws_address(&ws)) != MOE_OK) return st;
    return moe_layer(dims, weights, x, token_ids, y, ws, stream);
}
