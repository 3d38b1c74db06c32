// kan_fixed_scratch.cu -- a forward entry point that allocates nothing.
//
// Some callers cannot allocate device memory at the point where they run the
// layer: code whose memory is handed out only by a framework's own caching
// allocator, long-running serving loops that must not stall on an allocation
// (cudaMalloc can synchronise the device and take driver locks), and hosts
// that budget all device memory up front.  kan_forward needs caller-provided
// workspace on the tensor-core path (split-K partial sums, and for fp32 the
// fp16 hi/lo copies of the coefficients).  kan_forward_fixed_scratch runs the
// same forward with that workspace taken from a fixed array that lives in this
// library's device image instead.
//
// Trade-offs, stated for users:
//   * every GPU that loads the library holds KAN_FIXED_SCRATCH_BYTES of device
//     memory for this array until the process exits;
//   * all calls share the one array, so two calls whose kernels overlap on
//     the GPU (different streams, no ordering between them) race on it; order
//     such calls on one stream or with events;
//   * the array keeps whatever the last call left in it; nothing the forward
//     reads from it needs to start at zero (every byte it reads was written
//     earlier in the same call);
//   * the first call on each device looks up the array's device address
//     (cudaGetSymbolAddress, with that device current); make that first call
//     before any stream capture begins.
#include <stdio.h>

#include <mutex>

#include "kan_internal.h"

namespace kan {
namespace {

// The fixed workspace.  In host code this name is only a stand-in for the
// symbol; its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_fixed_scratch[KAN_FIXED_SCRATCH_BYTES];

std::mutex g_mu;
void* g_addr[64] = {nullptr};

// Device address of g_fixed_scratch on the current device (looked up once per device).
kan_status fixed_scratch_address(void** out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_last_error(KAN_ERR_CUDA, "kan_forward_fixed_scratch: cudaGetDevice failed");
    if (dev < 0 || dev >= 64) return set_last_error(KAN_ERR_UNSUPPORTED, "kan_forward_fixed_scratch: device index >= 64");
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_fixed_scratch);
        if (e != cudaSuccess || !p) {
            char msg[256];
            snprintf(msg, sizeof(msg), "kan_forward_fixed_scratch: cudaGetSymbolAddress failed: %s",
                     cudaGetErrorString(e));
            return set_last_error(KAN_ERR_CUDA, msg);
        }
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return KAN_OK;
}

}  // namespace
}  // namespace kan

extern "C" kan_status kan_forward_fixed_scratch(const kan_shape* s, const void* x, const void* coef,
                                                const void* w_base, void* y, void* stream)
{
    size_t need = 0;
    kan_status st = kan_workspace_size(s, 0, &need);
    if (st != KAN_OK) return st;
    if (need > (size_t)KAN_FIXED_SCRATCH_BYTES) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "kan_forward_fixed_scratch: this shape needs %zu bytes of workspace, more than the %zu-byte fixed "
                 "scratch; call kan_forward with a caller-allocated workspace instead",
                 need, (size_t)KAN_FIXED_SCRATCH_BYTES);
        return kan::set_last_error(KAN_ERR_WORKSPACE, msg);
    }
    void* ws = nullptr;
    if (need > 0 && (st = kan::fixed_scratch_address(&ws)) != KAN_OK) return st;
    return kan_forward(s, x, coef, w_base, y, ws, need > 0 ? (size_t)KAN_FIXED_SCRATCH_BYTES : 0, stream);
}
