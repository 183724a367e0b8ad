// moe_noalloc.cu -- the layer forward for callers that cannot allocate device memory.
//
// Some callers have no way to obtain a device buffer for the workspace: a plugin
// that runs inside a host framework whose allocator owns all device memory and
// exposes no handle, a runtime that forbids cudaMalloc on its latency-critical
// path because an allocation may block or fail, or code that must not grow the
// process's memory footprint after start-up.  moe_forward_noalloc serves them:
// it takes the workspace from a fixed-size array that is part of this library's
// device image, so the caller passes only inputs and outputs.
//
// The array costs MOE_NOALLOC_SCRATCH_BYTES of memory on every GPU that loads the
// library, held until the process exits.  Its address is looked up once per
// device (cudaGetSymbolAddress, on the first call made with that device current)
// and handed to the same launch sequence moe_forward uses.  That sequence clears
// the parts that must start at zero (the status word and the work-claim
// counters) and writes every other part before reading it.  All calls share the
// one array: calls whose work overlaps on the GPU (different streams, different
// host threads without ordering) race on it and must be serialised by the caller.
#include <mutex>

#include "moe_internal.h"

namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address must come from the
// runtime; it is looked up once per device and cached for the life of the
// process (a reset of the device would make the cached address stale, so no call
// may follow one).
moe_status_t scratch_on_current_device(void **ptr)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *ptr = g_scratch_ptr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" moe_status_t moe_forward_noalloc(const moe_dims_t *d, const void *x, const void *router_w,
                                            const float *router_bias, const void *w_gate, const void *w_up,
                                            const void *w_down, void *out, void *stream)
{
    const size_t need = moe_workspace_size(d, MOE_DTYPE_BF16);
    if (need == 0)  // invalid dims: let the regular entry point name the error
        return moe_forward(d, x, router_w, router_bias, w_gate, w_up, w_down, out, nullptr, 0, stream);
    if (need > MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_TOO_LARGE;
    if (d->T == 0) return MOE_OK;
    void *ws = nullptr;
    const moe_status_t s = scratch_on_current_device(&ws);
    if (s != MOE_OK) return s;
    return moe_forward(d, x, router_w, router_bias, w_gate, w_up, w_down, out, ws, MOE_NOALLOC_SCRATCH_BYTES,
                       stream);
}

// The status word sits at the start of the scratch, as at the start of any workspace.
extern "C" moe_status_t moe_noalloc_get_device_status(void *stream)
{
    void *ws = nullptr;
    const moe_status_t s = scratch_on_current_device(&ws);
    if (s != MOE_OK) return s;
    return moe_get_device_status(ws, stream);
}
