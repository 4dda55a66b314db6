// still_hybrid_prefill_static: the prefill with its scratch in a fixed device array of this module
// instead of a caller-provided workspace, so that the call allocates no memory of any kind.
//
// The array lives in its own translation unit (its own CUDA module): under lazy module loading it is
// only reserved on a device once this entry point is first used there.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "still.h"
#include "still_internal.h"

static __device__ __align__(256) unsigned char g_prefill_scratch[STILL_STATIC_WORKSPACE_BYTES];

namespace {

constexpr int kMaxDevices = 128;  // device ordinals 0..127, as for the device status word
std::atomic<void *> g_scratch_addr[kMaxDevices];

// Address of the current device's copy of the array, looked up once per device with that device
// current.  The first lookup may load this module; it must not happen during stream capture.
still_status scratch_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return STILL_ERR_CUDA;
    void *p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_prefill_scratch) != cudaSuccess || !p) {
            (void)cudaGetLastError();
            return STILL_ERR_CUDA;
        }
        g_scratch_addr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return STILL_OK;
}

}  // namespace

extern "C" STILL_API still_status still_hybrid_prefill_static(const still_dims *dims, const void *q, const void *k,
                                                              const void *v, const void *Wq, const void *Wk, void *o,
                                                              const int32_t *idx_in, void *state, int state_capacity,
                                                              void *stream) {
    // the regular entry point's checks first, in its order, so that both report the same error
    bool empty = false;
    still_status chk = still::check_prefill_args(dims, q, k, v, Wq, Wk, o, idx_in, state, state_capacity, &empty);
    if (chk || empty) return chk;
    const size_t need = still_prefill_workspace_bytes(dims);
    if (need > (size_t)STILL_STATIC_WORKSPACE_BYTES) return STILL_ERR_WORKSPACE;
    void *scratch = nullptr;
    const still_status st = scratch_address(&scratch);
    if (st) return st;
    return still_hybrid_prefill(dims, q, k, v, Wq, Wk, o, idx_in, scratch, (size_t)STILL_STATIC_WORKSPACE_BYTES,
                                state, state_capacity, stream);
}
