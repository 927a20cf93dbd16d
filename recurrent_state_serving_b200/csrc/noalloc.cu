// dl_decode_step_noalloc: the decode step for callers that cannot allocate device
// memory.  Its arrival counters live in the fixed array below instead of a
// caller-allocated buffer.  The paper has no counterpart; see deltalog.h.
#include <cstdint>

#include <cuda_runtime.h>

#include "deltalog.h"
#include "dl_internal.h"

#define DL_API extern "C" __attribute__((visibility("default")))

namespace dl {
dl_status check_desc_without_arrive(const dl_pool_desc &d);
dl_status check_decode_args(const dl_pool_desc &desc, int32_t layer, const dl_step_args *args);
dl_status decode_step_on_desc(const dl_pool_desc &desc, int32_t *arrive, int32_t layer,
                              const dl_step_args *args, int32_t auto_merge, void *stream);
}

namespace {

// One arrival counter per (slot, layer).  Every GPU that loads the library holds
// this array (DL_NOALLOC_MAX_COUNTERS * 4 bytes) until the process exits.
static __device__ __align__(256) int32_t g_arrive_scratch[DL_NOALLOC_MAX_COUNTERS];

// Device address of g_arrive_scratch in the current device's context.  In host code
// the array's name only stands in for the symbol, so the address is looked up with
// cudaGetSymbolAddress on every call: nothing is cached, so no host-side state is
// shared between threads and no address outlives a context torn down and made again.
// The first lookup on a device can load the module, so that first call belongs
// outside stream capture.
dl_status scratch_on_current_device(int32_t **out) {
    void *addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_arrive_scratch) != cudaSuccess || !addr) return DL_ERR_CUDA;
    *out = static_cast<int32_t *>(addr);
    return DL_OK;
}

}  // namespace

DL_API dl_status dl_decode_step_noalloc(const dl_pool_desc *desc, int32_t layer,
                                        const dl_step_args *args, int32_t auto_merge,
                                        void *stream) {
    if (!desc || !args) return DL_ERR_INVALID_ARG;
    const dl_status v = dl::check_desc_without_arrive(*desc);
    if (v != DL_OK) return v;
    const long long counters = (long long)desc->n_slots * desc->n_layers;
    if (counters > DL_NOALLOC_MAX_COUNTERS) return DL_ERR_SHAPE;
    // the step's own host-side checks come before any CUDA call
    const dl_status a = dl::check_decode_args(*desc, layer, args);
    if (a != DL_OK || args->batch == 0) return a;
    int32_t *scratch = nullptr;
    if (args->batch > 0) {
        const dl_status s = scratch_on_current_device(&scratch);
        if (s != DL_OK) return s;
        // The counters must start at zero; the array keeps whatever the last call left.
        if (cudaMemsetAsync(scratch, 0, (size_t)counters * sizeof(int32_t),
                            static_cast<cudaStream_t>(stream)) != cudaSuccess)
            return DL_ERR_CUDA;
    }
    return dl::decode_step_on_desc(*desc, scratch, layer, args, auto_merge, stream);
}
