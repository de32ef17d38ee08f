// sbl_linear_noalloc: sbl_linear for callers that cannot allocate device memory.
//
// Some callers have no way to hand this library a workspace: a plugin whose
// host application owns the whole device-memory budget, a plain C caller with
// no allocator of its own, or a latency-critical path where a cudaMalloc could
// synchronise the device.  This entry point takes the same inputs and outputs
// as sbl_linear but keeps the scratch (the quantised activations and their
// per-token scales) in one fixed array of static device memory compiled into
// the library, so it allocates nothing at call time.
#include <cstdint>
#include <cuda_runtime.h>

#include "sbl.h"

namespace {

// The scratch array.  Every GPU that loads the library holds it until the
// process exits; all calls on a device share it.
static __device__ __align__(256) uint8_t g_noalloc_scratch[SBL_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the array on the current device.  The host-side symbol is
// only a stand-in: a kernel handed `g_noalloc_scratch` itself would fault or
// touch the wrong memory, so the address is asked for once per device.
sbl_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SBL_ERR_CUDA;
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SBL_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return SBL_OK;
}

}  // namespace

extern "C" sbl_status sbl_linear_noalloc(const uint16_t* x_bf16, int64_t T, int64_t K, const uint8_t* packed,
                                         const float* row_scale, int64_t O, int n, int m, void* y, int y_dtype,
                                         int32_t* acc_out, void* stream) {
    if (T < 0 || K <= 0) return SBL_ERR_INVALID_ARG;
    // quantised activations and token scales must fit; sbl_linear takes the
    // 2:4 sparse path only when the compressed weights fit as well
    const size_t need = ((static_cast<size_t>(T) * static_cast<size_t>(K) + 255) & ~static_cast<size_t>(255)) +
                        ((static_cast<size_t>(T) * 4 + 255) & ~static_cast<size_t>(255));
    if (need > static_cast<size_t>(SBL_NOALLOC_SCRATCH_BYTES)) return SBL_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (sbl_status s = scratch_address(&scratch)) return s;
    // Everything the kernels read from the scratch is written earlier in the
    // same call, so nothing needs clearing between calls.
    return sbl_linear(x_bf16, T, K, packed, row_scale, O, n, m, y, y_dtype, acc_out, scratch,
                      SBL_NOALLOC_SCRATCH_BYTES, stream);
}
