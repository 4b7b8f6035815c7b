// static_ws.cu -- a variant of gdn_chunk_prefill for callers that cannot allocate device
// memory: its scratch is a file-scope device array owned by the library, so the caller
// passes only inputs and outputs.
//
// Who needs it: code whose host side is not allowed to allocate on the device, for
// example a serving loop that runs under a no-allocation rule (an allocation can
// synchronise the device and stall every stream), or code called back from another
// framework that owns the device memory pool and hands out no allocator.  The price is a
// fixed block of device memory held by every GPU that loads this library, for as long
// as the process lives, and a cap on problem size.
#include <cuda_runtime.h>

#include <mutex>

#include "gdn.h"
#include "gdn_internal.cuh"

namespace {

// The scratch itself.  Its size is the cap on what one call may need
// (GDN_STATIC_SCRATCH_BYTES in gdn.h).
static __device__ __align__(256) uint8_t g_static_scratch[GDN_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device.  In host code the array's
// name only stands in for the symbol; the real address comes from cudaGetSymbolAddress,
// looked up once per device (with that device current) and cached.
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" gdn_status gdn_chunk_prefill_static_ws(
    const void* q, const void* k, const void* v, gdn_dtype io_dtype, const float* g, const float* beta,
    const float* initial_state, const int32_t* cu_seqlens, int32_t B, int64_t T, int32_t n_seqs, int32_t HK,
    int32_t HV, int32_t Dk, int32_t Dv, int32_t BT, float scale, int32_t qk_l2norm, void* o, float* final_state,
    void* stream) {
    // the sizes are checked as gdn_chunk_prefill checks them, so both return the same status
    const gdn_status sz =
        gdn::prefill_check_sizes(io_dtype, cu_seqlens != nullptr, B, T, n_seqs, HK, HV, Dk, Dv, BT);
    if (sz != GDN_OK) return sz;
    const size_t need =
        gdn_chunk_prefill_workspace_bytes((int64_t)B * T, n_seqs, HK, HV, Dk, Dv, BT, io_dtype);
    if (need > (size_t)GDN_STATIC_SCRATCH_BYTES) return GDN_ERR_WORKSPACE;   // problem too large
    void* scratch = nullptr;
    const cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    return gdn_chunk_prefill(q, k, v, io_dtype, g, beta, initial_state, cu_seqlens, B, T, n_seqs, HK, HV, Dk,
                             Dv, BT, scale, qk_l2norm, o, final_state, scratch,
                             (size_t)GDN_STATIC_SCRATCH_BYTES, stream);
}
