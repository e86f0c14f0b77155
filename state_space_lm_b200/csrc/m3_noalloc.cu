// m3_noalloc.cu -- the SISO chunked forward for callers that cannot allocate
// device memory.
//
// m3_siso_chunked_fwd takes its scratch from the caller.  Some callers have
// no allocator to get it from: code that runs inside a framework that owns
// all device memory, plugins and embedders that may not call cudaMalloc, and
// hosts that must not allocate between a warm-up and a latency-critical
// phase.  This entry point gives them the same computation with its scratch
// in a fixed buffer that is part of the library image: a file-scope
// __device__ array of M3_NOALLOC_SCRATCH_BYTES.  CUDA loads modules lazily,
// so a device commits the buffer at the first call there (the first symbol
// lookup loads this file's module) and keeps it until the process exits.
#include "m3_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[M3_NOALLOC_SCRATCH_BYTES];

// Device address of the buffer on the current device.  In host code the
// array's name is only a host-side stand-in, so the address comes from
// cudaGetSymbolAddress with that device current.  The lookup runs on every
// call (it allocates nothing once the module is loaded), so the address stays
// right after the caller resets the device and its context is recreated.
cudaError_t scratch_on_current_device(void **out) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    *out = p;
    return cudaSuccess;
}

}  // namespace

extern "C" m3_status m3_siso_chunked_fwd_noalloc(const void *x, const float *dt, const float *A, const float *lam,
                                                 const float *theta, const void *B, const void *C, const float *D,
                                                 m3_dtype dtype, const m3_bcnorm *norm, const float *h0,
                                                 const float *prevBx0, const float *angle0, m3_dims d, void *y,
                                                 float *h_final, float *prevBx_final, float *angle_final,
                                                 void *stream) {
    // sizes whose scratch exceeds the built-in buffer are rejected up front
    if (m3_workspace_bytes(M3_WS_SISO, d, dtype) > (size_t)M3_NOALLOC_SCRATCH_BYTES) return M3_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (scratch_on_current_device(&scratch) != cudaSuccess) return M3_ERR_CUDA;
    // Every part of the scratch that the kernels read is written earlier in the
    // same call, so no clearing is needed between calls.
    return m3_siso_chunked_fwd(x, dt, A, lam, theta, B, C, D, dtype, norm, h0, prevBx0, angle0, d, y, h_final,
                               prevBx_final, angle_final, scratch, (size_t)M3_NOALLOC_SCRATCH_BYTES, stream);
}
