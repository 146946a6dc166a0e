// noalloc.cu -- la_seg_forward_noalloc: the forward pass for callers that cannot allocate
// device memory.  Its scratch is one file-scope device array of LA_NOALLOC_SCRATCH_BYTES that
// the CUDA module reserves on every GPU where this library is loaded, for the life of the
// process.  Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <mutex>

#include <cuda_runtime.h>

#include "internal.h"
#include "la_seg.h"

namespace {

// The shared scratch.  Host code must not use this name as a device address: on the host it
// is only a stand-in symbol; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per device.
cudaError_t scratch_address(int dev, void **out) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" la_status la_seg_forward_noalloc(const void *q, const void *k, const void *v,
                                            const void *log_g, const float *S0, int B, int H,
                                            long long L, int dk, int dv, int P, int chunk,
                                            la_dtype dt, void *o, float *S_final,
                                            float *S_recv_save, int schedule, void *cuda_stream) {
    const size_t need = la_seg_workspace_bytes(B, H, L, dk, dv, P, chunk, dt, 0);
    if (need == 0)  // sizes the library rejects: let the regular entry point name the reason
        return la_seg_forward(q, k, v, log_g, S0, B, H, L, dk, dv, P, chunk, dt, o, S_final,
                              S_recv_save, schedule, nullptr, 0, cuda_stream);
    if (need > (size_t)LA_NOALLOC_SCRATCH_BYTES)
        return la::set_error(LA_ERR_WORKSPACE,
                             "la_seg_forward_noalloc: these sizes need %zu bytes of scratch but "
                             "the static scratch holds %zu; use la_seg_forward with a workspace",
                             need, (size_t)LA_NOALLOC_SCRATCH_BYTES);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return la::set_cuda_error(e, "la_seg_forward_noalloc: cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices)
        return la::set_error(LA_ERR_ARG, "la_seg_forward_noalloc: device %d out of range", dev);
    void *scratch = nullptr;
    e = scratch_address(dev, &scratch);
    if (e != cudaSuccess)
        return la::set_cuda_error(e, "la_seg_forward_noalloc: cudaGetSymbolAddress");
    return la_seg_forward(q, k, v, log_g, S0, B, H, L, dk, dv, P, chunk, dt, o, S_final,
                          S_recv_save, schedule, scratch, (size_t)LA_NOALLOC_SCRATCH_BYTES,
                          cuda_stream);
}
