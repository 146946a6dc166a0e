// noalloc.cu -- la_seg_forward_noalloc: the forward pass for callers that cannot allocate
// device memory.  Its scratch is one file-scope device array of LA_NOALLOC_SCRATCH_BYTES that
// the CUDA module reserves on every GPU where this library is loaded, for the life of the
// process.  Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "la_seg.h"

namespace {

// The shared scratch.  Host code must not use this name as a device address: on the host it
// is only a stand-in symbol; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LA_NOALLOC_SCRATCH_BYTES];

// The address is cached per device together with the unique id of the context it was looked
// up in.  cudaDeviceReset (or any other re-creation of the primary context) reloads the module,
// so the array may move; a changed context id makes the next call look it up again.
struct ScratchAddr {
    bool valid = false;
    unsigned long long ctx_id = 0;
    void *addr = nullptr;
};
std::mutex g_setup_mutex;
ScratchAddr g_scratch[la::kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

template <typename Fn>
Fn driver_fn(const char *name) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<Fn>(p);
}

// Unique id of the calling thread's current context; false when there is none (or the driver
// cannot say), in which case the caller looks the address up again.
bool current_ctx_id(unsigned long long *id) {
    static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    if (!get_current || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch on device `dev`, which must be current.  Looked up with
// cudaGetSymbolAddress on the first call per device and again whenever the device's context
// has been re-created since.
cudaError_t scratch_address(int dev, void **out) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    ScratchAddr &s = g_scratch[dev];
    unsigned long long id = 0;
    const bool have_id = current_ctx_id(&id);
    if (!s.valid || !have_id || s.ctx_id != id) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // creates the context if needed
        if (e != cudaSuccess) return e;
        s.valid = current_ctx_id(&s.ctx_id);  // cache only when the context is known
        s.addr = p;
    }
    *out = s.addr;
    return cudaSuccess;
}

la_status current_scratch(const char *who, void **scratch) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return la::set_cuda_error(e, who);
    if (dev < 0 || dev >= la::kMaxDevices)
        return la::set_error(LA_ERR_ARG, "%s: device %d is beyond the %d devices this library serves",
                             who, dev, la::kMaxDevices);
    e = scratch_address(dev, scratch);
    if (e != cudaSuccess) return la::set_cuda_error(e, who);
    return LA_OK;
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
    void *scratch = nullptr;
    la_status st = current_scratch("la_seg_forward_noalloc", &scratch);
    if (st != LA_OK) return st;
    return la_seg_forward(q, k, v, log_g, S0, B, H, L, dk, dv, P, chunk, dt, o, S_final,
                          S_recv_save, schedule, scratch, (size_t)LA_NOALLOC_SCRATCH_BYTES,
                          cuda_stream);
}

// The status word sits at the start of the static scratch, where la_seg_forward keeps it in a
// workspace; reading it needs the scratch's device address, which callers cannot name.
extern "C" la_status la_seg_noalloc_check_status(void *cuda_stream) {
    void *scratch = nullptr;
    la_status st = current_scratch("la_seg_noalloc_check_status", &scratch);
    if (st != LA_OK) return st;
    return la_seg_check_status(scratch, cuda_stream);
}
