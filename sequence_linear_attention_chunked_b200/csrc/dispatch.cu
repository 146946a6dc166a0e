// dispatch.cu -- picks the kernel family for one chunk pass: the tcgen05 kernels for the
// bf16 d=128 chunk=64 shape, the CUDA-core kernels for everything else (fp32 inputs, whose
// 1e-4 error bound bf16 tensor-core operands cannot meet, and the other d / chunk sizes).
#include "internal.h"

namespace la {

cudaError_t launch_pass(const PassArgs &a, PassMode mode, cudaStream_t st) {
    if (tc_pass_supported(a)) return launch_tc_pass(a, mode, st);
    return launch_simt_pass(a, mode, st);
}

cudaError_t launch_bwd_dstate(const BwdArgs &a, cudaStream_t st) { return launch_simt_dstate(a, st); }

cudaError_t launch_bwd_grad(const BwdArgs &a, cudaStream_t st) { return launch_simt_grad(a, st); }

}  // namespace la
