// dispatch.cu -- picks the kernel family for one chunk pass: the tcgen05 kernels for the
// bf16 d=128 chunk=64 shape, the CUDA-core kernels for everything else (fp32 inputs, whose
// 1e-4 error bound bf16 tensor-core operands cannot meet, and the other d / chunk sizes).
#include "internal.h"

namespace la {

cudaError_t launch_pass(const PassArgs &a, PassMode mode, cudaStream_t st) {
    if (tc_pass_supported(a)) return launch_tc_pass(a, mode, st);
    return launch_simt_pass(a, mode, st);
}

cudaError_t launch_bwd_dstate(const BwdArgs &a, cudaStream_t st) {
    PassArgs p = {};
    p.q = a.q; p.v = a.dO; p.g = a.g;  // the gradient-state pass reads dO through the v slot
    p.S_out = a.dSloc; p.logG = a.logG; p.status = a.status; p.flags = a.flags;
    p.L = a.L; p.T = a.T; p.BH = a.BH; p.NP = a.NP; p.dk = a.dk; p.dv = a.dv; p.chunk = a.chunk;
    p.dt = a.dt;
    if (tc_pass_supported(p)) return launch_tc_pass(p, kPassDState, st);
    return launch_simt_dstate(a, st);
}

// The tensor-core dq sweep also forms the fine parts' gradient states when a.dSloc and a.logG
// are given; the CUDA-core path runs the gradient-state pass over the fine split after it.
cudaError_t launch_bwd_dq(const BwdArgs &a, cudaStream_t st) {
    if (tc_bwd_supported(a)) return launch_tc_dq(a, st);
    cudaError_t e = launch_simt_dq(a, st);
    if (e != cudaSuccess || !a.dSloc || !a.logG) return e;
    BwdArgs f = a;
    f.NP = a.NP * a.fine;
    f.T = a.T / a.fine;
    f.fine = 1;
    return launch_bwd_dstate(f, st);
}

cudaError_t launch_bwd_dkv(const BwdArgs &a, cudaStream_t st) {
    return tc_bwd_supported(a) ? launch_tc_dkv(a, st) : launch_simt_dkv(a, st);
}

}  // namespace la
