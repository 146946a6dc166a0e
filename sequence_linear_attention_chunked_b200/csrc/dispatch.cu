// dispatch.cu -- picks the kernel family for one chunk pass.
#include "internal.h"

namespace la {

cudaError_t launch_pass(const PassArgs &a, PassMode mode, cudaStream_t st) {
    return launch_simt_pass(a, mode, st);
}

}  // namespace la
