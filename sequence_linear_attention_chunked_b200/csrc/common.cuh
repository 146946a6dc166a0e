// common.cuh -- small device/host helpers shared by the CUDA kernels of libla_seg.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "la_seg.h"

namespace la {

// Bits of the device status word kept at the start of the workspace.
enum : int { kStatusGateRange = 1, kStatusTimeout = 2 };

// Value a sub-segment of the single-pass forward publishes instead of its index when it has no
// received state to pass on (a wait before it gave up); larger than every index.
constexpr int kChainPoison = 0x7FFFFFF0;

// |sum of log_g over one chunk| above this makes exp(b_t - b_C) / exp(b_C - b_s) leave the
// range where the chunk factorisation is accurate; the kernels flag it instead of returning
// inf/NaN silently.
constexpr float kGateRangeLimit = 80.0f;

// B200: 148 SMs.  Used by the host-side sub-segment policy so that workspace sizes do not
// depend on a device query.
constexpr int kNumSMs = 148;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Geometry of one forward/backward launch after the sub-segment split.
struct Split {
    int BH;         // B * H
    int P;          // API segments
    int m;          // internal sub-segments per API segment
    int NP;         // P * m sub-segments per (b, h)
    long long T;    // tokens per sub-segment
    long long L;
};

}  // namespace la
