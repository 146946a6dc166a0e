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

// The chunk factorisation scales q by exp(b_t - b_C) and k by exp(b_C - b_s) (b the in-chunk
// cumsum of log_g, b_C its total).  For log_g <= 0 every such exponent lies in [-|b_C|, |b_C|],
// so a chunk is inside the factorisation's range when no log_g in it is positive and
// |b_C| <= kGateRangeLimit in every key dim (e^80 ~ 5.5e34 leaves headroom below the fp32 / bf16
// overflow at e^88.7).  Every other chunk -- a positive gate exponent, a strong decay, a
// non-finite value -- is flagged rather than returned as inf/NaN: marked for the exact
// token-by-token path when the caller runs one, otherwise reported as LA_ERR_GATE_RANGE.
constexpr float kGateRangeLimit = 80.0f;

// Running max, as signed 16-bit halves, of packed bf16 words: a bf16 is > 0 (or +inf, or a NaN
// with the sign bit clear) exactly when its bits read as a positive int16.
__device__ __forceinline__ uint32_t pos_bf16_max(uint32_t m, const uint4 &w) {
    return __vmaxs2(m, __vmaxs2(__vmaxs2(w.x, w.y), __vmaxs2(w.z, w.w)));
}
__device__ __forceinline__ bool any_pos_bf16(uint32_t m) { return __vmaxs2(m, 0u) != 0u; }

// A unit (a segment or fine part) met a chunk outside the range: mark units [unit, unit + n) for
// the exact path when the caller passed flags, else OR kStatusGateRange into the status word.
__device__ __forceinline__ void flag_range(int *flags, long long unit, int n, int *status) {
    if (flags) {
        for (int i = 0; i < n; ++i) flags[unit + i] = 1;
    } else if (status) {
        atomicOr(status, kStatusGateRange);
    }
}

// B200: 148 SMs.  Used by the host-side sub-segment policy so that workspace sizes do not
// depend on a device query.
constexpr int kNumSMs = 148;

// Devices (by runtime ordinal) that the per-device state of the library covers: the overlap
// schedule's second stream and the no-alloc entry point's scratch address.
constexpr int kMaxDevices = 64;

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
