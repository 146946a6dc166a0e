// tc_common.cuh -- pieces shared by the tcgen05 chunk kernels (forward and backward):
// tile geometry, swizzled-tile addressing, UMMA descriptors for the two operand majors,
// bf16 packing, the fast exp2, and the TMA tensor-map encoder.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "sm100.cuh"

namespace la {
namespace tc {

using namespace sm100;

constexpr int D = 128;                 // d_k = d_v
constexpr int CH = 64;                 // tokens per chunk
constexpr int kHalfBytes = CH * 64 * 2;  // one 64-column swizzle half of a tile: 8 KB
constexpr int kTileBytes = 2 * kHalfBytes;
constexpr float kLog2e = 1.4426950408889634f;

constexpr uint32_t kTmemCols = 512;  // every tensor-core kernel allocates all of it

// Byte offset of element (t, i) of a [64 x 128] bf16 tile TMA-loaded as two 64-column halves
// with the 128-byte swizzle (16-byte chunk index XOR row % 8).
__device__ __forceinline__ uint32_t tile_off(int t, int i) {
    const int half = i >> 6, ii = i & 63;
    return (uint32_t)(half * kHalfBytes + t * 128 + (((ii >> 3) ^ (t & 7)) << 4) + ((ii & 7) << 1));
}

// Descriptor of a K-major operand (rows x 128 K-elements, two swizzle halves) at K-step kk.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t base, int kk) {
    return smem_desc_sw128(base + (uint32_t)((kk >> 2) * kHalfBytes + (kk & 3) * 32), 16, 1024);
}
// Descriptor of an MN-major operand ([64 K-rows] x 128 MN-elements, two halves) at K-step kk.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t base, int kk) {
    return smem_desc_sw128(base + (uint32_t)(kk * 2048), kHalfBytes, 1024);
}

__device__ __forceinline__ bool wait_drain(uint64_t *bar, uint32_t parity) {
    int dummy = 0;
    return mbar_wait(bar, parity, &dummy);
}

// Waits by a whole warp; the answer is the same in every lane.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
    return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, abort));
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        f[2 * e] = __uint_as_float(w[e] << 16);
        f[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// [rows, 128] bf16 view, 64 x 64 boxes, 128-byte swizzle.
inline cudaError_t make_map(CUtensorMap *m, const void *base, long long rows) {
    auto fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)CH};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// [rows, 128] fp32 view, 32 x 128 boxes (one 128-byte row segment per row), 128-byte swizzle.
inline cudaError_t make_map_f32_rows(CUtensorMap *m, const void *base, long long rows) {
    auto fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 4};
    const cuuint32_t box[2] = {32, 128};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace tc
}  // namespace la
