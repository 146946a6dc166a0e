// tc_common.cuh -- pieces shared by the tcgen05 chunk kernels (forward and backward):
// tile geometry, swizzled-tile addressing, UMMA descriptors for the two operand majors,
// bf16 packing, the fast exp2, the copy of interleaved token pairs into tensor memory, and the
// TMA tensor-map encoder.
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

// A chunk's 64 pairs (lo, hi) for each of this warp's 32 key dims, lo from the bf16 stage tile at
// tile_lo and hi from the one at tile_hi (both [64 tokens][128 dims], tile_off layout), into
// TMEM as one word lo | hi << 16 per (dim, token): lane = dim (the warp's quarter), column =
// token from taddr's column.  ldmatrix with .trans gives thread l tokens 2(l%4) and 2(l%4)+1 of
// dim l/4 in each 8x8 block, which is how the 16x256b store lays its registers out; the eight
// row reads of one block fall on eight different 16-byte bank groups under the swizzle.
__device__ __forceinline__ void copy_pairs_to_tmem(uint32_t tile_lo, uint32_t tile_hi,
                                                   uint32_t taddr, int quarter, int lane) {
    const int dim0 = quarter * 32 + (lane >> 3) * 8;  // block lane / 8: dims dim0 .. dim0 + 7
    const int r = lane & 7;                           // the block row this lane addresses
    const uint32_t row = (uint32_t)((dim0 >> 6) * kHalfBytes + r * 128 +
                                    ((((dim0 & 63) >> 3) ^ r) << 4));
#pragma unroll
    for (int t0 = 0; t0 < CH; t0 += 8) {  // tokens t0 .. t0+7 (row t0 + r, and (t0 + r) % 8 = r)
        uint32_t a[4], b[4];
        ldsm_x4_trans(tile_lo + row + t0 * 128, a);
        ldsm_x4_trans(tile_hi + row + t0 * 128, b);
        uint32_t w[8];  // per block: the pair of token 2(l%4), then of token 2(l%4)+1
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            w[2 * m] = __byte_perm(a[m], b[m], 0x5410);
            w[2 * m + 1] = __byte_perm(a[m], b[m], 0x7632);
        }
        const uint32_t ta = taddr + ((uint32_t)(quarter * 32) << 16) + (uint32_t)t0;
        tmem_st_16x256b(ta, w[0], w[1], w[2], w[3]);                // dims +0 .. +15
        tmem_st_16x256b(ta + (16u << 16), w[4], w[5], w[6], w[7]);  // dims +16 .. +31
    }
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
