// tc_common.cuh -- pieces shared by the tcgen05 chunk kernels (forward and backward):
// tile geometry, swizzled-tile addressing, UMMA descriptors for the two operand majors,
// bf16 packing and products, the fast exp2, the lane-pair output store, the layout of the q . dq
// hand-over, the copy of interleaved token pairs into tensor memory, and the TMA tensor-map
// encoder.
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
// with the 128-byte swizzle (16-byte chunk index XOR row % 8), the second half `hs` bytes after
// the first (kHalfBytes when the halves are adjacent).
__device__ __forceinline__ uint32_t tile_off(int t, int i, int hs = kHalfBytes) {
    const int half = i >> 6, ii = i & 63;
    return (uint32_t)(half * hs + t * 128 + (((ii >> 3) ^ (t & 7)) << 4) + ((ii & 7) << 1));
}

// Descriptor of a K-major operand (rows x 128 K-elements, two swizzle halves `hs` bytes apart)
// at K-step kk.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t base, int kk, int hs = kHalfBytes) {
    return smem_desc_sw128(base + (uint32_t)((kk >> 2) * hs + (kk & 3) * 32), 16, 1024);
}
// Descriptor of an MN-major operand ([64 K-rows] x 128 MN-elements, two halves `hs` bytes
// apart) at K-step kk.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t base, int kk, int hs = kHalfBytes) {
    return smem_desc_sw128(base + (uint32_t)(kk * 2048), (uint32_t)hs, 1024);
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

// Two bf16 products (low and high halves), each rounded once to nearest-even: the product of two
// bf16 values is exact in fp32, so this equals pack_bf16 of the fp32 products.
__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Tokens t0 and t0+1 of this lane's dim (a warp's 32 lanes hold 32 consecutive dims, lane l dim
// dim0 + l) into a row-major [tokens][128] bf16 tensor with one 4-byte store per lane: lanes l
// and l ^ 1 trade one half, so that the even lane writes dims l, l+1 of token t0 and the odd
// lane dims l-1, l of token t0+1.  `row0` points at element (t0, dim0).  Called by all 32 lanes.
__device__ __forceinline__ void st_pair_bf16(__nv_bfloat16 *row0, int lane, float v0, float v1) {
    const uint32_t p = pack_bf16(v0, v1);  // low half: token t0, high half: token t0+1
    const bool odd = lane & 1;
    const uint32_t got = __shfl_xor_sync(0xFFFFFFFFu, p, 1);
    // even: (own t0, partner t0) = dims l, l+1 of t0; odd: (partner t0+1, own t0+1)
    const uint32_t w = __byte_perm(p, got, odd ? 0x3276u : 0x5410u);
    *reinterpret_cast<uint32_t *>(row0 + (lane & 1) * D + (lane & ~1)) = w;
}

// The fp32 q . dq hand-over between the dq sweep and the reverse sweep is kept token-quad
// interleaved: element (row r, dim i) of a [rows][128] block at ((r / 4) * 128 + i) * 4 + r % 4,
// so that the thread owning dim i reads or writes four consecutive tokens as one float4 and a
// warp's 32 dims make one 512-byte access.  Returns the float4 of rows 4 rq .. 4 rq + 3.
__device__ __forceinline__ float4 *qdq_quad(float *ws, long long rq, int i) {
    return reinterpret_cast<float4 *>(ws) + rq * D + i;
}

// A chunk's 64 pairs (lo, hi) for each of this warp's 32 key dims, lo from the bf16 stage tile at
// tile_lo and hi from the one at tile_hi (both [64 tokens][128 dims], tile_off layout with the
// half strides hs_lo, hs_hi), into TMEM as one word lo | hi << 16 per (dim, token): lane = dim
// (the warp's quarter), column = token from taddr's column.  ldmatrix with .trans gives thread l tokens 2(l%4) and 2(l%4)+1 of
// dim l/4 in each 8x8 block, which is how the 16x256b store lays its registers out; the eight
// row reads of one block fall on eight different 16-byte bank groups under the swizzle.
__device__ __forceinline__ void copy_pairs_to_tmem(uint32_t tile_lo, uint32_t tile_hi,
                                                   uint32_t taddr, int quarter, int lane,
                                                   int hs_lo = kHalfBytes, int hs_hi = kHalfBytes) {
    const int dim0 = quarter * 32 + (lane >> 3) * 8;  // block lane / 8: dims dim0 .. dim0 + 7
    const int r = lane & 7;                           // the block row this lane addresses
    const uint32_t row = (uint32_t)(r * 128 + ((((dim0 & 63) >> 3) ^ r) << 4));
    const uint32_t lo = tile_lo + (uint32_t)((dim0 >> 6) * hs_lo) + row;
    const uint32_t hi = tile_hi + (uint32_t)((dim0 >> 6) * hs_hi) + row;
#pragma unroll
    for (int t0 = 0; t0 < CH; t0 += 8) {  // tokens t0 .. t0+7 (row t0 + r, and (t0 + r) % 8 = r)
        uint32_t a[4], b[4];
        ldsm_x4_trans(lo + t0 * 128, a);
        ldsm_x4_trans(hi + t0 * 128, b);
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
