// scan.cu -- exclusive decayed scan of fp32 dk x dv states across segments.
//
// The All-Scan state update of the ZeCO review ("key machinery", Alg. 2 as the referee
// corrects it: the accumulated state moves on, not the local one), run on one device:
//
//   acc = init;  for p in order:  out[p] = acc;  acc = exp(log_gamma[p][i]) * acc + S_in[p]
//
// Rows i (and columns j) are independent, so the scan is element-parallel over (bh, i, j) and
// sequential over p.  It is HBM-bound.  The main kernel (scan_bulk_kernel, below) streams the
// states through shared memory by bulk copies; the per-thread kernel (scan_kernel) takes the
// shapes its 1024-float slices do not cover, each thread streaming float4 states with the loads
// of kUnroll segments issued before the dependent FMA chain consumes them.  Both keep one fma
// per element and segment in the same order, so they agree bit for bit.  Splitting d_k into
// blocks (the review's K blocks of All-Scan) changes nothing here: each element's chain is the
// same whatever the block split.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace la {
namespace {

using namespace sm100;

// Per-thread kernel: 128-thread blocks, and a 4-deep batch for the carry variant, so that a
// grid of ~7 blocks per SM stays at one wave.
constexpr int kScanThreads = 128;
constexpr int kUnroll = 8;

// With `carry` (the backward's reverse scan): carry[bh][p][i] = sum_j S_end_p[i][j] out[p][i][j],
// S_end_p = S_next[p+1] (p < NP-1) or S_last (p = NP-1; null: zero) -- the dlog_g carry of part
// p.  The threads of one row i are dv4 consecutive lanes of a warp, so the sum over j is a
// segmented warp reduction.  The xor butterfly over offsets below dv4 keeps to one row only
// when dv4 = dv / 4 is a power of two that divides 32 (dv in {4, 8, .., 128}) and rows start
// on dv4-lane boundaries (dk * dv4 a multiple of 32); launch_scan and la_seg_scan refuse any
// other dv with a carry.
template <bool CARRY>
__global__ void __launch_bounds__(kScanThreads)
scan_kernel(const float4 *__restrict__ S_in, const float *__restrict__ log_gamma,
            const float4 *__restrict__ init, int BH, int NP, int dk, int dv4, int reverse,
            float4 *__restrict__ out, float4 *__restrict__ final_state,
            const float4 *__restrict__ S_next, const float4 *__restrict__ S_last,
            float *__restrict__ carry) {
    const long long e = (long long)blockIdx.x * kScanThreads + threadIdx.x;  // (bh, i, j4)
    const long long per_bh = (long long)dk * dv4;
    if (e >= (long long)BH * per_bh) return;
    const long long bh = e / per_bh;
    const long long ij = e % per_bh;
    const int i = (int)(ij / dv4);
    const float4 *src = S_in + bh * NP * per_bh + ij;
    float4 *dst = out + bh * NP * per_bh + ij;
    const float *lg = log_gamma + bh * (long long)NP * dk + i;

    float4 acc = init ? init[bh * per_bh + ij] : make_float4(0.f, 0.f, 0.f, 0.f);
    constexpr int kU = CARRY ? 4 : kUnroll;
    for (int p0 = 0; p0 < NP; p0 += kU) {
        float4 x[kU], se[CARRY ? kU : 1];
        float gm[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int p = p0 + u;
            if (p < NP) {
                const int pp = reverse ? NP - 1 - p : p;
                x[u] = __ldcs(src + (long long)pp * per_bh);
                gm[u] = __expf(lg[(long long)pp * dk]);
                if (CARRY) {
                    const float4 *e4 = pp + 1 < NP ? S_next + (bh * NP + pp + 1) * per_bh + ij
                                                   : (S_last ? S_last + bh * per_bh + ij : nullptr);
                    se[CARRY ? u : 0] = e4 ? *e4 : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int p = p0 + u;
            if (p < NP) {
                const int pp = reverse ? NP - 1 - p : p;
                __stcs(dst + (long long)pp * per_bh, acc);
                if (CARRY) {
                    const float4 &v = se[CARRY ? u : 0];
                    float sum = fmaf(v.w, acc.w, fmaf(v.z, acc.z, fmaf(v.y, acc.y, v.x * acc.x)));
                    for (int o = 1; o < dv4; o <<= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
                    if (ij % dv4 == 0) carry[(bh * NP + pp) * dk + i] = sum;
                }
                acc.x = fmaf(gm[u], acc.x, x[u].x);
                acc.y = fmaf(gm[u], acc.y, x[u].y);
                acc.z = fmaf(gm[u], acc.z, x[u].z);
                acc.w = fmaf(gm[u], acc.w, x[u].w);
            }
        }
    }
    if (final_state) final_state[bh * per_bh + ij] = acc;
}

// ---- the scan fed by bulk copies ------------------------------------------------------------
// One CTA per (bh, slice of kSlice consecutive floats of the dk x dv state).  A producer thread
// streams each segment's slice and the log-decays of the slice's rows (and, for the carry, the
// matching slice of the segment's end state) into a ring of shared memory with bulk copies: the
// copy engine keeps the bytes of many segments in flight, where per-thread loads capped a
// 16-head scan at about half the bandwidth a plain copy reaches.  Thread t of the 128 carries
// elements 8t .. 8t+7 of the slice (one row, since dv >= 32) through the recurrence and stores
// out[p] straight to HBM.  12 stages (6 with the end states) keep four CTAs per SM resident, so
// a 32-head grid of 512 CTAs is a single wave.
constexpr int kSlice = 1024, kSliceThreads = 128;
constexpr int kSliceBytes = kSlice * 4, kLgBytes = 128;  // a slice has kSlice / dv <= 32 rows

template <bool CARRY> struct SliceRing {
    static constexpr int stages = CARRY ? 6 : 12;
    static constexpr int off_end = kSliceBytes;                       // end-state slice (carry)
    static constexpr int off_lg = kSliceBytes * (CARRY ? 2 : 1);
    static constexpr int stage = off_lg + kLgBytes;
    static constexpr int smem = stages * stage + 2 * stages * 8 + 16;
};

__device__ __forceinline__ float4 vfma4(float g, const float4 &a, const float4 &x) {
    return make_float4(fmaf(g, a.x, x.x), fmaf(g, a.y, x.y), fmaf(g, a.z, x.z), fmaf(g, a.w, x.w));
}

// With CARRY (the backward's reverse scan): carry[bh][p][i] = sum_j S_end_p[i][j] out[p][i][j],
// S_end_p = S_next[p+1] (p < NP-1) or S_last (p = NP-1; null: zero), summed in the order of the
// per-thread kernel: a 4-term fma chain per group of 4 columns, then a pairwise tree over the
// row's groups (the thread's two groups first, then across the dv / 8 lanes of the row), which
// la_seg_dkv_pass reproduces when it forms the carry itself.
template <bool CARRY>
__global__ void __launch_bounds__(kSliceThreads + 32)
scan_bulk_kernel(const float *__restrict__ S_in, const float *__restrict__ log_gamma,
                 const float *__restrict__ init, int NP, int dk, int dv, int reverse,
                 float *__restrict__ out, float *__restrict__ final_state,
                 const float *__restrict__ S_next, const float *__restrict__ S_last,
                 float *__restrict__ carry, int *status) {
    using R = SliceRing<CARRY>;
    extern __shared__ __align__(128) uint8_t sm[];
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + R::stages * R::stage);
    uint64_t *empty = full + R::stages;
    volatile int *abort = reinterpret_cast<volatile int *>(empty + R::stages);
    const int nsl = dk * dv / kSlice;
    const long long bh = blockIdx.x / nsl;
    const int sl = blockIdx.x % nsl;
    const int rows = kSlice / dv, row0 = sl * rows;
    const long long state = (long long)dk * dv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < R::stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kSliceThreads / 32);
        }
        *abort = 0;
        mbar_fence_init();
    }
    __syncthreads();
    if (warp == kSliceThreads / 32) {  // the producer
        if (lane == 0) {
            int issued = 0;
            for (int p = 0; p < NP; ++p) {
                const int s = p % R::stages;
                if (p >= R::stages && !mbar_wait(&empty[s], ((p / R::stages) - 1) & 1, abort))
                    break;
                const long long pp = reverse ? NP - 1 - p : p;
                uint8_t *st = sm + s * R::stage;
                const float *end = nullptr;
                if (CARRY)
                    end = pp + 1 < NP ? S_next + (bh * NP + pp + 1) * state
                                      : (S_last ? S_last + bh * state : nullptr);
                mbar_arrive_expect_tx(&full[s], kSliceBytes + rows * 4 + (end ? kSliceBytes : 0));
                bulk_load(st, S_in + (bh * NP + pp) * state + (long long)sl * kSlice, kSliceBytes,
                          &full[s]);
                bulk_load(st + R::off_lg, log_gamma + (bh * NP + pp) * dk + row0, rows * 4,
                          &full[s]);
                if (end) bulk_load(st + R::off_end, end + (long long)sl * kSlice, kSliceBytes, &full[s]);
                issued = p + 1;
            }
            if (*abort) {  // let the copies this CTA started land before it exits
                int ignore = 0;
                for (int p = issued > R::stages ? issued - R::stages : 0; p < issued; ++p)
                    mbar_wait(&full[p % R::stages], (p / R::stages) & 1, &ignore);
            }
        }
        return;
    }
    const int e0 = threadIdx.x * 8;
    const int r = e0 / dv;
    const long long gofs = (long long)sl * kSlice + e0;
    float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
    if (init) {
        const float4 *ip = reinterpret_cast<const float4 *>(init + bh * state + gofs);
        a0 = ip[0];
        a1 = ip[1];
    }
    const int row_lanes = dv / 8;  // lanes that share a row: a power of two dividing 32
    bool ok = true;
    for (int p = 0; p < NP; ++p) {
        const int s = p % R::stages;
        if (!(ok = __all_sync(0xFFFFFFFFu, mbar_wait(&full[s], (p / R::stages) & 1, abort))))
            break;
        const long long pp = reverse ? NP - 1 - p : p;
        const uint8_t *st = sm + s * R::stage;
        const float4 x0 = *reinterpret_cast<const float4 *>(st + e0 * 4);
        const float4 x1 = *reinterpret_cast<const float4 *>(st + e0 * 4 + 16);
        const float g = __expf(*reinterpret_cast<const float *>(st + R::off_lg + r * 4));
        float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
        if (CARRY && (pp + 1 < NP || S_last)) {
            v0 = *reinterpret_cast<const float4 *>(st + R::off_end + e0 * 4);
            v1 = *reinterpret_cast<const float4 *>(st + R::off_end + e0 * 4 + 16);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);  // this warp's reads of the stage are done
        float4 *op = reinterpret_cast<float4 *>(out + (bh * NP + pp) * state + gofs);
        __stcs(op, a0);
        __stcs(op + 1, a1);
        if (CARRY) {
            float sum = fmaf(v0.w, a0.w, fmaf(v0.z, a0.z, fmaf(v0.y, a0.y, v0.x * a0.x))) +
                        fmaf(v1.w, a1.w, fmaf(v1.z, a1.z, fmaf(v1.y, a1.y, v1.x * a1.x)));
            for (int o = 1; o < row_lanes; o <<= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
            if ((lane & (row_lanes - 1)) == 0) carry[(bh * NP + pp) * dk + row0 + r] = sum;
        }
        a0 = vfma4(g, a0, x0);
        a1 = vfma4(g, a1, x1);
    }
    if (!ok) {
        if (status && lane == 0) atomicOr(status, kStatusTimeout);
        return;
    }
    if (final_state) {
        float4 *fp = reinterpret_cast<float4 *>(final_state + bh * state + gofs);
        fp[0] = a0;
        fp[1] = a1;
    }
}

__global__ void gather_states_kernel(const float4 *__restrict__ src, int BH, int NP, int m,
                                     long long per_state4, float4 *__restrict__ dst) {
    const int P = NP / m;
    const long long n = (long long)BH * P * per_state4;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x) {
        const long long bhp = e / per_state4, r = e % per_state4;
        const long long bh = bhp / P, p = bhp % P;
        dst[e] = src[(bh * NP + p * m) * per_state4 + r];
    }
}

__global__ void copy_state_kernel(const float4 *__restrict__ src, long long n4,
                                  float4 *__restrict__ dst) {
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n4;
         e += (long long)gridDim.x * blockDim.x)
        dst[e] = src ? src[e] : make_float4(0.f, 0.f, 0.f, 0.f);
}

}  // namespace

cudaError_t launch_scan(const float *S_in, const float *log_gamma, const float *init, int BH,
                        int NP, int dk, int dv, int reverse, float *out, float *final_state,
                        cudaStream_t st, const float *S_next, const float *S_last, float *carry,
                        int *status) {
    // bulk path: whole slices of whole rows, >= 4 rows per slice (16-byte log-decay copies; a
    // row's lanes within one warp), 16-byte aligned log-decay rows
    if (dk % 4 == 0 && (dk * dv) % kSlice == 0 && kSlice % dv == 0 && kSlice / dv >= 4 &&
        kSlice / dv * 4 <= kLgBytes && reinterpret_cast<uintptr_t>(log_gamma) % 16 == 0) {
        const long long nblk = (long long)BH * (dk * dv / kSlice);
        if (nblk == 0 || NP == 0) {
            if (NP == 0 && final_state && BH > 0)  // no segments: the final state is the start
                return launch_copy_state(init, BH, dk, dv, final_state, st);
            return cudaSuccess;
        }
        auto kern = carry ? scan_bulk_kernel<true> : scan_bulk_kernel<false>;
        const int smem = carry ? SliceRing<true>::smem : SliceRing<false>::smem;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)nblk, kSliceThreads + 32, smem, st>>>(S_in, log_gamma, init, NP, dk, dv,
                                                              reverse, out, final_state, S_next,
                                                              S_last, carry, status);
        return cudaGetLastError();
    }
    if (carry && (dv % 4 || 32 % (dv / 4) || (dk * (dv / 4)) % 32)) return cudaErrorInvalidValue;
    const int dv4 = dv / 4;
    const long long n = (long long)BH * dk * dv4;
    if (n == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((n + kScanThreads - 1) / kScanThreads);
    auto S_in4 = reinterpret_cast<const float4 *>(S_in);
    auto init4 = reinterpret_cast<const float4 *>(init);
    auto out4 = reinterpret_cast<float4 *>(out);
    auto fin4 = reinterpret_cast<float4 *>(final_state);
    if (carry)  // whole warps per row: dv4 divides 32 and blocks hold whole rows
        scan_kernel<true><<<blocks, kScanThreads, 0, st>>>(
            S_in4, log_gamma, init4, BH, NP, dk, dv4, reverse, out4, fin4,
            reinterpret_cast<const float4 *>(S_next), reinterpret_cast<const float4 *>(S_last), carry);
    else
        scan_kernel<false><<<blocks, kScanThreads, 0, st>>>(S_in4, log_gamma, init4, BH, NP, dk,
                                                            dv4, reverse, out4, fin4, nullptr,
                                                            nullptr, nullptr);
    return cudaGetLastError();
}

cudaError_t launch_gather_states(const float *src, int BH, int NP, int m, int dk, int dv,
                                 float *dst, cudaStream_t st) {
    const long long per4 = (long long)dk * dv / 4;
    const long long n = (long long)BH * (NP / m) * per4;
    if (n == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
    gather_states_kernel<<<blocks, 256, 0, st>>>(reinterpret_cast<const float4 *>(src), BH, NP, m,
                                                 per4, reinterpret_cast<float4 *>(dst));
    return cudaGetLastError();
}

cudaError_t launch_copy_state(const float *src, int BH, int dk, int dv, float *dst,
                              cudaStream_t st) {
    const long long n4 = (long long)BH * dk * dv / 4;
    if (n4 == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((n4 + 255) / 256 < 4096 ? (n4 + 255) / 256 : 4096);
    copy_state_kernel<<<blocks, 256, 0, st>>>(reinterpret_cast<const float4 *>(src), n4,
                                              reinterpret_cast<float4 *>(dst));
    return cudaGetLastError();
}

}  // namespace la

namespace la {
namespace {
__global__ void chain_reset_kernel(const float4 *__restrict__ S0, int BH, long long per4,
                                   float4 *__restrict__ states, int *__restrict__ ready) {
    const int bh = blockIdx.x;
    for (long long e = threadIdx.x; e < per4; e += blockDim.x)
        states[(long long)bh * 2 * per4 + e] = S0 ? S0[(long long)bh * per4 + e]
                                                  : make_float4(0.f, 0.f, 0.f, 0.f);
    if (threadIdx.x == 0) {
        ready[bh] = 0;
        if (bh == 0) ready[BH] = 0;
    }
}
}  // namespace

cudaError_t launch_chain_reset(const float *S0, int BH, int dk, int dv, float *states, int *ready,
                               cudaStream_t st) {
    if (BH == 0) return cudaSuccess;
    chain_reset_kernel<<<BH, 256, 0, st>>>(reinterpret_cast<const float4 *>(S0), BH,
                                           (long long)dk * dv / 4,
                                           reinterpret_cast<float4 *>(states), ready);
    return cudaGetLastError();
}

namespace {
__global__ void broadcast_state_kernel(const float4 *__restrict__ src, int BH, int P,
                                       long long per4, float4 *__restrict__ dst) {
    const long long n = (long long)BH * P * per4;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x) {
        const long long bhp = e / per4, r = e % per4;
        const long long bh = bhp / P;
        dst[e] = src ? src[bh * per4 + r] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
}
}  // namespace

cudaError_t launch_broadcast_state(const float *src, int BH, int P, int dk, int dv, float *dst,
                                   cudaStream_t st) {
    const long long per4 = (long long)dk * dv / 4;
    const long long n = (long long)BH * P * per4;
    if (n == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
    broadcast_state_kernel<<<blocks, 256, 0, st>>>(reinterpret_cast<const float4 *>(src), BH, P,
                                                   per4, reinterpret_cast<float4 *>(dst));
    return cudaGetLastError();
}
}  // namespace la
