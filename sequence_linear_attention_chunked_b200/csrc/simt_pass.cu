// simt_pass.cu -- chunkwise GLA passes on the CUDA cores (FFMA), every dtype / d / chunk.
//
// This is the fp32 path (tensor cores cannot hold a 1e-4 relative error bound) and the
// generic path for shapes the tcgen05 kernels do not cover.  One CTA walks one (b, h,
// sub-segment) chunk by chunk.  Per chunk of C tokens with in-chunk inclusive log-gate
// cumsum b_t and chunk total b_C (GLA chunkwise form; ZeCO review "key machinery" for the
// decayed state update):
//
//   Qbar'_t = q_t . exp(b_t - b_C)        Ktil_s = k_s . exp(b_C - b_s)
//   S'      = diag(exp(b_C)) S                          (state decayed to the chunk end)
//   o_t     = sum_{s<=t} (Qbar'_t . Ktil_s) v_s + Qbar'_t S'
//   S       = S' + Ktil^T V
//
// Qbar'_t Ktil_s = sum_i q_ti k_si exp(b_ti - b_si), and Qbar'_t S' = (q_t . exp(b_t)) S,
// which is the token recurrence summed over the chunk.  With log_g <= 0 every exponent is
// bounded by the chunk's |b_C|; a chunk with a positive log_g or |b_C| > kGateRangeLimit is
// flagged (flag_range).
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace la {
namespace {

constexpr int kThreads = 256;

template <int DK, int DV, int C>
struct SimtSmem {
    static constexpr int DKP = DK + 1;  // padded rows: lanes that vary the token index stay
    static constexpr int CP = C + 1;    // on distinct banks
    static constexpr int q = 0;
    static constexpr int k = q + C * DKP;
    static constexpr int g = k + C * DKP;
    static constexpr int v = g + C * DKP;
    static constexpr int A = v + C * DV;
    static constexpr int S = A + C * CP;
    static constexpr int eC = S + DK * DV;
    static constexpr int bC = eC + DK;
    static constexpr int total = bC + DK;  // floats
    static constexpr size_t bytes = sizeof(float) * total;
};

template <typename T, int DK, int DV, int C, int MODE>
__global__ void __launch_bounds__(kThreads) simt_pass_kernel(PassArgs a) {
    using L = SimtSmem<DK, DV, C>;
    constexpr int DKP = L::DKP, CP = L::CP;
    extern __shared__ float smem[];
    float *sq = smem + L::q, *sk = smem + L::k, *sg = smem + L::g, *sv = smem + L::v;
    float *sA = smem + L::A, *sS = smem + L::S, *seC = smem + L::eC, *sbC = smem + L::bC;

    const int tid = threadIdx.x;
    const int bh = blockIdx.x / a.NP;
    const int j = blockIdx.x % a.NP;
    const long long tok0 = (long long)j * a.T;
    const T *q = static_cast<const T *>(a.q) + ((long long)bh * a.L + tok0) * DK;
    const T *k = static_cast<const T *>(a.k) + ((long long)bh * a.L + tok0) * DK;
    const T *g = static_cast<const T *>(a.g) + ((long long)bh * a.L + tok0) * DK;
    const T *v = static_cast<const T *>(a.v) + ((long long)bh * a.L + tok0) * DV;
    T *o = a.o ? static_cast<T *>(a.o) + ((long long)bh * a.L + tok0) * DV : nullptr;

    constexpr bool kUsesQ = MODE != kPassState;
    constexpr bool kUsesKV = MODE != kPassCorrect;
    constexpr bool kWritesState = MODE == kPassState || MODE == kPassLocal;

    // Initial state: the received state for output/correct passes, zero for local passes.
    const float *Sin = (MODE == kPassOutput || MODE == kPassCorrect) && a.S_init
                           ? a.S_init + ((long long)bh * a.NP + j) * DK * DV
                           : nullptr;
    for (int idx = tid; idx < DK * DV; idx += kThreads) sS[idx] = Sin ? Sin[idx] : 0.f;

    float logG = 0.f;  // meaningful in threads tid < DK
    bool range_bad = false;
    const int nchunks = (int)(a.T / C);
    for (int c = 0; c < nchunks; ++c) {
        const long long r0 = (long long)c * C;
        __syncthreads();  // previous chunk fully consumed
        for (int idx = tid; idx < C * DK; idx += kThreads) {
            const int t = idx / DK, i = idx % DK;
            sg[t * DKP + i] = to_f32(g[(r0 + t) * DK + i]);
            if (kUsesQ) sq[t * DKP + i] = to_f32(q[(r0 + t) * DK + i]);
            if (kUsesKV) sk[t * DKP + i] = to_f32(k[(r0 + t) * DK + i]);
        }
        if (kUsesKV)
            for (int idx = tid; idx < C * DV; idx += kThreads) {
                const int t = idx / DV, jj = idx % DV;
                sv[t * DV + jj] = to_f32(v[(r0 + t) * DV + jj]);
            }
        __syncthreads();
        // In-chunk inclusive cumsum of the log-gates, one key dim per thread.
        if (tid < DK) {
            float acc = 0.f;
            for (int t = 0; t < C; ++t) {
                const float x = sg[t * DKP + tid];
                range_bad |= !(x <= 0.f);  // a positive (or NaN) gate exponent
                acc += x;
                sg[t * DKP + tid] = acc;
            }
            sbC[tid] = acc;
            seC[tid] = __expf(acc);
            logG += acc;
            range_bad |= !(fabsf(acc) <= kGateRangeLimit);
        }
        __syncthreads();
        // Decay factors folded into the operands; state decayed to the chunk end.
        for (int idx = tid; idx < C * DK; idx += kThreads) {
            const int t = idx / DK, i = idx % DK;
            const float b = sg[t * DKP + i], bc = sbC[i];
            if (kUsesQ) sq[t * DKP + i] *= __expf(b - bc);
            if (kUsesKV) sk[t * DKP + i] *= __expf(bc - b);
        }
        for (int idx = tid; idx < DK * DV; idx += kThreads) sS[idx] *= seC[idx / DV];
        __syncthreads();
        if (MODE == kPassOutput || MODE == kPassLocal) {
            // Intra-chunk scores, causal mask including the diagonal.
            for (int idx = tid; idx < C * C; idx += kThreads) {
                const int t = idx / C, s = idx % C;
                float acc = 0.f;
                if (s <= t) {
#pragma unroll 8
                    for (int i = 0; i < DK; ++i) acc += sq[t * DKP + i] * sk[s * DKP + i];
                }
                sA[t * CP + s] = acc;
            }
            __syncthreads();
            for (int idx = tid; idx < C * DV; idx += kThreads) {
                const int t = idx / DV, jj = idx % DV;
                float acc = 0.f;
                for (int s = 0; s <= t; ++s) acc += sA[t * CP + s] * sv[s * DV + jj];
#pragma unroll 8
                for (int i = 0; i < DK; ++i) acc += sq[t * DKP + i] * sS[i * DV + jj];
                o[(r0 + t) * DV + jj] = from_f32<T>(acc);
            }
        } else if (MODE == kPassCorrect) {
            for (int idx = tid; idx < C * DV; idx += kThreads) {
                const int t = idx / DV, jj = idx % DV;
                float acc = to_f32(o[(r0 + t) * DV + jj]);
#pragma unroll 8
                for (int i = 0; i < DK; ++i) acc += sq[t * DKP + i] * sS[i * DV + jj];
                o[(r0 + t) * DV + jj] = from_f32<T>(acc);
            }
        }
        if (kUsesKV) {
            __syncthreads();  // outputs read S' before it is updated
            for (int idx = tid; idx < DK * DV; idx += kThreads) {
                const int i = idx / DV, jj = idx % DV;
                float acc = sS[idx];
                for (int s = 0; s < C; ++s) acc += sk[s * DKP + i] * sv[s * DV + jj];
                sS[idx] = acc;
            }
        }
    }
    __syncthreads();
    if (kWritesState && a.S_out) {  // null: a local pass whose states are not wanted
        float *Sout = a.S_out + ((long long)bh * a.NP + j) * DK * DV;
        for (int idx = tid; idx < DK * DV; idx += kThreads) Sout[idx] = sS[idx];
    }
    if (kWritesState && a.logG && tid < DK) a.logG[((long long)bh * a.NP + j) * DK + tid] = logG;
    if (range_bad) flag_range(a.flags, (long long)bh * a.NP + j, 1, a.status);
}

template <typename T, int DK, int DV, int C, int MODE>
cudaError_t launch_t(const PassArgs &a, cudaStream_t st) {
    auto kern = simt_pass_kernel<T, DK, DV, C, MODE>;
    const size_t smem = SimtSmem<DK, DV, C>::bytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long nblk = (long long)a.BH * a.NP;
    if (nblk == 0) return cudaSuccess;
    kern<<<(unsigned)nblk, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <typename T, int DK, int DV, int C>
cudaError_t launch_mode(const PassArgs &a, PassMode mode, cudaStream_t st) {
    switch (mode) {
        case kPassState: return launch_t<T, DK, DV, C, kPassState>(a, st);
        case kPassOutput: return launch_t<T, DK, DV, C, kPassOutput>(a, st);
        case kPassLocal: return launch_t<T, DK, DV, C, kPassLocal>(a, st);
        case kPassCorrect: return launch_t<T, DK, DV, C, kPassCorrect>(a, st);
    }
    return cudaErrorInvalidValue;
}

template <typename T, int D>
cudaError_t launch_chunk(const PassArgs &a, PassMode mode, cudaStream_t st) {
    switch (a.chunk) {
        case 16: return launch_mode<T, D, D, 16>(a, mode, st);
        case 32: return launch_mode<T, D, D, 32>(a, mode, st);
        case 64: return launch_mode<T, D, D, 64>(a, mode, st);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t launch_d(const PassArgs &a, PassMode mode, cudaStream_t st) {
    if (a.dk != a.dv) return cudaErrorInvalidValue;
    switch (a.dk) {
        case 32: return launch_chunk<T, 32>(a, mode, st);
        case 64: return launch_chunk<T, 64>(a, mode, st);
        case 128: return launch_chunk<T, 128>(a, mode, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_simt_pass(const PassArgs &a, PassMode mode, cudaStream_t st) {
    if (a.dt == LA_F32) return launch_d<float>(a, mode, st);
    return launch_d<__nv_bfloat16>(a, mode, st);
}

}  // namespace la
