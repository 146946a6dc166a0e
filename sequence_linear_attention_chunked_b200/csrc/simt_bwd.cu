// simt_bwd.cu -- backward chunk passes on the CUDA cores (FFMA), every dtype / d / chunk.
//
// Loss = <o, dO> + <S_final, dS_final>.  For a segment j of T tokens that receives the state
// S_recv_j and whose end state S_end_j has gradient dX_j (from the reverse exclusive scan),
// chunk by chunk with in-chunk cumsum b_t, total b_C, S' = diag(e^{b_C}) S,
// Qbar'_t = q_t e^{b_t - b_C}, Ktil_s = k_s e^{b_C - b_s}, M_ts = [s<=t] dO_t . v_s and
// A_ts = [s<=t] Qbar'_t . Ktil_s:
//
//   forward sweep   dq_t  = e^{b_t - b_C} (dO_t S'^T + sum_s M_ts Ktil_s);  S = S' + Ktil^T V
//                   (one kernel; it also stores q_t . dq_t in fp32 for the reverse sweep)
//   reverse sweep   (a second kernel)
//                   dk_s  = e^{b_C - b_s} (sum_t M_ts Qbar'_t + v_s dS^T)
//                   dv_s  = sum_t A_ts dO_t + Ktil_s dS
//                   dS   <- diag(e^{b_C}) (dS + Qbar'^T dO)           (dS starts at dX_j)
//                   dlog_g_t = sum_{u>=t in segment} (q_u dq_u - k_u dk_u) + rowsum(S_end_j . dX_j)
//
// The last term is dlog_g at the next segment's first token: the sensitivity of the loss to
// a shift of all later log-gates, which the exact token recurrence gives as the row sums of
// (state . state gradient) at the boundary (ZeCO review, "forward implications": the
// backward reuses the forward's global states).  A separate pass forms each segment's
// gradient state dSloc_j = sum_t diag(e^{B_t}) q_t^T dO_t (B from the segment start).
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace la {
namespace {

constexpr int kThreads = 256;

// ------------------------------------------------------------------ gradient-state pass
template <int DK, int DV, int C>
struct DstSmem {
    static constexpr int DKP = DK + 1;
    static constexpr int q = 0;
    static constexpr int g = q + C * DKP;
    static constexpr int dO = g + C * DKP;
    static constexpr int R = dO + C * DV;
    static constexpr int B0 = R + DK * DV;
    static constexpr int total = B0 + DK;
    static constexpr size_t bytes = sizeof(float) * total;
};

template <typename T, int DK, int DV, int C>
__global__ void __launch_bounds__(kThreads) simt_dstate_kernel(BwdArgs a) {
    using L = DstSmem<DK, DV, C>;
    constexpr int DKP = L::DKP;
    extern __shared__ float smem[];
    float *sq = smem + L::q, *sg = smem + L::g, *sd = smem + L::dO, *sR = smem + L::R,
          *sB0 = smem + L::B0;
    const int tid = threadIdx.x;
    const int bh = blockIdx.x / a.NP, j = blockIdx.x % a.NP;
    const long long base = (long long)bh * a.L + (long long)j * a.T;
    const T *q = static_cast<const T *>(a.q) + base * DK;
    const T *g = static_cast<const T *>(a.g) + base * DK;
    const T *dO = static_cast<const T *>(a.dO) + base * DV;
    for (int idx = tid; idx < DK * DV; idx += kThreads) sR[idx] = 0.f;
    if (tid < DK) sB0[tid] = 0.f;
    bool range_bad = false;
    for (long long r0 = 0; r0 < a.T; r0 += C) {
        __syncthreads();
        for (int idx = tid; idx < C * DK; idx += kThreads) {
            const int t = idx / DK, i = idx % DK;
            sq[t * DKP + i] = to_f32(q[(r0 + t) * DK + i]);
            sg[t * DKP + i] = to_f32(g[(r0 + t) * DK + i]);
        }
        for (int idx = tid; idx < C * DV; idx += kThreads)
            sd[idx] = to_f32(dO[(r0 + idx / DV) * DV + idx % DV]);
        __syncthreads();
        if (tid < DK) {  // running log-decay from the segment start, inclusive
            float acc = sB0[tid];
            const float start = acc;
            for (int t = 0; t < C; ++t) {
                const float x = sg[t * DKP + tid];
                range_bad |= !(x <= 0.f);  // a positive (or NaN) gate exponent
                acc += x;
                sg[t * DKP + tid] = acc;
            }
            range_bad |= !(fabsf(acc - start) <= kGateRangeLimit);
            sB0[tid] = acc;
        }
        __syncthreads();
        for (int idx = tid; idx < C * DK; idx += kThreads) {
            const int t = idx / DK, i = idx % DK;
            sq[t * DKP + i] *= __expf(sg[t * DKP + i]);
        }
        __syncthreads();
        for (int idx = tid; idx < DK * DV; idx += kThreads) {
            const int i = idx / DV, jj = idx % DV;
            float acc = sR[idx];
            for (int t = 0; t < C; ++t) acc += sq[t * DKP + i] * sd[t * DV + jj];
            sR[idx] = acc;
        }
    }
    __syncthreads();
    float *R = a.dSloc + ((long long)bh * a.NP + j) * DK * DV;
    for (int idx = tid; idx < DK * DV; idx += kThreads) R[idx] = sR[idx];
    if (tid < DK) a.logG[((long long)bh * a.NP + j) * DK + tid] = sB0[tid];
    if (range_bad) flag_range(a.flags, (long long)blockIdx.x, 1, a.status);
}

// ------------------------------------------------------------------ gradient pass
template <int DK, int DV, int C>
struct GradSmem {
    static constexpr int DKP = DK + 1, CP = C + 1;
    static constexpr int q = 0;
    static constexpr int k = q + C * DKP;
    static constexpr int v = k + C * DKP;
    static constexpr int b = v + C * DV;
    static constexpr int dO = b + C * DKP;
    static constexpr int M = dO + C * DV;
    static constexpr int A = M + C * CP;
    static constexpr int S = A + C * CP;
    static constexpr int cg = S + DK * DV;
    static constexpr int eC = cg + C * DKP;
    static constexpr int bC = eC + DK;
    static constexpr int accg = bC + DK;
    static constexpr int total = accg + DK;
    static constexpr size_t bytes = sizeof(float) * total;
};

template <typename T, int DK, int DV, int C>
__global__ void __launch_bounds__(kThreads) simt_dq_kernel(BwdArgs a) {
    using L = GradSmem<DK, DV, C>;
    constexpr int DKP = L::DKP, CP = L::CP;
    extern __shared__ float smem[];
    float *sq = smem + L::q, *sk = smem + L::k, *sv = smem + L::v, *sb = smem + L::b,
          *sd = smem + L::dO, *sM = smem + L::M, *sA = smem + L::A, *sS = smem + L::S,
          *scg = smem + L::cg, *seC = smem + L::eC, *sbC = smem + L::bC, *saccg = smem + L::accg;
    const int tid = threadIdx.x;
    const int bh = blockIdx.x / a.NP, j = blockIdx.x % a.NP;
    const long long base = (long long)bh * a.L + (long long)j * a.T;
    const T *q = static_cast<const T *>(a.q) + base * DK;
    const T *k = static_cast<const T *>(a.k) + base * DK;
    const T *g = static_cast<const T *>(a.g) + base * DK;
    const T *v = static_cast<const T *>(a.v) + base * DV;
    const T *dO = static_cast<const T *>(a.dO) + base * DV;
    float *dqw = a.dq_ws + base * DK;
    T *dqo = static_cast<T *>(a.dq_out) + base * DK;
    const long long sidx = ((long long)bh * a.NP + j) * DK * DV;

    // cumsum of the chunk's log-gates (threads < DK), then e^{b_C}; returns after a barrier
    bool range_bad = false;
    auto gates = [&](long long r0) {
        if (tid < DK) {
            float acc = 0.f;
            for (int t = 0; t < C; ++t) {
                const float x = sb[t * DKP + tid];
                range_bad |= !(x <= 0.f);  // a positive (or NaN) gate exponent
                acc += x;
                sb[t * DKP + tid] = acc;
            }
            sbC[tid] = acc;
            seC[tid] = __expf(acc);
            range_bad |= !(fabsf(acc) <= kGateRangeLimit);
        }
        __syncthreads();
    };

    // ---- forward sweep: dq, and q . dq (fp32) for the reverse sweep's dlog_g
    for (int idx = tid; idx < DK * DV; idx += kThreads) sS[idx] = a.S_recv ? a.S_recv[sidx + idx] : 0.f;
    const long long Tf = a.T / a.fine;
    for (long long r0 = 0; r0 < a.T; r0 += C) {
        __syncthreads();
        if (a.S_fine && r0 % Tf == 0) {  // the state entering fine part r0 / Tf of this segment
            float *Sf = a.S_fine + (((long long)bh * a.NP + j) * a.fine + r0 / Tf) * DK * DV;
            for (int idx = tid; idx < DK * DV; idx += kThreads) Sf[idx] = sS[idx];
        }
        for (int idx = tid; idx < C * DK; idx += kThreads) {
            const int t = idx / DK, i = idx % DK;
            sk[t * DKP + i] = to_f32(k[(r0 + t) * DK + i]);
            sb[t * DKP + i] = to_f32(g[(r0 + t) * DK + i]);
        }
        for (int idx = tid; idx < C * DV; idx += kThreads) {
            sv[idx] = to_f32(v[(r0 + idx / DV) * DV + idx % DV]);
            sd[idx] = to_f32(dO[(r0 + idx / DV) * DV + idx % DV]);
        }
        __syncthreads();
        gates(r0);
        for (int idx = tid; idx < C * DK; idx += kThreads) {
            const int t = idx / DK, i = idx % DK;
            sk[t * DKP + i] *= __expf(sbC[i] - sb[t * DKP + i]);
        }
        for (int idx = tid; idx < DK * DV; idx += kThreads) sS[idx] *= seC[idx / DV];
        for (int idx = tid; idx < C * C; idx += kThreads) {
            const int t = idx / C, s = idx % C;
            float acc = 0.f;
            if (s <= t)
                for (int jj = 0; jj < DV; ++jj) acc += sd[t * DV + jj] * sv[s * DV + jj];
            sM[t * CP + s] = acc;
        }
        __syncthreads();
        for (int idx = tid; idx < C * DK; idx += kThreads) {
            const int t = idx / DK, i = idx % DK;
            float acc = 0.f;
            for (int jj = 0; jj < DV; ++jj) acc += sd[t * DV + jj] * sS[i * DV + jj];
            for (int s = 0; s <= t; ++s) acc += sM[t * CP + s] * sk[s * DKP + i];
            const float dqv = acc * __expf(sb[t * DKP + i] - sbC[i]);
            dqo[(r0 + t) * DK + i] = from_f32<T>(dqv);
            dqw[(r0 + t) * DK + i] = to_f32(q[(r0 + t) * DK + i]) * dqv;  // q . dq for dlog_g
        }
        __syncthreads();
        for (int idx = tid; idx < DK * DV; idx += kThreads) {
            const int i = idx / DV, jj = idx % DV;
            float acc = sS[idx];
            for (int s = 0; s < C; ++s) acc += sk[s * DKP + i] * sv[s * DV + jj];
            sS[idx] = acc;
        }
    }
    __syncthreads();
    if (range_bad)  // every fine part of the segment: the state runs through them
        flag_range(a.flags, ((long long)bh * a.NP + j) * a.fine, a.fine, a.status);
}

template <typename T, int DK, int DV, int C>
__global__ void __launch_bounds__(kThreads) simt_dkv_kernel(BwdArgs a) {
    using L = GradSmem<DK, DV, C>;
    constexpr int DKP = L::DKP, CP = L::CP;
    extern __shared__ float smem[];
    float *sq = smem + L::q, *sk = smem + L::k, *sv = smem + L::v, *sb = smem + L::b,
          *sd = smem + L::dO, *sM = smem + L::M, *sA = smem + L::A, *sS = smem + L::S,
          *scg = smem + L::cg, *seC = smem + L::eC, *sbC = smem + L::bC, *saccg = smem + L::accg;
    const int tid = threadIdx.x;
    const int bh = blockIdx.x / a.NP, j = blockIdx.x % a.NP;
    const long long base = (long long)bh * a.L + (long long)j * a.T;
    const T *q = static_cast<const T *>(a.q) + base * DK;
    const T *k = static_cast<const T *>(a.k) + base * DK;
    const T *g = static_cast<const T *>(a.g) + base * DK;
    const T *v = static_cast<const T *>(a.v) + base * DV;
    const T *dO = static_cast<const T *>(a.dO) + base * DV;
    float *dqw = a.dq_ws + base * DK;
    const long long sidx = ((long long)bh * a.NP + j) * DK * DV;

    // cumsum of the chunk's log-gates (threads < DK), then e^{b_C}; returns after a barrier
    bool range_bad = false;
    auto gates = [&](long long r0) {
        if (tid < DK) {
            float acc = 0.f;
            for (int t = 0; t < C; ++t) {
                const float x = sb[t * DKP + tid];
                range_bad |= !(x <= 0.f);  // a positive (or NaN) gate exponent
                acc += x;
                sb[t * DKP + tid] = acc;
            }
            sbC[tid] = acc;
            seC[tid] = __expf(acc);
            range_bad |= !(fabsf(acc) <= kGateRangeLimit);
        }
        __syncthreads();
    };

    // ---- reverse sweep: dk, dv, dlog_g
    __syncthreads();
    const float *dX = a.dX + sidx;
    for (int idx = tid; idx < DK * DV; idx += kThreads) sS[idx] = dX[idx];
    if (tid < DK) {
        float acc = 0.f;
        const float *Se = nullptr;
        if (j < a.NP - 1) {
            if (a.S_end_next) Se = a.S_end_next + sidx + (long long)DK * DV;
        } else if (a.S_fin) {
            Se = a.S_fin + (long long)bh * DK * DV;
        }
        if (Se)
            for (int jj = 0; jj < DV; ++jj) acc += Se[tid * DV + jj] * dX[tid * DV + jj];
        saccg[tid] = acc;
    }
    T *dk = static_cast<T *>(a.dk_out) + base * DK;
    T *dv = static_cast<T *>(a.dv_out) + base * DV;
    T *dg = static_cast<T *>(a.dg_out) + base * DK;
    for (long long r0 = a.T - C; r0 >= 0; r0 -= C) {
        __syncthreads();
        for (int idx = tid; idx < C * DK; idx += kThreads) {
            const int t = idx / DK, i = idx % DK;
            sq[t * DKP + i] = to_f32(q[(r0 + t) * DK + i]);
            sk[t * DKP + i] = to_f32(k[(r0 + t) * DK + i]);
            sb[t * DKP + i] = to_f32(g[(r0 + t) * DK + i]);
        }
        for (int idx = tid; idx < C * DV; idx += kThreads) {
            sv[idx] = to_f32(v[(r0 + idx / DV) * DV + idx % DV]);
            sd[idx] = to_f32(dO[(r0 + idx / DV) * DV + idx % DV]);
        }
        __syncthreads();
        gates(r0);
        for (int idx = tid; idx < C * DK; idx += kThreads) {
            const int t = idx / DK, i = idx % DK;
            const float x = sb[t * DKP + i] - sbC[i];
            sq[t * DKP + i] *= __expf(x);
            sk[t * DKP + i] *= __expf(-x);
        }
        __syncthreads();
        for (int idx = tid; idx < C * C; idx += kThreads) {
            const int t = idx / C, s = idx % C;
            float m = 0.f, aa = 0.f;
            if (s <= t) {
                for (int jj = 0; jj < DV; ++jj) m += sd[t * DV + jj] * sv[s * DV + jj];
                for (int i = 0; i < DK; ++i) aa += sq[t * DKP + i] * sk[s * DKP + i];
            }
            sM[t * CP + s] = m;
            sA[t * CP + s] = aa;
        }
        __syncthreads();
        for (int idx = tid; idx < C * DK; idx += kThreads) {  // dk and the dlog_g contribution
            const int s = idx / DK, i = idx % DK;
            float acc = 0.f;
            for (int t = s; t < C; ++t) acc += sM[t * CP + s] * sq[t * DKP + i];
            for (int jj = 0; jj < DV; ++jj) acc += sS[i * DV + jj] * sv[s * DV + jj];
            const float dks = acc * __expf(sbC[i] - sb[s * DKP + i]);
            dk[(r0 + s) * DK + i] = from_f32<T>(dks);
            scg[s * DKP + i] = dqw[(r0 + s) * DK + i] - to_f32(k[(r0 + s) * DK + i]) * dks;
        }
        for (int idx = tid; idx < C * DV; idx += kThreads) {  // dv
            const int s = idx / DV, jj = idx % DV;
            float acc = 0.f;
            for (int t = s; t < C; ++t) acc += sA[t * CP + s] * sd[t * DV + jj];
            for (int i = 0; i < DK; ++i) acc += sk[s * DKP + i] * sS[i * DV + jj];
            dv[(r0 + s) * DV + jj] = from_f32<T>(acc);
        }
        __syncthreads();
        if (tid < DK) {  // suffix sums of the contributions, carried across chunks
            float acc = saccg[tid];
            for (int t = C - 1; t >= 0; --t) {
                acc += scg[t * DKP + tid];
                dg[(r0 + t) * DK + tid] = from_f32<T>(acc);
            }
            saccg[tid] = acc;
        }
        for (int idx = tid; idx < DK * DV; idx += kThreads) {  // dS <- diag(e^{b_C}) (dS + Qbar'^T dO)
            const int i = idx / DV, jj = idx % DV;
            float acc = sS[idx];
            for (int t = 0; t < C; ++t) acc += sq[t * DKP + i] * sd[t * DV + jj];
            sS[idx] = acc * seC[i];
        }
    }
    if (range_bad) flag_range(a.flags, (long long)blockIdx.x, 1, a.status);
}

template <typename Kern>
cudaError_t launch_k(Kern kern, size_t smem, const BwdArgs &a, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long nblk = (long long)a.BH * a.NP;
    if (nblk == 0) return cudaSuccess;
    kern<<<(unsigned)nblk, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <typename T, int D, int C>
cudaError_t launch_c(const BwdArgs &a, int which, cudaStream_t st) {
    if (which == 0) return launch_k(simt_dstate_kernel<T, D, D, C>, DstSmem<D, D, C>::bytes, a, st);
    constexpr int CG = (D == 128 && C > 32) ? 32 : C;  // d = 128: 32-token blocks fit shared memory
    if (which == 1) return launch_k(simt_dq_kernel<T, D, D, CG>, GradSmem<D, D, CG>::bytes, a, st);
    return launch_k(simt_dkv_kernel<T, D, D, CG>, GradSmem<D, D, CG>::bytes, a, st);
}

template <typename T, int D>
cudaError_t launch_d(const BwdArgs &a, int which, cudaStream_t st) {
    switch (a.chunk) {
        case 16: return launch_c<T, D, 16>(a, which, st);
        case 32: return launch_c<T, D, 32>(a, which, st);
        case 64: return launch_c<T, D, 64>(a, which, st);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t launch_t(const BwdArgs &a, int which, cudaStream_t st) {
    switch (a.dk) {
        case 32: return launch_d<T, 32>(a, which, st);
        case 64: return launch_d<T, 64>(a, which, st);
        case 128: return launch_d<T, 128>(a, which, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_simt_dstate(const BwdArgs &a, cudaStream_t st) {
    return a.dt == LA_F32 ? launch_t<float>(a, 0, st) : launch_t<__nv_bfloat16>(a, 0, st);
}

cudaError_t launch_simt_dq(const BwdArgs &a, cudaStream_t st) {
    return a.dt == LA_F32 ? launch_t<float>(a, 1, st) : launch_t<__nv_bfloat16>(a, 1, st);
}

cudaError_t launch_simt_dkv(const BwdArgs &a, cudaStream_t st) {
    return a.dt == LA_F32 ? launch_t<float>(a, 2, st) : launch_t<__nv_bfloat16>(a, 2, st);
}

}  // namespace la
