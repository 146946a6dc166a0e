// exact.cu -- the exact token-by-token path for units that the chunk factorisation cannot hold.
//
// The chunk kernels scale q and k by exp(+-(b_t - b_C)) (b the in-chunk cumsum of log_g); a
// chunk with a positive log_g, or one whose decay over the chunk exceeds e^80 in some key dim
// (strong or complete forgetting, a = exp(log_g) down to 0), cannot be represented that way
// in fp32 / bf16 -- the K-bar = K . Gamma versus K / Lambda normalisation that the ZeCO review's
// referee flags (minor comment 4) breaks down there.  Those kernels mark the unit (a segment or
// one fine part of it) in a flag array, and the kernels here recompute every marked unit with
// the recurrence itself (the GLA state update of the review's "key machinery"):
//
//     S_t = diag(a_t) S_{t-1} + k_t^T v_t,   a_t = exp(log_g_t),   o_t = q_t S_t,
//
// and its exact adjoint, in fp32 on the CUDA cores.  The only exponentials formed are a_t and
// exp(B_t) (B a cumsum of log_g), so nothing overflows while log_g <= 0, whatever the decay;
// with a positive log_g the recurrence itself grows, and so does its result.
//
// One CTA of 16 warps holds the d x d fp32 state in registers, d^2 / 512 elements per thread:
//  - layout A (forward): lane l owns rows l + 32r, warp w owns columns w (d/16) + c, so the
//    column sums o_t[j] = sum_i q_t[i] S[i][j] are warp reductions;
//  - layout B (backward): warp w owns rows w (d/16) + r, lane l owns columns l + 32c, so the row
//    sums dq_t[i] and dk_t[i] are warp reductions; the column sums dv_t[j] go across the warps
//    through shared memory.
// A warp reduces its N = d/16 partial sums across the 32 lanes by reduce-scatter (halving the
// set at each of log2 N steps), then a butterfly over the remaining lane bits: log2 N + (5 -
// log2 N) + ... shuffles instead of 5 N.  Tokens are staged in batches of kTB through shared
// memory as fp32, and outputs leave through shared memory as whole rows.  The grid is
// persistent (one CTA per SM) and walks the units; an unmarked unit costs one flag read, so the
// launch that follows every chunk pass costs a few microseconds when nothing is marked.
#include <type_traits>

#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace la {
namespace {

constexpr int kXThreads = 512, kXWarps = 16, kTB = 8;

template <typename T>
__device__ __forceinline__ float ldx(const T *p) { return to_f32(*p); }

// Reduce-scatter of N per-lane values over the warp: returns in every lane the total (over all
// 32 lanes) of value index slot(lane), where slot takes the lane's top log2(N) bits.
template <int N>
__device__ __forceinline__ float warp_reduce_scatter(float (&x)[N], int lane) {
    static_assert(N == 1 || N == 2 || N == 4 || N == 8, "N");
#pragma unroll
    for (int half = N / 2, off = 16; half >= 1; half >>= 1, off >>= 1) {
        const bool upper = lane & off;
#pragma unroll
        for (int m = 0; m < half; ++m) {
            const float send = upper ? x[m] : x[m + half];
            const float keep = upper ? x[m + half] : x[m];
            x[m] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, off);
        }
    }
    float v = x[0];
#pragma unroll
    for (int off = 32 / N / 2; off >= 1; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
    return v;
}

// Index (0 .. N-1) of the value warp_reduce_scatter<N> leaves in this lane.
template <int N>
__device__ __forceinline__ int scatter_slot(int lane) {
    int s = 0;
#pragma unroll
    for (int b = 0, off = 16; b < (N == 8 ? 3 : N == 4 ? 2 : N == 2 ? 1 : 0); ++b, off >>= 1)
        s = (s << 1) | ((lane & off) ? 1 : 0);
    return s;
}
// The lanes that write a reduced value (one per slot).
template <int N>
__device__ __forceinline__ bool scatter_writer(int lane) { return (lane & (32 / N - 1)) == 0; }

// Stages rows [t0, t0 + n) of a [*, D] tensor (element type T) into dst[kTB][D] as fp32 (rows
// past n are zero); f maps each value (exp for the gates).
template <int D, typename T, typename F>
__device__ __forceinline__ void stage(float *dst, const T *src, long long t0, int n, F f) {
    for (int idx = threadIdx.x; idx < kTB * D; idx += kXThreads) {
        const int t = idx / D;
        dst[idx] = t < n ? f(ldx(src + (t0 + t) * D + idx % D)) : 0.f;
    }
}
struct Id { __device__ float operator()(float x) const { return x; } };
struct Exp { __device__ float operator()(float x) const { return __expf(x); } };

// ------------------------------------------------------------------ forward (layout A)
// One unit = tokens [tok0, tok0 + n) of sequence bh.  S (layout A) enters as the unit's start
// state and leaves as its end state; o (nullable) gets the outputs, lgs (nullable, per lane
// rows) the summed log-gates.
template <int D, typename T>
struct FwdUnit {
    float *sq, *sk, *sa, *sv, *sg, *so;  // kTB x D each
};

template <int D, typename T>
__device__ void fwd_tokens(const FwdUnit<D, T> &u, const PassArgs &a, int bh, long long tok0,
                           long long n, float (&S)[D / 32][D / 16], float (&lgs)[D / 32],
                           bool want_o) {
    constexpr int RL = D / 32, CW = D / 16;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const long long base = (long long)bh * a.L + tok0;
    const T *q = static_cast<const T *>(a.q) + base * D;
    const T *k = static_cast<const T *>(a.k) + base * D;
    const T *v = static_cast<const T *>(a.v) + base * D;
    const T *g = static_cast<const T *>(a.g) + base * D;
    T *o = want_o ? static_cast<T *>(a.o) + base * D : nullptr;
    for (long long b0 = 0; b0 < n; b0 += kTB) {
        const int nb = (int)(n - b0 < kTB ? n - b0 : kTB);
        __syncthreads();  // the previous batch's rows are read and its outputs written
        if (want_o) stage<D>(u.sq, q, b0, nb, Id());
        stage<D>(u.sk, k, b0, nb, Id());
        stage<D>(u.sv, v, b0, nb, Id());
        stage<D>(u.sg, g, b0, nb, Id());
        stage<D>(u.sa, g, b0, nb, Exp());
        __syncthreads();
        for (int t = 0; t < nb; ++t) {
            float vj[CW];
#pragma unroll
            for (int c = 0; c < CW; ++c) vj[c] = u.sv[t * D + w * CW + c];
            float part[CW];
#pragma unroll
            for (int c = 0; c < CW; ++c) part[c] = 0.f;
#pragma unroll
            for (int r = 0; r < RL; ++r) {
                const int i = lane + 32 * r;
                const float ai = u.sa[t * D + i], ki = u.sk[t * D + i];
                lgs[r] += u.sg[t * D + i];
                const float qi = want_o ? u.sq[t * D + i] : 0.f;
#pragma unroll
                for (int c = 0; c < CW; ++c) {
                    S[r][c] = fmaf(ai, S[r][c], ki * vj[c]);
                    part[c] = fmaf(qi, S[r][c], part[c]);
                }
            }
            if (want_o) {
                const float tot = warp_reduce_scatter<CW>(part, lane);
                if (scatter_writer<CW>(lane)) u.so[t * D + w * CW + scatter_slot<CW>(lane)] = tot;
            }
        }
        if (want_o) {
            __syncthreads();
            for (int idx = threadIdx.x; idx < nb * D; idx += kXThreads)
                o[(b0 + idx / D) * D + idx % D] = from_f32<T>(u.so[idx]);
        }
    }
}

template <int D>
__device__ void load_state_A(float (&S)[D / 32][D / 16], const float *src) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int r = 0; r < D / 32; ++r)
#pragma unroll
        for (int c = 0; c < D / 16; ++c)
            S[r][c] = src ? src[(lane + 32 * r) * D + w * (D / 16) + c] : 0.f;
}
template <int D>
__device__ void store_state_A(const float (&S)[D / 32][D / 16], float *dst) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int r = 0; r < D / 32; ++r)
#pragma unroll
        for (int c = 0; c < D / 16; ++c) dst[(lane + 32 * r) * D + w * (D / 16) + c] = S[r][c];
}

// Units of the chunk passes (one per (bh, sub-segment j)).  MODE kPassState: S_out and logG of
// the unit from a zero start; kPassOutput / kPassCorrect: o of the unit from S_init[j] (the
// whole output, so it also replaces a correction pass's o_local + correction); kPassLocal: o
// and the local state from zero.
template <int D, typename T, int MODE>
__global__ void __launch_bounds__(kXThreads, 1) exact_pass_kernel(const PassArgs a) {
    extern __shared__ float xs[];
    FwdUnit<D, T> u{xs, xs + kTB * D, xs + 2 * kTB * D, xs + 3 * kTB * D, xs + 4 * kTB * D,
                    xs + 5 * kTB * D};
    constexpr bool want_o = MODE != kPassState;
    constexpr bool from_init = MODE == kPassOutput || MODE == kPassCorrect;
    constexpr bool write_state = MODE == kPassState || MODE == kPassLocal;
    const long long units = (long long)a.BH * a.NP;
    for (long long un = blockIdx.x; un < units; un += gridDim.x) {
        if (!a.flags[un]) continue;  // uniform over the CTA
        const int bh = (int)(un / a.NP), j = (int)(un % a.NP);
        float S[D / 32][D / 16], lgs[D / 32];
        load_state_A<D>(S, from_init && a.S_init ? a.S_init + un * D * D : nullptr);
#pragma unroll
        for (int r = 0; r < D / 32; ++r) lgs[r] = 0.f;
        fwd_tokens<D, T>(u, a, bh, (long long)j * a.T, a.T, S, lgs, want_o);
        if (write_state && a.S_out) store_state_A<D>(S, a.S_out + un * D * D);
        if (write_state && a.logG && (threadIdx.x >> 5) == 0)
#pragma unroll
            for (int r = 0; r < D / 32; ++r) a.logG[un * D + (threadIdx.x & 31) + 32 * r] = lgs[r];
        __syncthreads();  // shared rows free for the next unit
    }
}

// Whole sequences (the single-pass schedule): every (b, h) with a marked sub-segment runs its
// L tokens from S0, writing o, the state entering every save_every-th sub-segment and S_final.
template <int D, typename T>
__global__ void __launch_bounds__(kXThreads, 1)
exact_sequence_kernel(const PassArgs a, const float *S0, float *S_final, float *S_save,
                      int save_every) {
    extern __shared__ float xs[];
    FwdUnit<D, T> u{xs, xs + kTB * D, xs + 2 * kTB * D, xs + 3 * kTB * D, xs + 4 * kTB * D,
                    xs + 5 * kTB * D};
    for (int bh = blockIdx.x; bh < a.BH; bh += gridDim.x) {
        int mark = 0;
        for (int j = threadIdx.x; j < a.NP; j += kXThreads) mark |= a.flags[(long long)bh * a.NP + j];
        if (!__syncthreads_or(mark)) continue;
        float S[D / 32][D / 16], lgs[D / 32] = {};
        load_state_A<D>(S, S0 ? S0 + (long long)bh * D * D : nullptr);
        for (int j = 0; j < a.NP; ++j) {
            if (S_save && j % save_every == 0)
                store_state_A<D>(S, S_save + ((long long)bh * (a.NP / save_every) + j / save_every) * D * D);
            fwd_tokens<D, T>(u, a, bh, (long long)j * a.T, a.T, S, lgs, true);
        }
        if (S_final) store_state_A<D>(S, S_final + (long long)bh * D * D);
        __syncthreads();
    }
}

// ------------------------------------------------------------------ backward (layout B)
template <int D>
__device__ void load_state_B(float (&S)[D / 16][D / 32], const float *src) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int r = 0; r < D / 16; ++r)
#pragma unroll
        for (int c = 0; c < D / 32; ++c)
            S[r][c] = src ? src[(w * (D / 16) + r) * D + lane + 32 * c] : 0.f;
}
template <int D>
__device__ void store_state_B(const float (&S)[D / 16][D / 32], float *dst) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int r = 0; r < D / 16; ++r)
#pragma unroll
        for (int c = 0; c < D / 32; ++c) dst[(w * (D / 16) + r) * D + lane + 32 * c] = S[r][c];
}

// Sum over the whole warp, every lane getting the total.
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, off);
    return x;
}

// The per-token terms of dlog_g.  dlog_g_t = sum_{u >= t} (q_u . dq_u - k_u . dk_u) + carry, and
// both q_u . dq_u and k_u . dk_u hold the same q_u k_u (v_u . dO_u): under strong decay that
// common part dwarfs their difference, and forming the two separately would cancel it in fp32.
// With S_u = a_u S_{u-1} + k_u^T v_u and dS_u = q_u^T dO_u + dS+_u (dS+_u the gradient of S_u
// from the tokens after u) the difference is, exactly,
//     q_u . dq_u - k_u . dk_u = q_u . (a_u S_{u-1} dO_u^T) - k_u . (dS+_u v_u^T),
// so the dq sweep hands over qdq'_u = q_u . a_u (S_{u-1} dO_u^T) and the reverse sweep subtracts
// kdk'_u = k_u . (dS+_u v_u^T): two small terms, no cancellation.

// Element (row r, dim i) of the q . dq hand-over, rows counted from a block start that is a
// multiple of 4 rows: token-quad interleaved (((r / 4) D + i) 4 + r % 4) when the tensor-core
// sweeps exchange it, row-major otherwise.
__device__ __forceinline__ long long qdq_index(long long r, int i, int D, int quad) {
    return quad ? ((r >> 2) * D + i) * 4 + (r & 3) : r * D + i;
}

// dq sweep of one segment (bh, j) whose fine parts are marked: from S_recv[j] (or zero), per
// token dq_t = dO_t S_t^T = a_t (S_{t-1} dO_t^T) + k_t (v_t . dO_t) and qdq'_t; at each fine
// part's start its entering state (S_fine), and over each fine part its gradient state
// sum_t diag(e^{B_t}) q_t^T dO_t (B_t the inclusive cumsum from the part's first token) and its
// log-decay sum.
template <int D, typename T>
__global__ void __launch_bounds__(kXThreads, 1) exact_dq_kernel(const BwdArgs a) {
    constexpr int RW = D / 16, CL = D / 32;
    extern __shared__ float xs[];
    float *sq = xs, *sk = xs + kTB * D, *sa = xs + 2 * kTB * D, *sv = xs + 3 * kTB * D,
          *sd = xs + 4 * kTB * D, *sg = xs + 5 * kTB * D, *sdq = xs + 6 * kTB * D,
          *sqd = xs + 7 * kTB * D;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const long long units = (long long)a.BH * a.NP;
    const long long Tf = a.T / a.fine;
    for (long long un = blockIdx.x; un < units; un += gridDim.x) {
        int mark = 0;
        for (int f = threadIdx.x; f < a.fine; f += kXThreads) mark |= a.flags[un * a.fine + f];
        if (!__syncthreads_or(mark)) continue;
        const int bh = (int)(un / a.NP), j = (int)(un % a.NP);
        const long long base = (long long)bh * a.L + (long long)j * a.T;
        const T *q = static_cast<const T *>(a.q) + base * D;
        const T *k = static_cast<const T *>(a.k) + base * D;
        const T *v = static_cast<const T *>(a.v) + base * D;
        const T *g = static_cast<const T *>(a.g) + base * D;
        const T *dO = static_cast<const T *>(a.dO) + base * D;
        T *dq = static_cast<T *>(a.dq_out) + base * D;
        float *qdq = a.dq_ws + base * D;
        float S[RW][CL], R[RW][CL], B[RW];
        load_state_B<D>(S, a.S_recv ? a.S_recv + un * D * D : nullptr);
        for (int f = 0; f < a.fine; ++f) {
            const long long uf = un * a.fine + f;
            if (a.S_fine) store_state_B<D>(S, a.S_fine + uf * D * D);
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                B[r] = 0.f;
#pragma unroll
                for (int c = 0; c < CL; ++c) R[r][c] = 0.f;
            }
            for (long long b0 = f * Tf; b0 < (f + 1) * Tf; b0 += kTB) {
                const int nb = (int)((f + 1) * Tf - b0 < kTB ? (f + 1) * Tf - b0 : kTB);
                __syncthreads();
                stage<D>(sq, q, b0, nb, Id());
                stage<D>(sk, k, b0, nb, Id());
                stage<D>(sv, v, b0, nb, Id());
                stage<D>(sd, dO, b0, nb, Id());
                stage<D>(sg, g, b0, nb, Id());
                stage<D>(sa, g, b0, nb, Exp());
                __syncthreads();
                for (int t = 0; t < nb; ++t) {
                    float vj[CL], dj[CL], pre[RW], vdo = 0.f;
#pragma unroll
                    for (int c = 0; c < CL; ++c) {
                        vj[c] = sv[t * D + lane + 32 * c];
                        dj[c] = sd[t * D + lane + 32 * c];
                        vdo = fmaf(vj[c], dj[c], vdo);
                    }
                    vdo = warp_sum(vdo);
#pragma unroll
                    for (int r = 0; r < RW; ++r) {
                        const int i = w * RW + r;
                        const float ai = sa[t * D + i], ki = sk[t * D + i], qi = sq[t * D + i];
                        B[r] += sg[t * D + i];
                        const float eq = __expf(B[r]) * qi;
                        pre[r] = 0.f;
#pragma unroll
                        for (int c = 0; c < CL; ++c) {
                            pre[r] = fmaf(S[r][c], dj[c], pre[r]);  // S_{t-1} dO_t^T
                            S[r][c] = fmaf(ai, S[r][c], ki * vj[c]);
                            R[r][c] = fmaf(eq, dj[c], R[r][c]);
                        }
                    }
                    const float p = warp_reduce_scatter<RW>(pre, lane);
                    if (scatter_writer<RW>(lane)) {
                        const int i = w * RW + scatter_slot<RW>(lane);
                        const float ap = sa[t * D + i] * p;
                        sdq[t * D + i] = fmaf(sk[t * D + i], vdo, ap);
                        sqd[t * D + i] = sq[t * D + i] * ap;
                    }
                }
                __syncthreads();
                for (int idx = threadIdx.x; idx < nb * D; idx += kXThreads) {
                    const long long r = b0 + idx / D;
                    dq[r * D + idx % D] = from_f32<T>(sdq[idx]);
                    qdq[qdq_index(r, idx % D, D, a.qdq_quad)] = sqd[idx];
                }
            }
            if (a.dSloc) store_state_B<D>(R, a.dSloc + uf * D * D);
            if (a.logG && lane == 0)
#pragma unroll
                for (int r = 0; r < RW; ++r) a.logG[uf * D + w * RW + r] = B[r];
        }
        __syncthreads();
    }
}

// Reverse sweep of one marked fine part (bh, jf): dS from dX[jf] (the gradient of the part's end
// state); per token, last to first,
//   dk_t = dS_t v_t^T = dS+_t v_t^T + q_t (dO_t . v_t),   dS_t = dS+_t + q_t^T dO_t,
//   dv_t = k_t dS_t,   dS+_{t-1} = diag(a_t) dS_t,
// and dlog_g_t = sum_{u >= t in the part} (qdq'_u - kdk'_u) + carry[jf] (qdq' from the exact dq
// sweep, kdk'_u = k_u . (dS+_u v_u^T): see above).
template <int D, typename T>
__global__ void __launch_bounds__(kXThreads, 1) exact_dkv_kernel(const BwdArgs a) {
    constexpr int RW = D / 16, CL = D / 32;
    extern __shared__ float xs[];
    float *sq = xs, *sk = xs + kTB * D, *sa = xs + 2 * kTB * D, *sv = xs + 3 * kTB * D,
          *sd = xs + 4 * kTB * D, *sqdq = xs + 5 * kTB * D, *sdk = xs + 6 * kTB * D,
          *sdg = xs + 7 * kTB * D, *spv = xs + 8 * kTB * D;  // spv: [kXWarps][kTB][D]
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const long long units = (long long)a.BH * a.NP;
    for (long long un = blockIdx.x; un < units; un += gridDim.x) {
        if (!a.flags[un]) continue;
        const int bh = (int)(un / a.NP), j = (int)(un % a.NP);
        const long long base = (long long)bh * a.L + (long long)j * a.T;
        const T *q = static_cast<const T *>(a.q) + base * D;
        const T *k = static_cast<const T *>(a.k) + base * D;
        const T *v = static_cast<const T *>(a.v) + base * D;
        const T *g = static_cast<const T *>(a.g) + base * D;
        const T *dO = static_cast<const T *>(a.dO) + base * D;
        const float *qdq = a.dq_ws + base * D;
        T *dk = static_cast<T *>(a.dk_out) + base * D;
        T *dv = static_cast<T *>(a.dv_out) + base * D;
        T *dg = static_cast<T *>(a.dg_out) + base * D;
        float dS[RW][CL];
        load_state_B<D>(dS, a.dX + un * D * D);
        // the dlog_g suffix sum of row w RW + scatter_slot(lane), kept by its writer lane
        float acc = a.carry[un * D + w * RW + scatter_slot<RW>(lane)];
        for (long long b0 = ((a.T - 1) / kTB) * kTB; b0 >= 0; b0 -= kTB) {
            const int nb = (int)(a.T - b0 < kTB ? a.T - b0 : kTB);
            __syncthreads();
            stage<D>(sq, q, b0, nb, Id());
            stage<D>(sk, k, b0, nb, Id());
            stage<D>(sv, v, b0, nb, Id());
            stage<D>(sd, dO, b0, nb, Id());
            stage<D>(sa, g, b0, nb, Exp());
            for (int idx = threadIdx.x; idx < kTB * D; idx += kXThreads)
                sqdq[idx] = idx / D < nb ? qdq[qdq_index(b0 + idx / D, idx % D, D, a.qdq_quad)] : 0.f;
            __syncthreads();
            for (int t = nb - 1; t >= 0; --t) {
                float vj[CL], dj[CL], pre[RW], pv[CL], vdo = 0.f;
#pragma unroll
                for (int c = 0; c < CL; ++c) {
                    vj[c] = sv[t * D + lane + 32 * c];
                    dj[c] = sd[t * D + lane + 32 * c];
                    vdo = fmaf(vj[c], dj[c], vdo);
                    pv[c] = 0.f;
                }
                vdo = warp_sum(vdo);
#pragma unroll
                for (int r = 0; r < RW; ++r) {
                    const int i = w * RW + r;
                    const float qi = sq[t * D + i], ki = sk[t * D + i], ai = sa[t * D + i];
                    pre[r] = 0.f;
#pragma unroll
                    for (int c = 0; c < CL; ++c) {
                        pre[r] = fmaf(dS[r][c], vj[c], pre[r]);  // dS+_t v_t^T
                        dS[r][c] = fmaf(qi, dj[c], dS[r][c]);
                        pv[c] = fmaf(ki, dS[r][c], pv[c]);
                        dS[r][c] *= ai;
                    }
                }
#pragma unroll
                for (int c = 0; c < CL; ++c) spv[(w * kTB + t) * D + lane + 32 * c] = pv[c];
                const float p = warp_reduce_scatter<RW>(pre, lane);
                if (scatter_writer<RW>(lane)) {
                    const int i = w * RW + scatter_slot<RW>(lane);
                    const float ki = sk[t * D + i];
                    acc += sqdq[t * D + i] - ki * p;
                    sdk[t * D + i] = fmaf(sq[t * D + i], vdo, p);
                    sdg[t * D + i] = acc;
                }
            }
            __syncthreads();
            for (int idx = threadIdx.x; idx < nb * D; idx += kXThreads) {
                const int t = idx / D, col = idx % D;
                float s = 0.f;
#pragma unroll
                for (int ww = 0; ww < kXWarps; ++ww) s += spv[(ww * kTB + t) * D + col];
                const long long e = (b0 + t) * D + col;
                dv[e] = from_f32<T>(s);
                dk[e] = from_f32<T>(sdk[idx]);
                dg[e] = from_f32<T>(sdg[idx]);
            }
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------ host side
constexpr int kXBlocksPerSM = 1;

unsigned grid_for(long long units) {
    const long long cap = (long long)kNumSMs * kXBlocksPerSM;
    return (unsigned)(units < cap ? units : cap);
}

template <typename Kern>
cudaError_t launch_x(Kern kern, size_t smem, unsigned grid, cudaStream_t st, const PassArgs &a) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess || grid == 0) return e;
    kern<<<grid, kXThreads, smem, st>>>(a);
    return cudaGetLastError();
}
template <typename Kern>
cudaError_t launch_xb(Kern kern, size_t smem, unsigned grid, cudaStream_t st, const BwdArgs &a) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess || grid == 0) return e;
    kern<<<grid, kXThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <int D, typename T>
cudaError_t exact_pass_dt(const PassArgs &a, PassMode mode, cudaStream_t st) {
    const size_t smem = 6 * kTB * D * sizeof(float);
    const unsigned grid = grid_for((long long)a.BH * a.NP);
    switch (mode) {
        case kPassState: return launch_x(exact_pass_kernel<D, T, kPassState>, smem, grid, st, a);
        case kPassOutput: return launch_x(exact_pass_kernel<D, T, kPassOutput>, smem, grid, st, a);
        case kPassLocal: return launch_x(exact_pass_kernel<D, T, kPassLocal>, smem, grid, st, a);
        case kPassCorrect: return launch_x(exact_pass_kernel<D, T, kPassCorrect>, smem, grid, st, a);
        default: return cudaErrorInvalidValue;
    }
}

template <typename F>
cudaError_t by_shape(int d, la_dtype dt, F f) {
    if (dt == LA_F32) {
        if (d == 32) return f(std::integral_constant<int, 32>(), float());
        if (d == 64) return f(std::integral_constant<int, 64>(), float());
        if (d == 128) return f(std::integral_constant<int, 128>(), float());
    } else {
        if (d == 32) return f(std::integral_constant<int, 32>(), __nv_bfloat16());
        if (d == 64) return f(std::integral_constant<int, 64>(), __nv_bfloat16());
        if (d == 128) return f(std::integral_constant<int, 128>(), __nv_bfloat16());
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_exact_pass(const PassArgs &a, PassMode mode, cudaStream_t st) {
    if (!a.flags || a.dk != a.dv) return cudaErrorInvalidValue;
    return by_shape(a.dk, a.dt, [&](auto dc, auto tv) {
        return exact_pass_dt<decltype(dc)::value, decltype(tv)>(a, mode, st);
    });
}

cudaError_t launch_exact_sequence(const PassArgs &a, const float *S0, float *S_final,
                                  float *S_save, int save_every, cudaStream_t st) {
    if (!a.flags || a.dk != a.dv || save_every < 1) return cudaErrorInvalidValue;
    return by_shape(a.dk, a.dt, [&](auto dc, auto tv) -> cudaError_t {
        constexpr int D = decltype(dc)::value;
        auto kern = exact_sequence_kernel<D, decltype(tv)>;
        const size_t smem = 6 * kTB * D * sizeof(float);
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        const unsigned grid = grid_for(a.BH);
        if (e != cudaSuccess || grid == 0) return e;
        kern<<<grid, kXThreads, smem, st>>>(a, S0, S_final, S_save, save_every);
        return cudaGetLastError();
    });
}

cudaError_t launch_exact_dq(const BwdArgs &a_in, cudaStream_t st) {
    if (!a_in.flags || a_in.dk != a_in.dv || a_in.fine < 1) return cudaErrorInvalidValue;
    BwdArgs a = a_in;
    a.qdq_quad = tc_bwd_supported(a_in);  // the layout the dq sweep of these arguments writes
    return by_shape(a.dk, a.dt, [&](auto dc, auto tv) {
        constexpr int D = decltype(dc)::value;
        return launch_xb(exact_dq_kernel<D, decltype(tv)>, 8 * kTB * D * sizeof(float),
                         grid_for((long long)a.BH * a.NP), st, a);
    });
}

cudaError_t launch_exact_dkv(const BwdArgs &a_in, cudaStream_t st) {
    if (!a_in.flags || !a_in.carry || a_in.dk != a_in.dv) return cudaErrorInvalidValue;
    BwdArgs a = a_in;
    a.qdq_quad = tc_bwd_supported(a_in);
    return by_shape(a.dk, a.dt, [&](auto dc, auto tv) {
        constexpr int D = decltype(dc)::value;
        return launch_xb(exact_dkv_kernel<D, decltype(tv)>,
                         (8 + kXWarps) * kTB * D * sizeof(float),
                         grid_for((long long)a.BH * a.NP), st, a);
    });
}

}  // namespace la
