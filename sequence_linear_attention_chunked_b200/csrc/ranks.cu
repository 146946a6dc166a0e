// ranks.cu -- the All-Scan between devices: the steps that combine the (Gamma, S) pairs of
// whole sequence blocks held by different ranks (ZeCO review, "key machinery": each device
// applies the decayed update S_recv_{p+1} = Gamma_p S_recv_p + S_p to the state it receives and
// passes the accumulated state on; referee major comment 4 fixes that the accumulated state,
// not the local one, moves on).  A rank reduces its own sub-segments to one pair (log Gamma_r,
// S_r) with la_seg_scan and la_seg_log_gamma_total; the pairs of all ranks meet in local HBM
// (an all-gather, or the tree's point-to-point exchanges); the kernels here turn them into the
// state a rank receives.  The recurrence is element-wise over the d_k x d_v state, so every
// kernel is a coalesced float4 stream; they move kilobytes to megabytes.
#include "common.cuh"
#include "internal.h"

namespace la {
namespace {

constexpr int kThreads = 256;

__global__ void log_gamma_total_kernel(const float *__restrict__ lg, int BH, int NP, int dk,
                                       float *__restrict__ out) {
    const long long e = (long long)blockIdx.x * kThreads + threadIdx.x;  // (bh, i)
    if (e >= (long long)BH * dk) return;
    const long long bh = e / dk, i = e % dk;
    const float *p = lg + bh * (long long)NP * dk + i;
    float s = 0.f;
    for (int q = 0; q < NP; ++q) s += p[(long long)q * dk];  // in segment order
    out[e] = s;
}

// Element (bh, i, 4 j) of the exclusive scan over ranks, in rank order (reverse: from the last
// rank down): acc = init; for every rank r' before `rank`: acc = exp(lg[r']) acc + S[r'].
__global__ void rank_scan_kernel(const float4 *__restrict__ S, const float *__restrict__ lg,
                                 const float4 *__restrict__ init, int N, int BH, int dk, int dv4,
                                 int rank, int reverse, float4 *__restrict__ S_in,
                                 float4 *__restrict__ total) {
    const long long per = (long long)dk * dv4, n = (long long)BH * per;
    const long long e = (long long)blockIdx.x * kThreads + threadIdx.x;
    if (e >= n) return;
    const long long bh = e / per, i = (e % per) / dv4;
    float4 acc = init ? init[e] : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k = 0; k < N; ++k) {
        const int r = reverse ? N - 1 - k : k;
        if (r == rank) {
            S_in[e] = acc;
            if (!total) return;
        }
        const float g = __expf(lg[((long long)r * BH + bh) * dk + i]);
        const float4 x = S[(long long)r * n + e];
        acc = make_float4(fmaf(g, acc.x, x.x), fmaf(g, acc.y, x.y), fmaf(g, acc.z, x.z),
                          fmaf(g, acc.w, x.w));
    }
    if (total) total[e] = acc;
}

// (lg_a, S_a) followed by (lg_b, S_b): lg = lg_a + lg_b, S = exp(lg_b) S_a + S_b.  S_out may be
// S_b (each element is read before it is written by the same thread); lg_out is distinct from
// both inputs, since the lanes of a row read lg_b while its first lane writes lg_out.
__global__ void combine_kernel(const float *__restrict__ lga, const float4 *__restrict__ Sa,
                               const float *__restrict__ lgb, const float4 *Sb, int BH, int dk,
                               int dv4, float *__restrict__ lgo, float4 *So) {
    const long long per = (long long)dk * dv4, n = (long long)BH * per;
    const long long e = (long long)blockIdx.x * kThreads + threadIdx.x;
    if (e >= n) return;
    const long long bh = e / per, i = (e % per) / dv4, j4 = e % dv4;
    const long long gi = bh * dk + i;
    const float lb = lgb[gi];
    const float g = __expf(lb);
    const float4 a = Sa[e], b = Sb[e];
    So[e] = make_float4(fmaf(g, a.x, b.x), fmaf(g, a.y, b.y), fmaf(g, a.z, b.z), fmaf(g, a.w, b.w));
    if (j4 == 0) lgo[gi] = lga[gi] + lb;
}

unsigned blocks_for(long long n) { return (unsigned)((n + kThreads - 1) / kThreads); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace
}  // namespace la

extern "C" {

la_status la_seg_log_gamma_total(const float *log_gamma, int BH, int NP, int dk,
                                 float *log_gamma_total, void *cuda_stream) {
    if (BH < 0 || NP < 0 || dk < 1) return la::set_error(LA_ERR_SHAPE, "need BH, NP >= 0, dk >= 1");
    if ((long long)BH * dk > 0 && (!log_gamma_total || (NP > 0 && !log_gamma)))
        return la::set_error(LA_ERR_ARG, "log_gamma and log_gamma_total must be non-null");
    const long long n = (long long)BH * dk;
    if (n == 0) return LA_OK;
    la::log_gamma_total_kernel<<<la::blocks_for(n), la::kThreads, 0,
                                 static_cast<cudaStream_t>(cuda_stream)>>>(log_gamma, BH, NP, dk,
                                                                          log_gamma_total);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? LA_OK : la::set_cuda_error(e, "log-gamma total");
}

la_status la_seg_rank_scan(const float *S_ranks, const float *log_gamma_ranks, const float *init,
                           int N, int BH, int dk, int dv, int rank, int reverse, float *S_in,
                           float *total, void *cuda_stream) {
    if (N < 1 || BH < 0 || dk < 1 || dv < 4 || dv % 4 || rank < 0 || rank >= N)
        return la::set_error(LA_ERR_SHAPE, "need N >= 1, 0 <= rank < N, BH >= 0, dk >= 1, dv a "
                                           "positive multiple of 4 (N=%d rank=%d dv=%d)", N, rank, dv);
    if (BH > 0 && (!S_ranks || !log_gamma_ranks || !S_in))
        return la::set_error(LA_ERR_ARG, "S_ranks, log_gamma_ranks and S_in must be non-null");
    const void *p16[] = {S_ranks, init, S_in, total};
    for (const void *p : p16)
        if (p && !la::aligned16(p)) return la::set_error(LA_ERR_ALIGN, "states must be 16-byte aligned");
    const long long n = (long long)BH * dk * (dv / 4);
    if (n == 0) return LA_OK;
    la::rank_scan_kernel<<<la::blocks_for(n), la::kThreads, 0, static_cast<cudaStream_t>(cuda_stream)>>>(
        reinterpret_cast<const float4 *>(S_ranks), log_gamma_ranks,
        reinterpret_cast<const float4 *>(init), N, BH, dk, dv / 4, rank, reverse,
        reinterpret_cast<float4 *>(S_in), reinterpret_cast<float4 *>(total));
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? LA_OK : la::set_cuda_error(e, "rank scan");
}

la_status la_seg_combine(const float *log_gamma_a, const float *S_a, const float *log_gamma_b,
                         const float *S_b, int BH, int dk, int dv, float *log_gamma_out,
                         float *S_out, void *cuda_stream) {
    if (BH < 0 || dk < 1 || dv < 4 || dv % 4)
        return la::set_error(LA_ERR_SHAPE, "need BH >= 0, dk >= 1, dv a positive multiple of 4");
    if (BH > 0 && (!log_gamma_a || !S_a || !log_gamma_b || !S_b || !log_gamma_out || !S_out))
        return la::set_error(LA_ERR_ARG, "every pointer of la_seg_combine must be non-null");
    const void *p16[] = {S_a, S_b, S_out};
    for (const void *p : p16)
        if (p && !la::aligned16(p)) return la::set_error(LA_ERR_ALIGN, "states must be 16-byte aligned");
    if (S_out == S_a || log_gamma_out == log_gamma_a || log_gamma_out == log_gamma_b)
        return la::set_error(LA_ERR_ARG, "S_out may alias S_b only; log_gamma_out aliases nothing");
    const long long n = (long long)BH * dk * (dv / 4);
    if (n == 0) return LA_OK;
    la::combine_kernel<<<la::blocks_for(n), la::kThreads, 0, static_cast<cudaStream_t>(cuda_stream)>>>(
        log_gamma_a, reinterpret_cast<const float4 *>(S_a), log_gamma_b,
        reinterpret_cast<const float4 *>(S_b), BH, dk, dv / 4, log_gamma_out,
        reinterpret_cast<float4 *>(S_out));
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? LA_OK : la::set_cuda_error(e, "combine");
}

}  // extern "C"
