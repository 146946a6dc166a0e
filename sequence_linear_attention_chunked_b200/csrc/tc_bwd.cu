// tc_bwd.cu -- backward chunk passes on the 5th-generation tensor cores (bf16, d = 128,
// chunk = 64): the dq sweep (forward over chunks) and the reverse sweep (dk, dv, dlog_g).
//
// dq sweep, per chunk with in-chunk cumsum b_t, total b_C, Ktil_s = k_s e^{b_C - b_s},
// S' = diag(e^{b_C}) S (S the state entering the chunk, rows = key dims on TMEM lanes):
//
//   M    = dO V^T                       M=64  (t)  N=64  (s)  K=128 (j)   -> masked s <= t, bf16
//   dS   = Ktil^T V                     M=128 (i)  N=128 (j)  K=64  (s)
//   dq^T = S' dO^T + Ktil^T M^T         M=128 (i)  N=64  (t)  K=128 (j) / 64 (s)
//   dq[t,i] = e^{b_t,i - b_C,i} dq^T[i,t];   S <- S' + dS
//
// The gate warps write e^{b_t - b_C} over the log_g tile (bf16, same swizzled layout) for the
// epilogue's output scaling.  The epilogue also stores q . dq in fp32, which the reverse sweep
// needs for dlog_g.  Role layout, bounded waits and the abort path follow tc_pass.cu.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tc_common.cuh"

namespace la {
namespace {

using namespace sm100;
using namespace tc;

constexpr int kEpiWarps = 8, kGateWarps = 4;
constexpr int kTmaWarp = 12, kMmaWarp = 13;
constexpr int kThreads = 32 * (kEpiWarps + kGateWarps + 2);

// Shared-memory accesses of the output stages as explicit instructions in program order; they
// carry no compiler memory clobber, so the compiler may schedule other work around them.  Each
// kernel reads its factors from tiles it does not write and stages its outputs in tiles that no
// MMA reads any more.
__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ void sts_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v));
}

// Stores the bf16 values of tokens s and s+1 of this lane's dim x into a [64 x 128] swizzled
// tile.  Lanes x and x^1 swap one value so that each writes one 4-byte word (dims x & ~1 and
// x | 1): the even lane row s, the odd lane row s+1.  Two-byte stores would put two lanes on
// each 4-byte word and take two shared-memory wavefronts per instruction.
__device__ __forceinline__ void store_pair(uint32_t tile, int s, int x, float a, float b) {
    const uint32_t p = pack_bf16(a, b);  // low half: token s, high half: token s+1
    const bool odd = x & 1;
    const uint32_t send = odd ? (p & 0xFFFFu) : (p >> 16);
    const uint32_t recv = __shfl_xor_sync(0xFFFFFFFFu, send, 1);
    const uint32_t w = odd ? (recv | (p & 0xFFFF0000u)) : ((p & 0xFFFFu) | (recv << 16));
    sts_u32(tile + tile_off(s + (odd ? 1 : 0), x & ~1), w);
}

// ------------------------------------------------------------------ dq sweep
namespace dqs {

// R^T: the gradient-state sum of the current fine part (when the sweep also produces it).
constexpr uint32_t kColDS = 0, kColDQ = 128, kColSA = 192, kColM = 256, kColR = 320;
constexpr int kStages = 2;
constexpr int off_k = 0, off_v = kTileBytes, off_do = 2 * kTileBytes, off_g = 3 * kTileBytes,
              off_q = 4 * kTileBytes,   // q only feeds the epilogue's q . dq
              off_qh = 5 * kTileBytes;  // Qhat = q e^{B + b_t}, B: log-decay since the part's start
constexpr int kStageBytes = 6 * kTileBytes;
constexpr int off_m = kStages * kStageBytes;
constexpr int off_ec = off_m + CH * CH * 2;
constexpr int off_bar = off_ec + kStages * D * 4;
constexpr int kBars = 3 * kStages + 14;
constexpr int off_misc = off_bar + kBars * 8;
constexpr int kSmemBytes = off_misc + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Bars {
    uint64_t *full, *gated, *empty;
    uint64_t *m_full, *m_free, *p_full, *ds_full, *ds_free, *sa_full, *sa_free, *dq_full,
        *dq_free, *r_full, *r_free, *fin;
};

__device__ void producer(uint8_t *smem, const Bars &b, volatile int *abort, const CUtensorMap *tk,
                         const CUtensorMap *tv, const CUtensorMap *tdo, const CUtensorMap *tg,
                         const CUtensorMap *tq, long long row0, int nchunks) {
    int issued = 0;
    for (int c = 0; c < nchunks; ++c) {
        const int s = c % kStages;
        if (c >= kStages && !mbar_wait(&b.empty[s], ((c / kStages) - 1) & 1, abort)) break;
        mbar_arrive_expect_tx(&b.full[s], 5 * kTileBytes);
        uint8_t *st = smem + s * kStageBytes;
        const int y = (int)(row0 + (long long)c * CH);
        tma_load_2d(st + off_k, tk, 0, y, &b.full[s]);
        tma_load_2d(st + off_k + kHalfBytes, tk, 64, y, &b.full[s]);
        tma_load_2d(st + off_v, tv, 0, y, &b.full[s]);
        tma_load_2d(st + off_v + kHalfBytes, tv, 64, y, &b.full[s]);
        tma_load_2d(st + off_do, tdo, 0, y, &b.full[s]);
        tma_load_2d(st + off_do + kHalfBytes, tdo, 64, y, &b.full[s]);
        tma_load_2d(st + off_g, tg, 0, y, &b.full[s]);
        tma_load_2d(st + off_g + kHalfBytes, tg, 64, y, &b.full[s]);
        tma_load_2d(st + off_q, tq, 0, y, &b.full[s]);
        tma_load_2d(st + off_q + kHalfBytes, tq, 64, y, &b.full[s]);
        issued = c + 1;
    }
    if (*abort)
        for (int c = issued > kStages ? issued - kStages : 0; c < issued; ++c)
            wait_drain(&b.full[c % kStages], (c / kStages) & 1);
}

__device__ void mma_issuer(uint8_t *smem, const Bars &b, volatile int *abort, uint32_t tmem,
                           int nchunks, bool dstate, int cpf) {
    constexpr uint32_t i_m = idesc_bf16_f32(64, 64, 0, 0);
    constexpr uint32_t i_ds = idesc_bf16_f32(128, 128, 1, 1);
    constexpr uint32_t i_dqb = idesc_bf16_f32(128, 64, 1, 0);
    constexpr uint32_t i_dqa = idesc_bf16_f32(128, 64, 0, 0);
    const uint32_t m_addr = smem_u32(smem + off_m);
    for (int c = 0; c < nchunks; ++c) {
        const int s = c % kStages;
        const uint32_t st = smem_u32(smem + s * kStageBytes);
        const uint32_t ka = st + off_k, va = st + off_v, da = st + off_do;
        // M = dO V^T reads untouched tiles: it runs while the gate warps rescale k
        if (!warp_wait(&b.full[s], (c / kStages) & 1, abort)) break;
        if (c > 0 && !warp_wait(b.m_free, (c - 1) & 1, abort)) break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_ss(tmem + kColM, desc_kmajor(da, kk), desc_kmajor(va, kk), i_m, kk > 0);
            mma_commit(b.m_full);
        }
        __syncwarp();
        if (!warp_wait(&b.gated[s], (c / kStages) & 1, abort)) break;
        if (c > 0 && !warp_wait(b.ds_free, (c - 1) & 1, abort)) break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // dS = Ktil^T V
                mma_ss(tmem + kColDS, desc_mnmajor(ka, kk), desc_mnmajor(va, kk), i_ds, kk > 0);
            mma_commit(b.ds_full);
        }
        __syncwarp();
        if (dstate) {  // R^T += dO^T Qhat over the fine part; before dq so that dq_full covers it
            const int part = c / cpf;
            const bool first = c % cpf == 0;
            if (first && part > 0 && !warp_wait(b.r_free, (part - 1) & 1, abort)) break;
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ss(tmem + kColR, desc_mnmajor(da, kk), desc_mnmajor(st + off_qh, kk), i_ds,
                           (!first || kk > 0) ? 1u : 0u);
                if (c % cpf == cpf - 1) mma_commit(b.r_full);
            }
            __syncwarp();
        }
        if (c > 0 && !warp_wait(b.dq_free, (c - 1) & 1, abort)) break;
        if (!warp_wait(b.p_full, c & 1, abort)) break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // dq^T = Ktil^T M^T
                mma_ss(tmem + kColDQ, desc_mnmajor(ka, kk), smem_desc_sw128(m_addr + kk * 32, 16, 1024),
                       i_dqb, kk > 0);
        }
        __syncwarp();
        if (!warp_wait(b.sa_full, c & 1, abort)) break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // dq^T += S' dO^T, A from tensor memory
                mma_ts(tmem + kColDQ, tmem + kColSA + kk * 8, desc_kmajor(da, kk), i_dqa, 1u);
            mma_commit(b.dq_full);
            mma_commit(b.sa_free);
            mma_commit(&b.empty[s]);
        }
        __syncwarp();
    }
    if (elect_one()) mma_commit(b.fin);
    __syncwarp();
    wait_drain(b.fin, 0);
}

// Gate warps: cumsum as in the forward pass, Ktil in place of k, e^{b_t - b_C} in place of
// log_g, e^{b_C} per key dim for the state decay; with the gradient-state sum, also
// Qhat = q e^{B + b_t} (B: log-decay from the fine part's start to the chunk's start, so that
// e^{B + b_t} = e^{B + b_C} e^{b_t - b_C}) and each part's log-decay sum.
__device__ void gate_role(uint8_t *smem, const Bars &b, volatile int *abort, const BwdArgs &a,
                          int nchunks, bool dstate, int cpf, int bh, int j) {
    const int gw = (threadIdx.x >> 5) - kEpiWarps;
    const int lane = threadIdx.x & 31;
    const int tg = lane >> 2, ig = lane & 3;
    const int i0 = gw * 32 + ig * 8;
    float *ec = reinterpret_cast<float *>(smem + off_ec);
    bool range_bad = false;
    float logB[8];  // log-decay from the fine part's start through the current chunk
#pragma unroll
    for (int e = 0; e < 8; ++e) logB[e] = 0.f;
    for (int c = 0; c < nchunks; ++c) {
        const int s = c % kStages;
        if (!mbar_wait(&b.full[s], (c / kStages) & 1, abort)) break;
        uint8_t *st = smem + s * kStageBytes;
        float bt[8][8];
        {
            uint4 graw[8];
#pragma unroll
            for (int r = 0; r < 8; ++r)
                graw[r] = *reinterpret_cast<const uint4 *>(st + off_g + tile_off(tg * 8 + r, i0));
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                float f[8];
                unpack8(graw[r], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) bt[r][e] = (r ? bt[r - 1][e] : 0.f) + f[e];
            }
        }
        float incl[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) incl[e] = bt[7][e];
#pragma unroll
        for (int d = 1; d < 8; d <<= 1) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float up = __shfl_up_sync(0xFFFFFFFFu, incl[e], 4 * d);
                if (tg >= d) incl[e] += up;
            }
        }
        float nbCl[8], eB[8];
        const bool part_start = c % cpf == 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float bC = __shfl_sync(0xFFFFFFFFu, incl[e], 28 + ig);
            const float off = incl[e] - bt[7][e];
#pragma unroll
            for (int r = 0; r < 8; ++r) bt[r][e] += off;
            nbCl[e] = -bC * kLog2e;
            range_bad |= !(fabsf(bC) <= kGateRangeLimit);
            logB[e] = (part_start ? 0.f : logB[e]) + bC;
            eB[e] = dstate ? ex2_approx(logB[e] * kLog2e) : 0.f;
        }
        if (dstate && c % cpf == cpf - 1 && tg == 0) {  // the part's log-decay sum
            const long long jf = (long long)j * a.fine + c / cpf;
            float4 *lg = reinterpret_cast<float4 *>(a.logG + ((long long)bh * a.NP * a.fine + jf) * D + i0);
            lg[0] = make_float4(logB[0], logB[1], logB[2], logB[3]);
            lg[1] = make_float4(logB[4], logB[5], logB[6], logB[7]);
        }
        if (tg == 0) {
            float4 *e4 = reinterpret_cast<float4 *>(ec + s * D + i0);
            e4[0] = make_float4(ex2_approx(-nbCl[0]), ex2_approx(-nbCl[1]), ex2_approx(-nbCl[2]),
                                ex2_approx(-nbCl[3]));
            e4[1] = make_float4(ex2_approx(-nbCl[4]), ex2_approx(-nbCl[5]), ex2_approx(-nbCl[6]),
                                ex2_approx(-nbCl[7]));
        }
#pragma unroll
        for (int r0 = 0; r0 < 8; r0 += 2) {
            uint4 kr[2], qr[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const uint32_t off = tile_off(tg * 8 + r0 + r, i0);
                kr[r] = *reinterpret_cast<const uint4 *>(st + off_k + off);
                if (dstate) qr[r] = *reinterpret_cast<const uint4 *>(st + off_q + off);
            }
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const uint32_t off = tile_off(tg * 8 + r0 + r, i0);
                float x[8], f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = fmaf(bt[r0 + r][e], kLog2e, nbCl[e]);
                unpack8(kr[r], f);
                uint32_t wk[4], wf[4], wq[4];
                float fq[8];
                if (dstate) unpack8(qr[r], fq);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float u0 = ex2_approx(x[2 * e]), u1 = ex2_approx(x[2 * e + 1]);
                    wk[e] = pack_bf16(f[2 * e] * ex2_approx(-x[2 * e]), f[2 * e + 1] * ex2_approx(-x[2 * e + 1]));
                    wf[e] = pack_bf16(u0, u1);
                    if (dstate)
                        wq[e] = pack_bf16(fq[2 * e] * u0 * eB[2 * e], fq[2 * e + 1] * u1 * eB[2 * e + 1]);
                }
                *reinterpret_cast<uint4 *>(st + off_k + off) = make_uint4(wk[0], wk[1], wk[2], wk[3]);
                *reinterpret_cast<uint4 *>(st + off_g + off) = make_uint4(wf[0], wf[1], wf[2], wf[3]);
                if (dstate)
                    *reinterpret_cast<uint4 *>(st + off_qh + off) = make_uint4(wq[0], wq[1], wq[2], wq[3]);
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&b.gated[s]);
    }
    if (range_bad && a.status) atomicOr(a.status, kStatusGateRange);
}

// Epilogue warps: thread (w, lane) owns key dim i = 32 (w % 4) + lane (its TMEM lane) and the
// half h = w / 4 of the state row (value dims 64h .. 64h+63) and of each chunk's 64 tokens.
__device__ void epilogue_role(uint8_t *smem, const Bars &b, volatile int *abort, const BwdArgs &a,
                              uint32_t tmem, int bh, int j, long long row0, int nchunks,
                              bool dstate) {
    constexpr int HD = D / 2;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int quarter = warp & 3, h = warp >> 2;
    const int i = quarter * 32 + lane;
    const uint32_t lrow = (uint32_t)(quarter * 32) << 16;
    const float *ec = reinterpret_cast<const float *>(smem + off_ec);

    float S[HD];  // S[i][64h + e]
    if (a.S_recv) {
        const float4 *Si = reinterpret_cast<const float4 *>(
            a.S_recv + ((long long)bh * a.NP + j) * D * D + (long long)i * D + h * HD);
#pragma unroll
        for (int e4 = 0; e4 < HD / 4; ++e4) {
            const float4 v = Si[e4];
            S[4 * e4] = v.x; S[4 * e4 + 1] = v.y; S[4 * e4 + 2] = v.z; S[4 * e4 + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int e = 0; e < HD; ++e) S[e] = 0.f;
    }
    const int cpf = nchunks / a.fine;  // chunks per fine part
    for (int c = 0; c < nchunks; ++c) {
        const int s = c % kStages;
        uint8_t *st = smem + s * kStageBytes;
        uint32_t r[32];

        if (a.S_fine && c % cpf == 0) {  // the state entering fine part c / cpf
            float4 *Sf = reinterpret_cast<float4 *>(
                a.S_fine + (((long long)bh * a.NP + j) * a.fine + c / cpf) * D * D + (long long)i * D + h * HD);
#pragma unroll
            for (int e4 = 0; e4 < HD / 4; ++e4)
                Sf[e4] = make_float4(S[4 * e4], S[4 * e4 + 1], S[4 * e4 + 2], S[4 * e4 + 3]);
        }
        {  // (a) M -> causal mask -> bf16 tile (K-major rows t)
            if (!mbar_wait(b.m_full, c & 1, abort)) break;
            tc_fence_after();
            tmem_ld32(tmem + lrow + kColM + h * 32, r);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(b.m_free);
            if (lane < 16) {
                const int t = quarter * 16 + lane;
                uint8_t *mrow = smem + off_m + t * 128;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    uint32_t w4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int sl = jj * 8 + 2 * e, s0 = h * 32 + sl;
                        w4[e] = pack_bf16(s0 <= t ? __uint_as_float(r[sl]) : 0.f,
                                          s0 + 1 <= t ? __uint_as_float(r[sl + 1]) : 0.f);
                    }
                    *reinterpret_cast<uint4 *>(mrow + (((h * 4 + jj) ^ (t & 7)) << 4)) =
                        make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(b.p_full);
        }
        // (b) S' = diag(e^{b_C}) S; bf16 copy into tensor memory (A of dq^T += S' dO^T)
        if (!mbar_wait(&b.gated[s], (c / kStages) & 1, abort)) break;
        const float e_i = ec[s * D + i];
#pragma unroll
        for (int e = 0; e < HD; ++e) S[e] *= e_i;
        if (c > 0 && !mbar_wait(b.sa_free, (c - 1) & 1, abort)) break;
        tc_fence_after();
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = pack_bf16(S[2 * e], S[2 * e + 1]);
        tmem_st32(tmem + lrow + kColSA + h * 32, r);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(b.sa_full);
        // (c) S = S' + dS
        if (!mbar_wait(b.ds_full, c & 1, abort)) break;
        tc_fence_after();
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            tmem_ld32(tmem + lrow + kColDS + h * HD + p * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) S[p * 32 + e] += __uint_as_float(r[e]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(b.ds_free);
        // (d) dq rows t = 32h .. 32h+31, column i, and q . dq, stored straight from registers:
        // q . dq (fp32) as one 128-byte line per warp and token, dq (bf16) as 4-byte words
        // (lanes i and i^1 swap one token, so each writes dims i & ~1, i | 1 of one token)
        if (!mbar_wait(b.dq_full, c & 1, abort)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(st);
        const long long tok0 = row0 + (long long)c * CH + h * 32;
        __nv_bfloat16 *dq = static_cast<__nv_bfloat16 *>(a.dq_out);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint32_t r16[16];
            tmem_ld16(tmem + lrow + kColDQ + h * 32 + hh * 16, r16);
            tmem_wait_ld();
            if (hh == 1) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(b.dq_free);
            }
#pragma unroll
            for (int t0 = 0; t0 < 16; t0 += 8) {
                uint32_t fq[8];  // factor e^{b_t - b_C} (low half) and q (high half), bf16
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t off = tile_off(h * 32 + hh * 16 + t0 + e, i);
                    fq[e] = lds_u16(sa + off_g + off) | (lds_u16(sa + off_q + off) << 16);
                }
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const long long t = tok0 + hh * 16 + t0 + e;
                    const float v0 = __uint_as_float(r16[t0 + e]) * __uint_as_float(fq[e] << 16);
                    const float v1 = __uint_as_float(r16[t0 + e + 1]) * __uint_as_float(fq[e + 1] << 16);
                    a.dq_ws[t * D + i] = __uint_as_float(fq[e] & 0xFFFF0000u) * v0;
                    a.dq_ws[(t + 1) * D + i] = __uint_as_float(fq[e + 1] & 0xFFFF0000u) * v1;
                    const uint32_t p = pack_bf16(v0, v1);  // low: token t, high: token t+1
                    const bool odd = i & 1;
                    const uint32_t recv = __shfl_xor_sync(0xFFFFFFFFu, odd ? (p & 0xFFFFu) : (p >> 16), 1);
                    const uint32_t w = odd ? (recv | (p & 0xFFFF0000u)) : ((p & 0xFFFFu) | (recv << 16));
                    *reinterpret_cast<uint32_t *>(dq + (t + (odd ? 1 : 0)) * D + (i & ~1)) = w;
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&b.empty[s]);  // this warp's reads of the stage are done
        if (dstate && c % cpf == cpf - 1) {  // the fine part's gradient state R[i'][j] = R^T[j][i']
            if (!mbar_wait(b.r_full, (c / cpf) & 1, abort)) break;
            tc_fence_after();
            const long long jf = (long long)j * a.fine + c / cpf;
            float *Ro = a.dSloc + ((long long)bh * a.NP * a.fine + jf) * D * D + (h * HD) * D + i;
#pragma unroll 1
            for (int p = 0; p < 4; ++p, Ro += 16 * D) {  // key dims h HD + 16p .. +15
                uint32_t r16[16];
                tmem_ld16(tmem + lrow + kColR + h * HD + p * 16, r16);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) Ro[e * D] = __uint_as_float(r16[e]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(b.r_free);
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
tc_dq_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
             const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_g,
             const __grid_constant__ CUtensorMap tm_q, const BwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + off_bar);
    Bars b;
    b.full = bar;
    b.gated = bar + kStages;
    b.empty = bar + 2 * kStages;
    uint64_t *x = bar + 3 * kStages;
    b.m_full = x + 0; b.m_free = x + 1; b.p_full = x + 2; b.ds_full = x + 3; b.ds_free = x + 4;
    b.sa_full = x + 5; b.sa_free = x + 6; b.dq_full = x + 7; b.dq_free = x + 8;
    b.r_full = x + 9; b.r_free = x + 10; b.fin = x + 11;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + off_misc);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + off_misc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x / a.NP, j = blockIdx.x % a.NP;
    const long long row0 = (long long)bh * a.L + (long long)j * a.T;
    const int nchunks = (int)(a.T / CH);
    const bool dstate = a.dSloc && a.logG;  // also the fine parts' gradient states
    const int cpf = nchunks / a.fine;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&b.full[s], 1);
            mbar_init(&b.gated[s], kGateWarps);
            mbar_init(&b.empty[s], 1 + kEpiWarps);
        }
        mbar_init(b.m_full, 1);
        mbar_init(b.m_free, kEpiWarps);
        mbar_init(b.p_full, kEpiWarps);
        mbar_init(b.ds_full, 1);
        mbar_init(b.ds_free, kEpiWarps);
        mbar_init(b.sa_full, kEpiWarps);
        mbar_init(b.sa_free, 1);
        mbar_init(b.dq_full, 1);
        mbar_init(b.dq_free, kEpiWarps);
        mbar_init(b.r_full, 1);
        mbar_init(b.r_free, kEpiWarps);
        mbar_init(b.fin, 1);
        *abort = 0;
        mbar_fence_init();
    }
    if (warp == kTmaWarp && lane == 0) {
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_do);
        prefetch_tmap(&tm_g);
        prefetch_tmap(&tm_q);
    }
    if (warp == kMmaWarp) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (warp == kTmaWarp) {
        if (lane == 0) producer(smem, b, abort, &tm_k, &tm_v, &tm_do, &tm_g, &tm_q, row0, nchunks);
    } else if (warp == kMmaWarp) {
        mma_issuer(smem, b, abort, tmem, nchunks, dstate, cpf);
    } else if (warp >= kEpiWarps) {
        gate_role(smem, b, abort, a, nchunks, dstate, cpf, bh, j);
    } else {
        epilogue_role(smem, b, abort, a, tmem, bh, j, row0, nchunks, dstate);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (threadIdx.x == 0 && *abort && a.status) atomicOr(a.status, kStatusTimeout);
}

}  // namespace dqs

// ------------------------------------------------------------------ reverse sweep
// Per chunk, last to first, with dS the gradient of the state at the chunk's end (rows = key
// dims; starts at dX of the part), Qbar'_t = q_t e^{b_t - b_C}, Ktil_s = k_s e^{b_C - b_s}:
//
//   M     = dO V^T,  A = Qbar' Ktil^T   M=64  (t) N=64 (s) K=128          -> masked s <= t, bf16
//   dk^T  = Qbar'^T M + dS V^T          M=128 (i) N=64 (s) K=64 (t) / 128 (j)
//   dv^T  = dO^T A + dS^T Ktil^T        M=128 (j) N=64 (s) K=64 (t) / 128 (i)
//   dS   += Qbar'^T dO                  M=128 (i) N=128 (j) K=64 (t), accumulated in TMEM
//   dk[s,i] = e^{b_C,i - b_s,i} dk^T[i,s];   dS <- diag(e^{b_C}) dS
//   dlog_g_s = rowsum(S_end . dX) + sum_{u >= s in the part} (q_u dq_u - k_u dk_u)
//
// Roles (448 threads): warps 0-3 carry dS -- the fp32 dS lives in tensor memory (row i on lane
// i), they apply the decay, write its bf16 copy into a shared [i][j] tile (read by the MMAs as
// the K-major A operand of dS V^T and the MN-major A operand of dS^T Ktil^T) and turn M and A
// into masked bf16 tiles (double-buffered); warps 4-7 read dk^T and dv^T (double-buffered in
// TMEM; thread x owns key / value dim x for all 64 tokens of the chunk, so the dlog_g suffix
// sums need no exchange), stage dk, dlog_g and dv in the stage's v, q and dO tiles (free by then)
// and write them with TMA stores; warps 8-11 gates; 12 TMA; 13 MMA.
namespace dkv {

constexpr int kStateWarps = 4, kOutWarps = 4;
constexpr uint32_t kColM = 0, kColA = 64, kColDK = 128, kColDV = 256, kColDS = 384;
constexpr int kStages = 2;
constexpr int off_q = 0, off_k = kTileBytes, off_v = 2 * kTileBytes, off_do = 3 * kTileBytes,
              off_g = 4 * kTileBytes;
constexpr int kStageBytes = 5 * kTileBytes;
constexpr int kDsHalf = 128 * 128;            // one 64-column half of the [128 x 128] bf16 dS tile
constexpr int kMaskBytes = CH * CH * 2;       // one masked 64 x 64 bf16 tile
constexpr int off_ma = kStages * kStageBytes;  // 2 buffers x (M tile, A tile)
constexpr int off_ds = off_ma + 4 * kMaskBytes;
constexpr int off_ec = off_ds + 2 * kDsHalf;
constexpr int off_bar = off_ec + kStages * D * 4;
constexpr int kBars = 3 * kStages + 15;
constexpr int off_misc = off_bar + kBars * 8;
constexpr int kSmemBytes = off_misc + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Bars {
    uint64_t *full, *gated, *empty;
    uint64_t *mm_full, *mm_free, *p_full, *dst_full, *dk_full, *dk_free, *dv_full, *dv_free,
        *dsn_full, *osync, *fin;
};

// [128 rows][128 cols] bf16 tile as two 64-column halves of 16 KiB, 128-byte swizzle.
__device__ __forceinline__ uint32_t ds_off(int row, int col) {
    const int half = col >> 6, cc = col & 63;
    return (uint32_t)(half * kDsHalf + row * 128 + (((cc >> 3) ^ (row & 7)) << 4) + ((cc & 7) << 1));
}

__device__ void producer(uint8_t *smem, const Bars &b, volatile int *abort, const CUtensorMap *tq,
                         const CUtensorMap *tk, const CUtensorMap *tv, const CUtensorMap *tdo,
                         const CUtensorMap *tg, const float *qdq, long long row0, int nchunks) {
    int issued = 0;
    for (int it = 0; it < nchunks; ++it) {
        const int s = it % kStages;
        const int c = nchunks - 1 - it;  // last chunk first
        // the chunk's q . dq rows (read with plain loads by the output warps) on their way to L2
        bulk_prefetch_l2(qdq + (row0 + (long long)c * CH) * D, CH * D * 4);
        if (it >= kStages && !mbar_wait(&b.empty[s], ((it / kStages) - 1) & 1, abort)) break;
        mbar_arrive_expect_tx(&b.full[s], kStageBytes);
        uint8_t *st = smem + s * kStageBytes;
        const int y = (int)(row0 + (long long)c * CH);
        tma_load_2d(st + off_q, tq, 0, y, &b.full[s]);
        tma_load_2d(st + off_q + kHalfBytes, tq, 64, y, &b.full[s]);
        tma_load_2d(st + off_k, tk, 0, y, &b.full[s]);
        tma_load_2d(st + off_k + kHalfBytes, tk, 64, y, &b.full[s]);
        tma_load_2d(st + off_v, tv, 0, y, &b.full[s]);
        tma_load_2d(st + off_v + kHalfBytes, tv, 64, y, &b.full[s]);
        tma_load_2d(st + off_do, tdo, 0, y, &b.full[s]);
        tma_load_2d(st + off_do + kHalfBytes, tdo, 64, y, &b.full[s]);
        tma_load_2d(st + off_g, tg, 0, y, &b.full[s]);
        tma_load_2d(st + off_g + kHalfBytes, tg, 64, y, &b.full[s]);
        issued = it + 1;
    }
    if (*abort)
        for (int it = issued > kStages ? issued - kStages : 0; it < issued; ++it)
            wait_drain(&b.full[it % kStages], (it / kStages) & 1);
}

// The whole warp walks the loop; one elected lane issues.  Per chunk: dk^T and dv^T into
// buffer it % 2 after the dS update (so that dk_full also frees the q tile), then the next
// chunk's M and A (so that they are ready when the dS warps finish the decay).
__device__ void mma_issuer(uint8_t *smem, const Bars &b, volatile int *abort, uint32_t tmem,
                           int nchunks) {
    constexpr uint32_t i_sq = idesc_bf16_f32(64, 64, 0, 0);      // M, A
    constexpr uint32_t i_dsn = idesc_bf16_f32(128, 128, 1, 1);   // Qbar'^T dO
    constexpr uint32_t i_dka = idesc_bf16_f32(128, 64, 1, 1);    // Qbar'^T M
    constexpr uint32_t i_dkb = idesc_bf16_f32(128, 64, 0, 0);    // dS V^T
    constexpr uint32_t i_dva = idesc_bf16_f32(128, 64, 1, 1);    // dO^T A
    constexpr uint32_t i_dvb = idesc_bf16_f32(128, 64, 1, 0);    // dS^T Ktil^T
    const uint32_t base = smem_u32(smem);
    const uint32_t ma_addr = base + off_ma, ds_addr = base + off_ds;
    auto stage = [&](int it) { return base + (uint32_t)((it % kStages) * kStageBytes); };
    auto issue_ma = [&](int it) {
        const uint32_t st = stage(it);
        if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // M = dO V^T
                mma_ss(tmem + kColM, desc_kmajor(st + off_do, kk), desc_kmajor(st + off_v, kk), i_sq,
                       kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // A = Qbar' Ktil^T
                mma_ss(tmem + kColA, desc_kmajor(st + off_q, kk), desc_kmajor(st + off_k, kk), i_sq,
                       kk > 0);
            mma_commit(b.mm_full);
        }
        __syncwarp();
    };
    bool ok = nchunks > 0 && warp_wait(&b.gated[0], 0, abort);
    tc_fence_after();
    if (ok) issue_ma(0);
    for (int it = 0; ok && it < nchunks; ++it) {
        const int s = it % kStages, bb = it & 1;
        const uint32_t st = stage(it);
        const uint32_t qa = st + off_q, ka = st + off_k, va = st + off_v, da = st + off_do;
        const uint32_t mt = ma_addr + bb * 2 * kMaskBytes, at = mt + kMaskBytes;
        if (!(ok = warp_wait(b.p_full, it & 1, abort))) break;
        if (!(ok = warp_wait(b.dst_full, it & 1, abort))) break;
        if (it >= 2) {
            if (!(ok = warp_wait(&b.dk_free[bb], ((it >> 1) - 1) & 1, abort))) break;
            if (!(ok = warp_wait(&b.dv_free[bb], ((it >> 1) - 1) & 1, abort))) break;
        }
        tc_fence_after();
        if (elect_one()) {
            const uint32_t dk_col = tmem + kColDK + bb * 64, dv_col = tmem + kColDV + bb * 64;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // dS += Qbar'^T dO  (dk and dv read the old dS tile)
                mma_ss(tmem + kColDS, desc_mnmajor(qa, kk), desc_mnmajor(da, kk), i_dsn, 1u);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // dk^T = Qbar'^T M   (B: M tile read MN-major)
                mma_ss(dk_col, desc_mnmajor(qa, kk), smem_desc_sw128(mt + kk * 2048, kHalfBytes, 1024),
                       i_dka, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // dk^T += dS V^T   (A: dS tile K-major, 128 rows)
                mma_ss(dk_col, smem_desc_sw128(ds_addr + (kk >> 2) * kDsHalf + (kk & 3) * 32, 16, 1024),
                       desc_kmajor(va, kk), i_dkb, 1u);
            mma_commit(&b.dk_full[bb]);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // dv^T = dO^T A   (B: A tile read MN-major)
                mma_ss(dv_col, desc_mnmajor(da, kk), smem_desc_sw128(at + kk * 2048, kHalfBytes, 1024),
                       i_dva, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // dv^T += dS^T Ktil^T   (A: dS tile read MN-major)
                mma_ss(dv_col, smem_desc_sw128(ds_addr + kk * 2048, kDsHalf, 1024), desc_kmajor(ka, kk),
                       i_dvb, 1u);
            mma_commit(&b.dv_full[bb]);
            mma_commit(b.dsn_full);  // the dS tile is read out as well
            mma_commit(&b.empty[s]);
        }
        __syncwarp();
        if (it + 1 < nchunks) {  // the next chunk's M and A, once its tiles are gated
            if (!(ok = warp_wait(&b.gated[(it + 1) % kStages], ((it + 1) / kStages) & 1, abort))) break;
            if (!(ok = warp_wait(b.mm_free, it & 1, abort))) break;
            tc_fence_after();
            issue_ma(it + 1);
        }
    }
    if (elect_one()) mma_commit(b.fin);
    __syncwarp();
    wait_drain(b.fin, 0);
}

// Gate warps: Qbar' and Ktil in place of q and k, e^{b_C - b_t} in place of log_g (the dk
// output factor), e^{b_C} per key dim.
__device__ void gate_role(uint8_t *smem, const Bars &b, volatile int *abort, const BwdArgs &a,
                          int nchunks) {
    const int gw = (threadIdx.x >> 5) - kEpiWarps;
    const int lane = threadIdx.x & 31;
    const int tg = lane >> 2, ig = lane & 3;
    const int i0 = gw * 32 + ig * 8;
    float *ec = reinterpret_cast<float *>(smem + off_ec);
    bool range_bad = false;
    for (int it = 0; it < nchunks; ++it) {
        const int s = it % kStages;
        if (!mbar_wait(&b.full[s], (it / kStages) & 1, abort)) break;
        uint8_t *st = smem + s * kStageBytes;
        float bt[8][8];
        {
            uint4 graw[8];
#pragma unroll
            for (int r = 0; r < 8; ++r)
                graw[r] = *reinterpret_cast<const uint4 *>(st + off_g + tile_off(tg * 8 + r, i0));
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                float f[8];
                unpack8(graw[r], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) bt[r][e] = (r ? bt[r - 1][e] : 0.f) + f[e];
            }
        }
        float incl[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) incl[e] = bt[7][e];
#pragma unroll
        for (int d = 1; d < 8; d <<= 1) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float up = __shfl_up_sync(0xFFFFFFFFu, incl[e], 4 * d);
                if (tg >= d) incl[e] += up;
            }
        }
        float nbCl[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float bC = __shfl_sync(0xFFFFFFFFu, incl[e], 28 + ig);
            const float off = incl[e] - bt[7][e];
#pragma unroll
            for (int r = 0; r < 8; ++r) bt[r][e] += off;
            nbCl[e] = -bC * kLog2e;
            range_bad |= !(fabsf(bC) <= kGateRangeLimit);
        }
        if (tg == 0) {
            float4 *e4 = reinterpret_cast<float4 *>(ec + s * D + i0);
            e4[0] = make_float4(ex2_approx(-nbCl[0]), ex2_approx(-nbCl[1]), ex2_approx(-nbCl[2]),
                                ex2_approx(-nbCl[3]));
            e4[1] = make_float4(ex2_approx(-nbCl[4]), ex2_approx(-nbCl[5]), ex2_approx(-nbCl[6]),
                                ex2_approx(-nbCl[7]));
        }
#pragma unroll
        for (int r0 = 0; r0 < 8; r0 += 2) {
            uint4 qr[2], kr[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const uint32_t off = tile_off(tg * 8 + r0 + r, i0);
                qr[r] = *reinterpret_cast<const uint4 *>(st + off_q + off);
                kr[r] = *reinterpret_cast<const uint4 *>(st + off_k + off);
            }
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const uint32_t off = tile_off(tg * 8 + r0 + r, i0);
                float x[8], fq[8], fk[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = fmaf(bt[r0 + r][e], kLog2e, nbCl[e]);
                unpack8(qr[r], fq);
                unpack8(kr[r], fk);
                uint32_t wq[4], wk[4], wf[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float u0 = ex2_approx(x[2 * e]), u1 = ex2_approx(x[2 * e + 1]);
                    const float d0 = ex2_approx(-x[2 * e]), d1 = ex2_approx(-x[2 * e + 1]);
                    wq[e] = pack_bf16(fq[2 * e] * u0, fq[2 * e + 1] * u1);
                    wk[e] = pack_bf16(fk[2 * e] * d0, fk[2 * e + 1] * d1);
                    wf[e] = pack_bf16(d0, d1);
                }
                *reinterpret_cast<uint4 *>(st + off_q + off) = make_uint4(wq[0], wq[1], wq[2], wq[3]);
                *reinterpret_cast<uint4 *>(st + off_k + off) = make_uint4(wk[0], wk[1], wk[2], wk[3]);
                *reinterpret_cast<uint4 *>(st + off_g + off) = make_uint4(wf[0], wf[1], wf[2], wf[3]);
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&b.gated[s]);
    }
    if (range_bad && a.status) atomicOr(a.status, kStatusGateRange);
}

// Writes a masked (s <= t) bf16 copy of a M=64 TMEM accumulator half into a 64x64 tile.
__device__ __forceinline__ void masked_tile(uint8_t *tile, const uint32_t (&r)[32], int quarter,
                                            int h, int lane) {
    if (lane < 16) {
        const int t = quarter * 16 + lane;
        uint8_t *row = tile + t * 128;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int sl = jj * 8 + 2 * e, s0 = h * 32 + sl;
                w4[e] = pack_bf16(s0 <= t ? __uint_as_float(r[sl]) : 0.f,
                                  s0 + 1 <= t ? __uint_as_float(r[sl + 1]) : 0.f);
            }
            *reinterpret_cast<uint4 *>(row + (((h * 4 + jj) ^ (t & 7)) << 4)) =
                make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
    }
}

// Warps 0-3: thread i owns row i of dS (TMEM lane i).  Per chunk: the decay by the previous
// chunk's e^{b_C} (S_new = diag(e^{b_C}) (dS + Qbar'^T dO), the sum formed by the MMA), the
// bf16 copy of row i into the dS tile, then the masked M and A tiles of the chunk.
__device__ void state_role(uint8_t *smem, const Bars &b, volatile int *abort, const BwdArgs &a,
                           uint32_t tmem, int bh, int j, int nchunks) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = warp * 32 + lane;
    const uint32_t lrow = (uint32_t)(warp * 32) << 16;
    const float *ec = reinterpret_cast<const float *>(smem + off_ec);
    uint32_t r[32];
    {  // dS at the part's end: dX
        const float4 *x4 = reinterpret_cast<const float4 *>(a.dX + ((long long)bh * a.NP + j) * D * D +
                                                            (long long)i * D);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) {
                const float4 v = x4[p * 8 + e4];
                r[4 * e4] = __float_as_uint(v.x); r[4 * e4 + 1] = __float_as_uint(v.y);
                r[4 * e4 + 2] = __float_as_uint(v.z); r[4 * e4 + 3] = __float_as_uint(v.w);
            }
            tmem_st32(tmem + lrow + kColDS + p * 32, r);
        }
        tmem_wait_st();
        tc_fence_before();
    }
    for (int it = 0; it < nchunks; ++it) {
        // (1) dS of this chunk's end: decayed unless it is the part's end
        if (it > 0) {
            if (!mbar_wait(b.dsn_full, (it - 1) & 1, abort)) break;
        }
        tc_fence_after();
        const uint64_t e2 = it > 0 ? (uint64_t)__float_as_uint(ec[((it - 1) % kStages) * D + i]) * 0x100000001ull
                                   : 0ull;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            tmem_ld32(tmem + lrow + kColDS + p * 32, r);
            tmem_wait_ld();
            if (it > 0) {
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const uint64_t x = mul_f32x2(((uint64_t)r[2 * e + 1] << 32) | r[2 * e], e2);
                    r[2 * e] = (uint32_t)x;
                    r[2 * e + 1] = (uint32_t)(x >> 32);
                }
                tmem_st32(tmem + lrow + kColDS + p * 32, r);
            }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const uint32_t *x = r + jj * 8;
                *reinterpret_cast<uint4 *>(smem + off_ds + ds_off(i, p * 32 + jj * 8)) =
                    make_uint4(pack_bf16(__uint_as_float(x[0]), __uint_as_float(x[1])),
                               pack_bf16(__uint_as_float(x[2]), __uint_as_float(x[3])),
                               pack_bf16(__uint_as_float(x[4]), __uint_as_float(x[5])),
                               pack_bf16(__uint_as_float(x[6]), __uint_as_float(x[7])));
            }
        }
        if (it > 0) tmem_wait_st();
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(b.dst_full);
            if (it > 0) mbar_arrive(&b.empty[(it - 1) % kStages]);  // its e^{b_C} is used
        }
        // (2) masked M and A tiles of this chunk (M=64 layout: lanes 0-15 hold row 16 warp + lane)
        if (!mbar_wait(b.mm_full, it & 1, abort)) break;
        tc_fence_after();
        uint8_t *mt = smem + off_ma + (it & 1) * 2 * kMaskBytes;
#pragma unroll
        for (int t = 0; t < 4; ++t) {  // M half 0, M half 1, A half 0, A half 1
            tmem_ld32(tmem + lrow + (t < 2 ? kColM : kColA) + (t & 1) * 32, r);
            tmem_wait_ld();
            if (t == 3) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(b.mm_free);
            }
            masked_tile(mt + (t >> 1) * kMaskBytes, r, warp, t & 1, lane);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(b.p_full);
    }
}

// Warps 4-7: thread x = 32 (warp - 4) + lane owns key dim x of dk / dlog_g and value dim x of
// dv for all 64 tokens of the chunk.
__device__ void out_role(uint8_t *smem, const Bars &b, volatile int *abort, const BwdArgs &a,
                         uint32_t tmem, int bh, int j, long long row0, int nchunks,
                         const CUtensorMap *tdk, const CUtensorMap *tdv, const CUtensorMap *tdg) {
    const int quarter = (threadIdx.x >> 5) & 3, lane = threadIdx.x & 31;
    const int x = quarter * 32 + lane;
    const uint32_t lrow = (uint32_t)(quarter * 32) << 16;
    const bool storer = threadIdx.x == 32 * kStateWarps;
    const long long sidx = ((long long)bh * a.NP + j) * D * D;
    // carry: rowsum(S_end . dX), the gradient reaching this part from its end state
    float carry = 0.f;
    {
        const float *Se = nullptr;
        if (j < a.NP - 1) {
            if (a.S_end_next) Se = a.S_end_next + sidx + (long long)D * D;
        } else if (a.S_fin) {
            Se = a.S_fin + (long long)bh * D * D;
        }
        if (Se) {
            const float4 *x4 = reinterpret_cast<const float4 *>(a.dX + sidx + (long long)x * D);
            const float4 *s4 = reinterpret_cast<const float4 *>(Se + (long long)x * D);
#pragma unroll 8
            for (int e4 = 0; e4 < D / 4; ++e4) {
                const float4 v = x4[e4], u = s4[e4];
                carry += u.x * v.x + u.y * v.y + u.z * v.z + u.w * v.w;
            }
        }
    }
    uint32_t r[16];
    float qv[16], qn[16];
    for (int it = 0; it < nchunks; ++it) {
        const int s = it % kStages, bb = it & 1;
        const int c = nchunks - 1 - it;
        uint8_t *st = smem + s * kStageBytes;
        const float *qdq = a.dq_ws + (row0 + (long long)c * CH) * D + x;
        // q . dq of the chunk's last 16 tokens (L2-prefetched with the chunk's tiles), in flight
        // while this thread waits for dk; each later group is loaded one group ahead
#pragma unroll
        for (int t = 0; t < 16; ++t) qn[t] = qdq[(48 + t) * D];
        if (it > 0 && storer) {  // the previous chunk's output tiles are read out: release its stage
            bulk_wait_read();
            mbar_arrive(&b.empty[(it - 1) % kStages]);
        }
        // (1) dk and the dlog_g suffix sums: tokens last to first, 16 at a time.  dk_full also
        // means the dS update is done, so the v and q tiles are free for dk and dlog_g.
        if (!mbar_wait(&b.dk_full[bb], (it >> 1) & 1, abort)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(st);
        uint32_t fk[16];  // next group's factors and Ktil, bf16 pairs (f low, Ktil high)
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            const uint32_t off = tile_off(48 + t, x);
            fk[t] = lds_u16(sa + off_g + off) | (lds_u16(sa + off_k + off) << 16);
        }
#pragma unroll
        for (int g = 3; g >= 0; --g) {
            tmem_ld16(tmem + lrow + kColDK + bb * 64 + g * 16, r);
#pragma unroll
            for (int t = 0; t < 16; ++t) qv[t] = qn[t];
            if (g > 0) {
#pragma unroll
                for (int t = 0; t < 16; ++t) qn[t] = qdq[((g - 1) * 16 + t) * D];
            }
            // dk = e^{b_C - b_s} acc and the contribution q . dq - k . dk (k . dk = Ktil . acc,
            // Ktil = k e^{b_C - b_s} the MMA operand); then the suffix sums
            float f[16], c[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                f[t] = __uint_as_float(fk[t] << 16);
                c[t] = __uint_as_float(fk[t] & 0xFFFF0000u);
            }
            if (g > 0) {  // the next group's loads go out before this group's stores
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const uint32_t off = tile_off((g - 1) * 16 + t, x);
                    fk[t] = lds_u16(sa + off_g + off) | (lds_u16(sa + off_k + off) << 16);
                }
            }
            tmem_wait_ld();
            if (g == 0) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&b.dk_free[bb]);
            }
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                const float acc = __uint_as_float(r[t]);
                f[t] *= acc;                  // dk
                c[t] = qv[t] - c[t] * acc;    // contribution
            }
#pragma unroll
            for (int t = 15; t >= 0; --t) {
                carry += c[t];
                c[t] = carry;                 // dlog_g
            }
#pragma unroll
            for (int t = 0; t < 16; t += 2) {
                store_pair(sa + off_v, g * 16 + t, x, f[t], f[t + 1]);
                store_pair(sa + off_q, g * 16 + t, x, c[t], c[t + 1]);
            }
        }
        // (2) dv into the dO tile (its last readers, the dv MMAs, are done)
        if (!mbar_wait(&b.dv_full[bb], (it >> 1) & 1, abort)) break;
        tc_fence_after();
#pragma unroll 1
        for (int g = 0; g < 4; ++g) {
            tmem_ld16(tmem + lrow + kColDV + bb * 64 + g * 16, r);
            tmem_wait_ld();
            if (g == 3) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&b.dv_free[bb]);
            }
#pragma unroll
            for (int t = 0; t < 16; t += 2)
                store_pair(sa + off_do, g * 16 + t, x, __uint_as_float(r[t]), __uint_as_float(r[t + 1]));
        }
        // (3) once all four warps' values are in the tiles, one thread stores them
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(b.osync);
        if (!mbar_wait(b.osync, it & 1, abort)) break;
        if (storer) {
            const int y = (int)(row0 + (long long)c * CH);
            tma_store_2d(tdk, 0, y, st + off_v);
            tma_store_2d(tdk, 64, y, st + off_v + kHalfBytes);
            tma_store_2d(tdg, 0, y, st + off_q);
            tma_store_2d(tdg, 64, y, st + off_q + kHalfBytes);
            tma_store_2d(tdv, 0, y, st + off_do);
            tma_store_2d(tdv, 64, y, st + off_do + kHalfBytes);
            bulk_commit();
        }
    }
    if (storer) bulk_wait_all();
}

__global__ void __launch_bounds__(kThreads, 1)
tc_dkv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_dk,
              const __grid_constant__ CUtensorMap tm_dv, const __grid_constant__ CUtensorMap tm_dg,
              const BwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + off_bar);
    Bars b;
    b.full = bar;
    b.gated = bar + kStages;
    b.empty = bar + 2 * kStages;
    uint64_t *x = bar + 3 * kStages;
    b.mm_full = x + 0; b.mm_free = x + 1; b.p_full = x + 2; b.dst_full = x + 3; b.dk_full = x + 4;
    b.dk_free = x + 6; b.dv_full = x + 8; b.dv_free = x + 10; b.dsn_full = x + 12; b.osync = x + 13;
    b.fin = x + 14;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + off_misc);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + off_misc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x / a.NP, j = blockIdx.x % a.NP;
    const long long row0 = (long long)bh * a.L + (long long)j * a.T;
    const int nchunks = (int)(a.T / CH);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&b.full[s], 1);
            mbar_init(&b.gated[s], kGateWarps);
            mbar_init(&b.empty[s], 1 + kStateWarps + 1);  // MMA, dS warps, output storer
        }
        uint64_t *one[] = {b.mm_full, b.dk_full, b.dk_full + 1, b.dv_full, b.dv_full + 1,
                           b.dsn_full, b.fin};
        uint64_t *st4[] = {b.mm_free, b.p_full, b.dst_full};
        uint64_t *out4[] = {b.dk_free, b.dk_free + 1, b.dv_free, b.dv_free + 1, b.osync};
        for (uint64_t *p : one) mbar_init(p, 1);
        for (uint64_t *p : st4) mbar_init(p, kStateWarps);
        for (uint64_t *p : out4) mbar_init(p, kOutWarps);
        *abort = 0;
        mbar_fence_init();
    }
    if (warp == kTmaWarp && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_do);
        prefetch_tmap(&tm_g);
        prefetch_tmap(&tm_dk);
        prefetch_tmap(&tm_dv);
        prefetch_tmap(&tm_dg);
    }
    if (warp == kMmaWarp) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (warp == kTmaWarp) {
        if (lane == 0)
            producer(smem, b, abort, &tm_q, &tm_k, &tm_v, &tm_do, &tm_g, a.dq_ws, row0, nchunks);
    } else if (warp == kMmaWarp) {
        mma_issuer(smem, b, abort, tmem, nchunks);
    } else if (warp >= kEpiWarps) {
        gate_role(smem, b, abort, a, nchunks);
    } else if (warp < kStateWarps) {
        state_role(smem, b, abort, a, tmem, bh, j, nchunks);
    } else {
        out_role(smem, b, abort, a, tmem, bh, j, row0, nchunks, &tm_dk, &tm_dv, &tm_dg);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (threadIdx.x == 0 && *abort && a.status) atomicOr(a.status, kStatusTimeout);
}

}  // namespace dkv

}  // namespace

bool tc_bwd_supported(const BwdArgs &a) {
    return a.dt == LA_BF16 && a.dk == D && a.dv == D && a.chunk == CH && a.T % CH == 0 &&
           (long long)a.BH * a.L <= 0x7FFFFFFFLL;
}

cudaError_t launch_tc_dq(const BwdArgs &a, cudaStream_t st) {
    const long long rows = (long long)a.BH * a.L;
    CUtensorMap mk, mv, mdo, mg, mq;
    cudaError_t e;
    if ((e = make_map(&mk, a.k, rows)) != cudaSuccess) return e;
    if ((e = make_map(&mv, a.v, rows)) != cudaSuccess) return e;
    if ((e = make_map(&mdo, a.dO, rows)) != cudaSuccess) return e;
    if ((e = make_map(&mg, a.g, rows)) != cudaSuccess) return e;
    if ((e = make_map(&mq, a.q, rows)) != cudaSuccess) return e;
    e = cudaFuncSetAttribute(dqs::tc_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             dqs::kSmemBytes);
    if (e != cudaSuccess) return e;
    const long long nblk = (long long)a.BH * a.NP;
    if (nblk == 0) return cudaSuccess;
    dqs::tc_dq_kernel<<<(unsigned)nblk, kThreads, dqs::kSmemBytes, st>>>(mk, mv, mdo, mg, mq, a);
    return cudaGetLastError();
}

cudaError_t launch_tc_dkv(const BwdArgs &a, cudaStream_t st) {
    const long long rows = (long long)a.BH * a.L;
    CUtensorMap mq, mk, mv, mdo, mg, mdk, mdv, mdg;
    cudaError_t e;
    if ((e = make_map(&mq, a.q, rows)) != cudaSuccess) return e;
    if ((e = make_map(&mk, a.k, rows)) != cudaSuccess) return e;
    if ((e = make_map(&mv, a.v, rows)) != cudaSuccess) return e;
    if ((e = make_map(&mdo, a.dO, rows)) != cudaSuccess) return e;
    if ((e = make_map(&mg, a.g, rows)) != cudaSuccess) return e;
    if ((e = make_map(&mdk, a.dk_out, rows)) != cudaSuccess) return e;
    if ((e = make_map(&mdv, a.dv_out, rows)) != cudaSuccess) return e;
    if ((e = make_map(&mdg, a.dg_out, rows)) != cudaSuccess) return e;
    e = cudaFuncSetAttribute(dkv::tc_dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             dkv::kSmemBytes);
    if (e != cudaSuccess) return e;
    const long long nblk = (long long)a.BH * a.NP;
    if (nblk == 0) return cudaSuccess;
    dkv::tc_dkv_kernel<<<(unsigned)nblk, kThreads, dkv::kSmemBytes, st>>>(mq, mk, mv, mdo, mg, mdk,
                                                                          mdv, mdg, a);
    return cudaGetLastError();
}

}  // namespace la
