// tc_dq.cu -- the backward's dq sweep on the tensor cores (bf16, d_k = d_v = 128, chunk 64):
// forward over the chunks of each (b, h, segment), from the state the segment received.
//
// Per chunk, with b_t the inclusive in-chunk cumsum of log_g, b_C its total, the state S
// entering the chunk (rows i = key dims on the TMEM lanes, fp32, resident in tensor memory for
// the whole segment), S' = diag(e^{b_C}) S and Ktil_s = k_s e^{b_C - b_s}:
//
//   M    = dO V^T                    M=64  (t) N=64  (s) K=128 (j)  -> masked s <= t, bf16 tile
//   S   <- S' + Ktil^T V             M=128 (i) N=128 (j) K=64  (s)  accumulated onto S' in TMEM
//   dq^T = S' dO^T + Ktil^T M^T      M=128 (i) N=64  (t) K=128 (j) / 64 (s), A = S' from TMEM
//   dq[t,i] = e^{b_t,i - b_C,i} dq^T[i,t];   q . dq (fp32) for the reverse sweep's dlog_g,
//   formed as bf16(q F) dq^T with F = bf16(e^{b_t - b_C}) (see the read-out)
//
// (the gradient of o_t = q_t S_t with respect to q_t, in the chunk factorisation of the
// forward).  The sweep also records the state entering each of the segment's `fine` equal
// parts, and -- when asked -- forms each fine part's gradient state
// R = sum_t diag(e^{B_t}) q_t^T dO_t (B_t: inclusive log-decay from the part's start), as
// R^T += dO^T Qhat with Qhat = q e^{B + b_t} = q e^{B + b_C} e^{b_t - b_C} written by the gates,
// and the part's log-decay sum.
//
// Warp roles (576 threads): 0-3 state (one TMEM row i per thread: decay, bf16 copy as the A
// operand of S' dO^T, fine-part records), 4-7 output (M -> masked P tile, dq and q . dq
// read-out), 8-15 gates, 16 TMA producer, 17 MMA issuer / TMEM owner.  Every wait is bounded
// (about a second of clock), after which the CTA stops, drains what it issued, frees its TMEM
// and reports kStatusTimeout.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tc_common.cuh"

namespace la {
namespace {

using namespace sm100;
using namespace tc;

constexpr int kStateWarps = 4, kOutWarps = 4, kEpiWarps = kStateWarps + kOutWarps, kGateWarps = 8;
constexpr int kTmaWarp = kEpiWarps + kGateWarps, kMmaWarp = kTmaWarp + 1;
constexpr int kThreads = 32 * (kMmaWarp + 1);

// Tensor-memory columns: the fp32 state, dq^T, the bf16 S' copy, the chunk's (F, q) pairs for
// the output warps, M (M=64 layout), R^T.
constexpr uint32_t kColS = 0, kColDQ = 128, kColSA = 192, kColFQ = 256, kColM = 320, kColR = 384;

constexpr int kStages = 2;
constexpr int off_k = 0, off_v = kTileBytes, off_do = 2 * kTileBytes, off_g = 3 * kTileBytes,
              off_q = 4 * kTileBytes,   // read by the output warps (q . dq) and the gates (Qhat)
              off_qh = 5 * kTileBytes;  // Qhat, written by the gates
constexpr int kStageBytes = 6 * kTileBytes;
constexpr int off_p = kStages * kStageBytes;  // two masked M tiles
constexpr int off_ec = off_p + 2 * CH * CH * 2;
constexpr int off_bar = off_ec + kStages * D * 4;
constexpr int off_misc = off_bar + 24 * 8;  // room for kNumBars
constexpr int kSmemBytes = off_misc + 16 + 1024;  // + slack to align the base to 1 KB
static_assert(kSmemBytes <= 232448, "shared memory budget");

// Barriers by index from one base pointer (addresses are recomputed where used rather than
// held in registers): ring barriers per stage, then the single and paired ones.
enum : int {
    kFull = 0, kGated = kFull + kStages, kEmpty = kGated + kStages, kMFull = kEmpty + kStages,
    kMFree, kPFull, kDsFull = kPFull + 2, kSaFull, kSaFree, kDqFull = kSaFree + 2, kDqFree,
    kRFull, kRFree, kFin, kFullB, kEcFull = kFullB + kStages, kNumBars = kEcFull + kStages
};
static_assert(kNumBars <= 24, "barrier area");
struct Bars {
    uint64_t *base;
    __device__ __forceinline__ uint64_t *operator[](int k) const { return base + k; }
};

struct Sweep {           // per-CTA constants shared by the roles
    int bh, j, nchunks;  // (b, h), segment, chunks in the segment
    int cpf;             // chunks per fine part
    bool dstate;         // also the fine parts' gradient states
    long long row0;      // first token row of the segment
};

// ------------------------------------------------------------------ TMA producer (1 thread)
__device__ void producer(uint8_t *smem, const Bars &b, volatile int *abort, const CUtensorMap *tk,
                         const CUtensorMap *tv, const CUtensorMap *tdo, const CUtensorMap *tg,
                         const CUtensorMap *tq, const Sweep &w) {
    int issued = 0;
    for (int c = 0; c < w.nchunks; ++c) {
        const int s = c % kStages;
        if (c >= kStages && !mbar_wait(b[kEmpty + s], ((c / kStages) - 1) & 1, abort)) break;
        uint8_t *st = smem + s * kStageBytes;
        const int y = (int)(w.row0 + (long long)c * CH);
        // the gates' tiles first, on their own barrier (the gates start as soon as they land);
        // dO and v, read only by the tensor cores, behind them
        const CUtensorMap *maps[5] = {tg, tk, tq, tdo, tv};
        const int offs[5] = {off_g, off_k, off_q, off_do, off_v};
        mbar_arrive_expect_tx(b[kFull + s], 3 * kTileBytes);
        mbar_arrive_expect_tx(b[kFullB + s], 2 * kTileBytes);
#pragma unroll
        for (int m = 0; m < 5; ++m) {
            uint64_t *bar = b[(m < 3 ? kFull : kFullB) + s];
            tma_load_2d(st + offs[m], maps[m], 0, y, bar);
            tma_load_2d(st + offs[m] + kHalfBytes, maps[m], 64, y, bar);
        }
        issued = c + 1;
    }
    if (*abort)  // let every copy this CTA started land before it exits
        for (int c = issued > kStages ? issued - kStages : 0; c < issued; ++c) {
            wait_drain(b[kFull + c % kStages], (c / kStages) & 1);
            wait_drain(b[kFullB + c % kStages], (c / kStages) & 1);
        }
}

// ------------------------------------------------------------------ MMA issuer (1 warp)
// The whole warp walks the loop and waits; one elected lane issues.  Per chunk: M as soon as
// the tiles land (it reads untouched tiles, so it overlaps the gates), R^T once Qhat is written,
// the state increment onto S' once the state warps have scaled S, then dq^T.
__device__ void mma_issuer(uint8_t *smem, const Bars &b, volatile int *abort, uint32_t tmem,
                           const Sweep &w) {
    constexpr uint32_t i_m = idesc_bf16_f32(64, 64, 0, 0);     // dO V^T
    constexpr uint32_t i_ss = idesc_bf16_f32(128, 128, 1, 1);  // Ktil^T V, dO^T Qhat
    constexpr uint32_t i_qa = idesc_bf16_f32(128, 64, 0, 0);   // S' dO^T (A from TMEM)
    constexpr uint32_t i_qb = idesc_bf16_f32(128, 64, 1, 0);   // Ktil^T M^T
    const uint32_t base = smem_u32(smem);
    bool ok = true;
    for (int c = 0; ok && c < w.nchunks; ++c) {
        const int s = c % kStages, pb = c & 1;
        const uint32_t st = base + (uint32_t)(s * kStageBytes);
        const uint32_t ka = st + off_k, va = st + off_v, da = st + off_do;
        if (!(ok = warp_wait(b[kFullB + s], (c / kStages) & 1, abort))) break;  // dO, v
        if (c > 0 && !(ok = warp_wait(b[kMFree], (c - 1) & 1, abort))) break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // M = dO V^T
                mma_ss(tmem + kColM, desc_kmajor(da, kk), desc_kmajor(va, kk), i_m, kk > 0);
            mma_commit(b[kMFull]);
        }
        __syncwarp();
        if (!(ok = warp_wait(b[kGated + s], (c / kStages) & 1, abort))) break;
        tc_fence_after();
        if (w.dstate) {  // R^T += dO^T Qhat over the fine part
            const int part = c / w.cpf;
            const bool first = c % w.cpf == 0;
            if (first && part > 0 && !(ok = warp_wait(b[kRFree], (part - 1) & 1, abort))) break;
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ss(tmem + kColR, desc_mnmajor(da, kk), desc_mnmajor(st + off_qh, kk), i_ss,
                           (!first || kk > 0) ? 1u : 0u);
                if (c % w.cpf == w.cpf - 1) mma_commit(b[kRFull]);
            }
            __syncwarp();
        }
        if (!(ok = warp_wait(b[kSaFull], c & 1, abort))) break;  // S' and its bf16 copy in place
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // S = S' + Ktil^T V
                mma_ss(tmem + kColS, desc_mnmajor(ka, kk), desc_mnmajor(va, kk), i_ss, 1u);
            mma_commit(b[kDsFull]);
        }
        __syncwarp();
        if (c > 0 && !(ok = warp_wait(b[kDqFree], (c - 1) & 1, abort))) break;
        if (!(ok = warp_wait(b[kPFull + pb], (c >> 1) & 1, abort))) break;
        tc_fence_after();
        if (elect_one()) {
            const uint32_t pa = base + off_p + pb * (CH * CH * 2);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // dq^T = S' dO^T
                mma_ts(tmem + kColDQ, tmem + kColSA + kk * 8, desc_kmajor(da, kk), i_qa, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // dq^T += Ktil^T M^T   (B: masked M tile, K-major)
                mma_ss(tmem + kColDQ, desc_mnmajor(ka, kk), smem_desc_sw128(pa + kk * 32, 16, 1024),
                       i_qb, 1u);
            mma_commit(b[kDqFull]);
            mma_commit(b[kSaFree]);
            mma_commit(b[kEmpty + s]);
        }
        __syncwarp();
    }
    if (elect_one()) mma_commit(b[kFin]);  // nothing of this CTA may still run at dealloc
    __syncwarp();
    wait_drain(b[kFin], 0);
}

// ------------------------------------------------------------------ gate warps (256 threads)
// Warp gw owns key dims 16gw .. 16gw+15; lane = 2 tg + ig owns rows 4tg .. 4tg+3 and the 16-byte
// key chunk ig, visiting its rows in the order 4tg + (k ^ sw), sw = tg & 2, which keeps every
// warp-wide 16-byte shared access at the minimum wavefront count.  Per chunk: the in-chunk
// cumsum (row-pair sums + a 4-step shuffle scan over the 16 token groups), then in place
// Ktil = k e^{b_C - b_t} over k and F = e^{b_t - b_C} over log_g (the output warps' dq factor),
// e^{b_C} per key dim for the state warps, and with the gradient-state sum Qhat = q F e^{B + b_C}.
// (Kept out of line: inlined beside the other roles it pushes the kernel over its register
// budget of 96 per thread.)
__device__ __noinline__ void gate_role(uint8_t *smem, const Bars &b, volatile int *abort,
                                       const BwdArgs &a, const Sweep &w) {
    const int gw = (threadIdx.x >> 5) - kEpiWarps;
    const int lane = threadIdx.x & 31;
    const int tg = lane >> 1, ig = lane & 1;
    const int i0 = gw * 16 + ig * 8;  // first key dim of this thread's chunk
    const int sw = tg & 2;            // step k visits row 4tg + (k ^ sw)
    float *ec = reinterpret_cast<float *>(smem + off_ec);
    float logB[8];  // log-decay from the fine part's start through the current chunk
#pragma unroll
    for (int e = 0; e < 8; ++e) logB[e] = 0.f;
    bool range_bad = false;
    uint32_t posm = 0x80008000u;  // running int16 max of the log_g bits: > 0 means a positive gate exponent
    for (int c = 0; c < w.nchunks; ++c) {
        const int s = c % kStages;
        if (!mbar_wait(b[kFull + s], (c / kStages) & 1, abort)) break;
        uint8_t *st = smem + s * kStageBytes;
        // bk[k]: inclusive cumsum, from the group's first row, of the row visited at step k
        float bk[4][8], tot[8];
        {
            uint4 graw[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                graw[k] = *reinterpret_cast<const uint4 *>(st + off_g + tile_off(tg * 4 + (k ^ sw), i0));
#pragma unroll
            for (int k = 0; k < 4; ++k) posm = pos_bf16_max(posm, graw[k]);
            float f[4][8];
#pragma unroll
            for (int k = 0; k < 4; ++k) unpack8(graw[k], f[k]);
#pragma unroll
            for (int e = 0; e < 8; e += 2) {  // two key dims per f32x2 instruction
                // steps (0,1) and (2,3) each visit one row pair in order; the pair of rows
                // 4tg, 4tg+1 is at steps 0,1 when sw == 0, at steps 2,3 otherwise
                float p01[2], p23[2];
                add_x2(p01[0], p01[1], f[0][e], f[0][e + 1], f[1][e], f[1][e + 1]);
                add_x2(p23[0], p23[1], f[2][e], f[2][e + 1], f[3][e], f[3][e + 1]);
                const float o01a = sw ? p23[0] : 0.f, o01b = sw ? p23[1] : 0.f;
                const float o23a = sw ? 0.f : p01[0], o23b = sw ? 0.f : p01[1];
                add_x2(bk[0][e], bk[0][e + 1], f[0][e], f[0][e + 1], o01a, o01b);
                add_x2(bk[1][e], bk[1][e + 1], p01[0], p01[1], o01a, o01b);
                add_x2(bk[2][e], bk[2][e + 1], f[2][e], f[2][e + 1], o23a, o23b);
                add_x2(bk[3][e], bk[3][e + 1], p23[0], p23[1], o23a, o23b);
                add_x2(tot[e], tot[e + 1], p01[0], p01[1], p23[0], p23[1]);
            }
        }
        float incl[8];  // inclusive scan of the group totals across tg (lanes ig, ig+2, ...)
#pragma unroll
        for (int e = 0; e < 8; ++e) incl[e] = tot[e];
#pragma unroll
        for (int d = 1; d < 16; d <<= 1) {
            float up[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) up[e] = __shfl_up_sync(0xFFFFFFFFu, incl[e], 2 * d);
            if (tg >= d) {
#pragma unroll
                for (int e = 0; e < 8; e += 2)
                    add_x2(incl[e], incl[e + 1], incl[e], incl[e + 1], up[e], up[e + 1]);
            }
        }
        float nbCl[8], eB[8];
        const bool part_start = c % w.cpf == 0;
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            const float bC0 = __shfl_sync(0xFFFFFFFFu, incl[e], 30 + ig);
            const float bC1 = __shfl_sync(0xFFFFFFFFu, incl[e + 1], 30 + ig);
            float off[2];  // exclusive prefix of this token group
            sub_x2(off[0], off[1], incl[e], incl[e + 1], tot[e], tot[e + 1]);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                add_x2(bk[k][e], bk[k][e + 1], bk[k][e], bk[k][e + 1], off[0], off[1]);
            mul_x2(nbCl[e], nbCl[e + 1], -bC0, -bC1, kLog2e, kLog2e);
            range_bad |= !(fabsf(bC0) <= kGateRangeLimit) || !(fabsf(bC1) <= kGateRangeLimit);
            logB[e] = (part_start ? 0.f : logB[e]) + bC0;
            logB[e + 1] = (part_start ? 0.f : logB[e + 1]) + bC1;
            eB[e] = w.dstate ? ex2_approx(logB[e] * kLog2e) : 0.f;
            eB[e + 1] = w.dstate ? ex2_approx(logB[e + 1] * kLog2e) : 0.f;
        }
        if (tg == 0) {
            float4 *e4 = reinterpret_cast<float4 *>(ec + s * D + i0);
            e4[0] = make_float4(ex2_approx(-nbCl[0]), ex2_approx(-nbCl[1]), ex2_approx(-nbCl[2]),
                                ex2_approx(-nbCl[3]));
            e4[1] = make_float4(ex2_approx(-nbCl[4]), ex2_approx(-nbCl[5]), ex2_approx(-nbCl[6]),
                                ex2_approx(-nbCl[7]));
            if (w.dstate && c % w.cpf == w.cpf - 1) {  // the fine part's log-decay sum
                const long long jf = (long long)w.j * a.fine + c / w.cpf;
                float4 *lg = reinterpret_cast<float4 *>(a.logG + ((long long)w.bh * a.NP * a.fine + jf) * D + i0);
                lg[0] = make_float4(logB[0], logB[1], logB[2], logB[3]);
                lg[1] = make_float4(logB[4], logB[5], logB[6], logB[7]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(b[kEcFull + s]);  // e^{b_C}: the state warps' decay can start
#pragma unroll
        for (int k = 0; k < 4; ++k) {  // one row at a time, dims in pairs (register budget)
            const uint32_t off = tile_off(tg * 4 + (k ^ sw), i0);
            const uint4 kr = *reinterpret_cast<const uint4 *>(st + off_k + off);
            const uint4 qr = w.dstate ? *reinterpret_cast<const uint4 *>(st + off_q + off) : kr;
            const uint32_t kw[4] = {kr.x, kr.y, kr.z, kr.w}, qw[4] = {qr.x, qr.y, qr.z, qr.w};
            uint32_t wk[4], wf[4], wq[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float x0, x1, k0, k1;
                fma_x2(x0, x1, bk[k][2 * e], bk[k][2 * e + 1], kLog2e, kLog2e, nbCl[2 * e],
                       nbCl[2 * e + 1]);
                const float u0 = ex2_approx(x0), u1 = ex2_approx(x1);
                mul_x2(k0, k1, __uint_as_float(kw[e] << 16), __uint_as_float(kw[e] & 0xFFFF0000u),
                       ex2_approx(-x0), ex2_approx(-x1));
                wk[e] = pack_bf16(k0, k1);
                wf[e] = pack_bf16(u0, u1);
                float h0, h1;  // Qhat = (q u) e^B
                mul_x2(h0, h1, __uint_as_float(qw[e] << 16), __uint_as_float(qw[e] & 0xFFFF0000u), u0, u1);
                mul_x2(h0, h1, h0, h1, eB[2 * e], eB[2 * e + 1]);
                wq[e] = pack_bf16(h0, h1);
            }
            *reinterpret_cast<uint4 *>(st + off_k + off) = make_uint4(wk[0], wk[1], wk[2], wk[3]);
            *reinterpret_cast<uint4 *>(st + off_g + off) = make_uint4(wf[0], wf[1], wf[2], wf[3]);
            if (w.dstate)
                *reinterpret_cast<uint4 *>(st + off_qh + off) = make_uint4(wq[0], wq[1], wq[2], wq[3]);
        }
        fence_proxy_async_smem();  // the tensor cores read these tiles through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(b[kGated + s]);
    }
    if (range_bad || any_pos_bf16(posm))  // every fine part of the segment: the state runs through them
        flag_range(a.flags, ((long long)w.bh * a.NP + w.j) * a.fine, a.fine, a.status);
}

// ------------------------------------------------------------------ state warps (0-3)
// Thread i (= TMEM lane) owns row i of the fp32 state.  Per chunk c it records the row when c
// starts a fine part, scales it by the chunk's decay e^{b_C,i} (S' = diag(e^{b_C}) S), stores
// S' back for the MMA to accumulate Ktil^T V onto, and stores the bf16 copy into S' buffer
// c % 2, the A operand of S' dO^T.  At a fine part's end it reads the part's R^T out.
__device__ void state_role(uint8_t *smem, const Bars &b, volatile int *abort, const BwdArgs &a,
                           uint32_t tmem, const Sweep &w) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = warp * 32 + lane;
    const uint32_t lrow = (uint32_t)(warp * 32) << 16;
    const float *ec = reinterpret_cast<const float *>(smem + off_ec);
    uint32_t r[32];
    {  // the state the segment receives (or zero)
        const float *Si = a.S_recv ? a.S_recv + (((long long)w.bh * a.NP + w.j) * D + i) * D : nullptr;
#pragma unroll 1
        for (int p = 0; p < 4; ++p) {
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) {
                const float4 v = Si ? reinterpret_cast<const float4 *>(Si)[p * 8 + e4]
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                r[4 * e4] = __float_as_uint(v.x); r[4 * e4 + 1] = __float_as_uint(v.y);
                r[4 * e4 + 2] = __float_as_uint(v.z); r[4 * e4 + 3] = __float_as_uint(v.w);
            }
            tmem_st32(tmem + lrow + kColS + p * 32, r);
        }
        tmem_wait_st();
        tc_fence_before();
    }
    for (int c = 0; c < w.nchunks; ++c) {
        const int s = c % kStages;
        // the decay needs only e^{b_C}, published by the gates before they rescale the tiles
        if (!mbar_wait(b[kEcFull + s], (c / kStages) & 1, abort)) break;
        if (c > 0 && !mbar_wait(b[kDsFull], (c - 1) & 1, abort)) break;
        if (c >= 1 && !mbar_wait(b[kSaFree], (c - 1) & 1, abort)) break;
        tc_fence_after();
        const uint64_t e2 = (uint64_t)__float_as_uint(ec[s * D + i]) * 0x100000001ull;
        if (a.S_fine && c % w.cpf == 0) {  // the state entering a fine part, to HBM
            // read through the 16x256b shape, so that one warp-wide store covers whole 32-byte
            // sectors of 8 rows (thread l: rows r and r + 8, two adjacent columns per 8), where
            // a thread writing its own row spread every store over 32 rows
            float *rec = a.S_fine + (((long long)w.bh * a.NP + w.j) * a.fine + c / w.cpf) * D * D;
            const int c2 = 2 * (lane & 3);
#pragma unroll 1
            for (int hq = 0; hq < 2; ++hq) {
                const int ra = warp * 32 + 16 * hq + (lane >> 2);
#pragma unroll 1
                for (int p = 0; p < 4; ++p) {
                    uint32_t q16[16];
                    tmem_ld_16x256b_x4(tmem + ((uint32_t)(warp * 32 + 16 * hq) << 16) + kColS + p * 32,
                                       q16);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int col = p * 32 + 8 * k + c2;
                        *reinterpret_cast<float2 *>(rec + (long long)ra * D + col) =
                            make_float2(__uint_as_float(q16[4 * k]), __uint_as_float(q16[4 * k + 1]));
                        *reinterpret_cast<float2 *>(rec + (long long)(ra + 8) * D + col) =
                            make_float2(__uint_as_float(q16[4 * k + 2]), __uint_as_float(q16[4 * k + 3]));
                    }
                }
            }
        }
        const uint32_t sa = tmem + lrow + kColSA;
#pragma unroll 1
        for (int p = 0; p < 4; ++p) {  // value dims 32p .. 32p+31
            tmem_ld32(tmem + lrow + kColS + p * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const uint64_t x = mul_f32x2(((uint64_t)r[2 * e + 1] << 32) | r[2 * e], e2);
                r[2 * e] = (uint32_t)x;
                r[2 * e + 1] = (uint32_t)(x >> 32);
            }
            tmem_st32(tmem + lrow + kColS + p * 32, r);
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = pack_bf16(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
            tmem_st16(sa + p * 16, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(b[kSaFull]);
            mbar_arrive(b[kEmpty + s]);  // this chunk's e^{b_C} is used
        }
        if (w.dstate && c % w.cpf == w.cpf - 1) {  // R[i'][j] = R^T[j][i'] of the fine part
            if (!mbar_wait(b[kRFull], (c / w.cpf) & 1, abort)) break;
            tc_fence_after();
            const long long jf = (long long)w.j * a.fine + c / w.cpf;
            float *Ro = a.dSloc + ((long long)w.bh * a.NP * a.fine + jf) * D * D + i;  // + i' D
#pragma unroll 1
            for (int p = 0; p < 4; ++p, Ro += 32 * D) {
                tmem_ld32(tmem + lrow + kColR + p * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) Ro[e * D] = __uint_as_float(r[e]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(b[kRFree]);
        }
    }
}

// ------------------------------------------------------------------ output warps (4-7)
// (a) M -> causal mask -> bf16 P tile (buffer c % 2); (b) the chunk's (F, q) pairs copied from
// the stage into TMEM, which releases the stage; (d) dq^T read-out: thread i owns key dim i;
// dq = F . dq^T with F = e^{b_t - b_C} from the gates, q . dq in fp32 -- stored straight from
// registers (q . dq as one 128-byte line per warp and token, dq as 2-byte stores per token).
// Chunk c's copy and read-out come before M of chunk c+1 is masked, since M(c+1) can only be
// formed once chunk c+1 has landed.
__device__ void out_role(uint8_t *smem, const Bars &b, volatile int *abort, const BwdArgs &a,
                         uint32_t tmem, const Sweep &w) {
    const int quarter = (threadIdx.x >> 5) & 3, lane = threadIdx.x & 31;
    const int i = quarter * 32 + lane;
    const uint32_t lrow = (uint32_t)(quarter * 32) << 16;
    __nv_bfloat16 *dq = static_cast<__nv_bfloat16 *>(a.dq_out);
    auto make_p = [&](int c) -> bool {  // M=64 accumulator: lanes 0-15 hold rows 16 quarter + lane
        if (!mbar_wait(b[kMFull], c & 1, abort)) return false;
        tc_fence_after();
        const int t = quarter * 16 + lane, pb = c & 1;
        uint8_t *prow = smem + off_p + pb * (CH * CH * 2) + t * 128;
        uint32_t r[32];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            tmem_ld32(tmem + lrow + kColM + h * 32, r);
            tmem_wait_ld();
            if (h == 1) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(b[kMFree]);
            }
            if (lane < 16) {
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    uint32_t w4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int sl = jj * 8 + 2 * e, s0 = h * 32 + sl;
                        w4[e] = pack_bf16(s0 <= t ? __uint_as_float(r[sl]) : 0.f,
                                          s0 + 1 <= t ? __uint_as_float(r[sl + 1]) : 0.f);
                    }
                    *reinterpret_cast<uint4 *>(prow + (((h * 4 + jj) ^ (t & 7)) << 4)) =
                        make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(b[kPFull + pb]);
        return true;
    };
    if (w.nchunks > 0 && !make_p(0)) return;
    for (int c = 0; c < w.nchunks; ++c) {
        const int s = c % kStages;
        // (b) once the gates are done, this dim's 64 (F, q) pairs into its TMEM lane: the
        // stage is released before the read-out instead of after it
        if (!warp_wait(b[kGated + s], (c / kStages) & 1, abort)) break;
        {  // factor (low half) and q (high half), bf16
            const uint32_t sa = smem_u32(smem + s * kStageBytes);
            copy_pairs_to_tmem(sa + off_g, sa + off_q, tmem + kColFQ, quarter, lane);
            tmem_wait_st();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(b[kEmpty + s]);  // this warp's reads of the stage are done
        // (d) dq and q . dq
        if (!mbar_wait(b[kDqFull], c & 1, abort)) break;
        tc_fence_after();
        const long long tok0 = w.row0 + (long long)c * CH;
#pragma unroll 1
        for (int g = 0; g < 4; ++g) {  // tokens 16g .. 16g+15
            uint32_t r16[16], fq[16];
            tmem_ld16(tmem + lrow + kColDQ + g * 16, r16);
            tmem_ld16(tmem + lrow + kColFQ + g * 16, fq);
            tmem_wait_ld();
            if (g == 3) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(b[kDqFree]);
            }
            float dqv[16], qd[16];
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
                const float F0 = __uint_as_float(fq[e] << 16), F1 = __uint_as_float(fq[e + 1] << 16);
                const float a0 = __uint_as_float(r16[e]), a1 = __uint_as_float(r16[e + 1]);
                mul_x2(dqv[e], dqv[e + 1], a0, a1, F0, F1);
                // q . dq handed over as Qbar' dq^T, Qbar' = bf16(q F) -- bit for bit the operand
                // the reverse sweep's MMAs use -- so that the diagonal term (q_t . k_t)(v_t . dO_t)
                // of q . dq and of k . dk is the same exact fp32 product in both sweeps and
                // cancels in dlog_g down to fp32 accumulation error
                const uint32_t qb = mul_bf16x2(__byte_perm(fq[e], fq[e + 1], 0x7632),
                                               __byte_perm(fq[e], fq[e + 1], 0x5410));
                mul_x2(qd[e], qd[e + 1], __uint_as_float(qb << 16), __uint_as_float(qb & 0xFFFF0000u),
                       a0, a1);
            }
            const long long t0 = tok0 + g * 16;
#pragma unroll
            for (int m = 0; m < 4; ++m) {  // four tokens per float4, two per pair store
                *qdq_quad(a.dq_ws, (t0 >> 2) + m, i) =
                    make_float4(qd[4 * m], qd[4 * m + 1], qd[4 * m + 2], qd[4 * m + 3]);
                st_pair_bf16(dq + (t0 + 4 * m) * D + quarter * 32, lane, dqv[4 * m], dqv[4 * m + 1]);
                st_pair_bf16(dq + (t0 + 4 * m + 2) * D + quarter * 32, lane, dqv[4 * m + 2],
                             dqv[4 * m + 3]);
            }
        }
        if (c + 1 < w.nchunks && !make_p(c + 1)) break;
    }
}

// ------------------------------------------------------------------ the kernel
__global__ void __launch_bounds__(kThreads, 1)
tc_dq_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
             const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_g,
             const __grid_constant__ CUtensorMap tm_q, const BwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    Bars b;
    b.base = reinterpret_cast<uint64_t *>(smem + off_bar);
    static_assert(kNumBars <= 24, "barrier area");
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + off_misc);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + off_misc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    Sweep w;
    w.bh = blockIdx.x / a.NP;
    w.j = blockIdx.x % a.NP;
    w.nchunks = (int)(a.T / CH);
    w.cpf = w.nchunks / a.fine;
    w.dstate = a.dSloc && a.logG;
    w.row0 = (long long)w.bh * a.L + (long long)w.j * a.T;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(b[kFull + s], 1);
            mbar_init(b[kFullB + s], 1);
            mbar_init(b[kEcFull + s], kGateWarps);
            mbar_init(b[kGated + s], kGateWarps);
            mbar_init(b[kEmpty + s], 1 + kStateWarps + kOutWarps);
        }
        mbar_init(b[kMFull], 1);
        mbar_init(b[kMFree], kOutWarps);
        mbar_init(b[kDsFull], 1);
        mbar_init(b[kSaFull], kStateWarps);
        mbar_init(b[kDqFull], 1);
        mbar_init(b[kDqFree], kOutWarps);
        mbar_init(b[kRFull], 1);
        mbar_init(b[kRFree], kStateWarps);
        for (int k = 0; k < 2; ++k) {
            mbar_init(b[kPFull + k], kOutWarps);
            mbar_init(b[kSaFree + k], 1);
        }
        mbar_init(b[kFin], 1);
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
        if (lane == 0) producer(smem, b, abort, &tm_k, &tm_v, &tm_do, &tm_g, &tm_q, w);
    } else if (warp == kMmaWarp) {
        mma_issuer(smem, b, abort, tmem, w);
    } else if (warp >= kEpiWarps) {
        gate_role(smem, b, abort, a, w);
    } else if (warp < kStateWarps) {
        state_role(smem, b, abort, a, tmem, w);
    } else {
        out_role(smem, b, abort, a, tmem, w);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (threadIdx.x == 0 && *abort && a.status) atomicOr(a.status, kStatusTimeout);
}

}  // namespace

cudaError_t launch_tc_dq(const BwdArgs &a, cudaStream_t st) {
    const long long rows = (long long)a.BH * a.L;
    CUtensorMap mk, mv, mdo, mg, mq;
    cudaError_t e;
    if ((e = make_map(&mk, a.k, rows)) != cudaSuccess) return e;
    if ((e = make_map(&mv, a.v, rows)) != cudaSuccess) return e;
    if ((e = make_map(&mdo, a.dO, rows)) != cudaSuccess) return e;
    if ((e = make_map(&mg, a.g, rows)) != cudaSuccess) return e;
    if ((e = make_map(&mq, a.q, rows)) != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tc_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    const long long nblk = (long long)a.BH * a.NP;
    if (nblk == 0) return cudaSuccess;
    tc_dq_kernel<<<(unsigned)nblk, kThreads, kSmemBytes, st>>>(mk, mv, mdo, mg, mq, a);
    return cudaGetLastError();
}

}  // namespace la
