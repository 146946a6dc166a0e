// tc_bwd.cu -- the backward's reverse sweep on the 5th-generation tensor cores (bf16, d = 128,
// chunk = 64): dk, dv and dlog_g, walking each fine part's chunks last to first (the dq sweep
// is in tc_dq.cu).  Bounded waits and the abort path follow tc_pass.cu.
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

// ------------------------------------------------------------------ reverse sweep
// Per chunk, last to first, with dS the gradient of the state at the chunk's end (rows = key
// dims; starts at dX of the part), Qbar'_t = q_t e^{b_t - b_C}, Ktil_s = k_s e^{b_C - b_s}:
//
//   [M *; * A] = [dO; Qbar'] [V; Ktil]^T  M=128 N=128 K=128: M = dO V^T and A = Qbar' Ktil^T
//                                       are its diagonal 64 x 64 blocks  -> masked s <= t, bf16
//   dk^T  = Qbar'^T M + dS V^T          M=128 (i) N=64 (s) K=64 (t) / 128 (j)
//   dv^T  = dO^T A + dS^T Ktil^T        M=128 (j) N=64 (s) K=64 (t) / 128 (i)
//   dS   += Qbar'^T dO                  M=128 (i) N=128 (j) K=64 (t), accumulated in TMEM
//   dk[s,i] = e^{b_C,i - b_s,i} dk^T[i,s];   dS <- diag(e^{b_C}) dS
//   dlog_g_s = rowsum(S_end . dX) + sum_{u >= s in the part} (q_u dq_u - k_u dk_u)
//
// The (dO, Qbar') and (V, Ktil) tiles of a stage sit with their 64-column halves interleaved,
// [dO h0][Qbar' h0][dO h1][Qbar' h1], so that each pair is also one 128-row K-major operand:
// M and A come from 8 MMA instructions of full width instead of 16 of half width (the
// off-diagonal blocks are computed and ignored).
//
// Roles (448 threads): warps 0-3 carry dS -- the fp32 dS lives in tensor memory (row i on lane
// i), they apply the decay, write its bf16 copy into a shared [i][j] tile (read by the MMAs as
// the K-major A operand of dS V^T and the MN-major A operand of dS^T Ktil^T), turn M and A into
// masked bf16 tiles (double-buffered) and write dv from dv^T; warps 4-7 read dk^T
// (double-buffered in TMEM) and write dk and dlog_g (thread x owns key dim x for all 64 tokens
// of the chunk, so the dlog_g suffix sums need no exchange); warps 8-11 gate the chunks; 12 TMA;
// 13 MMA.  A stage is released once the tensor cores are done with it and the dS and output
// warps have copied the per-key factors they need into registers or TMEM.
namespace dkv {

constexpr int kStateWarps = 4, kOutWarps = 4;
// Tensor-memory columns: [M *; * A] (128 x 128), dk^T x 2, dv^T, the chunk's
// (e^{b_C - b_s}, Ktil) pairs for the output warps, dS.
constexpr uint32_t kColMA = 0, kColDK = 128, kColDV = 256, kColFK = 320, kColDS = 384;
constexpr int kStages = 2;
constexpr int kPairHalf = 2 * kHalfBytes;  // distance between a paired tile's two halves
constexpr int off_do = 0, off_q = kHalfBytes, off_v = 2 * kTileBytes,
              off_k = 2 * kTileBytes + kHalfBytes, off_g = 4 * kTileBytes;
constexpr int kStageBytes = 5 * kTileBytes;
constexpr int kDsHalf = 128 * 128;            // one 64-column half of the [128 x 128] bf16 dS tile
constexpr int kMaskBytes = CH * CH * 2;       // one masked 64 x 64 bf16 tile
constexpr int off_ma = kStages * kStageBytes;  // 2 buffers x (M tile, A tile)
constexpr int off_ds = off_ma + 4 * kMaskBytes;
constexpr int off_ec = off_ds + 2 * kDsHalf;
constexpr int off_bar = off_ec + kStages * D * 4;
constexpr int kBars = 4 * kStages + 17;
constexpr int off_misc = off_bar + kBars * 8;
constexpr int kSmemBytes = off_misc + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Bars {
    uint64_t *full, *full_b, *gated, *empty;  // full: log_g, q, k (the gates); full_b: v, dO
    uint64_t *ma_full, *ma_free, *p_full, *dst_full, *dk_full, *dk_free, *dv_full, *dv_free,
        *dsn_full, *fin, *dx_full;
};

// At a CTA's start the part's dX (fp32 [128 x 128], 64 KiB) is TMA-loaded as four 32-column
// boxes with the 128-byte swizzle into the masked-tile and dS-tile area, which the first chunk
// only writes later: row i of box b at kDxStage + b * 16 KiB + i * 128, 16-byte chunk e stored
// at chunk e ^ (i % 8), so that the dS warps' row reads are free of bank conflicts.
constexpr int kDxStage = off_ma;
static_assert(off_ds + 2 * kDsHalf - off_ma == 4 * 16384, "dX staging area");

// [128 rows][128 cols] bf16 tile as two 64-column halves of 16 KiB, 128-byte swizzle.
__device__ __forceinline__ uint32_t ds_off(int row, int col) {
    const int half = col >> 6, cc = col & 63;
    return (uint32_t)(half * kDsHalf + row * 128 + (((cc >> 3) ^ (row & 7)) << 4) + ((cc & 7) << 1));
}

__device__ void producer(uint8_t *smem, const Bars &b, volatile int *abort, const BwdArgs &a,
                         const CUtensorMap *tq, const CUtensorMap *tk, const CUtensorMap *tv,
                         const CUtensorMap *tdo, const CUtensorMap *tg, const CUtensorMap *tdx,
                         int dx_row, long long row0, int nchunks) {
    mbar_arrive_expect_tx(b.dx_full, 4 * 16384);
    for (int bx = 0; bx < 4; ++bx)
        tma_load_2d(smem + kDxStage + bx * 16384, tdx, 32 * bx, dx_row, b.dx_full);
    int issued = 0;
    for (int it = 0; it < nchunks; ++it) {
        const int s = it % kStages;
        const int c = nchunks - 1 - it;  // last chunk first
        // the chunk's q . dq block (read with plain loads by the output warps) on its way to L2
        bulk_prefetch_l2(a.dq_ws + (row0 + (long long)c * CH) * D, CH * D * 4);
        if (it >= kStages && !mbar_wait(&b.empty[s], ((it / kStages) - 1) & 1, abort)) break;
        uint8_t *st = smem + s * kStageBytes;
        const int y = (int)(row0 + (long long)c * CH);
        // the gates' tiles first, on their own barrier (the gates start as soon as they land);
        // v and dO, read only by the tensor cores, behind them
        const CUtensorMap *maps[5] = {tg, tq, tk, tv, tdo};
        const int offs[5] = {off_g, off_q, off_k, off_v, off_do};
        mbar_arrive_expect_tx(&b.full[s], 3 * kTileBytes);
        mbar_arrive_expect_tx(&b.full_b[s], 2 * kTileBytes);
#pragma unroll
        for (int m = 0; m < 5; ++m) {
            uint64_t *bar = m < 3 ? &b.full[s] : &b.full_b[s];
            tma_load_2d(st + offs[m], maps[m], 0, y, bar);
            tma_load_2d(st + offs[m] + (m == 0 ? kHalfBytes : kPairHalf), maps[m], 64, y, bar);
        }
        issued = it + 1;
    }
    if (*abort) {
        wait_drain(b.dx_full, 0);
        for (int it = issued > kStages ? issued - kStages : 0; it < issued; ++it) {
            wait_drain(&b.full[it % kStages], (it / kStages) & 1);
            wait_drain(&b.full_b[it % kStages], (it / kStages) & 1);
        }
    }
}

// The whole warp walks the loop; one elected lane issues.  Per chunk: dk^T and dv^T into
// buffer it % 2 after the dS update (so that dk_full also frees the q tile), then the next
// chunk's M and A once it is gated (so that they are ready when the dS warps finish the decay).
__device__ void mma_issuer(uint8_t *smem, const Bars &b, volatile int *abort, uint32_t tmem,
                           int nchunks) {
    constexpr uint32_t i_ma = idesc_bf16_f32(128, 128, 0, 0);    // [M *; * A]
    constexpr uint32_t i_dsn = idesc_bf16_f32(128, 128, 1, 1);   // Qbar'^T dO
    constexpr uint32_t i_dka = idesc_bf16_f32(128, 64, 1, 1);    // Qbar'^T M
    constexpr uint32_t i_dkb = idesc_bf16_f32(128, 64, 0, 0);    // dS V^T
    constexpr uint32_t i_dva = idesc_bf16_f32(128, 64, 1, 1);    // dO^T A
    constexpr uint32_t i_dvb = idesc_bf16_f32(128, 64, 1, 0);    // dS^T Ktil^T
    const uint32_t base = smem_u32(smem);
    const uint32_t ma_addr = base + off_ma, ds_addr = base + off_ds;
    auto stage = [&](int it) { return base + (uint32_t)((it % kStages) * kStageBytes); };
    // [dO; Qbar'] [V; Ktil]^T: both 128-row operands are K-major pairs of interleaved tiles
    auto issue_ma = [&](int it) -> bool {
        const uint32_t st = stage(it);
        if (!warp_wait(&b.full_b[it % kStages], (it / kStages) & 1, abort)) return false;  // v, dO
        if (!warp_wait(&b.gated[it % kStages], (it / kStages) & 1, abort)) return false;
        if (it > 0 && !warp_wait(b.ma_free, (it - 1) & 1, abort)) return false;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_ss(tmem + kColMA, desc_kmajor(st + off_do, kk, kPairHalf),
                       desc_kmajor(st + off_v, kk, kPairHalf), i_ma, kk > 0);
            mma_commit(b.ma_full);
        }
        __syncwarp();
        return true;
    };
    bool ok = nchunks > 0 && issue_ma(0);
    for (int it = 0; ok && it < nchunks; ++it) {
        const int s = it % kStages, bb = it & 1;
        const uint32_t st = stage(it);
        const uint32_t qa = st + off_q, ka = st + off_k, va = st + off_v, da = st + off_do;
        const uint32_t mt = ma_addr + bb * 2 * kMaskBytes, at = mt + kMaskBytes;
        if (!(ok = warp_wait(b.p_full, it & 1, abort))) break;
        if (!(ok = warp_wait(b.dst_full, it & 1, abort))) break;
        if (it >= 2 && !(ok = warp_wait(&b.dk_free[bb], ((it >> 1) - 1) & 1, abort))) break;
        if (it >= 1 && !(ok = warp_wait(b.dv_free, (it - 1) & 1, abort))) break;
        tc_fence_after();
        if (elect_one()) {
            const uint32_t dk_col = tmem + kColDK + bb * 64, dv_col = tmem + kColDV;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // dS += Qbar'^T dO  (dk and dv read the old dS tile)
                mma_ss(tmem + kColDS, desc_mnmajor(qa, kk, kPairHalf), desc_mnmajor(da, kk, kPairHalf),
                       i_dsn, 1u);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // dk^T = Qbar'^T M   (B: M tile read MN-major)
                mma_ss(dk_col, desc_mnmajor(qa, kk, kPairHalf),
                       smem_desc_sw128(mt + kk * 2048, kHalfBytes, 1024), i_dka, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // dk^T += dS V^T   (A: dS tile K-major, 128 rows)
                mma_ss(dk_col, smem_desc_sw128(ds_addr + (kk >> 2) * kDsHalf + (kk & 3) * 32, 16, 1024),
                       desc_kmajor(va, kk, kPairHalf), i_dkb, 1u);
            mma_commit(&b.dk_full[bb]);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // dv^T = dO^T A   (B: A tile read MN-major)
                mma_ss(dv_col, desc_mnmajor(da, kk, kPairHalf),
                       smem_desc_sw128(at + kk * 2048, kHalfBytes, 1024), i_dva, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // dv^T += dS^T Ktil^T   (A: dS tile read MN-major)
                mma_ss(dv_col, smem_desc_sw128(ds_addr + kk * 2048, kDsHalf, 1024),
                       desc_kmajor(ka, kk, kPairHalf), i_dvb, 1u);
            mma_commit(b.dv_full);
            mma_commit(b.dsn_full);  // the dS tile is read out as well
            mma_commit(&b.empty[s]);
        }
        __syncwarp();
        if (it + 1 < nchunks && !(ok = issue_ma(it + 1))) break;  // the next chunk's M and A
    }
    if (elect_one()) mma_commit(b.fin);
    __syncwarp();
    wait_drain(b.fin, 0);
}

// dv of one chunk from dv^T (thread x = TMEM lane x owns value dim x), straight to HBM (`dvc`
// points at the chunk's first token, dim 32 w for warp w); releases the accumulator after the
// last tensor-memory read.  The dS warps run it after the next chunk's decay, while the next
// chunk's M and A are formed: that chunk's dv^T MMA waits for it (one dv^T buffer).
__device__ __forceinline__ bool dv_readout(const Bars &b, volatile int *abort, uint32_t tmem,
                                           uint32_t lrow, int parity, __nv_bfloat16 *dvc,
                                           int lane) {
    if (!mbar_wait(b.dv_full, parity, abort)) return false;
    tc_fence_after();
    uint32_t r[16];
#pragma unroll 1
    for (int g = 0; g < 4; ++g) {
        tmem_ld16(tmem + lrow + kColDV + g * 16, r);
        tmem_wait_ld();
        if (g == 3) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(b.dv_free);
        }
#pragma unroll
        for (int t = 0; t < 16; t += 2)
            st_pair_bf16(dvc + (g * 16 + t) * D, lane, __uint_as_float(r[t]), __uint_as_float(r[t + 1]));
    }
    return true;
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
    uint32_t posm = 0x80008000u;  // running int16 max of the log_g bits: > 0 means a positive gate exponent
    for (int it = 0; it < nchunks; ++it) {
        const int s = it % kStages;
        if (!mbar_wait(&b.full[s], (it / kStages) & 1, abort)) break;
        uint8_t *st = smem + s * kStageBytes;
        // The in-chunk cumsum reproduces the dq sweep's bit for bit -- the same sums within
        // groups of 4 rows and the same Hillis-Steele tree over the 16 group totals (this
        // thread holds groups 2 tg and 2 tg + 1) -- so that both sweeps form identical bf16
        // operands Ktil and Qbar' = bf16(q bf16(e^x)); the diagonal term of q . dq and k . dk is
        // then the same fp32 product in both and cancels exactly in dlog_g.
        float bt[8][8], tot[2][8];
        {
            uint4 graw[8];
#pragma unroll
            for (int r = 0; r < 8; ++r)
                graw[r] = *reinterpret_cast<const uint4 *>(st + off_g + tile_off(tg * 8 + r, i0));
#pragma unroll
            for (int r = 0; r < 8; ++r) posm = pos_bf16_max(posm, graw[r]);
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // rows 8 tg + 4 h .. + 3
                float f[4][8];
#pragma unroll
                for (int k = 0; k < 4; ++k) unpack8(graw[4 * h + k], f[k]);
#pragma unroll
                for (int e = 0; e < 8; e += 2) {  // two key dims per f32x2 instruction
                    float p01[2], p23[2];
                    add_x2(p01[0], p01[1], f[0][e], f[0][e + 1], f[1][e], f[1][e + 1]);
                    add_x2(p23[0], p23[1], f[2][e], f[2][e + 1], f[3][e], f[3][e + 1]);
                    bt[4 * h][e] = f[0][e];
                    bt[4 * h][e + 1] = f[0][e + 1];
                    bt[4 * h + 1][e] = p01[0];
                    bt[4 * h + 1][e + 1] = p01[1];
                    add_x2(bt[4 * h + 2][e], bt[4 * h + 2][e + 1], f[2][e], f[2][e + 1], p01[0], p01[1]);
                    add_x2(bt[4 * h + 3][e], bt[4 * h + 3][e + 1], p23[0], p23[1], p01[0], p01[1]);
                    add_x2(tot[h][e], tot[h][e + 1], p01[0], p01[1], p23[0], p23[1]);
                }
            }
        }
        float ia[8], ib[8];  // inclusive scan of the group totals: groups 2 tg, 2 tg + 1
#pragma unroll
        for (int e = 0; e < 8; e += 2) {  // step 1: group g adds group g - 1
            const float u0 = __shfl_up_sync(0xFFFFFFFFu, tot[1][e], 4);
            const float u1 = __shfl_up_sync(0xFFFFFFFFu, tot[1][e + 1], 4);
            add_x2(ia[e], ia[e + 1], tot[0][e], tot[0][e + 1], u0, u1);
            if (tg < 1) {
                ia[e] = tot[0][e];
                ia[e + 1] = tot[0][e + 1];
            }
            add_x2(ib[e], ib[e + 1], tot[1][e], tot[1][e + 1], tot[0][e], tot[0][e + 1]);
        }
#pragma unroll
        for (int dd = 1; dd < 8; dd <<= 1) {  // steps 2, 4, 8: group g adds group g - 2 dd
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
                const float a0 = __shfl_up_sync(0xFFFFFFFFu, ia[e], 4 * dd);
                const float a1 = __shfl_up_sync(0xFFFFFFFFu, ia[e + 1], 4 * dd);
                const float b0 = __shfl_up_sync(0xFFFFFFFFu, ib[e], 4 * dd);
                const float b1 = __shfl_up_sync(0xFFFFFFFFu, ib[e + 1], 4 * dd);
                if (tg >= dd) {
                    add_x2(ia[e], ia[e + 1], ia[e], ia[e + 1], a0, a1);
                    add_x2(ib[e], ib[e + 1], ib[e], ib[e + 1], b0, b1);
                }
            }
        }
        float nbCl[8];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            const float bC0 = __shfl_sync(0xFFFFFFFFu, ib[e], 28 + ig);  // group 15
            const float bC1 = __shfl_sync(0xFFFFFFFFu, ib[e + 1], 28 + ig);
            float offa[2], offb[2];
            sub_x2(offa[0], offa[1], ia[e], ia[e + 1], tot[0][e], tot[0][e + 1]);
            sub_x2(offb[0], offb[1], ib[e], ib[e + 1], tot[1][e], tot[1][e + 1]);
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                add_x2(bt[r][e], bt[r][e + 1], bt[r][e], bt[r][e + 1], offa[0], offa[1]);
                add_x2(bt[4 + r][e], bt[4 + r][e + 1], bt[4 + r][e], bt[4 + r][e + 1], offb[0], offb[1]);
            }
            mul_x2(nbCl[e], nbCl[e + 1], -bC0, -bC1, kLog2e, kLog2e);
            range_bad |= !(fabsf(bC0) <= kGateRangeLimit) || !(fabsf(bC1) <= kGateRangeLimit);
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
                const uint32_t off = tile_off(tg * 8 + r0 + r, i0, kPairHalf);
                qr[r] = *reinterpret_cast<const uint4 *>(st + off_q + off);
                kr[r] = *reinterpret_cast<const uint4 *>(st + off_k + off);
            }
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const uint32_t off = tile_off(tg * 8 + r0 + r, i0, kPairHalf);
                float x[8], fk[8];
#pragma unroll
                for (int e = 0; e < 8; e += 2)
                    fma_x2(x[e], x[e + 1], bt[r0 + r][e], bt[r0 + r][e + 1], kLog2e, kLog2e, nbCl[e],
                           nbCl[e + 1]);
                unpack8(kr[r], fk);
                const uint32_t qw[4] = {qr[r].x, qr[r].y, qr[r].z, qr[r].w};
                uint32_t wq[4], wk[4], wf[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float u0 = ex2_approx(x[2 * e]), u1 = ex2_approx(x[2 * e + 1]);
                    const float d0 = ex2_approx(-x[2 * e]), d1 = ex2_approx(-x[2 * e + 1]);
                    const uint32_t fw = pack_bf16(u0, u1);  // F = bf16(e^x), as the dq sweep has it
                    wq[e] = mul_bf16x2(qw[e], fw);  // bf16(q F): the bf16 product is exact in fp32
                    float k0, k1;
                    mul_x2(k0, k1, fk[2 * e], fk[2 * e + 1], d0, d1);
                    wk[e] = pack_bf16(k0, k1);
                    wf[e] = pack_bf16(d0, d1);
                }
                *reinterpret_cast<uint4 *>(st + off_q + off) = make_uint4(wq[0], wq[1], wq[2], wq[3]);
                *reinterpret_cast<uint4 *>(st + off_k + off) = make_uint4(wk[0], wk[1], wk[2], wk[3]);
                *reinterpret_cast<uint4 *>(st + off_g + tile_off(tg * 8 + r0 + r, i0)) =
                    make_uint4(wf[0], wf[1], wf[2], wf[3]);
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&b.gated[s]);
    }
    if (range_bad || any_pos_bf16(posm))  // this CTA's unit is fine part blockIdx.x = bh * NP + j
        flag_range(a.flags, (long long)blockIdx.x, 1, a.status);
}

// Writes columns 32 h .. 32 h + 31 of row t of a 64 x 64 tile as its masked (s <= t) bf16 copy.
__device__ __forceinline__ void masked_row(uint8_t *tile, const uint32_t (&r)[32], int t, int h) {
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

// Warps 0-3: thread i owns row i of dS (TMEM lane i).  Per chunk: the decay by the previous
// chunk's e^{b_C} (S_new = diag(e^{b_C}) (dS + Qbar'^T dO), the sum formed by the MMA), the
// bf16 copy of row i into the dS tile, dv of the previous chunk (value dim i; M and A of this
// chunk are formed meanwhile), the masked M and A tiles; the stage is released as soon as its
// e^{b_C} is in a register.
__device__ void state_role(uint8_t *smem, const Bars &b, volatile int *abort, const BwdArgs &a,
                           uint32_t tmem, int bh, int j, int nchunks) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = warp * 32 + lane;
    const uint32_t lrow = (uint32_t)(warp * 32) << 16;
    const float *ec = reinterpret_cast<const float *>(smem + off_ec);
    __nv_bfloat16 *dv = static_cast<__nv_bfloat16 *>(a.dv_out) +
                        ((long long)bh * a.L + (long long)j * a.T) * D + warp * 32;
    uint32_t r[32];
    // dS at the part's end: dX, row i from the swizzled staging boxes.  Column groups go last to
    // first: the bf16 copy of group p lands on row i of box 2 + p / 2 (the dS tile's halves
    // overlay boxes 2 and 3), which this thread has read by then; no other thread reads row i.
    const bool dx_ok = warp_wait(b.dx_full, 0, abort);
#pragma unroll
    for (int p = 3; p >= 0; --p) {
        if (!dx_ok) break;
        const uint8_t *row = smem + kDxStage + p * 16384 + i * 128;
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
            const uint4 v = *reinterpret_cast<const uint4 *>(row + ((e4 ^ (i & 7)) << 4));
            r[4 * e4] = v.x; r[4 * e4 + 1] = v.y; r[4 * e4 + 2] = v.z; r[4 * e4 + 3] = v.w;
        }
        tmem_st32(tmem + lrow + kColDS + p * 32, r);
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
    tmem_wait_st();
    tc_fence_before();
    // the first masked tiles overwrite boxes 0 and 1, whose rows the other dS warps read (every
    // dS warp reaches this barrier, also when its wait gave up)
    named_sync(1, kStateWarps * 32);
    if (!dx_ok) return;
    uint64_t e2 = 0;  // e^{b_C,i} of the previous chunk, in both halves
    for (int it = 0; it < nchunks; ++it) {
        // (1) dS of this chunk's end: the decayed dS of the chunk after it (the part's last
        // chunk starts from dX, stored above)
        if (it > 0) {
            if (!mbar_wait(b.dsn_full, (it - 1) & 1, abort)) break;
            tc_fence_after();
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                tmem_ld32(tmem + lrow + kColDS + p * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const uint64_t x = mul_f32x2(((uint64_t)r[2 * e + 1] << 32) | r[2 * e], e2);
                    r[2 * e] = (uint32_t)x;
                    r[2 * e + 1] = (uint32_t)(x >> 32);
                }
                tmem_st32(tmem + lrow + kColDS + p * 32, r);
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
            tmem_wait_st();
        }
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(b.dst_full);
        // dv of the previous chunk: its MMAs completed with dsn_full
        if (it > 0 && !dv_readout(b, abort, tmem, lrow, (it - 1) & 1,
                                  dv + (long long)(nchunks - it) * CH * D, lane))
            break;
        // (2) masked M and A tiles of this chunk: TMEM lane 32 w + l is row 32 w + l of
        // [M *; * A], so warps 0-1 hold rows t = 32 w + l of M (columns 0-63) and warps 2-3 rows
        // t = 32 (w - 2) + l of A (columns 64-127)
        if (!mbar_wait(b.ma_full, it & 1, abort)) break;
        tc_fence_after();
        {
            const int blk = warp >> 1, t = (warp & 1) * 32 + lane;
            uint8_t *mt = smem + off_ma + ((it & 1) * 2 + blk) * kMaskBytes;
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                tmem_ld32(tmem + lrow + kColMA + blk * 64 + h * 32, r);
                tmem_wait_ld();
                if (h == 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(b.ma_free);
                }
                masked_row(mt, r, t, h);
            }
        }
        fence_proxy_async_smem();
        // the chunk's e^{b_C} is this role's last read of the stage
        e2 = (uint64_t)__float_as_uint(ec[(it % kStages) * D + i]) * 0x100000001ull;
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(b.p_full);
            mbar_arrive(&b.empty[it % kStages]);
        }
    }
    if (!*abort && nchunks > 0)  // dv of the part's first chunk
        dv_readout(b, abort, tmem, lrow, (nchunks - 1) & 1, dv, lane);
}

// Warps 4-7: thread x = 32 (warp - 4) + lane owns key dim x of dk and dlog_g for all 64 tokens
// of the chunk.  As soon as the gates are done with a chunk, each thread copies its dim's 64
// (e^{b_C - b_s}, Ktil) pairs from the stage into its TMEM lane and releases the stage; the dk
// loop then reads them back from TMEM beside the dk^T accumulator.  Outputs go straight from
// registers to HBM, each lane of a pair writing two dims of one token.
__device__ void out_role(uint8_t *smem, const Bars &b, volatile int *abort, const BwdArgs &a,
                         uint32_t tmem, int bh, int j, long long row0, int nchunks) {
    const int quarter = (threadIdx.x >> 5) & 3, lane = threadIdx.x & 31;
    const int x = quarter * 32 + lane;
    const uint32_t lrow = (uint32_t)(quarter * 32) << 16;
    __nv_bfloat16 *dk = static_cast<__nv_bfloat16 *>(a.dk_out);
    __nv_bfloat16 *dg = static_cast<__nv_bfloat16 *>(a.dg_out);
    const long long sidx = ((long long)bh * a.NP + j) * D * D;
    // carry: rowsum(S_end . dX), the gradient reaching this part from its end state (formed by
    // the reverse scan when it is given)
    float carry = 0.f;
    if (a.carry) {
        carry = a.carry[((long long)bh * a.NP + j) * D + x];
    } else {
        const float *Se = nullptr;
        if (j < a.NP - 1) {
            if (a.S_end_next) Se = a.S_end_next + sidx + (long long)D * D;
        } else if (a.S_fin) {
            Se = a.S_fin + (long long)bh * D * D;
        }
        if (Se) {  // summed in the reverse scan's order (per 4 columns, then a pairwise tree)
            const float4 *x4 = reinterpret_cast<const float4 *>(a.dX + sidx + (long long)x * D);
            const float4 *s4 = reinterpret_cast<const float4 *>(Se + (long long)x * D);
            float part[D / 4];
#pragma unroll
            for (int e4 = 0; e4 < D / 4; ++e4) {
                const float4 v = x4[e4], u = s4[e4];
                part[e4] = fmaf(u.w, v.w, fmaf(u.z, v.z, fmaf(u.y, v.y, u.x * v.x)));
            }
#pragma unroll
            for (int o = 1; o < D / 4; o <<= 1) {
#pragma unroll
                for (int k = 0; k < D / 4; k += 2 * o) part[k] += part[k + o];
            }
            carry = part[0];
        }
    }
    // q . dq (token-quad interleaved, float4 = 4 tokens of dim x): two buffers of one 16-token
    // group each; a group's loads go out as soon as the group two before it has been used
    auto load_qdq = [&](float4 (&dst)[4], long long rq) {
#pragma unroll
        for (int m = 0; m < 4; ++m) dst[m] = *qdq_quad(a.dq_ws, rq + m, x);
    };
    const int dim0 = quarter * 32;
    for (int it = 0; it < nchunks; ++it) {
        const int s = it % kStages, bb = it & 1;
        const int c = nchunks - 1 - it;
        const long long tq = (row0 + (long long)c * CH) >> 2;  // the chunk's first token quad
        float4 qb[2][4];
        load_qdq(qb[0], tq + 12);  // tokens 48 .. 63, then 32 .. 47 (L2-prefetched with the tiles)
        load_qdq(qb[1], tq + 8);
        // (1) the chunk's factors and Ktil into this lane of TMEM; then the stage is released
        if (!warp_wait(&b.gated[s], (it / kStages) & 1, abort)) break;
        const uint32_t sa = smem_u32(smem + s * kStageBytes);
        copy_pairs_to_tmem(sa + off_g, sa + off_k, tmem + kColFK, quarter, lane, kHalfBytes, kPairHalf);
        tmem_wait_st();
        __syncwarp();
        if (lane == 0) mbar_arrive(&b.empty[s]);
        // (2) dk and the dlog_g suffix sums: tokens last to first, 16 at a time
        if (!mbar_wait(&b.dk_full[bb], (it >> 1) & 1, abort)) break;
        tc_fence_after();
#pragma unroll
        for (int g = 3; g >= 0; --g) {
            uint32_t r[16], fk[16];
            tmem_ld16(tmem + lrow + kColDK + bb * 64 + g * 16, r);
            tmem_ld16(tmem + lrow + kColFK + g * 16, fk);
            tmem_wait_ld();
            if (g == 0) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&b.dk_free[bb]);
            }
            const float4 *qv = qb[(3 - g) & 1];
            // dk = e^{b_C - b_s} acc and the contribution q . dq - k . dk (k . dk = Ktil . acc,
            // Ktil = k e^{b_C - b_s} the MMA operand); then the suffix sums
            float fd[16], cg[16];  // dk, then contributions / dlog_g
#pragma unroll
            for (int t = 0; t < 16; t += 2) {  // two tokens per f32x2 instruction
                const float a0 = __uint_as_float(r[t]), a1 = __uint_as_float(r[t + 1]);
                const float4 &q4 = qv[t >> 2];
                const float q0 = (t & 3) == 0 ? q4.x : q4.z, q1 = (t & 3) == 0 ? q4.y : q4.w;
                mul_x2(fd[t], fd[t + 1], __uint_as_float(fk[t] << 16), __uint_as_float(fk[t + 1] << 16),
                       a0, a1);  // dk
                fma_x2(cg[t], cg[t + 1], -__uint_as_float(fk[t] & 0xFFFF0000u),
                       -__uint_as_float(fk[t + 1] & 0xFFFF0000u), a0, a1, q0, q1);  // contribution
            }
            if (g >= 2) load_qdq(qb[(3 - g) & 1], tq + 4 * (g - 2));  // group g - 2
#pragma unroll
            for (int t = 15; t >= 0; --t) {
                carry += cg[t];
                cg[t] = carry;                 // dlog_g
            }
            const long long e0 = (row0 + (long long)c * CH + g * 16) * D + dim0;  // (t0, dim0)
#pragma unroll
            for (int t = 0; t < 16; t += 2) {
                st_pair_bf16(dk + e0 + t * D, lane, fd[t], fd[t + 1]);
                st_pair_bf16(dg + e0 + t * D, lane, cg[t], cg[t + 1]);
            }
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
tc_dkv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_dx,
              const BwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + off_bar);
    Bars b;
    b.full = bar;
    b.gated = bar + kStages;
    b.empty = bar + 2 * kStages;
    b.full_b = bar + 3 * kStages;
    uint64_t *x = bar + 4 * kStages;
    b.ma_full = x + 0; b.ma_free = x + 1; b.p_full = x + 2; b.dst_full = x + 3; b.dk_full = x + 4;
    b.dk_free = x + 6; b.dv_full = x + 8; b.dv_free = x + 10; b.dsn_full = x + 12; b.fin = x + 13;
    b.dx_full = x + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + off_misc);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + off_misc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x / a.NP, j = blockIdx.x % a.NP;
    const long long row0 = (long long)bh * a.L + (long long)j * a.T;
    const int nchunks = (int)(a.T / CH);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&b.full[s], 1);
            mbar_init(&b.full_b[s], 1);
            mbar_init(&b.gated[s], kGateWarps);
            mbar_init(&b.empty[s], 1 + kStateWarps + kOutWarps);
        }
        uint64_t *one[] = {b.ma_full, b.dk_full, b.dk_full + 1, b.dv_full, b.dsn_full,
                           b.fin, b.dx_full};
        uint64_t *st4[] = {b.ma_free, b.p_full, b.dst_full, b.dv_free};
        uint64_t *out4[] = {b.dk_free, b.dk_free + 1};
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
        prefetch_tmap(&tm_dx);
    }
    if (warp == kMmaWarp) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (warp == kTmaWarp) {
        if (lane == 0)
            producer(smem, b, abort, a, &tm_q, &tm_k, &tm_v, &tm_do, &tm_g, &tm_dx,
                     (int)(((long long)bh * a.NP + j) * D), row0, nchunks);
    } else if (warp == kMmaWarp) {
        mma_issuer(smem, b, abort, tmem, nchunks);
    } else if (warp >= kEpiWarps) {
        gate_role(smem, b, abort, a, nchunks);
    } else if (warp < kStateWarps) {
        state_role(smem, b, abort, a, tmem, bh, j, nchunks);
    } else {
        out_role(smem, b, abort, a, tmem, bh, j, row0, nchunks);
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

cudaError_t launch_tc_dkv(const BwdArgs &a, cudaStream_t st) {
    const long long rows = (long long)a.BH * a.L;
    CUtensorMap mq, mk, mv, mdo, mg;
    cudaError_t e;
    if ((e = make_map(&mq, a.q, rows)) != cudaSuccess) return e;
    if ((e = make_map(&mk, a.k, rows)) != cudaSuccess) return e;
    if ((e = make_map(&mv, a.v, rows)) != cudaSuccess) return e;
    if ((e = make_map(&mdo, a.dO, rows)) != cudaSuccess) return e;
    if ((e = make_map(&mg, a.g, rows)) != cudaSuccess) return e;
    CUtensorMap mdx;  // dX as [BH * NP * dk rows, dv] fp32
    if ((long long)a.BH * a.NP * D > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
    if ((e = make_map_f32_rows(&mdx, a.dX, (long long)a.BH * a.NP * D)) != cudaSuccess) return e;
    e = cudaFuncSetAttribute(dkv::tc_dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             dkv::kSmemBytes);
    if (e != cudaSuccess) return e;
    const long long nblk = (long long)a.BH * a.NP;
    if (nblk == 0) return cudaSuccess;
    dkv::tc_dkv_kernel<<<(unsigned)nblk, kThreads, dkv::kSmemBytes, st>>>(mq, mk, mv, mdo, mg, mdx,
                                                                           a);
    return cudaGetLastError();
}

}  // namespace la
