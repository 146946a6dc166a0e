// internal.h -- launchers shared between the translation units of libla_seg.so (C++ only,
// never part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "common.cuh"

namespace la {

// What one chunk-pass launch computes for each (b, h, sub-segment j), starting from state
// S_init[j] (or zero) and walking the sub-segment chunk by chunk:
enum PassMode : int {
    kPassState = 0,    // local state S_j (from zero) + log-decay sum only; reads k, v, log_g
    kPassOutput = 1,   // o from S_init[j]; reads q, k, v, log_g; writes o
    kPassLocal = 2,    // o_local from zero, local state and log-decay sum; writes o, S, logG
    kPassCorrect = 3,  // o += (q . exp(B_seg)) S_init[j]; reads q, log_g, o
    kPassDState = 4,   // backward gradient state sum_t diag(e^{B_t}) q_t^T dO_t (dO passed as v)
};

struct PassArgs {
    const void *q, *k, *v, *g;
    void *o;
    const float *S_init;  // [BH, NP, dk, dv] or null (zero)
    float *S_out;         // [BH, NP, dk, dv] (kPassState / kPassLocal; null: not written)
    float *logG;          // [BH, NP, dk]    (kPassState / kPassLocal; null: not written)
    int *status;
    int *flags;           // [BH, NP] units met outside the factorisation's range (null: status)
    long long L, T;       // tokens per (b, h), tokens per sub-segment
    int BH, NP, dk, dv, chunk;
    la_dtype dt;
};

// Arguments of the backward chunk passes (one CTA per (b, h, segment j)).  The dq sweep runs
// over NP segments of T tokens and records the state entering every one of its `fine` equal
// parts in S_fine; the gradient-state pass and the reverse sweep run over those fine parts
// (NP and T then describe the fine split), so that the exact dlog_g carry
// rowsum(S_end . dX) is re-anchored every T tokens.
struct BwdArgs {
    const void *q, *k, *v, *g, *dO;
    void *dq_out, *dk_out, *dv_out, *dg_out;
    const float *S_recv;      // dq sweep: [BH, NP, dk, dv] state each segment receives (null: zero)
    float *S_fine;            // dq sweep output: [BH, NP * fine, dk, dv] (null: not recorded)
    const float *S_end_next;  // reverse sweep: S_end_j = S_end_next[j+1] for j < NP-1 (null: no carry)
    const float *S_fin;       // [BH, dk, dv] state after the last token (null: no carry there)
    const float *dX;          // [BH, NP, dk, dv] gradient of each segment's end state
    float *dq_ws;             // [BH, L, dk] fp32 q . dq, from the dq sweep to the reverse sweep:
                              // token-quad interleaved on the tensor-core path, row-major on
                              // the SIMT path
    float *dSloc;             // [BH, NP, dk, dv] per-segment gradient states (dstate pass)
    float *logG;              // [BH, NP, dk] per-segment log-decay sums (dstate pass)
    const float *carry;       // reverse sweep: [BH, NP, dk] dlog_g carry per part (null: computed)
    int *status;
    int *flags;               // [BH, NP * fine] fine parts met outside the factorisation's range
                              // (null: status); the dq sweep marks every part of its segment
    long long L, T;
    int BH, NP, dk, dv, chunk, fine;
    la_dtype dt;
    int qdq_quad;             // exact path only: dq_ws is token-quad interleaved (set by its
                              // launchers from tc_bwd_supported)
};

// The single-pass forward's chain through the sub-segments of every (b, h) sequence.
struct ChainArgs {
    float *states;   // [BH, 2, dk, dv]: two slots for the state a sub-segment receives; sub-segment
                     // j reads slot j % 2 and writes the state after it into slot (j + 1) % 2
    int *ready;      // [BH + 1]: ready[bh] = the latest sub-segment j whose received state is in
                     // its slot (kChainPoison after a failure); ready[BH] = ticket counter
    float *S_final;  // [BH, dk, dv] state after the last sub-segment, or null
    float *S_save;   // [BH, NP / save_every, dk, dv] received state of every save_every-th
                     // sub-segment, or null
    int save_every;
};

// Single-pass forward (bf16, d = 128, chunk 64): state pass, chained scan and output pass in
// one kernel.  ready and slot 0 of states must be set up by launch_chain_reset.
cudaError_t launch_tc_chain(const PassArgs &a, const ChainArgs &ch, cudaStream_t st);

// Slot 0 of every sequence's chain = S0 (or zeros), ready[bh] = 0, ticket counter = 0.
cudaError_t launch_chain_reset(const float *S0, int BH, int dk, int dv, float *states, int *ready,
                               cudaStream_t st);

// Backward passes for these arguments (tensor-core kernels where they apply, else SIMT).
cudaError_t launch_bwd_dstate(const BwdArgs &a, cudaStream_t st);
cudaError_t launch_bwd_dq(const BwdArgs &a, cudaStream_t st);
cudaError_t launch_bwd_dkv(const BwdArgs &a, cudaStream_t st);

// tcgen05 backward passes (bf16, d = 128, chunk 64).
bool tc_bwd_supported(const BwdArgs &a);
cudaError_t launch_tc_dq(const BwdArgs &a, cudaStream_t st);
cudaError_t launch_tc_dkv(const BwdArgs &a, cudaStream_t st);

// Generic CUDA-core backward passes.
cudaError_t launch_simt_dstate(const BwdArgs &a, cudaStream_t st);
cudaError_t launch_simt_dq(const BwdArgs &a, cudaStream_t st);
cudaError_t launch_simt_dkv(const BwdArgs &a, cudaStream_t st);

// Generic CUDA-core (FFMA) chunk pass: any supported dtype, d and chunk.
cudaError_t launch_simt_pass(const PassArgs &a, PassMode mode, cudaStream_t st);

// tcgen05 / TMEM chunk pass (bf16, d_k = d_v = 128, chunk 64).
bool tc_pass_supported(const PassArgs &a);
cudaError_t launch_tc_pass(const PassArgs &a, PassMode mode, cudaStream_t st);

// The chunk pass for these arguments: the tensor-core kernels where they apply, else SIMT.
cudaError_t launch_pass(const PassArgs &a, PassMode mode, cudaStream_t st);

// The exact token-by-token path (exact.cu) over the units a chunk kernel marked in a.flags:
//  launch_exact_pass      units (bh, j) of a chunk pass: kPassState rewrites S_out and logG,
//                         kPassOutput / kPassCorrect rewrite o from S_init[j] (the whole output),
//                         kPassLocal rewrites o, S_out and logG from zero;
//  launch_exact_sequence  every (b, h) with a marked sub-segment, from S0 over all L tokens: o,
//                         S_final and the state entering every save_every-th sub-segment;
//  launch_exact_dq        segments with a marked fine part: dq, q . dq, S_fine, dSloc, logG;
//  launch_exact_dkv       marked fine parts: dk, dv, dlog_g (needs a.carry).
cudaError_t launch_exact_pass(const PassArgs &a, PassMode mode, cudaStream_t st);
cudaError_t launch_exact_sequence(const PassArgs &a, const float *S0, float *S_final,
                                  float *S_save, int save_every, cudaStream_t st);
cudaError_t launch_exact_dq(const BwdArgs &a, cudaStream_t st);
cudaError_t launch_exact_dkv(const BwdArgs &a, cudaStream_t st);

// Exclusive decayed scan over NP sub-segments (see la_seg_scan in la_seg.h).  With `carry`
// (fp32 [BH, NP, dk]) it also writes the reverse sweep's dlog_g carry of every part p,
// rowsum(S_end_p . out[p]), S_end_p = S_next[p+1] for p < NP-1 and S_last (nullable: zero) for
// the last part.  Without a carry (and for d_k x d_v states of whole 1024-float slices) the
// scan streams the states by bulk copies; a wait there that gives up sets kStatusTimeout in
// *status (nullable).
cudaError_t launch_scan(const float *S_in, const float *log_gamma, const float *init, int BH,
                        int NP, int dk, int dv, int reverse, float *out, float *final_state,
                        cudaStream_t st, const float *S_next = nullptr,
                        const float *S_last = nullptr, float *carry = nullptr,
                        int *status = nullptr);

// Copies the per-sub-segment states at API-segment boundaries: dst[bh][p] = src[bh][p*m].
cudaError_t launch_gather_states(const float *src, int BH, int NP, int m, int dk, int dv,
                                 float *dst, cudaStream_t st);

// dst[bh][p] = src[bh] (or zeros when src is null) for p < P; dst is [BH, P, dk, dv].
cudaError_t launch_broadcast_state(const float *src, int BH, int P, int dk, int dv, float *dst,
                                   cudaStream_t st);

// Record the calling thread's error detail (printf-style) and return s / LA_ERR_CUDA.
la_status set_error(la_status s, const char *fmt, ...);
la_status set_cuda_error(cudaError_t e, const char *what);

// Copies S0 (or zeros) into dst [BH, dk, dv].
cudaError_t launch_copy_state(const float *src, int BH, int dk, int dv, float *dst,
                              cudaStream_t st);

}  // namespace la
