// la_seg_api.cu -- the C ABI of libla_seg.so: argument checks, workspace layout, the
// sub-segment split and the launch sequence of each schedule.  No allocation, no host sync
// (except la_seg_check_status), no C++ exception across the boundary.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <initializer_list>
#include <utility>

#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "la_seg.h"

namespace {

thread_local char g_detail[512] = "no error";

la_status fail(la_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
    va_end(ap);
    return s;
}

la_status cuda_fail(cudaError_t e, const char *what) {
    return fail(LA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Shapes accepted by every entry point.
la_status check_shape(int B, int H, long long L, int dk, int dv, int P, int chunk, la_dtype dt) {
    if (dt != LA_F32 && dt != LA_BF16) return fail(LA_ERR_DTYPE, "unknown la_dtype %d", (int)dt);
    if (B < 1 || H < 1 || P < 1 || L < 0)
        return fail(LA_ERR_SHAPE, "need B, H, P >= 1 and L >= 0 (got B=%d H=%d P=%d L=%lld)", B, H,
                    P, L);
    if (!(dk == 32 || dk == 64 || dk == 128) || dv != dk)
        return fail(LA_ERR_SHAPE, "need dk == dv in {32, 64, 128} (got dk=%d dv=%d)", dk, dv);
    if (!(chunk == 16 || chunk == 32 || chunk == 64))
        return fail(LA_ERR_SHAPE, "chunk must be 16, 32 or 64 (got %d)", chunk);
    if (L % P != 0) return fail(LA_ERR_SHAPE, "L=%lld is not a multiple of P=%d", L, P);
    if ((L / P) % chunk != 0)
        return fail(LA_ERR_SHAPE, "segment length L/P=%lld is not a multiple of chunk=%d", L / P,
                    chunk);
    if ((long long)B * H > (1LL << 24) || L > (1LL << 40))
        return fail(LA_ERR_SHAPE, "sizes out of range");
    return LA_OK;
}

// Internal split of every API segment into m equal sub-segments (the linear-decomposition
// identity makes the result independent of the split).  Chooses the m (a power of two that
// divides the chunks of a segment) with the fewest estimated CTA-waves x chunks per CTA, so
// that small B*H*P still fill the 148 SMs while large ones keep whole segments.
la::Split make_split(int B, int H, long long L, int P, int chunk) {
    la::Split s;
    s.BH = B * H;
    s.P = P;
    s.L = L;
    const long long chunks_per_seg = (L / P) / chunk;
    const long long bhp = (long long)s.BH * P;
    int best_m = 1;
    double best_cost = 1e300;
    for (long long m = 1; chunks_per_seg > 0 && m <= chunks_per_seg; m *= 2) {
        if (chunks_per_seg % m) break;
        const long long ctas = bhp * m;
        const long long waves = (ctas + la::kNumSMs - 1) / la::kNumSMs;
        const double cost = (double)waves * ((double)(chunks_per_seg / m) + 2.0);
        if (cost < best_cost * 0.97) {
            best_cost = cost;
            best_m = (int)m;
        }
    }
    s.m = best_m;
    s.NP = P * best_m;
    s.T = (L / P) / best_m;
    return s;
}

// Both layouts start with the status word and the flag arrays of the exact path, which each
// call clears with one memset of the bytes before S_loc.
struct FwdLayout {
    size_t status, flags, S_loc, logG, S_recv, chain_states, chain_ready, total;
};

FwdLayout fwd_layout(const la::Split &s, int dk, int dv) {
    FwdLayout w;
    const size_t states = (size_t)s.BH * s.NP * dk * dv * sizeof(float);
    const size_t gam = (size_t)s.BH * s.NP * dk * sizeof(float);
    w.status = 0;
    w.flags = 256;  // [BH, NP] sub-segments marked for the exact path
    w.S_loc = align_up(w.flags + (size_t)s.BH * s.NP * sizeof(int), 256);
    w.logG = align_up(w.S_loc + states, 256);
    w.S_recv = align_up(w.logG + gam, 256);
    w.chain_states = align_up(w.S_recv + states, 256);
    w.chain_ready = align_up(w.chain_states + (size_t)s.BH * 2 * dk * dv * sizeof(float), 256);
    w.total = align_up(w.chain_ready + (size_t)(s.BH + 1) * sizeof(int), 256);
    return w;
}

// Fine parts per segment for the backward's reverse sweep: the largest power-of-two split
// into parts of at most kMaxPartTokens tokens (whole chunks).  dlog_g is re-anchored on the
// exact carry rowsum(S_end . dX) at every part boundary, which keeps the rounding of the
// per-token terms it sums from accumulating over long segments.  With the sweeps' shared bf16
// operands the measured dlog_g error is <= 0.67% of max at 1024-token parts, <= 0.86% at 2048
// and <= 1.06% at 4096 (bound 2%); 2048 halves the reverse scan and the part-boundary state
// stores of 1024 and keeps a 2.3x margin.
constexpr long long kMaxPartTokens = 2048;
int fine_factor(long long T, int chunk) {
    int r = 1;
    while (T / r > kMaxPartTokens && T % (2LL * r) == 0 && (T / (2LL * r)) % chunk == 0) r *= 2;
    return r;
}

struct BwdLayout {
    size_t status, flags_s, flags_f, S_loc, logG, S_recv, S_fin, S_fine, dSloc, logG_f, dX, carry,
        qdq, total;
};

BwdLayout bwd_layout(const la::Split &s, int r, int dk, int dv) {
    BwdLayout w;
    const size_t states = (size_t)s.BH * s.NP * dk * dv * sizeof(float);
    const size_t fine_states = states * r;
    const size_t gam = (size_t)s.BH * s.NP * dk * sizeof(float);
    w.status = 0;
    w.flags_s = 256;  // [BH, NP] segments of the recomputed state pass marked for the exact path
    w.flags_f = align_up(w.flags_s + (size_t)s.BH * s.NP * sizeof(int), 256);  // [BH, NP * r] fine parts
    w.S_loc = align_up(w.flags_f + (size_t)s.BH * s.NP * r * sizeof(int), 256);
    w.logG = align_up(w.S_loc + states, 256);
    w.S_recv = align_up(w.logG + gam, 256);
    w.S_fin = align_up(w.S_recv + states, 256);
    w.S_fine = align_up(w.S_fin + (size_t)s.BH * dk * dv * sizeof(float), 256);
    w.dSloc = align_up(w.S_fine + fine_states, 256);
    w.logG_f = align_up(w.dSloc + fine_states, 256);
    w.dX = align_up(w.logG_f + gam * r, 256);
    w.carry = align_up(w.dX + fine_states, 256);
    w.qdq = align_up(w.carry + gam * r, 256);
    w.total = align_up(w.qdq + (size_t)s.BH * s.L * dk * sizeof(float), 256);
    return w;
}

// LA_SCHED_OVERLAP's second stream (highest priority, so that the scan's blocks are placed
// beside the local pass's CTAs as SMs free up) and its fork / join events: one set per host
// thread and device, created on first use and kept for the thread's lifetime.
struct Aux {
    int device = -1;
    cudaStream_t stream = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};

cudaError_t aux_streams(Aux **out) {
    static thread_local Aux per_device[la::kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= la::kMaxDevices) return cudaErrorInvalidDevice;
    Aux &x = per_device[dev];
    if (x.device != dev) {
        int lo = 0, hi = 0;
        if ((e = cudaDeviceGetStreamPriorityRange(&lo, &hi)) != cudaSuccess) return e;
        if ((e = cudaStreamCreateWithPriority(&x.stream, cudaStreamNonBlocking, hi)) != cudaSuccess)
            return e;
        if ((e = cudaEventCreateWithFlags(&x.fork, cudaEventDisableTiming)) != cudaSuccess ||
            (e = cudaEventCreateWithFlags(&x.join, cudaEventDisableTiming)) != cudaSuccess)
            return e;
        x.device = dev;
    }
    *out = &x;
    return cudaSuccess;
}

la::Split whole_segments(const la::Split &s) {
    la::Split w = s;
    w.m = 1;
    w.NP = s.P;
    w.T = s.L / s.P;
    return w;
}

template <typename Ptr>
char *at(Ptr base, size_t off) {
    return static_cast<char *>(const_cast<void *>(static_cast<const void *>(base))) + off;
}

}  // namespace

namespace la {

la_status set_error(la_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
    va_end(ap);
    return s;
}

la_status set_cuda_error(cudaError_t e, const char *what) { return cuda_fail(e, what); }

}  // namespace la

extern "C" {

size_t la_seg_workspace_bytes(int B, int H, long long L, int dk, int dv, int P, int chunk,
                              la_dtype dt, int backward) {
    if (check_shape(B, H, L, dk, dv, P, chunk, dt) != LA_OK) return 0;
    const la::Split s = make_split(B, H, L, P, chunk);
    if (!backward) return fwd_layout(s, dk, dv).total;
    // la_seg_backward keeps whole segments when it reuses saved states
    const la::Split whole = whole_segments(s);
    const size_t a = bwd_layout(s, fine_factor(s.T, chunk), dk, dv).total;
    const size_t b = bwd_layout(whole, fine_factor(whole.T, chunk), dk, dv).total;
    return a > b ? a : b;
}

}  // extern "C"

// ---- per-step entry points ---------------------------------------------------------
namespace {

la_status check_pass(int B, int H, long long L, int dk, int dv, int NP, int chunk, la_dtype dt,
                     std::initializer_list<std::pair<const void *, const char *>> need,
                     std::initializer_list<std::pair<const void *, const char *>> opt) {
    la_status st = check_shape(B, H, L, dk, dv, NP, chunk, dt);
    if (st != LA_OK) return st;
    for (auto &p : need) {
        if (L > 0 && !p.first) return fail(LA_ERR_ARG, "%s must be non-null", p.second);
        if (p.first && !aligned(p.first, 16))
            return fail(LA_ERR_ALIGN, "%s is not 16-byte aligned", p.second);
    }
    for (auto &p : opt)
        if (p.first && !aligned(p.first, 16))
            return fail(LA_ERR_ALIGN, "%s is not 16-byte aligned", p.second);
    return LA_OK;
}

la::PassArgs pass_args(const void *q, const void *k, const void *v, const void *g, void *o,
                       const float *S_init, float *S_out, float *logG, int *status, int B, int H,
                       long long L, int dk, int dv, int NP, int chunk, la_dtype dt) {
    la::PassArgs a = {};
    a.q = q; a.k = k; a.v = v; a.g = g; a.o = o;
    a.S_init = S_init; a.S_out = S_out; a.logG = logG; a.status = status;
    a.L = L; a.T = NP > 0 ? L / NP : 0; a.BH = B * H; a.NP = NP;
    a.dk = dk; a.dv = dv; a.chunk = chunk; a.dt = dt;
    return a;
}

la_status run_pass(const la::PassArgs &a, la::PassMode mode, cudaStream_t st, const char *what) {
    if (a.L == 0) return LA_OK;
    cudaError_t e = la::launch_pass(a, mode, st);
    return e == cudaSuccess ? LA_OK : cuda_fail(e, what);
}

}  // namespace

extern "C" {

la_status la_seg_state_pass(const void *k, const void *v, const void *log_g, int B, int H,
                            long long L, int dk, int dv, int NP, int chunk, la_dtype dt,
                            float *S_loc, float *log_gamma, int *status, void *cuda_stream) {
    la_status st = check_pass(B, H, L, dk, dv, NP, chunk, dt,
                              {{k, "k"}, {v, "v"}, {log_g, "log_g"}, {S_loc, "S_loc"}, {log_gamma, "log_gamma"}}, {});
    if (st != LA_OK) return st;
    return run_pass(pass_args(nullptr, k, v, log_g, nullptr, nullptr, S_loc, log_gamma, status, B,
                              H, L, dk, dv, NP, chunk, dt),
                    la::kPassState, static_cast<cudaStream_t>(cuda_stream), "state pass");
}

la_status la_seg_local_pass(const void *q, const void *k, const void *v, const void *log_g, int B,
                            int H, long long L, int dk, int dv, int NP, int chunk, la_dtype dt,
                            void *o, float *S_loc, float *log_gamma, int *status,
                            void *cuda_stream) {
    la_status st = check_pass(B, H, L, dk, dv, NP, chunk, dt,
                              {{q, "q"}, {k, "k"}, {v, "v"}, {log_g, "log_g"}, {o, "o"}},
                              {{S_loc, "S_loc"}, {log_gamma, "log_gamma"}});
    if (st != LA_OK) return st;
    if (!S_loc != !log_gamma) return fail(LA_ERR_ARG, "S_loc and log_gamma go together");
    return run_pass(pass_args(q, k, v, log_g, o, nullptr, S_loc, log_gamma, status, B, H, L, dk, dv,
                              NP, chunk, dt),
                    la::kPassLocal, static_cast<cudaStream_t>(cuda_stream), "local pass");
}

la_status la_seg_output_pass(const void *q, const void *k, const void *v, const void *log_g,
                             const float *S_recv, int B, int H, long long L, int dk, int dv,
                             int NP, int chunk, la_dtype dt, void *o, int *status,
                             void *cuda_stream) {
    la_status st = check_pass(B, H, L, dk, dv, NP, chunk, dt,
                              {{q, "q"}, {k, "k"}, {v, "v"}, {log_g, "log_g"}, {o, "o"}},
                              {{S_recv, "S_recv"}});
    if (st != LA_OK) return st;
    return run_pass(pass_args(q, k, v, log_g, o, S_recv, nullptr, nullptr, status, B, H, L, dk, dv,
                              NP, chunk, dt),
                    la::kPassOutput, static_cast<cudaStream_t>(cuda_stream), "output pass");
}

la_status la_seg_correct_pass(const void *q, const void *log_g, const float *S_recv, int B, int H,
                              long long L, int dk, int dv, int NP, int chunk, la_dtype dt, void *o,
                              int *status, void *cuda_stream) {
    la_status st = check_pass(B, H, L, dk, dv, NP, chunk, dt,
                              {{q, "q"}, {log_g, "log_g"}, {o, "o"}, {S_recv, "S_recv"}}, {});
    if (st != LA_OK) return st;
    return run_pass(pass_args(q, nullptr, nullptr, log_g, o, S_recv, nullptr, nullptr, status, B,
                              H, L, dk, dv, NP, chunk, dt),
                    la::kPassCorrect, static_cast<cudaStream_t>(cuda_stream), "correction pass");
}

la_status la_seg_dstate_pass(const void *q, const void *dO, const void *log_g, int B, int H,
                             long long L, int dk, int dv, int NP, int chunk, la_dtype dt,
                             float *dSloc, float *log_gamma, int *status, void *cuda_stream) {
    la_status st = check_pass(B, H, L, dk, dv, NP, chunk, dt,
                              {{q, "q"}, {dO, "dO"}, {log_g, "log_g"}, {dSloc, "dSloc"},
                               {log_gamma, "log_gamma"}}, {});
    if (st != LA_OK) return st;
    if (L == 0) return LA_OK;
    la::BwdArgs b = {};
    b.q = q; b.g = log_g; b.dO = dO; b.dSloc = dSloc; b.logG = log_gamma; b.status = status;
    b.fine = 1;
    b.L = L; b.T = L / NP; b.BH = B * H; b.NP = NP; b.dk = dk; b.dv = dv; b.chunk = chunk; b.dt = dt;
    cudaError_t e = la::launch_bwd_dstate(b, static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? LA_OK : cuda_fail(e, "gradient-state pass");
}

la_status la_seg_dq_pass(const void *q, const void *k, const void *v, const void *log_g,
                         const void *dO, const float *S_recv, int B, int H, long long L, int dk,
                         int dv, int NP, int fine, int chunk, la_dtype dt, void *dq, float *qdq,
                         float *S_fine, float *dSloc, float *log_gamma, int *status,
                         void *cuda_stream) {
    la_status st = check_pass(B, H, L, dk, dv, NP, chunk, dt,
                              {{q, "q"}, {k, "k"}, {v, "v"}, {log_g, "log_g"}, {dO, "dO"},
                               {dq, "dq"}, {qdq, "qdq"}},
                              {{S_recv, "S_recv"}, {S_fine, "S_fine"}, {dSloc, "dSloc"},
                               {log_gamma, "log_gamma"}});
    if (st != LA_OK) return st;
    if (!dSloc != !log_gamma) return fail(LA_ERR_ARG, "dSloc and log_gamma go together");
    if (fine < 1 || (L > 0 && ((L / NP) % fine != 0 || ((L / NP) / fine) % chunk != 0)))
        return fail(LA_ERR_SHAPE, "fine=%d must cut each segment into whole chunks", fine);
    if (L == 0) return LA_OK;
    la::BwdArgs b = {};
    b.q = q; b.k = k; b.v = v; b.g = log_g; b.dO = dO; b.dq_out = dq; b.dq_ws = qdq;
    b.S_recv = S_recv; b.S_fine = S_fine; b.dSloc = dSloc; b.logG = log_gamma; b.status = status;
    b.L = L; b.T = L / NP; b.BH = B * H; b.NP = NP; b.dk = dk; b.dv = dv; b.chunk = chunk;
    b.fine = fine; b.dt = dt;
    cudaError_t e = la::launch_bwd_dq(b, static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? LA_OK : cuda_fail(e, "dq pass");
}

la_status la_seg_dkv_pass(const void *q, const void *k, const void *v, const void *log_g,
                          const void *dO, const float *S_recv, const float *S_final,
                          const float *dX, const float *qdq, const float *carry, int B, int H,
                          long long L, int dk, int dv, int NP, int chunk, la_dtype dt, void *dk_,
                          void *dv_, void *dlog_g, int *status, void *cuda_stream) {
    la_status st = check_pass(B, H, L, dk, dv, NP, chunk, dt,
                              {{q, "q"}, {k, "k"}, {v, "v"}, {log_g, "log_g"}, {dO, "dO"},
                               {dX, "dX"}, {qdq, "qdq"}, {dk_, "dk"}, {dv_, "dv"},
                               {dlog_g, "dlog_g"}},
                              {{S_recv, "S_recv"}, {S_final, "S_final"}, {carry, "carry"}});
    if (st != LA_OK) return st;
    if (L == 0) return LA_OK;
    la::BwdArgs b = {};
    b.q = q; b.k = k; b.v = v; b.g = log_g; b.dO = dO;
    b.dk_out = dk_; b.dv_out = dv_; b.dg_out = dlog_g;
    b.S_end_next = S_recv; b.S_fin = S_final; b.dX = dX; b.dq_ws = const_cast<float *>(qdq);
    b.carry = carry;
    b.status = status;
    b.L = L; b.T = L / NP; b.BH = B * H; b.NP = NP; b.dk = dk; b.dv = dv; b.chunk = chunk;
    b.fine = 1; b.dt = dt;
    cudaError_t e = la::launch_bwd_dkv(b, static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? LA_OK : cuda_fail(e, "dkv pass");
}

int la_seg_backward_parts(int B, int H, long long L, int dk, int dv, int P, int chunk,
                          la_dtype dt, int reuse) {
    if (check_shape(B, H, L, dk, dv, P, chunk, dt) != LA_OK) return 0;
    const la::Split base = make_split(B, H, L, P, chunk);
    const la::Split s = reuse ? whole_segments(base) : base;
    return s.NP * fine_factor(s.T, chunk);
}

int la_seg_subsegments(int B, int H, long long L, int dk, int dv, int P, int chunk, la_dtype dt) {
    if (check_shape(B, H, L, dk, dv, P, chunk, dt) != LA_OK) return 0;
    return make_split(B, H, L, P, chunk).NP;
}

la_status la_seg_forward(const void *q, const void *k, const void *v, const void *log_g,
                         const float *S0, int B, int H, long long L, int dk, int dv, int P,
                         int chunk, la_dtype dt, void *o, float *S_final, float *S_recv_save,
                         int schedule, void *workspace, size_t ws_bytes, void *cuda_stream) {
    la_status st = check_shape(B, H, L, dk, dv, P, chunk, dt);
    if (st != LA_OK) return st;
    if (schedule != LA_SCHED_AUTO && schedule != LA_SCHED_TWO_PASS &&
        schedule != LA_SCHED_THREE_PHASE && schedule != LA_SCHED_SINGLE_PASS &&
        schedule != LA_SCHED_OVERLAP)
        return fail(LA_ERR_ARG, "unknown schedule %d", schedule);
    if (L > 0 && (!q || !k || !v || !log_g || !o))
        return fail(LA_ERR_ARG, "q, k, v, log_g and o must be non-null");
    const void *ptrs[] = {q, k, v, log_g, o, S0, S_final, S_recv_save};
    const char *names[] = {"q", "k", "v", "log_g", "o", "S0", "S_final", "S_recv_save"};
    for (int i = 0; i < 8; ++i)
        if (ptrs[i] && !aligned(ptrs[i], 16))
            return fail(LA_ERR_ALIGN, "%s is not 16-byte aligned", names[i]);
    const la::Split s = make_split(B, H, L, P, chunk);
    const FwdLayout w = fwd_layout(s, dk, dv);
    if (!workspace || ws_bytes < w.total)
        return fail(LA_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu%s)", w.total,
                    ws_bytes, workspace ? "" : ", null");
    if (!aligned(workspace, 256)) return fail(LA_ERR_ALIGN, "workspace is not 256-byte aligned");
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    int *status = reinterpret_cast<int *>(at(workspace, w.status));
    int *flags = reinterpret_cast<int *>(at(workspace, w.flags));
    cudaError_t e = cudaMemsetAsync(status, 0, w.S_loc, stream);  // status word and flags
    if (e != cudaSuccess) return cuda_fail(e, "status reset");

    if (L == 0) {
        if (S_final && (e = la::launch_copy_state(S0, s.BH, dk, dv, S_final, stream)) != cudaSuccess)
            return cuda_fail(e, "S_final copy");
        if (S_recv_save &&
            (e = la::launch_broadcast_state(S0, s.BH, P, dk, dv, S_recv_save, stream)) != cudaSuccess)
            return cuda_fail(e, "S_recv_save fill");
        return LA_OK;
    }

    float *S_loc = reinterpret_cast<float *>(at(workspace, w.S_loc));
    float *logG = reinterpret_cast<float *>(at(workspace, w.logG));
    float *S_recv = reinterpret_cast<float *>(at(workspace, w.S_recv));

    // Every chunk pass below marks the sub-segments whose chunks the factorisation cannot hold
    // in `flags`; the exact path then rewrites what those sub-segments produced: their local
    // states before the scan reads them, their outputs after the last pass.
    if (schedule == LA_SCHED_SINGLE_PASS) {  // same sub-segments as the other schedules
        la::PassArgs a = pass_args(q, k, v, log_g, o, nullptr, nullptr, nullptr, status, B, H, L,
                                   dk, dv, s.NP, chunk, dt);
        a.flags = flags;
        if (la::tc_pass_supported(a)) {
            la::ChainArgs ch;
            ch.states = reinterpret_cast<float *>(at(workspace, w.chain_states));
            ch.ready = reinterpret_cast<int *>(at(workspace, w.chain_ready));
            ch.S_final = S_final;
            ch.S_save = S_recv_save;
            ch.save_every = s.m;
            if ((e = la::launch_chain_reset(S0, s.BH, dk, dv, ch.states, ch.ready, stream)) !=
                cudaSuccess)
                return cuda_fail(e, "chain reset");
            if ((e = la::launch_tc_chain(a, ch, stream)) != cudaSuccess)
                return cuda_fail(e, "single pass");
            // a marked sub-segment's state runs on through the chain: its whole sequence again
            if ((e = la::launch_exact_sequence(a, S0, S_final, S_recv_save, s.m, stream)) != cudaSuccess)
                return cuda_fail(e, "exact path (sequences)");
            return LA_OK;
        }
        // other shapes: the two-pass order below (same result)
    }

    la::PassArgs a = pass_args(q, k, v, log_g, o, nullptr, S_loc, logG, status, B, H, L, dk, dv,
                               s.NP, chunk, dt);
    a.flags = flags;
    if (schedule == LA_SCHED_OVERLAP) {
        Aux *aux = nullptr;
        if ((e = aux_streams(&aux)) != cudaSuccess)
            return e == cudaErrorInvalidDevice
                       ? fail(LA_ERR_ARG, "LA_SCHED_OVERLAP: the current device is beyond the %d "
                              "devices this library serves", la::kMaxDevices)
                       : cuda_fail(e, "second stream");
        // 1. local states (state pass) on the caller's stream
        if ((e = la::launch_pass(a, la::kPassState, stream)) != cudaSuccess)
            return cuda_fail(e, "state pass");
        if ((e = la::launch_exact_pass(a, la::kPassState, stream)) != cudaSuccess)
            return cuda_fail(e, "exact path (states)");
        // 2. fork: the scan on the second stream, the local outputs on the caller's
        if ((e = cudaEventRecord(aux->fork, stream)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(aux->stream, aux->fork, 0)) != cudaSuccess)
            return cuda_fail(e, "stream fork");
        if ((e = la::launch_scan(S_loc, logG, S0, s.BH, s.NP, dk, dv, 0, S_recv, S_final,
                                 aux->stream, nullptr, nullptr, nullptr, status)) != cudaSuccess)
            return cuda_fail(e, "state scan");
        if ((e = cudaEventRecord(aux->join, aux->stream)) != cudaSuccess)
            return cuda_fail(e, "stream join");
        la::PassArgs loc = a;
        loc.S_out = nullptr;  // the state pass has them; the scan reads them meanwhile
        loc.logG = nullptr;
        if ((e = la::launch_pass(loc, la::kPassLocal, stream)) != cudaSuccess)
            return cuda_fail(e, "local pass");
        // 3. join, then the q . S_recv correction
        if ((e = cudaStreamWaitEvent(stream, aux->join, 0)) != cudaSuccess)
            return cuda_fail(e, "stream join");
        a.S_init = S_recv;
        if ((e = la::launch_pass(a, la::kPassCorrect, stream)) != cudaSuccess)
            return cuda_fail(e, "correction pass");
        if ((e = la::launch_exact_pass(a, la::kPassCorrect, stream)) != cudaSuccess)
            return cuda_fail(e, "exact path (outputs)");
        if (S_recv_save &&
            (e = la::launch_gather_states(S_recv, s.BH, s.NP, s.m, dk, dv, S_recv_save, stream)) !=
                cudaSuccess)
            return cuda_fail(e, "S_recv_save gather");
        return LA_OK;
    }
    const bool three = schedule == LA_SCHED_THREE_PHASE;
    // 1. per sub-segment: local state from zero (+ intra-chunk outputs for three-phase)
    if ((e = la::launch_pass(a, three ? la::kPassLocal : la::kPassState, stream)) != cudaSuccess)
        return cuda_fail(e, three ? "local pass" : "state pass");
    if ((e = la::launch_exact_pass(a, la::kPassState, stream)) != cudaSuccess)
        return cuda_fail(e, "exact path (states)");
    // 2. exclusive decayed scan across sub-segments
    if ((e = la::launch_scan(S_loc, logG, S0, s.BH, s.NP, dk, dv, 0, S_recv, S_final, stream,
                             nullptr, nullptr, nullptr, status)) !=
        cudaSuccess)
        return cuda_fail(e, "state scan");
    // 3. outputs from the received states (two-pass) or the q . S_recv correction (three-phase)
    a.S_init = S_recv;
    if ((e = la::launch_pass(a, three ? la::kPassCorrect : la::kPassOutput, stream)) != cudaSuccess)
        return cuda_fail(e, three ? "correction pass" : "output pass");
    if ((e = la::launch_exact_pass(a, la::kPassOutput, stream)) != cudaSuccess)
        return cuda_fail(e, "exact path (outputs)");
    if (S_recv_save &&
        (e = la::launch_gather_states(S_recv, s.BH, s.NP, s.m, dk, dv, S_recv_save, stream)) !=
            cudaSuccess)
        return cuda_fail(e, "S_recv_save gather");
    return LA_OK;
}

la_status la_seg_chain_reset(const float *S0, int B, int H, int dk, int dv, float *chain_states,
                             int *chain_ready, void *cuda_stream) {
    if (B < 1 || H < 1 || !(dk == 32 || dk == 64 || dk == 128) || dv != dk)
        return fail(LA_ERR_SHAPE, "need B, H >= 1 and dk == dv in {32, 64, 128}");
    if (!chain_states || !chain_ready)
        return fail(LA_ERR_ARG, "chain_states and chain_ready must be non-null");
    if (!aligned(chain_states, 16) || !aligned(chain_ready, 16) || (S0 && !aligned(S0, 16)))
        return fail(LA_ERR_ALIGN, "S0, chain_states and chain_ready must be 16-byte aligned");
    cudaError_t e = la::launch_chain_reset(S0, B * H, dk, dv, chain_states, chain_ready,
                                           static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? LA_OK : cuda_fail(e, "chain reset");
}

la_status la_seg_chain_pass(const void *q, const void *k, const void *v, const void *log_g, int B,
                            int H, long long L, int dk, int dv, int NP, int chunk, la_dtype dt,
                            float *chain_states, int *chain_ready, void *o, float *S_final,
                            float *S_recv_save, int save_every, int *status, void *cuda_stream) {
    la_status st = check_pass(B, H, L, dk, dv, NP, chunk, dt,
                              {{q, "q"}, {k, "k"}, {v, "v"}, {log_g, "log_g"}, {o, "o"},
                               {chain_states, "chain_states"}, {chain_ready, "chain_ready"}},
                              {{S_final, "S_final"}, {S_recv_save, "S_recv_save"}});
    if (st != LA_OK) return st;
    if (save_every < 1 || NP % save_every != 0)
        return fail(LA_ERR_ARG, "save_every=%d must divide NP=%d", save_every, NP);
    la::PassArgs a = pass_args(q, k, v, log_g, o, nullptr, nullptr, nullptr, status, B, H, L, dk,
                               dv, NP, chunk, dt);
    if (!la::tc_pass_supported(a))
        return fail(LA_ERR_SHAPE, "the single pass needs bf16, dk = dv = 128 and chunk = 64");
    if (L == 0) return LA_OK;
    la::ChainArgs ch;
    ch.states = chain_states;
    ch.ready = chain_ready;
    ch.S_final = S_final;
    ch.S_save = S_recv_save;
    ch.save_every = save_every;
    cudaError_t e = la::launch_tc_chain(a, ch, static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? LA_OK : cuda_fail(e, "single pass");
}

la_status la_seg_backward(const void *q, const void *k, const void *v, const void *log_g,
                          const float *S0, const float *S_recv_saved, const void *dO,
                          const float *dS_final, int B, int H, long long L, int dk, int dv, int P,
                          int chunk, la_dtype dt, void *dq, void *dk_, void *dv_, void *dlog_g,
                          float *dS0, void *workspace, size_t ws_bytes, void *cuda_stream) {
    la_status st = check_shape(B, H, L, dk, dv, P, chunk, dt);
    if (st != LA_OK) return st;
    if (L > 0 && (!q || !k || !v || !log_g || !dO || !dq || !dk_ || !dv_ || !dlog_g))
        return fail(LA_ERR_ARG, "q, k, v, log_g, dO, dq, dk, dv and dlog_g must be non-null");
    const void *ptrs[] = {q, k, v, log_g, dO, dq, dk_, dv_, dlog_g, S0, S_recv_saved, dS_final, dS0};
    const char *names[] = {"q", "k", "v", "log_g", "dO", "dq", "dk", "dv", "dlog_g", "S0",
                           "S_recv_saved", "dS_final", "dS0"};
    for (int i = 0; i < 13; ++i)
        if (ptrs[i] && !aligned(ptrs[i], 16))
            return fail(LA_ERR_ALIGN, "%s is not 16-byte aligned", names[i]);
    // Saved states are per API segment: when they can be reused (S_final not needed), the dq
    // sweep keeps whole segments so that every segment's received state is one the forward saved.
    const bool reuse = S_recv_saved && !dS_final;
    const la::Split base = make_split(B, H, L, P, chunk);
    const la::Split s = reuse ? whole_segments(base) : base;
    const int r = fine_factor(s.T, chunk);
    const BwdLayout w = bwd_layout(s, r, dk, dv);
    const size_t need = la_seg_workspace_bytes(B, H, L, dk, dv, P, chunk, dt, 1);
    if (!workspace || ws_bytes < need)
        return fail(LA_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu%s)", need,
                    ws_bytes, workspace ? "" : ", null");
    if (!aligned(workspace, 256)) return fail(LA_ERR_ALIGN, "workspace is not 256-byte aligned");
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    int *status = reinterpret_cast<int *>(at(workspace, w.status));
    int *flags_s = reinterpret_cast<int *>(at(workspace, w.flags_s));
    int *flags_f = reinterpret_cast<int *>(at(workspace, w.flags_f));
    cudaError_t e = cudaMemsetAsync(status, 0, w.S_loc, stream);  // status word and flags
    if (e != cudaSuccess) return cuda_fail(e, "status reset");
    if (L == 0) {  // no tokens: S_final = S0, so dS0 = dS_final
        if (dS0 && (e = la::launch_copy_state(dS_final, s.BH, dk, dv, dS0, stream)) != cudaSuccess)
            return cuda_fail(e, "dS0 copy");
        return LA_OK;
    }
    float *S_loc = reinterpret_cast<float *>(at(workspace, w.S_loc));
    float *logG = reinterpret_cast<float *>(at(workspace, w.logG));
    float *S_recv = reinterpret_cast<float *>(at(workspace, w.S_recv));
    float *S_fin = reinterpret_cast<float *>(at(workspace, w.S_fin));
    float *S_fine = reinterpret_cast<float *>(at(workspace, w.S_fine));
    float *dSloc = reinterpret_cast<float *>(at(workspace, w.dSloc));
    float *logG_f = reinterpret_cast<float *>(at(workspace, w.logG_f));
    float *dX = reinterpret_cast<float *>(at(workspace, w.dX));
    float *carry = reinterpret_cast<float *>(at(workspace, w.carry));
    float *qdq = reinterpret_cast<float *>(at(workspace, w.qdq));

    // 1. the states each segment receives: the forward's when given and S_final is not needed
    //    (dS_final = 0); otherwise recomputed (state pass + scan)
    const float *recv = reuse ? S_recv_saved : S_recv;
    if (!reuse) {
        la::PassArgs a = pass_args(nullptr, k, v, log_g, nullptr, nullptr, S_loc, logG, status, B,
                                   H, L, dk, dv, s.NP, chunk, dt);
        a.flags = flags_s;
        if ((e = la::launch_pass(a, la::kPassState, stream)) != cudaSuccess)
            return cuda_fail(e, "backward state pass");
        if ((e = la::launch_exact_pass(a, la::kPassState, stream)) != cudaSuccess)
            return cuda_fail(e, "exact path (states)");
        if ((e = la::launch_scan(S_loc, logG, S0, s.BH, s.NP, dk, dv, 0, S_recv, S_fin, stream,
                                 nullptr, nullptr, nullptr, status)) !=
            cudaSuccess)
            return cuda_fail(e, "backward state scan");
    }
    la::BwdArgs b = {};
    b.q = q; b.k = k; b.v = v; b.g = log_g; b.dO = dO;
    b.dq_out = dq; b.dk_out = dk_; b.dv_out = dv_; b.dg_out = dlog_g;
    b.S_recv = recv; b.S_fine = S_fine; b.S_end_next = S_fine; b.S_fin = reuse ? nullptr : S_fin;
    b.dX = dX; b.dq_ws = qdq; b.dSloc = dSloc; b.logG = logG_f; b.status = status;
    b.flags = flags_f;  // fine parts whose chunks the factorisation cannot hold: the exact path
    b.L = L; b.BH = s.BH; b.dk = dk; b.dv = dv; b.chunk = chunk; b.dt = dt;
    // 2. dq sweep over the segments; records the state entering each of their r fine parts,
    //    and forms every fine part's gradient state and log-decay sum
    b.NP = s.NP; b.T = s.T; b.fine = r;
    if ((e = la::launch_bwd_dq(b, stream)) != cudaSuccess) return cuda_fail(e, "dq pass");
    if ((e = la::launch_exact_dq(b, stream)) != cudaSuccess) return cuda_fail(e, "exact path (dq)");
    // 3-4 run over the fine parts
    b.NP = s.NP * r; b.T = s.T / r; b.fine = 1;
    // 3. reverse exclusive decayed scan: gradient of every part's end state, dS0, and each
    //    part's dlog_g carry rowsum(S_end . dX) (S_end: the state entering the next part)
    if ((e = la::launch_scan(dSloc, logG_f, dS_final, s.BH, b.NP, dk, dv, 1, dX, dS0, stream,
                             S_fine, b.S_fin, carry)) != cudaSuccess)
        return cuda_fail(e, "reverse state scan");
    b.carry = carry;
    // 4. dk, dv, dlog_g per part
    if ((e = la::launch_bwd_dkv(b, stream)) != cudaSuccess) return cuda_fail(e, "dkv pass");
    if ((e = la::launch_exact_dkv(b, stream)) != cudaSuccess) return cuda_fail(e, "exact path (dkv)");
    return LA_OK;
}

la_status la_seg_scan(const float *S_in, const float *log_gamma, const float *init, int BH,
                      int NP, int dk, int dv, int reverse, float *out, float *final_state,
                      const float *S_next, const float *S_last, float *carry, int *status,
                      void *cuda_stream) {
    if (BH < 0 || NP < 0 || dk < 1 || dv < 4 || dv % 4)
        return fail(LA_ERR_SHAPE, "need BH, NP >= 0, dk >= 1, dv a positive multiple of 4");
    if ((long long)BH * NP > 0 && (!S_in || !log_gamma || !out))
        return fail(LA_ERR_ARG, "S_in, log_gamma and out must be non-null");
    const void *ptrs[] = {S_in, init, out, final_state};
    const char *names[] = {"S_in", "init", "out", "final_state"};
    for (int i = 0; i < 4; ++i)
        if (ptrs[i] && !aligned(ptrs[i], 16))
            return fail(LA_ERR_ALIGN, "%s is not 16-byte aligned", names[i]);
    if (log_gamma && !aligned(log_gamma, 4)) return fail(LA_ERR_ALIGN, "log_gamma misaligned");
    if (S_in && out == S_in) return fail(LA_ERR_ARG, "out may not alias S_in");
    if (carry) {
        if (32 % (dv / 4) || (dk * (dv / 4)) % 32)
            return fail(LA_ERR_SHAPE, "carry needs dv / 4 to divide 32 (got dv=%d)", dv);
        if ((long long)BH * NP > 0 && !S_next)
            return fail(LA_ERR_ARG, "S_next must be non-null with carry");
        const void *cp[] = {S_next, S_last};
        for (const void *q : cp)
            if (q && !aligned(q, 16)) return fail(LA_ERR_ALIGN, "S_next / S_last misaligned");
        if (!aligned(carry, 4)) return fail(LA_ERR_ALIGN, "carry misaligned");
    }
    cudaError_t e = la::launch_scan(S_in, log_gamma, init, BH, NP, dk, dv, reverse, out,
                                    final_state, static_cast<cudaStream_t>(cuda_stream), S_next,
                                    S_last, carry, status);
    return e == cudaSuccess ? LA_OK : cuda_fail(e, "scan");
}

int la_seg_train_saved_states(int B, int H, long long L, int dk, int dv, int P, int chunk,
                              la_dtype dt) {
    return la_seg_subsegments(B, H, L, dk, dv, P, chunk, dt);
}

// The training pair saves and reuses the states at the library's own split: the same kernels and
// results as la_seg_forward / la_seg_backward called with P = la_seg_subsegments(P) (the result
// does not depend on P, and for that P the library keeps the same sub-segments), so the
// backward's dq sweep runs one CTA per sub-segment rather than per API segment.
la_status la_seg_train_forward(const void *q, const void *k, const void *v, const void *log_g,
                               const float *S0, int B, int H, long long L, int dk, int dv, int P,
                               int chunk, la_dtype dt, void *o, float *S_final, float *saved,
                               int schedule, void *workspace, size_t ws_bytes, void *cuda_stream) {
    const int NS = la_seg_subsegments(B, H, L, dk, dv, P, chunk, dt);
    if (NS == 0)  // rejected sizes: the regular entry point names the reason
        return la_seg_forward(q, k, v, log_g, S0, B, H, L, dk, dv, P, chunk, dt, o, S_final, saved,
                              schedule, workspace, ws_bytes, cuda_stream);
    return la_seg_forward(q, k, v, log_g, S0, B, H, L, dk, dv, NS, chunk, dt, o, S_final, saved,
                          schedule, workspace, ws_bytes, cuda_stream);
}

la_status la_seg_train_backward(const void *q, const void *k, const void *v, const void *log_g,
                                const float *S0, const float *saved, const void *dO,
                                const float *dS_final, int B, int H, long long L, int dk, int dv,
                                int P, int chunk, la_dtype dt, void *dq, void *dk_, void *dv_,
                                void *dlog_g, float *dS0, void *workspace, size_t ws_bytes,
                                void *cuda_stream) {
    const int NS = la_seg_subsegments(B, H, L, dk, dv, P, chunk, dt);
    return la_seg_backward(q, k, v, log_g, S0, saved, dO, dS_final, B, H, L, dk, dv,
                           NS == 0 ? P : NS, chunk, dt, dq, dk_, dv_, dlog_g, dS0, workspace,
                           ws_bytes, cuda_stream);
}

size_t la_seg_train_workspace_bytes(int B, int H, long long L, int dk, int dv, int P, int chunk,
                                    la_dtype dt, int backward) {
    const int NS = la_seg_subsegments(B, H, L, dk, dv, P, chunk, dt);
    return NS == 0 ? 0 : la_seg_workspace_bytes(B, H, L, dk, dv, NS, chunk, dt, backward);
}

la_status la_seg_gather_states(const float *src, int BH, int NP, int m, int dk, int dv, float *dst,
                               void *cuda_stream) {
    if (BH < 0 || NP < 0 || m < 1 || (NP % m) != 0 || dk < 1 || dv < 4 || dv % 4)
        return fail(LA_ERR_SHAPE, "need BH, NP >= 0, m >= 1 dividing NP, dk >= 1, dv a multiple of 4");
    if ((long long)BH * NP > 0 && (!src || !dst))
        return fail(LA_ERR_ARG, "src and dst must be non-null");
    if ((src && !aligned(src, 16)) || (dst && !aligned(dst, 16)))
        return fail(LA_ERR_ALIGN, "src and dst must be 16-byte aligned");
    cudaError_t e = la::launch_gather_states(src, BH, NP, m, dk, dv, dst,
                                             static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? LA_OK : cuda_fail(e, "state gather");
}

la_status la_seg_check_status(void *workspace, void *cuda_stream) {
    if (!workspace) return fail(LA_ERR_ARG, "workspace is null");
    int h = 0;
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    cudaError_t e = cudaMemcpyAsync(&h, workspace, sizeof(int), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e, "status read");
    if (h & la::kStatusTimeout) return fail(LA_ERR_TIMEOUT, "a device-side wait gave up");
    if (h & la::kStatusGateRange)
        return fail(LA_ERR_GATE_RANGE,
                    "some chunk has a positive log_g or |sum of log_g| > %.0f in a key dimension; "
                    "la_seg_forward / la_seg_backward compute such chunks exactly",
                    (double)la::kGateRangeLimit);
    return LA_OK;
}

la_status la_last_error_detail(char *buf, size_t n) {
    if (!buf || n == 0) return LA_ERR_ARG;
    strncpy(buf, g_detail, n - 1);
    buf[n - 1] = '\0';
    return LA_OK;
}

}  // extern "C"
