"""Pins of the fp64 oracle against things other than itself.

Each pin checks the oracle (any ``oracle.Oracle`` instance, so that deliberately broken
copies can be run through the same checks) against a fact fixed by the mathematics or by
the ZeCO pages, never against a retyped copy of its own loop:

* ``brute_force``   -- the quadratic masked-decay form with a global cumulative log-gate,
                       evaluated as one dense einsum (GLA's parallel form).
* ``no_gate``       -- log_g = 0 is plain causal linear attention: S_t = S0 + cumsum of k^T v.
* ``zero_gate``     -- a = 0 forgets everything: o_t = (q_t . k_t) v_t.
* ``closed_form``   -- d_k = d_v = 1, constant gate, k = v = 1: geometric series.
* ``segmented``     -- the linear-decomposition identity of the ZeCO review ("key
                       machinery"): per-segment local states from zero, the exclusive decayed
                       scan S_recv_p = Gamma_{p-1} S_recv_{p-1} + S_{p-1} and the correction
                       o += (q . exp(B_seg)) S_recv reproduce the unsegmented result, for
                       several P and chunk sizes (a separate chunkwise restatement).
* ``propagation``   -- P >= 3: the state segment 2 receives carries Gamma_1 Gamma_0 S0 +
                       Gamma_1 S_0 + S_1 (the accumulated state is forwarded, not only the
                       local one; the ZeCO review's referee flags Alg. 2 for exactly this).
* ``seg_backward``  -- a chunked, segmented restatement of the backward (per-segment gradient
                       states, a reverse exclusive decayed scan, forward and reverse chunk
                       sweeps, dlog_g from a chunk-local suffix sum plus the carry
                       rowsum(S_end . dX)) reproduces the oracle's gradients.
* ``finite_diff``   -- the backward equals central finite differences of the forward.
* ``dg_identity``   -- dlog_g_t = sum_{s>=t} (q_s . dq_s - k_s . dk_s) + rowsum(dS_final . S_final).
"""
from __future__ import annotations

import numpy as np


def rand_case(seed, B=1, H=2, L=24, dk=4, dv=3, gate=0.3, s0=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, L, dk))
    k = rng.standard_normal((B, H, L, dk))
    v = rng.standard_normal((B, H, L, dv))
    g = -gate * np.abs(rng.standard_normal((B, H, L, dk)))  # log of gates in (0, 1]
    S0 = rng.standard_normal((B, H, dk, dv)) if s0 else None
    return q, k, v, g, S0


def rel_err(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.max(np.abs(b))
    return float(np.max(np.abs(a - b)) / (den if den > 0 else 1.0))


# --------------------------------------------------------------------------- references
def brute_force(q, k, v, g, S0):
    """o_t = sum_{s<=t} sum_i q_ti k_si e^{B_ti - B_si} v_s + (q_t e^{B_t}) S0, B global cumsum."""
    Bc = np.cumsum(g, axis=2)
    L = q.shape[2]
    W = np.exp(Bc[:, :, :, None, :] - Bc[:, :, None, :, :])            # [b,h,t,s,i]
    A = np.einsum("bhti,bhsi,bhtsi->bhts", q, k, W) * np.tril(np.ones((L, L)))
    o = A @ v
    Sf = np.einsum("bhsi,bhsj->bhij", k * np.exp(Bc[:, :, -1:, :] - Bc), v)
    if S0 is not None:
        o = o + np.einsum("bhti,bhij->bhtj", q * np.exp(Bc), S0)
        Sf = Sf + np.exp(Bc[:, :, -1, :])[..., None] * S0
    return o, Sf


def chunked_segment_local(q, k, v, g, C):
    """One segment from a zero state, chunk by chunk (GLA chunkwise form): returns o_local,
    the local state and the segment's log-decay sum.  Shapes [T, d]."""
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv))
    o = np.zeros((T, dv))
    for c0 in range(0, T, C):
        qc, kc, vc, gc = q[c0:c0 + C], k[c0:c0 + C], v[c0:c0 + C], g[c0:c0 + C]
        b = np.cumsum(gc, axis=0)
        bC = b[-1]
        Qb = qc * np.exp(b)
        Kb = kc * np.exp(-b)
        intra = np.tril(Qb @ Kb.T) @ vc
        o[c0:c0 + C] = intra + Qb @ S
        S = np.exp(bC)[:, None] * S + (kc * np.exp(bC - b)).T @ vc
    return o, S, g.sum(axis=0)


def segmented(q, k, v, g, S0, P, C):
    """Segments -> local pass -> exclusive decayed scan -> correction (fp64)."""
    Bn, H, L, dk = q.shape
    dv = v.shape[-1]
    T = L // P
    o = np.zeros((Bn, H, L, dv))
    Sf = np.zeros((Bn, H, dk, dv))
    S_recv_all = np.zeros((Bn, H, P, dk, dv))
    for b in range(Bn):
        for h in range(H):
            S_loc, logG, o_loc = [], [], []
            for p in range(P):
                sl = slice(p * T, (p + 1) * T)
                ol, Sl, lg = chunked_segment_local(q[b, h, sl], k[b, h, sl], v[b, h, sl],
                                                   g[b, h, sl], C)
                S_loc.append(Sl)
                logG.append(lg)
                o_loc.append(ol)
            S_recv = np.zeros((dk, dv)) if S0 is None else S0[b, h].copy()
            for p in range(P):
                sl = slice(p * T, (p + 1) * T)
                Bseg = np.cumsum(g[b, h, sl], axis=0)
                o[b, h, sl] = o_loc[p] + (q[b, h, sl] * np.exp(Bseg)) @ S_recv
                S_recv_all[b, h, p] = S_recv
                S_recv = np.exp(logG[p])[:, None] * S_recv + S_loc[p]
            Sf[b, h] = S_recv
    return o, Sf, S_recv_all


def segmented_backward(q, k, v, g, dO, S0, dSf, P, C):
    """Gradients of loss = <o, dO> + <S_final, dSf> by segments and chunks (fp64)."""
    Bn, H, L, dk = q.shape
    dv = v.shape[-1]
    T = L // P
    out = [np.zeros_like(q), np.zeros_like(k), np.zeros_like(v), np.zeros_like(g)]
    dS0 = np.zeros((Bn, H, dk, dv))
    for b in range(Bn):
        for h in range(H):
            qq, kk, vv, gg, dd = q[b, h], k[b, h], v[b, h], g[b, h], dO[b, h]
            # forward: local states, decays, received states, final state
            S_loc, logG = [], []
            for p in range(P):
                sl = slice(p * T, (p + 1) * T)
                _, Sl, lg = chunked_segment_local(qq[sl], kk[sl], vv[sl], gg[sl], C)
                S_loc.append(Sl)
                logG.append(lg)
            S_recv = [np.zeros((dk, dv)) if S0 is None else S0[b, h].copy()]
            for p in range(P):
                S_recv.append(np.exp(logG[p])[:, None] * S_recv[p] + S_loc[p])
            # per-segment gradient states dSloc_p = sum_t diag(e^{B_t}) q_t^T dO_t
            dSloc = []
            for p in range(P):
                sl = slice(p * T, (p + 1) * T)
                Bseg = np.cumsum(gg[sl], axis=0)
                dSloc.append((qq[sl] * np.exp(Bseg)).T @ dd[sl])
            # reverse exclusive scan: dX_p = d loss / d S_end_p
            dX = [None] * P
            acc = np.zeros((dk, dv)) if dSf is None else dSf[b, h].copy()
            for p in range(P - 1, -1, -1):
                dX[p] = acc
                acc = np.exp(logG[p])[:, None] * acc + dSloc[p]
            dS0[b, h] = acc
            for p in range(P):
                sl = slice(p * T, (p + 1) * T)
                qs, ks, vs, gs, ds = qq[sl], kk[sl], vv[sl], gg[sl], dd[sl]
                dq = np.zeros_like(qs)
                S = S_recv[p].copy()
                for c0 in range(0, T, C):  # forward sweep: dq
                    cs = slice(c0, c0 + C)
                    bt = np.cumsum(gs[cs], axis=0)
                    bC = bt[-1]
                    Sp = np.exp(bC)[:, None] * S
                    Kt = ks[cs] * np.exp(bC - bt)
                    M = np.tril(ds[cs] @ vs[cs].T)
                    dq[cs] = np.exp(bt - bC) * (ds[cs] @ Sp.T + M @ Kt)
                    S = Sp + Kt.T @ vs[cs]
                dk_ = np.zeros_like(ks)
                dv_ = np.zeros_like(vs)
                dgs = np.zeros_like(gs)
                dS = dX[p].copy()
                acc_g = np.sum(S_recv[p + 1] * dX[p], axis=1)  # carry: rowsum(S_end . dX)
                for c0 in reversed(range(0, T, C)):  # reverse sweep: dk, dv, dlog_g
                    cs = slice(c0, c0 + C)
                    bt = np.cumsum(gs[cs], axis=0)
                    bC = bt[-1]
                    Qb = qs[cs] * np.exp(bt - bC)
                    Kt = ks[cs] * np.exp(bC - bt)
                    M = np.tril(ds[cs] @ vs[cs].T)
                    A = np.tril(Qb @ Kt.T)
                    dk_[cs] = np.exp(bC - bt) * (M.T @ Qb + vs[cs] @ dS.T)
                    dv_[cs] = A.T @ ds[cs] + Kt @ dS
                    contrib = qs[cs] * dq[cs] - ks[cs] * dk_[cs]
                    suffix = np.flip(np.cumsum(np.flip(contrib, 0), 0), 0)
                    dgs[cs] = suffix + acc_g
                    acc_g = acc_g + contrib.sum(axis=0)
                    dS = np.exp(bC)[:, None] * (dS + Qb.T @ ds[cs])
                out[0][b, h, sl], out[1][b, h, sl], out[2][b, h, sl], out[3][b, h, sl] = dq, dk_, dv_, dgs
    return out[0], out[1], out[2], out[3], dS0


# --------------------------------------------------------------------------- pins
def pin_brute_force(orc, tol=1e-12):
    worst = 0.0
    for seed, (L, dk, dv) in enumerate([(1, 1, 1), (7, 3, 2), (33, 8, 5), (64, 8, 8)]):
        q, k, v, g, S0 = rand_case(100 + seed, L=L, dk=dk, dv=dv)
        o, Sf, _ = orc.forward(q, k, v, g, S0)
        o_ref, Sf_ref = brute_force(q, k, v, g, S0)
        worst = max(worst, rel_err(o, o_ref), rel_err(Sf, Sf_ref))
    return worst <= tol, worst


def pin_no_gate(orc, tol=1e-12):
    q, k, v, g, S0 = rand_case(7, L=40, dk=5, dv=6)
    g = np.zeros_like(g)
    o, Sf, _ = orc.forward(q, k, v, g, S0)
    S_t = S0[:, :, None] + np.cumsum(k[..., :, None] * v[..., None, :], axis=2)  # [b,h,t,i,j]
    o_ref = np.einsum("bhti,bhtij->bhtj", q, S_t)
    err = max(rel_err(o, o_ref), rel_err(Sf, S_t[:, :, -1]))
    return err <= tol, err


def pin_zero_gate(orc, tol=1e-12):
    q, k, v, g, S0 = rand_case(8, L=20, dk=4, dv=4)
    g = np.full_like(g, -1.0e4)  # exp underflows to exactly 0
    o, Sf, _ = orc.forward(q, k, v, g, S0)
    o_ref = np.sum(q * k, axis=-1, keepdims=True) * v
    Sf_ref = k[:, :, -1, :, None] * v[:, :, -1, None, :]
    err = max(rel_err(o, o_ref), rel_err(Sf, Sf_ref))
    return err <= tol, err


def pin_closed_form(orc, tol=1e-12):
    L, a, s0 = 50, 0.9, 0.7
    q = np.linspace(-1.0, 1.0, L).reshape(1, 1, L, 1)
    ones = np.ones((1, 1, L, 1))
    g = np.full((1, 1, L, 1), np.log(a))
    o, Sf, _ = orc.forward(q, ones, ones, g, np.full((1, 1, 1, 1), s0))
    t = np.arange(L).reshape(1, 1, L, 1)
    s_t = a ** (t + 1) * s0 + (1 - a ** (t + 1)) / (1 - a)
    err = max(rel_err(o, q * s_t), rel_err(Sf, s_t[:, :, -1:, :]))
    return err <= tol, err


def pin_segmented(orc, tol=1e-12):
    worst = 0.0
    for seed, (L, P, C, s0) in enumerate([(64, 4, 16, True), (96, 3, 8, False), (128, 8, 4, True),
                                          (64, 1, 64, True)]):
        q, k, v, g, S0 = rand_case(200 + seed, L=L, dk=6, dv=5, s0=s0)
        o, Sf, S_seg = orc.forward(q, k, v, g, S0, seg_len=L // P)
        o_ref, Sf_ref, S_recv_ref = segmented(q, k, v, g, S0, P, C)
        worst = max(worst, rel_err(o, o_ref), rel_err(Sf, Sf_ref), rel_err(S_seg, S_recv_ref))
    return worst <= tol, worst


def pin_propagation(orc, tol=1e-12):
    L, P = 48, 4
    T = L // P
    q, k, v, g, S0 = rand_case(9, L=L, dk=4, dv=3, gate=0.05)
    _, _, S_seg = orc.forward(q, k, v, g, S0, seg_len=T)
    S_loc, Gam = [], []
    for p in range(P):
        sl = slice(p * T, (p + 1) * T)
        _, Sl, _ = orc.forward(q[:, :, sl], k[:, :, sl], v[:, :, sl], g[:, :, sl], None)
        S_loc.append(Sl)
        Gam.append(np.exp(g[:, :, sl].sum(axis=2))[..., None])
    expect2 = Gam[1] * Gam[0] * S0 + Gam[1] * S_loc[0] + S_loc[1]
    err = rel_err(S_seg[:, :, 2], expect2)
    # forwarding only the local state (S_recv_2 = S_loc_1) must be visibly different here
    distinct = rel_err(S_loc[1], expect2) > 1e-3
    return (err <= tol and distinct), err


def pin_seg_backward(orc, tol=1e-11):
    worst = 0.0
    for seed, (L, P, C, s0, dsf) in enumerate([(64, 4, 8, True, True), (96, 3, 16, False, False),
                                               (48, 1, 16, True, False), (128, 8, 4, False, True)]):
        q, k, v, g, S0 = rand_case(300 + seed, L=L, dk=5, dv=4, s0=s0)
        rng = np.random.default_rng(400 + seed)
        dO = rng.standard_normal(v.shape)
        dSf = rng.standard_normal((q.shape[0], q.shape[1], 5, 4)) if dsf else None
        ref = orc.backward(q, k, v, g, dO, S0, dSf)
        got = segmented_backward(q, k, v, g, dO, S0, dSf, P, C)
        worst = max(worst, *(rel_err(a, b) for a, b in zip(got, ref)))
    return worst <= tol, worst


def _loss(orc, q, k, v, g, S0, dO, dSf):
    o, Sf, _ = orc.forward(q, k, v, g, S0)
    return float(np.sum(o * dO) + np.sum(Sf * dSf))


def pin_finite_diff(orc, tol=1e-7, h=1e-6):
    q, k, v, g, S0 = rand_case(11, B=1, H=1, L=12, dk=3, dv=2)
    rng = np.random.default_rng(12)
    dO = rng.standard_normal((1, 1, 12, 2))
    dSf = rng.standard_normal((1, 1, 3, 2))
    grads = orc.backward(q, k, v, g, dO, S0, dSf)
    inputs = [q, k, v, g, S0]
    worst = 0.0
    for x, gx in zip(inputs, grads):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            lp = _loss(orc, *inputs, dO, dSf)
            x[idx] = old - h
            lm = _loss(orc, *inputs, dO, dSf)
            x[idx] = old
            fd[idx] = (lp - lm) / (2 * h)
        worst = max(worst, rel_err(gx, fd))
    return worst <= tol, worst


def pin_dg_identity(orc, tol=1e-11):
    worst = 0.0
    for seed, with_dsf in [(13, False), (14, True)]:
        q, k, v, g, S0 = rand_case(seed, L=30, dk=4, dv=5)
        rng = np.random.default_rng(seed + 50)
        dO = rng.standard_normal(v.shape)
        dSf = rng.standard_normal(S0.shape) if with_dsf else None
        dq, dk, dv, dg, _ = orc.backward(q, k, v, g, dO, S0, dSf)
        contrib = q * dq - k * dk
        ref = np.flip(np.cumsum(np.flip(contrib, axis=2), axis=2), axis=2)
        if with_dsf:
            _, Sf, _ = orc.forward(q, k, v, g, S0)
            ref = ref + np.sum(dSf * Sf, axis=-1)[:, :, None, :]
        worst = max(worst, rel_err(dg, ref))
    return worst <= tol, worst


ALL_PINS = {
    "brute_force": pin_brute_force,
    "no_gate": pin_no_gate,
    "zero_gate": pin_zero_gate,
    "closed_form": pin_closed_form,
    "segmented": pin_segmented,
    "propagation": pin_propagation,
    "seg_backward": pin_seg_backward,
    "finite_diff": pin_finite_diff,
    "dg_identity": pin_dg_identity,
}


def run_all(orc):
    return {name: fn(orc) for name, fn in ALL_PINS.items()}
