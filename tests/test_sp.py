"""Sequence parallelism across ranks (sp.py) on gloo ranks on the CPU.

The orchestration -- the split into sub-segments, each rank's reduction to one (log Gamma, S)
pair, the All-Scan across ranks (all-gather + scan, and the tree of point-to-point rounds), the
local scans with S0 / dS_final and the dlog_g carries at block ends -- runs unchanged on 2, 3
and 4 gloo ranks.  Its per-step calls are served by OracleSteps, which computes each step from
the fp64 oracle on that step's tokens (the chunk passes) or from the step's definition (the
scans), so the test checks how sp.py composes the steps: every rank's outputs and gradients,
put together, must equal the oracle on the whole sequence.  The GPU version of this test, with
the library's kernels, is tests/test_gpu_sp.py.
"""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from tests.parity import rel_err

NAMES = ("dq", "dk", "dv", "dlog_g")


def t64(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64))


class OracleSteps:
    """The steps sp.py needs, on fp64 CPU tensors: chunk passes from the oracle over the
    step's own tokens, scans from their definitions (la_seg.h)."""

    def subsegments(self, B, H, L, dk, dv, P, chunk, dt):
        return 2 * P  # a split of every segment, as the library makes

    def backward_parts(self, B, H, L, dk, dv, P, chunk, dt):
        return 2 * P

    def state_pass(self, k, v, g, NP, chunk):
        B, H, L, dk = k.shape
        T = L // NP
        S, lg = [], []
        for p in range(NP):
            sl = slice(p * T, (p + 1) * T)
            S.append(oracle.forward(k[:, :, sl], k[:, :, sl], v[:, :, sl], g[:, :, sl], None)[1])
            lg.append(g[:, :, sl].sum(dim=2).numpy())
        return t64(np.stack(S, axis=2)), t64(np.stack(lg, axis=2))

    def scan(self, S_in, lg, init, reverse, S_next=None, S_last=None):
        B, H, NP, dk, dv = S_in.shape
        acc = init.clone() if init is not None else torch.zeros((B, H, dk, dv), dtype=torch.float64)
        out = torch.empty_like(S_in)
        carry = torch.empty((B, H, NP, dk), dtype=torch.float64) if S_next is not None else None
        for k in range(NP):
            p = NP - 1 - k if reverse else k
            out[:, :, p] = acc
            if carry is not None:
                end = S_next[:, :, p + 1] if p + 1 < NP else (S_last if S_last is not None else torch.zeros_like(acc))
                carry[:, :, p] = (end * acc).sum(dim=-1)
            acc = torch.exp(lg[:, :, p])[..., None] * acc + S_in[:, :, p]
        return out, acc, carry

    def log_gamma_total(self, lg):
        return lg.sum(dim=2)

    def rank_scan(self, S_ranks, lg_ranks, rank, init, reverse):
        N = S_ranks.shape[0]
        acc = init.clone() if init is not None else torch.zeros_like(S_ranks[0])
        S_in = None
        for k in range(N):
            r = N - 1 - k if reverse else k
            if r == rank:
                S_in = acc.clone()
            acc = torch.exp(lg_ranks[r])[..., None] * acc + S_ranks[r]
        return S_in, acc

    def combine(self, lg_a, S_a, lg_b, S_b):
        return lg_a + lg_b, torch.exp(lg_b)[..., None] * S_a + S_b

    def output_pass(self, q, k, v, g, S_recv, NP, chunk):
        T = q.shape[2] // NP
        o = [oracle.forward(q[:, :, p * T:(p + 1) * T], k[:, :, p * T:(p + 1) * T],
                            v[:, :, p * T:(p + 1) * T], g[:, :, p * T:(p + 1) * T],
                            S_recv[:, :, p])[0] for p in range(NP)]
        return t64(np.concatenate(o, axis=2))

    def gather_states(self, S_recv, m):
        return S_recv[:, :, ::m].contiguous()

    def dq_pass(self, q, k, v, g, dO, S_recv, NP, fine, chunk):
        B, H, L, dk = q.shape
        T, Tf = L // NP, L // NP // fine
        dq, S_fine, dSloc, lgf = [], [], [], []
        for p in range(NP):
            sl = slice(p * T, (p + 1) * T)
            dq.append(oracle.backward(q[:, :, sl], k[:, :, sl], v[:, :, sl], g[:, :, sl], dO[:, :, sl],
                                      S_recv[:, :, p], None)[0])
            S = S_recv[:, :, p].numpy()
            for f in range(fine):
                fs = slice(p * T + f * Tf, p * T + (f + 1) * Tf)
                S_fine.append(S)
                grads = oracle.backward(q[:, :, fs], k[:, :, fs], v[:, :, fs], g[:, :, fs], dO[:, :, fs], S, None)
                dSloc.append(grads[4])
                lgf.append(g[:, :, fs].sum(dim=2).numpy())
                S = oracle.forward(q[:, :, fs], k[:, :, fs], v[:, :, fs], g[:, :, fs], S)[1]
        dq = t64(np.concatenate(dq, axis=2))
        return (dq, q * dq, t64(np.stack(S_fine, axis=2)), t64(np.stack(dSloc, axis=2)),
                t64(np.stack(lgf, axis=2)))

    def dkv_pass(self, q, k, v, g, dO, S_fine, dX, qdq, NPF, chunk, carry):
        Tf = q.shape[2] // NPF
        dk, dv, dg = [], [], []
        for f in range(NPF):
            fs = slice(f * Tf, (f + 1) * Tf)
            r = oracle.backward(q[:, :, fs], k[:, :, fs], v[:, :, fs], g[:, :, fs], dO[:, :, fs],
                                S_fine[:, :, f], dX[:, :, f])
            dk.append(r[1]); dv.append(r[2]); dg.append(r[3])
        return tuple(t64(np.concatenate(x, axis=2)) for x in (dk, dv, dg))

    def check(self):
        pass


def _inputs(seed, B, H, L, dk, dv):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, L, dk)) / np.sqrt(dk)
    k = rng.standard_normal((B, H, L, dk)) / np.sqrt(dk)
    v = rng.standard_normal((B, H, L, dv))
    g = np.log(1 / (1 + np.exp(-(rng.standard_normal((B, H, L, dk)) + 2.0)))) / 4
    dO = rng.standard_normal((B, H, L, dv))
    S0 = rng.standard_normal((B, H, dk, dv)) / 4
    dSf = rng.standard_normal((B, H, dk, dv))
    return q, k, v, g, dO, S0, dSf


CASE = dict(B=1, H=2, Lr=32, dk=4, dv=4, P=2)


def _worker(rank, world, port, method, with_s0, with_dsf, outdir):
    from sequence_linear_attention_chunked_b200 import sp
    import datetime
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        c = CASE
        q, k, v, g, dO, S0, dSf = _inputs(5, c["B"], c["H"], c["Lr"] * world, c["dk"], c["dv"])
        sl = slice(rank * c["Lr"], (rank + 1) * c["Lr"])
        blk = [t64(x[:, :, sl]) for x in (q, k, v, g, dO)]
        steps = OracleSteps()
        o, Sf, saved = sp.sp_forward(*blk[:4], t64(S0) if with_s0 else None, c["P"], 8,
                                     method=method, steps=steps)
        grads = sp.sp_backward(*blk, saved, t64(dSf) if with_dsf else None, c["P"], 8,
                               method=method, steps=steps)
        np.savez(os.path.join(outdir, f"r{rank}.npz"), o=o.numpy(), Sf=Sf.numpy(),
                 **{n: t.numpy() for n, t in zip(NAMES + ("dS0",), grads)})
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,method,with_s0,with_dsf", [
    (2, "gather", True, True), (2, "tree", False, False), (3, "gather", False, True),
    (3, "tree", True, True), (4, "tree", True, False), (4, "gather", True, True)])
def test_sp_matches_oracle_on_gloo_ranks(world, method, with_s0, with_dsf):
    with tempfile.TemporaryDirectory() as outdir:
        mp.start_processes(_worker, args=(world, _free_port(), method, with_s0, with_dsf, outdir),
                           nprocs=world, join=True, start_method="spawn")
        res = [dict(np.load(os.path.join(outdir, f"r{r}.npz"))) for r in range(world)]
    c = CASE
    q, k, v, g, dO, S0, dSf = _inputs(5, c["B"], c["H"], c["Lr"] * world, c["dk"], c["dv"])
    S0 = S0 if with_s0 else None
    dSf = dSf if with_dsf else None
    o_ref, Sf_ref, _ = oracle.forward(q, k, v, g, S0)
    ref = oracle.backward(q, k, v, g, dO, S0, dSf)
    assert rel_err(np.concatenate([r["o"] for r in res], axis=2), o_ref) < 1e-12
    for r in res:
        assert rel_err(r["Sf"], Sf_ref) < 1e-12
        assert rel_err(r["dS0"], ref[4]) < 1e-12
    for i, n in enumerate(NAMES):
        got = np.concatenate([r[n] for r in res], axis=2)
        assert rel_err(got, ref[i]) < 1e-11, n
