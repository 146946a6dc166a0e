"""Sequence parallelism across ranks (sp.py) with the library's kernels, against the oracle.

Two (and three) processes share cuda:0, each holding one block of every sequence and running
its own kernels; their (log Gamma, S) pairs cross through host memory on a gloo group (no
kernel waits on another process's).  Every rank's outputs and gradients, put together, match
the fp64 oracle on the whole sequence within the bf16 bound, for both All-Scans.
"""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from tests.parity import rel_err

pytestmark = pytest.mark.gpu
NAMES = ("dq", "dk", "dv", "dlog_g", "dS0")
B, H, LR, D, P, CHUNK = 1, 2, 1024, 128, 2, 64


def _worker(rank, world, port, method, with_s0, with_dsf, outdir):
    import datetime
    import torch.distributed as dist
    from sequence_linear_attention_chunked_b200 import sp
    from sequence_linear_attention_chunked_b200.inputs import Workload, make_inputs
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        dev = torch.device("cuda:0")
        w = Workload("sp", B, H, LR * world, D, D, P, CHUNK, "bf16", "weak", backward=True, seed=3)
        x = make_inputs(w, dev, with_s0=True)
        sl = slice(rank * LR, (rank + 1) * LR)
        blk = {n: x[n][:, :, sl].contiguous() for n in ("q", "k", "v", "log_g", "dO")}
        dSf = torch.randn((B, H, D, D), generator=torch.Generator(device=dev).manual_seed(9),
                          device=dev) if with_dsf else None
        o, Sf, saved = sp.sp_forward(blk["q"], blk["k"], blk["v"], blk["log_g"],
                                     x["S0"] if with_s0 else None, P, CHUNK, method=method)
        g = sp.sp_backward(blk["q"], blk["k"], blk["v"], blk["log_g"], blk["dO"], saved, dSf, P,
                           CHUNK, method=method)
        torch.cuda.synchronize()
        np.savez(os.path.join(outdir, f"r{rank}.npz"), o=o.float().cpu().numpy(),
                 Sf=Sf.cpu().numpy(), **{n: t.float().cpu().numpy() for n, t in zip(NAMES, g)})
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,method,with_s0,with_dsf", [(2, "gather", True, True),
                                                           (3, "tree", False, True)])
def test_sp_on_one_gpu_matches_oracle(cuda_device, world, method, with_s0, with_dsf):
    from sequence_linear_attention_chunked_b200.inputs import Workload, make_inputs
    with tempfile.TemporaryDirectory() as outdir:
        mp.start_processes(_worker, args=(world, _free_port(), method, with_s0, with_dsf, outdir),
                           nprocs=world, join=True, start_method="spawn")
        res = [dict(np.load(os.path.join(outdir, f"r{r}.npz"))) for r in range(world)]
    w = Workload("sp", B, H, LR * world, D, D, P, CHUNK, "bf16", "weak", backward=True, seed=3)
    x = make_inputs(w, cuda_device, with_s0=True)
    S0 = x["S0"] if with_s0 else None
    dSf = torch.randn((B, H, D, D), generator=torch.Generator(device=cuda_device).manual_seed(9),
                      device=cuda_device) if with_dsf else None
    o_ref, Sf_ref, _ = oracle.forward(x["q"], x["k"], x["v"], x["log_g"], S0)
    ref = oracle.backward(x["q"], x["k"], x["v"], x["log_g"], x["dO"], S0, dSf)
    tol = 2e-2
    assert np.abs(Sf_ref).max() > 0 and rel_err(np.concatenate([r["o"] for r in res], axis=2), o_ref) <= tol
    for r in res:
        assert rel_err(r["Sf"], Sf_ref) <= tol
        assert rel_err(r["dS0"], ref[4]) <= tol
    for i, n in enumerate(NAMES[:4]):
        assert rel_err(np.concatenate([r[n] for r in res], axis=2), ref[i]) <= tol, n
