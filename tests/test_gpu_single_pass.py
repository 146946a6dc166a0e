"""The single-pass forward (state pass, chained scan and output pass in one kernel) against the
fp64 oracle, through the C ABI; its bounded cross-CTA wait; agreement with the two-pass order."""
import numpy as np
import pytest
import torch

import oracle
from sequence_linear_attention_chunked_b200 import la_seg
from sequence_linear_attention_chunked_b200.inputs import WORKLOADS, Workload, make_inputs
from tests.parity import oracle_window, rel_err

pytestmark = pytest.mark.gpu

SINGLE = la_seg.SCHED_SINGLE_PASS


def forward(x, w, schedule=SINGLE):
    ws = la_seg.workspace(w.B, w.H, w.L, w.dk, w.dv, w.P, w.chunk,
                          la_seg.LA_F32 if w.dtype == "f32" else la_seg.LA_BF16, False,
                          x["q"].device)
    o, Sf, Sr = la_seg.la_seg_forward(x["q"], x["k"], x["v"], x["log_g"], x.get("S0"), w.P,
                                      w.chunk, schedule, want_S_recv=True, ws=ws)
    la_seg.la_seg_check_status(ws)
    return o, Sf, Sr


SHAPES = [  # (B, H, L, P, dist): bf16, d = 128, chunk 64 (the tensor-core shape); these few
    # sequences are split into sub-segments of one to three chunks: long chains
    (1, 2, 4096, 2, "gla"),
    (2, 3, 3072, 3, "gla"),     # P = 3
    (1, 1, 1536, 1, "gla"),
    (1, 2, 128, 2, "gla"),      # one chunk per segment
    (1, 4, 8192, 4, "weak"),    # the received states carry real signal
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_single_pass_parity(cuda_device, shape):
    B, H, L, P, dist = shape
    w = Workload("single", B, H, L, 128, 128, P, 64, "bf16", dist, seed=L + P)
    x = make_inputs(w, cuda_device, with_s0=(L % 3 == 0 or dist == "weak"))
    o, Sf, Sr = forward(x, w)
    o_ref, Sf_ref, Sr_ref = oracle.forward(x["q"], x["k"], x["v"], x["log_g"], x.get("S0"),
                                           seg_len=L // P)
    errs = (rel_err(o, o_ref), rel_err(Sf, Sf_ref), rel_err(Sr, Sr_ref))
    assert max(errs) <= 2e-2, errs
    if dist == "weak":
        assert np.abs(Sr_ref[:, :, 1:]).max() > 0.1


def test_other_shapes_run_two_pass(cuda_device):
    """fp32 and small d have no single-pass kernel: the schedule runs the two-pass order."""
    w = WORKLOADS["C0"]
    x = make_inputs(w, cuda_device, with_s0=True)
    a = forward(x, w, SINGLE)
    b = forward(x, w, la_seg.SCHED_TWO_PASS)
    for u, v in zip(a, b):
        assert torch.equal(u, v)


def test_chain_pass_one_chunk_links(cuda_device):
    """la_seg_chain_pass directly, with one-chunk sub-segments: a chain of 256 links per
    sequence, longer than the CTAs resident at once; S_recv_save every 32nd sub-segment."""
    w = Workload("chain", 1, 2, 16384, 128, 128, 8, 64, "bf16", "weak", seed=3)
    x = make_inputs(w, cuda_device, with_s0=True)
    NP, every = 256, 32
    states, ready = la_seg.chain_buffers(1, 2, 128, 128, cuda_device)
    status = torch.zeros(64, dtype=torch.int32, device=cuda_device)
    S_final = torch.empty((1, 2, 128, 128), dtype=torch.float32, device=cuda_device)
    S_save = torch.empty((1, 2, NP // every, 128, 128), dtype=torch.float32, device=cuda_device)
    la_seg.la_seg_chain_reset(x["S0"], 1, 2, 128, 128, states, ready)
    o = la_seg.la_seg_chain_pass(x["q"], x["k"], x["v"], x["log_g"], NP, 64, states, ready,
                                 S_final=S_final, S_recv_save=S_save, save_every=every,
                                 status=status)
    la_seg.la_seg_check_status(status)
    assert int(ready[:2].min()) == NP  # every sub-segment published
    o_ref, Sf_ref, Sr_ref = oracle.forward(x["q"], x["k"], x["v"], x["log_g"], x["S0"],
                                           seg_len=16384 // (NP // every))
    assert rel_err(o, o_ref) <= 2e-2
    assert rel_err(S_final, Sf_ref) <= 2e-2
    assert rel_err(S_save, Sr_ref) <= 2e-2


def test_chain_wait_gives_up(cuda_device):
    """A chain whose first state is never published: every wait is bounded, the call reports
    LA_ERR_TIMEOUT, the successors stop at the failure mark, and the context stays usable."""
    w = Workload("chain-timeout", 1, 2, 1024, 128, 128, 1, 64, "bf16", "gla", seed=5)
    x = make_inputs(w, cuda_device)
    states, ready = la_seg.chain_buffers(1, 2, 128, 128, cuda_device)
    status = torch.zeros(64, dtype=torch.int32, device=cuda_device)
    la_seg.la_seg_chain_reset(None, 1, 2, 128, 128, states, ready)
    ready[:2] = -1  # nothing ever publishes sub-segment 0's received state
    la_seg.la_seg_chain_pass(x["q"], x["k"], x["v"], x["log_g"], 2, 64, states, ready,
                             status=status)
    with pytest.raises(la_seg.LaSegError) as ei:
        la_seg.la_seg_check_status(status)
    assert ei.value.status == -7
    assert ready[:2].tolist() == [0x7FFFFFF0] * 2  # the failure mark reached every chain
    o, _, _ = forward(x, w)  # the device is still usable and the next call is right
    o_ref, _, _ = oracle.forward(x["q"], x["k"], x["v"], x["log_g"])
    assert rel_err(o, o_ref) <= 2e-2


def test_single_pass_deterministic_and_close_to_two_pass(cuda_device):
    w = WORKLOADS["C1"].with_(H=4, L=8192, P=2)
    x = make_inputs(w, cuda_device, with_s0=True)
    a = forward(x, w)
    b = forward(x, w)
    for u, v in zip(a, b):
        assert torch.equal(u, v)
    c = forward(x, w, la_seg.SCHED_TWO_PASS)
    for u, v in zip(a, c):
        assert rel_err(u, v.double().cpu().numpy()) <= 2e-2


def test_c2_single_pass_sampled(cuda_device):
    """C2 at full size through the single pass: windows at segment starts and inside."""
    w = WORKLOADS["C2"]
    x = make_inputs(w, cuda_device)
    ws = la_seg.workspace(w.B, w.H, w.L, w.dk, w.dv, w.P, w.chunk, la_seg.LA_BF16, False,
                          cuda_device)
    o, Sf, _ = la_seg.la_seg_forward(x["q"], x["k"], x["v"], x["log_g"], None, w.P, w.chunk,
                                     SINGLE, ws=ws)
    la_seg.la_seg_check_status(ws)
    T = w.L // w.P
    rng = np.random.default_rng(11)
    for h in (0, w.H - 1):
        for p in (0, 1, w.P - 1):
            for t0 in (p * T, p * T + int(rng.integers(0, T - 512)) // 64 * 64):
                ref = oracle_window(x, 0, h, t0, t0 + 512)
                assert rel_err(o[0, h, t0:t0 + 512], ref) <= 2e-2, (h, p, t0)
    del x, o
    torch.cuda.empty_cache()
