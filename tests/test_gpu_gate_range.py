"""Gates outside the chunk factorisation's range, against the fp64 oracle.

The chunk kernels scale q and k by exp(+-(b_t - b_C)) (b the in-chunk cumsum of log_g).  That
holds in fp32 / bf16 while no log_g in a chunk is positive and the chunk's decay stays within
e^-80 in every key dim.  Outside that range:

* the per-step entry points report LA_ERR_GATE_RANGE in their status word (the tensor-core
  kernels of every pass and sweep, and the CUDA-core ones), for a strong decay (chunk sum
  -96) and for a cumsum that rises and falls inside the chunk (chunk sum 0, peak +96);
* la_seg_forward and la_seg_backward route the marked units through the exact token-by-token
  path instead, so that complete forgetting (a = 0, log_g = -1e4, the oracle pin's case),
  log_g = -2 per token, positive gates and a single strongly decaying stretch inside an
  ordinary sequence all match the oracle, and sequences without such chunks stay bit for bit
  what the chunk kernels give.
Just inside the range (chunk sums of -75) the chunk kernels themselves keep the error bound.
"""
import pytest
import torch

import oracle
from sequence_linear_attention_chunked_b200 import la_seg
from sequence_linear_attention_chunked_b200.inputs import Workload, make_inputs
from tests.parity import TOL, rel_err

pytestmark = pytest.mark.gpu

GATE_RANGE = 1  # status bit behind LA_ERR_GATE_RANGE
NAMES = ("dq", "dk", "dv", "dlog_g", "dS0")
FWD_SCHEDULES = {"two_pass": la_seg.SCHED_TWO_PASS, "three_phase": la_seg.SCHED_THREE_PHASE,
                 "single_pass": la_seg.SCHED_SINGLE_PASS, "overlap": la_seg.SCHED_OVERLAP}


def gates(pattern, shape, device, dtype):
    """log_g of one of the test patterns (chunks of 64 tokens along dim -2)."""
    L = shape[-2]
    if pattern == "strong":          # chunk sum -96 < -80
        return torch.full(shape, -1.5, device=device).to(dtype)
    if pattern == "rise_fall":       # +3 for 32 tokens, then -3: chunk sum 0, peak +96
        t = torch.arange(L, device=device) % 64
        g = torch.where(t < 32, 3.0, -3.0).reshape(*([1] * (len(shape) - 2)), L, 1)
        return g.expand(shape).contiguous().to(dtype)
    if pattern == "near_limit":      # bf16(-1.17) = -1.171875: chunk sum -75, inside the range
        return torch.full(shape, -1.17, device=device).to(dtype)
    if pattern == "zero_gate":       # a = exp(-1e4) = 0: every token forgets all before it
        return torch.full(shape, -1.0e4, device=device).to(dtype)
    if pattern == "minus2":          # chunk sum -128
        return torch.full(shape, -2.0, device=device).to(dtype)
    if pattern == "positive":        # small positive gates: a > 1 for the first half of a chunk
        t = torch.arange(L, device=device) % 64
        g = torch.where(t < 32, 0.02, -0.05).reshape(*([1] * (len(shape) - 2)), L, 1)
        return g.expand(shape).contiguous().to(dtype)
    raise ValueError(pattern)


def status_word(device):
    return torch.zeros(1, dtype=torch.int32, device=device)


def tc_inputs(device, pattern, B=1, H=2, L=512):
    w = Workload("gates", B, H, L, 128, 128, 2, 64, "bf16", "gla", backward=True, seed=7)
    x = make_inputs(w, device)
    x["log_g"] = gates(pattern, x["log_g"].shape, device, torch.bfloat16)
    return w, x


# ----------------------------------------------------------------- per-step status reports
@pytest.mark.parametrize("pattern", ["strong", "rise_fall"])
def test_per_step_tc_calls_report_gate_range(cuda_device, pattern):
    """Every tensor-core pass and sweep reports a chunk outside the range (bf16, d=128, 64)."""
    w, x = tc_inputs(cuda_device, pattern)
    q, k, v, g, dO = x["q"], x["k"], x["v"], x["log_g"], x["dO"]
    NP, C = 2, 64
    BH = w.B * w.H
    calls = {
        "state": lambda st: la_seg.la_seg_state_pass(k, v, g, NP, C, status=st),
        "local": lambda st: la_seg.la_seg_local_pass(q, k, v, g, NP, C, status=st),
        "output": lambda st: la_seg.la_seg_output_pass(q, k, v, g, None, NP, C, status=st),
        "correct": lambda st: la_seg.la_seg_correct_pass(
            q, g, torch.zeros((w.B, w.H, NP, 128, 128), device=cuda_device), NP, C,
            torch.zeros_like(q), status=st),
        "dstate": lambda st: la_seg.la_seg_dstate_pass(q, dO, g, NP, C, status=st),
        "dq": lambda st: la_seg.la_seg_dq_pass(q, k, v, g, dO, None, NP, 2, C, status=st),
        "dkv": lambda st: la_seg.la_seg_dkv_pass(
            q, k, v, g, dO, None, None, torch.zeros((BH, NP, 128, 128), device=cuda_device),
            torch.zeros((w.B, w.H, w.L, 128), device=cuda_device), NP, C, status=st),
    }
    for name, call in calls.items():
        st = status_word(cuda_device)
        call(st)
        torch.cuda.synchronize()
        assert int(st.item()) & GATE_RANGE, (name, pattern)


def test_per_step_calls_clean_inside_the_range(cuda_device):
    """Ordinary gates and chunk sums of -75 leave the status word clear."""
    for pattern in ("ordinary", "near_limit"):
        w, x = tc_inputs(cuda_device, "near_limit")
        if pattern == "ordinary":
            x = make_inputs(w, cuda_device)
        st = status_word(cuda_device)
        la_seg.la_seg_state_pass(x["k"], x["v"], x["log_g"], 2, 64, status=st)
        la_seg.la_seg_output_pass(x["q"], x["k"], x["v"], x["log_g"], None, 2, 64, status=st)
        la_seg.la_seg_dq_pass(x["q"], x["k"], x["v"], x["log_g"], x["dO"], None, 2, 2, 64, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0, pattern


@pytest.mark.parametrize("pattern", ["strong", "rise_fall"])
def test_per_step_simt_calls_report_gate_range(cuda_device, pattern):
    """The CUDA-core passes (fp32, d = 32, chunk 16) report it too."""
    w = Workload("gates32", 1, 2, 256, 32, 32, 2, 16, "f32", "toy", backward=True, seed=3)
    x = make_inputs(w, cuda_device)
    g = x["log_g"]
    if pattern == "strong":
        g.fill_(-6.0)  # chunk sum -96
    else:
        t = torch.arange(w.L, device=cuda_device) % 16
        g.copy_(torch.where(t < 8, 12.0, -12.0).view(1, 1, -1, 1).expand_as(g))
    for name, call in {
        "state": lambda st: la_seg.la_seg_state_pass(x["k"], x["v"], g, 2, 16, status=st),
        "output": lambda st: la_seg.la_seg_output_pass(x["q"], x["k"], x["v"], g, None, 2, 16, status=st),
        "dq": lambda st: la_seg.la_seg_dq_pass(x["q"], x["k"], x["v"], g, x["dO"], None, 2, 1, 16,
                                               status=st),
    }.items():
        st = status_word(cuda_device)
        call(st)
        torch.cuda.synchronize()
        assert int(st.item()) & GATE_RANGE, (name, pattern)


# ----------------------------------------------------------------- whole calls vs the oracle
def forward_vs_oracle(x, w, schedule):
    ws = la_seg.workspace(w.B, w.H, w.L, w.dk, w.dv, w.P, w.chunk,
                          la_seg.LA_F32 if w.dtype == "f32" else la_seg.LA_BF16, False,
                          x["q"].device)
    o, Sf, Sr = la_seg.la_seg_forward(x["q"], x["k"], x["v"], x["log_g"], x.get("S0"), w.P,
                                      w.chunk, schedule, want_S_recv=True, ws=ws)
    la_seg.la_seg_check_status(ws)  # routed through the exact path: no error left behind
    ref = oracle.forward(x["q"], x["k"], x["v"], x["log_g"], x.get("S0"), seg_len=w.L // w.P)
    tol = TOL[w.torch_dtype]
    errs = [rel_err(got, r) for got, r in zip((o, Sf, Sr), ref)]
    assert all(e <= tol for e in errs), (w.describe(), errs)
    return o, Sf, Sr


def backward_vs_oracle(x, w, reuse):
    dt = la_seg.LA_F32 if w.dtype == "f32" else la_seg.LA_BF16
    Sr = None
    if reuse:
        _, _, Sr = la_seg.la_seg_forward(x["q"], x["k"], x["v"], x["log_g"], x.get("S0"), w.P,
                                         w.chunk, want_S_recv=True)
    ws = la_seg.workspace(w.B, w.H, w.L, w.dk, w.dv, w.P, w.chunk, dt, True, x["q"].device)
    got = la_seg.la_seg_backward(x["q"], x["k"], x["v"], x["log_g"], x["dO"], x.get("S0"), Sr,
                                 None, w.P, w.chunk, want_dS0=True, ws=ws)
    la_seg.la_seg_check_status(ws)
    ref = oracle.backward(x["q"], x["k"], x["v"], x["log_g"], x["dO"], x.get("S0"), None)
    tol = TOL[w.torch_dtype]
    errs = {n: rel_err(g, r) for n, g, r in zip(NAMES, got, ref)}
    assert all(e <= tol for e in errs.values()), (w.describe(), reuse, errs)
    return got


# (rise_fall is not among them: a state that grows by e^96 over half a chunk overflows fp32 in
# any implementation; it only serves the status checks above.)
@pytest.mark.parametrize("pattern", ["zero_gate", "minus2", "positive"])
@pytest.mark.parametrize("sched", list(FWD_SCHEDULES))
def test_forward_outside_the_range(cuda_device, pattern, sched):
    w, x = tc_inputs(cuda_device, pattern, B=1, H=2, L=1024)
    x["S0"] = torch.randn((1, 2, 128, 128), generator=torch.Generator(device=cuda_device).manual_seed(5),
                          device=cuda_device) / 16
    forward_vs_oracle(x, w, FWD_SCHEDULES[sched])


@pytest.mark.parametrize("pattern", ["zero_gate", "minus2", "positive"])
@pytest.mark.parametrize("reuse", [False, True])
def test_backward_outside_the_range(cuda_device, pattern, reuse):
    w, x = tc_inputs(cuda_device, pattern, B=1, H=2, L=1024)
    backward_vs_oracle(x, w, reuse)


def test_near_limit_on_the_chunk_kernels(cuda_device):
    """Chunk sums of -75 stay on the tensor-core path and keep the bf16 bound."""
    w, x = tc_inputs(cuda_device, "near_limit", B=1, H=2, L=1024)
    st = status_word(cuda_device)
    la_seg.la_seg_state_pass(x["k"], x["v"], x["log_g"], 2, 64, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0  # nothing was routed to the exact path
    for sched in FWD_SCHEDULES.values():
        forward_vs_oracle(x, w, sched)
    for reuse in (False, True):
        backward_vs_oracle(x, w, reuse)


def test_strong_stretch_inside_an_ordinary_sequence(cuda_device):
    """One sub-segment of head 1 forgets hard; the scan carries the exact path's state on, and
    the heads without such chunks are bit for bit what the chunk kernels alone give."""
    w = Workload("stretch", 1, 4, 8192, 128, 128, 2, 64, "bf16", "gla", backward=True, seed=11)
    x = make_inputs(w, cuda_device)
    clean = {n: t.clone() for n, t in x.items()}
    x["log_g"][0, 1, 3000:3100] = -5.0
    x["log_g"][0, 3, 6000:6064] = 0.25  # a positive stretch in another head
    o, Sf, Sr = forward_vs_oracle(x, w, la_seg.SCHED_AUTO)
    grads = backward_vs_oracle(x, w, reuse=True)
    o0, Sf0, Sr0 = la_seg.la_seg_forward(clean["q"], clean["k"], clean["v"], clean["log_g"], None,
                                         w.P, w.chunk, want_S_recv=True)
    g0 = la_seg.la_seg_backward(clean["q"], clean["k"], clean["v"], clean["log_g"], clean["dO"], None,
                                Sr0, None, w.P, w.chunk, want_dS0=True)
    for h in (0, 2):
        assert torch.equal(o[:, h], o0[:, h]) and torch.equal(Sf[:, h], Sf0[:, h])
        assert torch.equal(Sr[:, h], Sr0[:, h])
        for a, b in zip(grads, g0):
            assert torch.equal(a[:, h], b[:, h])


def test_fp32_strong_decay_on_the_cuda_core_path(cuda_device):
    """fp32, d = 32, chunk 16 with chunk sums of -128: the exact path keeps the 1e-4 bound."""
    w = Workload("strong32", 1, 2, 256, 32, 32, 4, 16, "f32", "toy", backward=True, seed=4)
    x = make_inputs(w, cuda_device, with_s0=True)
    x["log_g"].fill_(-8.0)
    for sched in FWD_SCHEDULES.values():
        forward_vs_oracle(x, w, sched)
    for reuse in (False, True):
        backward_vs_oracle(x, w, reuse)
