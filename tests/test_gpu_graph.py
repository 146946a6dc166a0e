"""The library's calls capture into a CUDA graph: they only queue work on the caller's stream
(kernels, a memset, and the overlap schedule's fork and join through events), so a captured
forward + backward replays bit for bit what the eager calls produce."""
import pytest
import torch

from sequence_linear_attention_chunked_b200 import la_seg
from sequence_linear_attention_chunked_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("schedule", [la_seg.SCHED_TWO_PASS, la_seg.SCHED_OVERLAP])
def test_forward_backward_graph_replay(cuda_device, schedule):
    w = WORKLOADS["C1"].with_(H=4, L=8192, P=2, backward=True)
    x = make_inputs(w, cuda_device)
    B, H, L, d = w.B, w.H, w.L, w.dk
    ws_f = la_seg.workspace(B, H, L, d, d, w.P, w.chunk, la_seg.LA_BF16, False, cuda_device)
    ws_b = la_seg.workspace(B, H, L, d, d, w.P, w.chunk, la_seg.LA_BF16, True, cuda_device)
    o = torch.empty_like(x["v"])
    S_final = torch.empty((B, H, d, d), dtype=torch.float32, device=cuda_device)
    S_recv = torch.empty((B, H, w.P, d, d), dtype=torch.float32, device=cuda_device)
    grads = [torch.empty_like(x[n]) for n in ("q", "k", "v", "log_g")]
    P_ = la_seg._ptr
    lib = la_seg.lib()

    def step(stream):
        s = la_seg._stream(stream)
        la_seg._check(lib.la_seg_forward(P_(x["q"]), P_(x["k"]), P_(x["v"]), P_(x["log_g"]), None,
                                         B, H, L, d, d, w.P, w.chunk, la_seg.LA_BF16, P_(o),
                                         P_(S_final), P_(S_recv), schedule, P_(ws_f),
                                         ws_f.numel(), s), "la_seg_forward")
        la_seg._check(lib.la_seg_backward(P_(x["q"]), P_(x["k"]), P_(x["v"]), P_(x["log_g"]),
                                          None, P_(S_recv), P_(x["dO"]), None, B, H, L, d, d,
                                          w.P, w.chunk, la_seg.LA_BF16, P_(grads[0]),
                                          P_(grads[1]), P_(grads[2]), P_(grads[3]), None,
                                          P_(ws_b), ws_b.numel(), s), "la_seg_backward")

    side = torch.cuda.Stream(device=cuda_device)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(side)  # eager, on the capture stream (also creates the overlap schedule's stream)
    side.synchronize()
    eager = [t.clone() for t in (o, S_final, S_recv, *grads)]
    for t in (o, S_final, S_recv, *grads):
        t.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        step(side)
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
        for a, b in zip(eager, (o, S_final, S_recv, *grads)):
            assert torch.equal(a, b)
    la_seg.la_seg_check_status(ws_f)
    la_seg.la_seg_check_status(ws_b)
    del g
