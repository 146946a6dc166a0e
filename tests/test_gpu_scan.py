"""The exclusive decayed scan kernel (through la_seg_scan) against fp64 references."""
import numpy as np
import pytest
import torch

from sequence_linear_attention_chunked_b200 import la_seg
from tests.parity import rel_err

pytestmark = pytest.mark.gpu


def ref_scan(S_in, lg, init, reverse):
    S_in = S_in.double().cpu().numpy()
    lg = lg.double().cpu().numpy()
    BH, NP, dk, dv = S_in.shape
    acc = np.zeros((BH, dk, dv)) if init is None else init.double().cpu().numpy().copy()
    out = np.zeros_like(S_in)
    order = range(NP - 1, -1, -1) if reverse else range(NP)
    for p in order:
        out[:, p] = acc
        acc = np.exp(lg[:, p])[..., None] * acc + S_in[:, p]
    return out, acc


def make(BH, NP, d, device, seed=0, scale=0.05):
    g = torch.Generator(device=device).manual_seed(seed)
    S = torch.randn((BH, NP, d, d), generator=g, device=device)
    lg = -scale * torch.rand((BH, NP, d), generator=g, device=device) * 64
    init = torch.randn((BH, d, d), generator=g, device=device)
    return S, lg, init


@pytest.mark.parametrize("BH,NP,d", [(1, 1, 32), (3, 5, 32), (16, 8, 128), (2, 37, 64), (4, 256, 128)])
@pytest.mark.parametrize("reverse", [False, True])
def test_scan_matches_reference(cuda_device, BH, NP, d, reverse):
    S, lg, init = make(BH, NP, d, cuda_device, seed=NP)
    out, fin = la_seg.la_seg_scan(S, lg, init, reverse)
    ref_out, ref_fin = ref_scan(S, lg, init, reverse)
    assert rel_err(out, ref_out) <= 1e-6
    assert rel_err(fin, ref_fin) <= 1e-6


def test_scan_without_init(cuda_device):
    S, lg, _ = make(2, 9, 64, cuda_device)
    out, fin = la_seg.la_seg_scan(S, lg, None)
    ref_out, ref_fin = ref_scan(S, lg, None, False)
    assert torch.count_nonzero(out[:, 0]) == 0
    assert rel_err(out, ref_out) <= 1e-6 and rel_err(fin, ref_fin) <= 1e-6


def test_dk_block_split_is_bit_identical(cuda_device):
    """All-Scan's split of the state into K blocks along d_k (ZeCO review, "key machinery")
    leaves every received state unchanged: rows scan independently."""
    S, lg, init = make(4, 16, 128, cuda_device, seed=3)
    out, fin = la_seg.la_seg_scan(S, lg, init)
    for K in (2, 4, 8):
        blk = 128 // K
        for kb in range(K):
            rows = slice(kb * blk, (kb + 1) * blk)
            o_b, f_b = la_seg.la_seg_scan(S[:, :, rows].contiguous(), lg[:, :, rows].contiguous(),
                                          init[:, rows].contiguous())
            assert torch.equal(o_b, out[:, :, rows]) and torch.equal(f_b, fin[:, rows])


def test_accumulated_state_propagates(cuda_device):
    """P >= 3: segment 2 receives Gamma_1 Gamma_0 S0 + Gamma_1 S_0 + S_1, not only S_1 (the
    referee's Alg. 2 comment in the ZeCO review)."""
    S, lg, init = make(2, 4, 32, cuda_device, seed=5, scale=0.001)
    out, _ = la_seg.la_seg_scan(S, lg, init)
    G = torch.exp(lg.double())[..., None]
    expect = G[:, 1] * G[:, 0] * init.double() + G[:, 1] * S[:, 0].double() + S[:, 1].double()
    assert rel_err(out[:, 2], expect.cpu().numpy()) <= 1e-6
    assert rel_err(S[:, 1], expect.cpu().numpy()) > 1e-2


def test_scan_empty(cuda_device):
    S = torch.zeros((0, 4, 32, 32), device=cuda_device)
    lg = torch.zeros((0, 4, 32), device=cuda_device)
    out, fin = la_seg.la_seg_scan(S, lg, None)
    assert out.numel() == 0 and fin.numel() == 0


def test_scan_carry(cuda_device):
    """The reverse scan's dlog_g carries: carry[p][i] = sum_j S_end_p[i][j] out[p][i][j], with
    S_end_p = S_next[p+1] and S_last for the last segment."""
    g = torch.Generator(device="cpu").manual_seed(5)
    BH, NP, d = 3, 9, 128
    S = torch.randn(BH, NP, d, d, generator=g).to(cuda_device)
    lg = (-torch.rand(BH, NP, d, generator=g)).to(cuda_device)
    init = torch.randn(BH, d, d, generator=g).to(cuda_device)
    S_next = torch.randn(BH, NP, d, d, generator=g).to(cuda_device)
    S_last = torch.randn(BH, d, d, generator=g).to(cuda_device)
    out, fin, carry = la_seg.la_seg_scan(S, lg, init, True, S_next=S_next, S_last=S_last)
    out_plain, fin_plain = la_seg.la_seg_scan(S, lg, init, True)
    assert torch.equal(out, out_plain) and torch.equal(fin, fin_plain)
    S_end = torch.cat([S_next[:, 1:], S_last[:, None]], dim=1).double()
    ref = (S_end * out.double()).sum(dim=-1)
    assert torch.allclose(carry.double(), ref, rtol=1e-5, atol=1e-4 * float(ref.abs().max()))
    _, _, carry0 = la_seg.la_seg_scan(S, lg, init, True, S_next=S_next)  # no S_last: zero there
    assert torch.equal(carry0[:, :-1], carry[:, :-1]) and torch.all(carry0[:, -1] == 0)


@pytest.mark.parametrize("dk,dv", [(6, 32), (4, 512), (128, 128)])
def test_scan_both_kernels(cuda_device, dk, dv):
    """Whole 1024-float slices of >= 4 rows with 16-byte aligned log-decays take the bulk-copy
    kernel, other shapes the per-thread one; a log_gamma view one float off alignment sends the
    same sizes to the per-thread kernel, and the two agree bit for bit (same fma order)."""
    g = torch.Generator(device=cuda_device).manual_seed(dk + dv)
    BH, NP = 3, 7
    S = torch.randn((BH, NP, dk, dv), generator=g, device=cuda_device)
    lg = -torch.rand((BH, NP, dk), generator=g, device=cuda_device)
    init = torch.randn((BH, dk, dv), generator=g, device=cuda_device)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    for reverse in (False, True):
        out, fin = la_seg.la_seg_scan(S, lg, init, reverse, status=status)
        ref_out, ref_fin = ref_scan(S, lg, init, reverse)
        assert rel_err(out, ref_out) <= 1e-6 and rel_err(fin, ref_fin) <= 1e-6
        buf = torch.empty(lg.numel() + 1, device=cuda_device)
        lg_off = buf[1:].view(BH, NP, dk)
        lg_off.copy_(lg)
        out2, fin2 = la_seg.la_seg_scan(S, lg_off, init, reverse, status=status)
        assert torch.equal(out, out2) and torch.equal(fin, fin2)
    assert int(status.item()) == 0
