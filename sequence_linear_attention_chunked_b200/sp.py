"""Sequence parallelism across ranks: the pages' own setting, one block of the sequence per GPU.

Rank r of N holds tokens [r L, (r + 1) L) of every (b, h) sequence (q, k, v, log_g and, for the
backward, dO, each [B, H, L, d] on its own device).  The forward follows ZeCO's order (ZeCO
review, "key machinery"; Alg. 1's two passes with the All-Scan between them):

1. the state pass over the rank's sub-segments gives their local states and log-decays;
2. the rank reduces them to one pair (log Gamma_r, S_r): the state its whole block would pass on
   from a zero start, and the block's log-decay;
3. the All-Scan across ranks gives S_in_r, the state the rank's block receives
   (S_in_0 = S0, S_in_{r+1} = Gamma_r S_in_r + S_r: the accumulated state moves on, as the
   referee's comment on Alg. 2 requires), and the sequence's final state;
4. the local scan from S_in_r gives every sub-segment's received state, and the output pass
   the outputs.

The backward reuses the forward's received states ("forward implications") and runs the same
pattern in reverse over the gradient states: dq sweep, reduction to (log Gamma_r, G_r), the
reverse All-Scan (which gives the gradient at the block's end and, on every rank, dS0), the
local reverse scan with the dlog_g carries, and the dk/dv sweep.

Two All-Scans: "gather" all-gathers the N pairs (d_k + d_k d_v floats per (b, h) and rank, about
1 MB per rank at 16 heads) into local HBM and scans them there (la_seg_rank_scan) -- one
collective, no chain; "tree" is the tree-structured form the review lists as future work
("pith inferences"): ceil(log2 N) rounds of point-to-point exchanges of running aggregates,
combined with la_seg_combine (Hillis-Steele), then one shift.  Either way every byte lands in
the rank's own memory before a kernel reads it: no kernel reads a peer's memory.

Every step is one of the library's kernels (through the C ABI); torch.distributed moves the
pairs.  The CUDA tensors go to NCCL as they are; with a gloo group they are staged through host
memory.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import la_seg


# ----------------------------------------------------------------------------- the steps
class LibrarySteps:
    """The per-step entry points of libla_seg.so that the orchestration uses."""

    def __init__(self):
        self.status = None

    def _st(self, device):
        if self.status is None or self.status.device != device:
            self.status = torch.zeros(1, dtype=torch.int32, device=device)
        return self.status

    def subsegments(self, B, H, L, dk, dv, P, chunk, dt):
        return la_seg.la_seg_subsegments(B, H, L, dk, dv, P, chunk, dt)

    def backward_parts(self, B, H, L, dk, dv, P, chunk, dt):
        return la_seg.la_seg_backward_parts(B, H, L, dk, dv, P, chunk, dt, True)

    def state_pass(self, k, v, g, NP, chunk):
        return la_seg.la_seg_state_pass(k, v, g, NP, chunk, status=self._st(k.device))

    def scan(self, S_in, lg, init, reverse, S_next=None, S_last=None):
        B, H, NP, dk, dv = S_in.shape
        flat = lambda t, *s: None if t is None else t.view(*s)
        r = la_seg.la_seg_scan(S_in.view(B * H, NP, dk, dv), lg.view(B * H, NP, dk),
                               flat(init, B * H, dk, dv), reverse,
                               S_next=flat(S_next, B * H, NP, dk, dv), S_last=flat(S_last, B * H, dk, dv),
                               status=self._st(S_in.device))
        out = r[0].view(B, H, NP, dk, dv)
        final = r[1].view(B, H, dk, dv)
        carry = r[2].view(B, H, NP, dk) if len(r) > 2 else None
        return out, final, carry

    def log_gamma_total(self, lg):
        return la_seg.la_seg_log_gamma_total(lg)

    def rank_scan(self, S_ranks, lg_ranks, rank, init, reverse):
        return la_seg.la_seg_rank_scan(S_ranks, lg_ranks, rank, init, reverse)

    def combine(self, lg_a, S_a, lg_b, S_b):
        return la_seg.la_seg_combine(lg_a, S_a, lg_b, S_b)

    def output_pass(self, q, k, v, g, S_recv, NP, chunk):
        return la_seg.la_seg_output_pass(q, k, v, g, S_recv, NP, chunk, status=self._st(q.device))

    def gather_states(self, S_recv, m):
        return la_seg.la_seg_gather_states(S_recv, m)

    def dq_pass(self, q, k, v, g, dO, S_recv, NP, fine, chunk):
        B, H, L, dk = q.shape
        dv = v.shape[-1]
        f32 = dict(dtype=torch.float32, device=q.device)
        S_fine = torch.empty((B, H, NP * fine, dk, dv), **f32)
        dSloc = torch.empty((B, H, NP * fine, dk, dv), **f32)
        lgf = torch.empty((B, H, NP * fine, dk), **f32)
        dq, qdq = la_seg.la_seg_dq_pass(q, k, v, g, dO, S_recv, NP, fine, chunk, S_fine=S_fine,
                                        dSloc=dSloc, log_gamma=lgf, status=self._st(q.device))
        return dq, qdq, S_fine, dSloc, lgf

    def dkv_pass(self, q, k, v, g, dO, S_fine, dX, qdq, NPF, chunk, carry):
        return la_seg.la_seg_dkv_pass(q, k, v, g, dO, S_fine, None, dX, qdq, NPF, chunk,
                                      carry=carry, status=self._st(q.device))

    def check(self):
        """Raises if a kernel reported a device-side condition (a gate outside the chunk kernels'
        range: the per-step calls report it rather than recompute)."""
        if self.status is None:
            return
        h = int(self.status.item())
        self.status.zero_()
        if h & 2:
            raise la_seg.LaSegError(-7, "sequence-parallel step", "a device-side wait gave up")
        if h & 1:
            raise la_seg.LaSegError(-6, "sequence-parallel step",
                                    "a chunk has a positive log_g or |sum of log_g| > 80")


# ----------------------------------------------------------------------------- collectives
class Exchange:
    """Moves (log Gamma, S) pairs between the ranks of `group`."""

    def __init__(self, group=None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.host = dist.get_backend(group) != "nccl"  # gloo: stage CUDA tensors through the host

    def _out(self, t):
        return t.cpu() if (self.host and t.is_cuda) else t

    def all_gather(self, t):
        """[N, *t.shape]: every rank's tensor, in rank order."""
        src = self._out(t.contiguous())
        if self.host:
            parts = [torch.empty_like(src) for _ in range(self.world)]
            dist.all_gather(parts, src, group=self.group)
            return torch.stack(parts).to(t.device)
        out = torch.empty((self.world, *src.shape), dtype=src.dtype, device=src.device)
        dist.all_gather_into_tensor(out, src, group=self.group)
        return out

    def shift(self, tensors, d):
        """Sends `tensors` to rank + d and returns those of rank - d (None at the edges)."""
        ops, recv = [], None
        peer = lambda r: dist.get_global_rank(self.group, r) if self.group is not None else r
        if self.rank + d < self.world:
            ops += [dist.P2POp(dist.isend, self._out(t.contiguous()), peer(self.rank + d), self.group)
                    for t in tensors]
        if self.rank - d >= 0:
            recv = [torch.empty_like(self._out(t)) for t in tensors]
            ops += [dist.P2POp(dist.irecv, r, peer(self.rank - d), self.group) for r in recv]
        if ops:
            for w in dist.batch_isend_irecv(ops):
                w.wait()
        if recv is None:
            return None
        return [r.to(t.device) for r, t in zip(recv, tensors)]

    def broadcast(self, t, src_rank):
        buf = self._out(t.contiguous())
        root = dist.get_global_rank(self.group, src_rank) if self.group is not None else src_rank
        dist.broadcast(buf, root, group=self.group)
        return buf.to(t.device)


def all_scan(steps, ex: Exchange, lg_r, S_r, init, reverse, method):
    """The state this rank's block receives and the scan's total over every rank.

    Forward (reverse = False): S_in = Gamma_{r-1} (... (Gamma_0 init + S_0) ...) + S_{r-1}.
    Reverse: the same from the last rank down (the gradient reaching the block's end).
    """
    N, r = ex.world, ex.rank
    if method == "gather":
        S_all = ex.all_gather(S_r)
        lg_all = ex.all_gather(lg_r)
        return steps.rank_scan(S_all, lg_all, r, init, reverse)
    if method != "tree":
        raise ValueError(f"unknown All-Scan {method!r} (gather or tree)")
    # Hillis-Steele over the ranks in scan order: position s = r (forward) or N-1-r (reverse).
    # After the round with distance d, (lg, S) spans positions s-2d+1 .. s.
    step = -1 if reverse else 1
    lg, S = lg_r, S_r
    d = 1
    while d < N:
        got = ex_shift(ex, (lg, S), d * step)
        if got is not None:
            lg, S = steps.combine(got[0], got[1], lg, S)  # the earlier span first
        d *= 2
    # exclusive prefix: the inclusive one of the previous position; identity at the first
    prev = ex_shift(ex, (lg, S), step)
    first = (r == N - 1) if reverse else (r == 0)
    if prev is None:  # the first position receives init (or zero) itself
        S_in = init.clone() if init is not None else torch.zeros_like(S_r)
    elif init is None:
        S_in = prev[1]
    else:
        S_in = steps.combine(torch.zeros_like(lg_r), init, prev[0], prev[1])[1]
    assert first == (prev is None)
    # the total: the last position's inclusive span, applied to init, on every rank
    last = 0 if reverse else N - 1
    lg_t, S_t = ex.broadcast(lg, last), ex.broadcast(S, last)
    total = S_t if init is None else steps.combine(torch.zeros_like(lg_r), init, lg_t, S_t)[1]
    return S_in, total


def ex_shift(ex: Exchange, tensors, d):
    """Exchange.shift with a signed distance (negative: towards lower ranks)."""
    if d >= 0:
        return ex.shift(list(tensors), d)
    # mirror: send to rank - |d|, receive from rank + |d|
    flipped = _Mirror(ex)
    return flipped.shift(list(tensors), -d)


class _Mirror(Exchange):
    """The same group with its ranks in reverse order (for the reverse All-Scan's shifts)."""

    def __init__(self, ex: Exchange):
        self.group, self.world, self.host = ex.group, ex.world, ex.host
        self.rank = ex.world - 1 - ex.rank

    def shift(self, tensors, d):
        ops, recv = [], None
        real = lambda m: (self.world - 1 - m)
        peer = lambda m: dist.get_global_rank(self.group, real(m)) if self.group is not None else real(m)
        if self.rank + d < self.world:
            ops += [dist.P2POp(dist.isend, self._out(t.contiguous()), peer(self.rank + d), self.group)
                    for t in tensors]
        if self.rank - d >= 0:
            recv = [torch.empty_like(self._out(t)) for t in tensors]
            ops += [dist.P2POp(dist.irecv, r_, peer(self.rank - d), self.group) for r_ in recv]
        if ops:
            for w in dist.batch_isend_irecv(ops):
                w.wait()
        if recv is None:
            return None
        return [r_.to(t.device) for r_, t in zip(recv, tensors)]


# ----------------------------------------------------------------------------- forward / backward
@dataclass
class Saved:
    """What the backward reuses from the forward on this rank."""
    S_recv: torch.Tensor   # fp32 [B, H, NS, dk, dv]: the state each of the rank's NS sub-segments
                           # receives (the library's split of its P segments)
    S_end: torch.Tensor    # fp32 [B, H, dk, dv]: the state after the rank's last token


def _dt(t):
    return la_seg.LA_F32 if t.dtype == torch.float32 else la_seg.LA_BF16


def sp_forward(q, k, v, log_g, S0=None, P=1, chunk=64, *, group=None, method="gather",
               steps=None, check=True):
    """o (this rank's block), S_final (the whole sequence's, on every rank), Saved.

    q, k, log_g [B, H, L, dk], v [B, H, L, dv]: this rank's block of every sequence.  S0 (fp32
    [B, H, dk, dv], the sequence's initial state) is given on every rank or on none (every rank
    takes the same collective steps); it enters the scan at rank 0.  P segments per rank.
    check: read the kernels' status word at the end (a host synchronisation)."""
    steps = steps or LibrarySteps()
    ex = Exchange(group)
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    NS = steps.subsegments(B, H, L, dk, dv, P, chunk, _dt(q))
    if NS == 0:
        raise la_seg.LaSegError(-2, "sp_forward", "sizes rejected by the library")
    S_loc, lg = steps.state_pass(k, v, log_g, NS, chunk)
    _, S_r, _ = steps.scan(S_loc, lg, None, False)          # the block from a zero start
    lg_r = steps.log_gamma_total(lg)                       # the block's log-decay
    init = S0
    S_in, S_final = all_scan(steps, ex, lg_r, S_r, init, False, method) if ex.world > 1 else \
        ((init if init is not None else torch.zeros_like(S_r)), None)
    S_recv, S_end, _ = steps.scan(S_loc, lg, S_in, False)
    if ex.world == 1:
        S_final = S_end
    o = steps.output_pass(q, k, v, log_g, S_recv, NS, chunk)
    if check:
        steps.check()
    return o, S_final, Saved(S_recv, S_end)  # the backward reuses them on the same split


def sp_backward(q, k, v, log_g, dO, saved: Saved, dS_final=None, P=1, chunk=64, *, group=None,
                method="gather", steps=None, check=True):
    """dq, dk, dv, dlog_g of this rank's block and dS0 (on every rank) for
    loss = <o, dO> + <S_final, dS_final> over the whole sequence.  dS_final (fp32
    [B, H, dk, dv]) is given on every rank or on none; it enters the reverse scan at the last
    rank."""
    steps = steps or LibrarySteps()
    ex = Exchange(group)
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    NS = saved.S_recv.shape[2]
    NPF = steps.backward_parts(B, H, L, dk, dv, NS, chunk, _dt(q))
    fine = NPF // NS
    dq, qdq, S_fine, dSloc, lgf = steps.dq_pass(q, k, v, log_g, dO, saved.S_recv, NS, fine, chunk)
    _, G_r, _ = steps.scan(dSloc, lgf, None, True)          # the block's start, from within it
    lg_r = steps.log_gamma_total(lgf)
    init = dS_final
    if ex.world > 1:
        dX_end, dS0 = all_scan(steps, ex, lg_r, G_r, init, True, method)
    else:
        dX_end, dS0 = (init if init is not None else torch.zeros_like(G_r)), None
    dX, dS_start, carry = steps.scan(dSloc, lgf, dX_end, True, S_next=S_fine, S_last=saved.S_end)
    if ex.world == 1:
        dS0 = dS_start
    dk_, dv_, dg = steps.dkv_pass(q, k, v, log_g, dO, S_fine, dX, qdq, NPF, chunk, carry)
    if check:
        steps.check()
    return dq, dk_, dv_, dg, dS0
