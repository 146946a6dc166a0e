"""Benchmark: segmented chunkwise gated linear attention on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload C1] [--schedule auto]
    python bench.py --impl reference ...      # the fp64 CPU oracle on this host's cores

A step is one pass of the whole path over one batch of the workload: la_seg_forward over the
workload's P segments, saving the states they receive, and for a fwd+bwd workload
la_seg_backward reusing them -- the calls a user makes, through the library's C ABI on the
current stream.  Inputs are resident in HBM and L2 is flushed (256 MiB write, untimed) before
every step; each step is bracketed by CUDA events.  The same kernels are also run through the
per-step entry points with events between the phases (checked bit for bit against the public
calls), which gives each kernel's time and roofline.  After the headline workload the forward
workloads C1-C3 are timed the same way into the line's "configs".
With N > 1 ranks (torchrun) the default is sequence parallelism across the ranks (sp.py, the
pages' setting): rank r holds block r of a global sequence of N x L tokens and the ranks
exchange their (log Gamma, S) pairs over NCCL between the passes ("weak" scaling: the tokens per
rank are fixed); --mode replicas runs independent copies instead.  The max over ranks of the
device time is reported.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

from sequence_linear_attention_chunked_b200.inputs import WORKLOADS, Workload, make_inputs  # noqa: E402

METRIC = "tokens/sec of gated linear attn fwd(+bwd) at 1 B200; % bf16 TC peak / % HBM BW"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- helpers
def max_over_ranks(value: float, world: int, device) -> float:
    """The largest of every rank's value: the job's device time is its slowest rank's."""
    t = torch.tensor([value], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step: float, world: int, steps: int, job_ms: float) -> float:
    """Units all ranks processed (each rank runs its own replica) per second of job time."""
    return units_per_rank_step * world * steps / (job_ms / 1e3)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# The sources each kernel's code is built from: a counter recorded for a kernel stays valid
# while these are unchanged (comments and whitespace aside).
KERNEL_SOURCES = {
    "dkv_pass": ["tc_bwd.cu"], "dq_pass": ["tc_dq.cu"], "state_pass": ["tc_pass.cu"],
    "output_pass": ["tc_pass.cu"], "local_pass": ["tc_pass.cu"], "correct_pass": ["tc_pass.cu"],
    "chain_kernel": ["tc_pass.cu"], "scan": ["scan.cu"],
}
SHARED_SOURCES = ["common.cuh", "internal.h", "tc_common.cuh", "sm100.cuh"]


def csrc_digest(kernel=None) -> str:
    """Digest of the code (comments and whitespace left out) of `kernel`'s sources and the
    headers every kernel shares, or of every source when kernel is None."""
    import re
    d = os.path.join(ROOT, "sequence_linear_attention_chunked_b200", "csrc")
    names = sorted(os.listdir(d)) if kernel is None else sorted(
        KERNEL_SOURCES.get(kernel, []) + SHARED_SOURCES)
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(d, name), encoding="utf-8") as f:
            src = f.read()
        code = re.sub(r"//[^\n]*|/\*.*?\*/", " ", src, flags=re.S)
        h.update(name.encode() + " ".join(code.split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it still matches the source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{kernel}@{workload}")
    if not e or e.get("csrc_digest") != csrc_digest(kernel):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, interval_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.interval = interval_s
        self._stop = threading.Event()
        self._thr = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                hi = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(hi)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    h = hi
            self.nvml, self.h = pynvml, h
            if h is not None:
                self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report no clocks rather than guess
            self.nvml, self.h, self.error = None, None, repr(e)

    def _run(self):
        while not self._stop.is_set():
            self.sample_once()
            time.sleep(self.interval)

    def sample_once(self):
        if self.h is None:
            return
        try:
            mhz = self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM)
            r = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            return
        self.samples.append(mhz)
        for bit, name in self.REASONS.items():
            if r & bit and name != "gpu_idle":
                self.reasons.add(name)

    def __enter__(self):
        self.sample_once()
        self._thr = threading.Thread(target=self._run, daemon=True)
        self._thr.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thr:
            self._thr.join()
        self.sample_once()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------- our arm
def dtype_code(la_seg, w):
    return la_seg.LA_F32 if w.dtype == "f32" else la_seg.LA_BF16


class Public:
    """The calls a user of the library makes for the workload, through the C ABI on the current
    stream: for a forward-only workload la_seg_forward over its P segments; for fwd+bwd the
    training pair, la_seg_train_forward over the P segments saving the received states at the
    library's own split, then la_seg_train_backward reusing them.  This is what the headline
    times."""

    def __init__(self, w: Workload, x, schedule: int, device):
        from sequence_linear_attention_chunked_b200 import la_seg
        self.la, self.w, self.x, self.schedule = la_seg, w, x, schedule
        dt = dtype_code(la_seg, w)
        f32 = dict(dtype=torch.float32, device=device)
        self.o = torch.empty((w.B, w.H, w.L, w.dv), dtype=w.torch_dtype, device=device)
        self.S_final = torch.empty((w.B, w.H, w.dk, w.dv), **f32)
        self.S_save = None
        if w.backward:
            NS = la_seg.lib().la_seg_train_saved_states(w.B, w.H, w.L, w.dk, w.dv, w.P, w.chunk, dt)
            self.ws = la_seg.train_workspace(w.B, w.H, w.L, w.dk, w.dv, w.P, w.chunk, dt, False, device)
            self.wsb = la_seg.train_workspace(w.B, w.H, w.L, w.dk, w.dv, w.P, w.chunk, dt, True, device)
            self.S_save = torch.empty((w.B, w.H, NS, w.dk, w.dv), **f32)
            self.grads = (torch.empty_like(x["q"]), torch.empty_like(x["k"]), torch.empty_like(x["v"]),
                          torch.empty_like(x["log_g"]), torch.empty_like(self.S_final))
        else:
            self.ws = la_seg.workspace(w.B, w.H, w.L, w.dk, w.dv, w.P, w.chunk, dt, False, device)
        self.ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        # kernels of this library per step: state pass, exact-path states, scan, output pass,
        # exact-path outputs; dq sweep, exact-path dq, reverse scan, dk/dv sweep, exact-path
        # dk/dv (the status / flag memsets are not counted)
        self.launches_per_step = 5 + (5 if w.backward else 0)

    def run(self, record=True):
        la, w, x, P = self.la, self.w, self.x, self.la._ptr
        st = la._stream(None)
        dt = dtype_code(la, w)
        if record:
            self.ev[0].record()
        fwd = la.lib().la_seg_train_forward if w.backward else la.lib().la_seg_forward
        la._check(fwd(
            P(x["q"]), P(x["k"]), P(x["v"]), P(x["log_g"]), None, w.B, w.H, w.L, w.dk, w.dv, w.P,
            w.chunk, dt, P(self.o), P(self.S_final), P(self.S_save), self.schedule, P(self.ws),
            self.ws.numel(), st), "forward")
        if w.backward:
            g = self.grads
            la._check(la.lib().la_seg_train_backward(
                P(x["q"]), P(x["k"]), P(x["v"]), P(x["log_g"]), None, P(self.S_save), P(x["dO"]),
                None, w.B, w.H, w.L, w.dk, w.dv, w.P, w.chunk, dt, P(g[0]), P(g[1]), P(g[2]),
                P(g[3]), P(g[4]), P(self.wsb), self.wsb.numel(), st), "la_seg_train_backward")
        if record:
            self.ev[1].record()

    def ms(self):
        return self.ev[0].elapsed_time(self.ev[1])

    def check_status(self):
        self.la.la_seg_check_status(self.ws)
        if self.w.backward:
            self.la.la_seg_check_status(self.wsb)


class Step:
    """The same device work as Public, composed of the C ABI's per-step entry points with CUDA
    events between the phases on the launching stream, so that each kernel can be timed and
    set against its roofline.  It reproduces the public calls' splits: the forward's passes over
    the library's sub-segments (state pass, state scan, output pass -- or the other schedules'
    passes); the backward, which reuses the received states the training forward saved at the
    same split: dq pass (which also forms the gradient states of the fine parts), reverse scan,
    dk/dv/dlog_g pass.  bench_ours checks that both give the same bits."""

    KERNEL_KEYS = {"chain reset": "chain_reset", "single pass": "chain_kernel",
                   "state pass": "state_pass", "output pass": "output_pass",
                   "local pass": "local_pass", "correction pass": "correct_pass",
                   "state scan": "scan", "dq pass": "dq_pass",
                   "reverse scan": "scan", "dkv pass": "dkv_pass"}

    def __init__(self, w: Workload, x, schedule: str, device):
        from sequence_linear_attention_chunked_b200 import la_seg
        self.la = la_seg
        self.w, self.x, self.dev = w, x, device
        dt = dtype_code(la_seg, w)
        self.NP = la_seg.la_seg_subsegments(w.B, w.H, w.L, w.dk, w.dv, w.P, w.chunk, dt)
        self.m = self.NP // w.P
        self.schedule = schedule
        B, H, L, dk, dv, NP = w.B, w.H, w.L, w.dk, w.dv, self.NP
        f32 = dict(dtype=torch.float32, device=device)
        self.o = torch.empty((B, H, L, dv), dtype=w.torch_dtype, device=device)
        self.S_loc = torch.empty((B, H, NP, dk, dv), **f32)
        self.logG = torch.empty((B, H, NP, dk), **f32)
        self.S_recv = torch.empty((B, H, NP, dk, dv), **f32)
        self.S_final = torch.empty((B, H, dk, dv), **f32)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        if schedule == "single":  # the same sub-segments; S_recv saved for the backward
            self.phases = ["chain reset", "single pass"]
            self.chain = la_seg.chain_buffers(B, H, dk, dv, device)
        elif schedule == "three":
            self.phases = ["local pass", "state scan", "correction pass"]
        elif schedule == "overlap":  # the scan on a second stream beside the local pass
            self.phases = ["state pass", "local pass", "correction pass", "state scan"]
            lo, hi = torch.cuda.Stream.priority_range()
            self.side = torch.cuda.Stream(device=device, priority=hi)
            self.fork, self.join = torch.cuda.Event(), torch.cuda.Event()
            self.scan_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        else:
            self.phases = ["state pass", "state scan", "output pass"]
        self.n_fwd = len(self.phases)
        if w.backward:
            # la_seg_train_backward: the library's sub-segments, each cut into fine parts
            self.NPD = NP
            self.NPF = la_seg.la_seg_backward_parts(w.B, w.H, w.L, w.dk, w.dv, NP, w.chunk, dt,
                                                    True)
            self.fine = self.NPF // self.NPD
            self.phases += ["dq pass", "reverse scan", "dkv pass"]
            NPF = self.NPF
            self.S_fine = torch.empty((B, H, NPF, dk, dv), **f32)
            self.dSloc = torch.empty((B, H, NPF, dk, dv), **f32)
            self.logG_b = torch.empty((B, H, NPF, dk), **f32)
            self.dX = torch.empty((B, H, NPF, dk, dv), **f32)
            self.carry = torch.empty((B, H, NPF, dk), **f32)  # the parts' dlog_g carries
            self.dS0 = torch.empty_like(self.S_final)
            self.grads = (torch.empty_like(x["q"]), torch.empty_like(x["k"]), torch.empty_like(x["v"]),
                          torch.empty_like(x["log_g"]))
            self.qdq = torch.empty((B, H, L, dk), **f32)
        # events between consecutive phases on the launching stream (the overlap schedule times
        # its scan on the side stream and spends that event after its join instead)
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(len(self.phases) + 1)]
        self.launches_per_step = len(self.phases)

    def run(self, record=True):
        la, x, w, NP = self.la, self.x, self.w, self.NP
        ev = self.events
        rec = (lambda i: ev[i].record()) if record else (lambda i: None)
        BH = w.B * w.H
        rec(0)
        if self.schedule == "overlap":
            la.la_seg_state_pass(x["k"], x["v"], x["log_g"], NP, w.chunk, S_loc=self.S_loc,
                                 log_gamma=self.logG, status=self.status)
            rec(1)
            cur = torch.cuda.current_stream()
            self.fork.record(cur)
            self.side.wait_event(self.fork)
            if record:
                self.scan_ev[0].record(self.side)
            la._check(la.lib().la_seg_scan(la._ptr(self.S_loc), la._ptr(self.logG), None, BH, NP,
                                           w.dk, w.dv, 0, la._ptr(self.S_recv),
                                           la._ptr(self.S_final), None, None, None,
                                           la._ptr(self.status), la._stream(self.side)),
                      "la_seg_scan")
            if record:
                self.scan_ev[1].record(self.side)
            self.join.record(self.side)
            la.la_seg_local_pass(x["q"], x["k"], x["v"], x["log_g"], NP, w.chunk, o=self.o,
                                 want_states=False, status=self.status)
            rec(2)
            cur.wait_event(self.join)
            rec(3)
            la.la_seg_correct_pass(x["q"], x["log_g"], self.S_recv, NP, w.chunk, self.o,
                                   status=self.status)
            rec(4)
        elif self.schedule == "single":
            la.la_seg_chain_reset(None, w.B, w.H, w.dk, w.dv, *self.chain)
            rec(1)
            la.la_seg_chain_pass(x["q"], x["k"], x["v"], x["log_g"], NP, w.chunk, *self.chain,
                                 o=self.o, S_final=self.S_final, S_recv_save=self.S_recv,
                                 save_every=1, status=self.status)
            rec(2)
        else:
            if self.schedule != "three":
                la.la_seg_state_pass(x["k"], x["v"], x["log_g"], NP, w.chunk, S_loc=self.S_loc,
                                     log_gamma=self.logG, status=self.status)
            else:
                la.la_seg_local_pass(x["q"], x["k"], x["v"], x["log_g"], NP, w.chunk, o=self.o,
                                     S_loc=self.S_loc, log_gamma=self.logG, status=self.status)
            rec(1)
            la._check(la.lib().la_seg_scan(la._ptr(self.S_loc), la._ptr(self.logG), None, BH, NP,
                                           w.dk, w.dv, 0, la._ptr(self.S_recv),
                                           la._ptr(self.S_final), None, None, None,
                                           la._ptr(self.status), la._stream(None)), "la_seg_scan")
            rec(2)
            if self.schedule != "three":
                la.la_seg_output_pass(x["q"], x["k"], x["v"], x["log_g"], self.S_recv, NP,
                                      w.chunk, o=self.o, status=self.status)
            else:
                la.la_seg_correct_pass(x["q"], x["log_g"], self.S_recv, NP, w.chunk, self.o,
                                       status=self.status)
            rec(3)
        if not w.backward:
            return
        f = self.n_fwd - 1
        la.la_seg_dq_pass(x["q"], x["k"], x["v"], x["log_g"], x["dO"], self.S_recv, self.NPD,
                          self.fine, w.chunk, dq=self.grads[0], qdq=self.qdq, S_fine=self.S_fine,
                          dSloc=self.dSloc, log_gamma=self.logG_b, status=self.status)
        rec(f + 2)
        NPF = self.NPF
        la._check(la.lib().la_seg_scan(la._ptr(self.dSloc), la._ptr(self.logG_b), None, BH, NPF,
                                       w.dk, w.dv, 1, la._ptr(self.dX), la._ptr(self.dS0),
                                       la._ptr(self.S_fine), None, la._ptr(self.carry),
                                       la._ptr(self.status), la._stream(None)), "la_seg_scan")
        rec(f + 3)
        la.la_seg_dkv_pass(x["q"], x["k"], x["v"], x["log_g"], x["dO"], self.S_fine, None, self.dX,
                           self.qdq, NPF, w.chunk, carry=self.carry, out=self.grads[1:],
                           status=self.status)
        rec(f + 4)

    def phase_ms(self):
        ev = self.events
        if self.schedule != "overlap":
            return [ev[i].elapsed_time(ev[i + 1]) for i in range(len(self.phases))]
        fwd = [ev[0].elapsed_time(ev[1]), ev[1].elapsed_time(ev[2]), ev[3].elapsed_time(ev[4]),
               self.scan_ev[0].elapsed_time(self.scan_ev[1])]
        return fwd + [ev[4 + i].elapsed_time(ev[5 + i]) for i in range(len(self.phases) - 4)]

    def overlap_fraction(self):
        """Share of the scan's window (side stream) that the local pass's window (launching
        stream) covers, from CUDA events on both streams (ZeCO review, skeptic critique's
        concrete test)."""
        ev, se = self.events, self.scan_ev
        s0, s1 = ev[0].elapsed_time(se[0]), ev[0].elapsed_time(se[1])
        l0, l1 = ev[0].elapsed_time(ev[1]), ev[0].elapsed_time(ev[2])
        return max(0.0, min(s1, l1) - max(s0, l0)) / max(s1 - s0, 1e-9)

    def algorithmic_bytes(self):
        """Bytes each phase must move at minimum (inputs read once, outputs written once)."""
        w = self.w
        e = 4 if w.dtype == "f32" else 2
        th = w.B * w.H * w.L
        st = w.B * w.H * self.NP * w.dk * w.dv * 4
        lg = w.B * w.H * self.NP * w.dk * 4
        fin = w.B * w.H * w.dk * w.dv * 4
        scan = 2 * st + lg + fin
        if self.schedule == "single":  # inputs read once, o and the saved states written once
            ab = {"chain reset": 2 * w.B * w.H * w.dk * w.dv * 4,
                  "single pass": th * (3 * w.dk + 2 * w.dv) * e + st + fin}
        elif self.schedule == "overlap":  # the local pass writes o only
            ab = {"state pass": th * (2 * w.dk + w.dv) * e + st + lg,
                  "local pass": th * (3 * w.dk + 2 * w.dv) * e,
                  "correction pass": th * (2 * w.dk + 2 * w.dv) * e + st, "state scan": scan}
        elif self.schedule != "three":
            ab = {"state pass": th * (2 * w.dk + w.dv) * e + st + lg, "state scan": scan,
                  "output pass": th * (3 * w.dk + 2 * w.dv) * e + st}
        else:
            ab = {"local pass": th * (3 * w.dk + 2 * w.dv) * e + st + lg, "state scan": scan,
                  "correction pass": th * (2 * w.dk + 2 * w.dv) * e + st}
        if w.backward:
            sts = st
            stf = w.B * w.H * self.NPF * w.dk * w.dv * 4
            lgf = w.B * w.H * self.NPF * w.dk * 4
            # reads q, k, v, dO, log_g and the received states; writes dq, S_fine, dSloc and
            # log_gamma (the fp32 q . dq hand-over to the dkv pass is not counted)
            ab["dq pass"] = th * (3 * w.dk + 2 * w.dv + w.dk) * e + sts + 2 * stf + lgf
            carry = w.B * w.H * self.NPF * w.dk * 4
            # reverse scan: the parts' gradient states in, their end-state gradients out, and the
            # dlog_g carries (end states read, one float per part and key dim written)
            ab["reverse scan"] = 3 * stf + lgf + fin + carry
            ab["dkv pass"] = th * (3 * w.dk + 2 * w.dv + 2 * w.dk + w.dv) * e + stf + carry
        return ab

    def flops(self):
        w = self.w
        th = w.B * w.H * w.L
        C, dk, dv = w.chunk, w.dk, w.dv
        intra = 2 * C * dk + 2 * C * dv  # QK^T and PV on full chunk tiles
        dd = 2 * dk * dv                 # one state-sized contraction per token
        if self.schedule == "single":
            fl = {"chain reset": 0, "single pass": th * (intra + 3 * dd)}
        elif self.schedule == "overlap":
            fl = {"state pass": th * dd, "local pass": th * (intra + 2 * dd),
                  "correction pass": th * dd, "state scan": 0}
        elif self.schedule != "three":
            fl = {"state pass": th * dd, "state scan": 0, "output pass": th * (intra + 2 * dd)}
        else:
            fl = {"local pass": th * (intra + 2 * dd), "state scan": 0, "correction pass": th * dd}
        if w.backward:
            fl["dq pass"] = th * (2 * C * dv + 2 * C * dk + 3 * dd)
            fl["reverse scan"] = 0
            fl["dkv pass"] = th * (3 * dd + 2 * C * (3 * dk + 2 * dv))
        return fl


SCHEDULE_CODES = {"auto": 0, "two": 1, "three": 2, "single": 3, "overlap": 4}


def check_same_bits(pub: Public, step: Step):
    """The composition must reproduce the public calls bit for bit."""
    w = pub.w
    pairs = [("o", pub.o, step.o), ("S_final", pub.S_final, step.S_final)]
    if w.backward:
        pairs += [("saved states", pub.S_save, step.S_recv)]
        pairs += [(n, a, b) for n, a, b in zip(("dq", "dk", "dv", "dlog_g"), pub.grads[:4], step.grads)]
        pairs += [("dS0", pub.grads[4], step.dS0)]
    bad = [n for n, a, b in pairs if not torch.equal(a, b)]
    if bad:
        raise RuntimeError(f"per-step composition differs from the public calls in {bad}")


def time_workload(w: Workload, args, device, world, steps: int, warmup: int):
    """Times the public calls (the throughput) and the per-step composition (the phases) on
    the workload, each step after an untimed L2 flush; returns the pieces of the JSON line."""
    x = make_inputs(w, device)
    pub = Public(w, x, SCHEDULE_CODES[args.schedule], device)
    step = Step(w, x, args.schedule, device)
    pub.run(record=False)
    pub.check_status()
    step.run(record=False)
    torch.cuda.synchronize()
    check_same_bits(pub, step)
    if int(step.status.item()) != 0:
        raise RuntimeError(f"device status {int(step.status.item())} after the check run")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    for _ in range(warmup):
        flush.zero_()
        pub.run()
        flush.zero_()
        step.run()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    pub_ms, step_ms, phase_ms, overlap = [], [], [], []
    # the headline steps first, on their own (the composition's extra work would heat the chip
    # between them), with the SM clock sampled while they run
    sampler = ClockSampler(device.index)
    with sampler:
        for _ in range(steps):
            flush.zero_()
            pub.run()
            torch.cuda.synchronize()  # read this step's events before the next one reuses them
            pub_ms.append(pub.ms())
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    comp_sampler = ClockSampler(device.index)
    with comp_sampler:
        for _ in range(steps):  # then the composition, for the phases
            flush.zero_()
            step.run()
            torch.cuda.synchronize()
            phase_ms.append(step.phase_ms())
            step_ms.append(step.events[0].elapsed_time(step.events[-1]))
            if args.schedule == "overlap":
                overlap.append(step.overlap_fraction())
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    total_ms = max_over_ranks(sum(pub_ms), world, device)
    comp_ms = max_over_ranks(sum(step_ms), world, device)
    value = job_throughput(w.B * w.L, world, steps, total_ms)

    mean_phase = [statistics.fmean(p[i] for p in phase_ms) for i in range(len(step.phases))]
    ab = step.algorithmic_bytes()
    fl = step.flops()
    peaks, peak_src = load_peaks()
    dom = max(range(len(step.phases)), key=lambda i: mean_phase[i])
    dname = step.phases[dom]
    achieved = ab[dname] / (mean_phase[dom] / 1e3) / 1e9
    phases = {}
    for i, name in enumerate(step.phases):
        sec = mean_phase[i] / 1e3
        phases[name] = {"ms": round(mean_phase[i], 5), "GB/s": round(ab[name] / sec / 1e9, 1),
                        "hbm_frac": round(ab[name] / sec / 1e9 / peaks["hbm_gbs"], 4),
                        "TFLOP/s": round(fl[name] / sec / 1e12, 2),
                        "tc_frac": round(fl[name] / sec / 1e12 / peaks["bf16_tflops"], 4)}
    roofline = {"bound": "hbm", "kernel": dname, "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "peak_source": f"{peak_src} hbm_gbs (burst copy)",
                "algorithmic_bytes_per_launch": ab[dname],
                "traffic": ncu_traffic(Step.KERNEL_KEYS[dname], w.name)}
    out = dict(x=x, pub=pub, step=step, value=value, total_ms=total_ms, comp_ms=comp_ms,
               pub_ms=pub_ms, phases=phases, roofline=roofline, sampler=sampler,
               comp_sampler=comp_sampler, mean_phase=mean_phase)
    if overlap:  # events on both streams: the scan's window and the local pass's
        out["overlap"] = {"scan_window_covered": round(statistics.median(overlap), 4),
                          "min": round(min(overlap), 4),
                          "scan_ms": round(mean_phase[step.phases.index("state scan")], 5),
                          "local_pass_ms": round(mean_phase[step.phases.index("local pass")], 5)}
    return out


def _clock_ratio(r):
    a, b = r["comp_sampler"].summary()["sm_mhz"], r["sampler"].summary()["sm_mhz"]
    if not a or not b:
        return None
    return round((r["comp_ms"] * a) / (r["total_ms"] * b), 4)


def bench_ours(args, rank, world, device):
    w = WORKLOADS[args.workload]
    r = time_workload(w, args, device, world, args.steps, args.warmup)
    step, pub = r["step"], r["pub"]
    line = {"metric": METRIC, "value": round(r["value"], 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(r["total_ms"] / args.steps, 5),
            "ms_per_step_median": round(statistics.median(r["pub_ms"]), 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": {"workload": w.describe(), "B": w.B, "H": w.H, "L": w.L, "d": w.dk, "P": w.P,
                       "chunk": w.chunk, "subsegments": step.NP, "schedule": args.schedule,
                       "timed": ("la_seg_train_forward(P, saving the received states at the "
                                 "library's split) + la_seg_train_backward(P, reusing them)")
                                if w.backward else "la_seg_forward(P)",
                       "l2": "flushed before every step (256 MiB write, untimed)",
                       "parallelism": f"replicas x{world}"},
            "composed": {"ms_per_step": round(r["comp_ms"] / args.steps, 5),
                         "vs_public": round(r["comp_ms"] / r["total_ms"], 4),
                         "sm_mhz": r["comp_sampler"].summary()["sm_mhz"],
                         # time x median SM clock: the two loops run one after the other, and the
                         # later one under more of the power cap
                         "vs_public_at_equal_clock": _clock_ratio(r),
                         "what": "the same kernels through the per-step entry points, bit-identical "
                                 "results; phases and roofline come from it"},
            "phases": r["phases"], "roofline": r["roofline"],
            "gpu_launches": pub.launches_per_step * args.steps,
            "clocks": r["sampler"].summary()}
    if "overlap" in r:
        line["overlap"] = r["overlap"]
    x = r["x"]
    if not args.no_e2e:
        line["e2e"] = bench_e2e(args, w, x, device, world)
    del r, x, step, pub
    torch.cuda.empty_cache()
    configs = [c for c in args.configs.split(",") if c and c != "none" and c != w.name]
    if configs:
        line["configs"] = {}
    for name in configs:
        cw = WORKLOADS[name]
        rc = time_workload(cw, args, device, world, args.config_steps, 3)
        entry = {"workload": cw.describe(), "tokens_per_s": round(rc["value"], 1),
                 "ms_per_step": round(rc["total_ms"] / args.config_steps, 5),
                 "composed_ms_per_step": round(rc["comp_ms"] / args.config_steps, 5),
                 "steps": args.config_steps, "phases": rc["phases"],
                 "roofline": {k: rc["roofline"][k] for k in ("kernel", "achieved", "frac", "unit")},
                 "clocks": rc["sampler"].summary()}
        if "state scan" in rc["phases"]:
            entry["scan"] = rc["phases"]["state scan"]
        line["configs"][name] = entry
        del rc
        torch.cuda.empty_cache()
    return line


def bench_sp(args, rank, world, device):
    """Sequence parallelism across the ranks (sp.py): rank r holds block r of every sequence of a
    global sequence of world x L tokens (the workload's L per rank, ZeCO's fixed tokens per
    device), runs the forward and backward passes on it, and the ranks exchange their (log Gamma,
    S) pairs over NCCL (all-gather, or the tree All-Scan).  The job time is the slowest rank's."""
    from sequence_linear_attention_chunked_b200 import sp
    w = WORKLOADS[args.workload]
    x = make_inputs(w.with_(seed=w.seed + rank), device)
    steps = sp.LibrarySteps()

    def one(check=False):
        o, Sf, saved = sp.sp_forward(x["q"], x["k"], x["v"], x["log_g"], None, w.P, w.chunk,
                                     method=args.all_scan, steps=steps, check=check)
        if w.backward:
            sp.sp_backward(x["q"], x["k"], x["v"], x["log_g"], x["dO"], saved, None, w.P, w.chunk,
                           method=args.all_scan, steps=steps, check=check)

    one(check=True)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    for _ in range(args.warmup):
        flush.zero_()
        one()
    torch.cuda.synchronize()
    dist.barrier()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ms = []
    sampler = ClockSampler(device.index)
    with sampler:
        for _ in range(args.steps):
            flush.zero_()
            dist.barrier()
            ev[0].record()
            one()
            ev[1].record()
            torch.cuda.synchronize()
            ms.append(ev[0].elapsed_time(ev[1]))
    steps.check()
    dist.barrier()
    total_ms = max_over_ranks(sum(ms), world, device)
    value = job_throughput(w.B * w.L, world, args.steps, total_ms)
    # the kernels' phases and roofline: the same workload through the per-step entry points on
    # every rank's own block (one GPU's work)
    r = time_workload(w, args, device, world, max(3, min(args.steps, 10)), 3)
    line = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 5),
            "ms_per_step_median": round(statistics.median(ms), 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": {"workload": w.describe() + f" per rank; global sequence {world} x {w.L}",
                       "B": w.B, "H": w.H, "L_per_rank": w.L, "L_global": world * w.L, "d": w.dk,
                       "P_per_rank": w.P, "chunk": w.chunk, "all_scan": args.all_scan,
                       "timed": "sp_forward" + (" + sp_backward" if w.backward else "") +
                                " (sequence parallel across the ranks, NCCL)",
                       "l2": "flushed before every step (256 MiB write, untimed)",
                       "parallelism": f"sp{world}"},
            "phases": r["phases"], "roofline": r["roofline"],
            # per step: state pass, block total (scan, log-decay sum), All-Scan (one rank scan, or
            # a combine per tree round), the scan from the received state, output pass; dq
            # sweep, block total (scan, log-decay sum), All-Scan, reverse scan, dk/dv sweep
            "gpu_launches": ((6 + (6 if w.backward else 0)) + (0 if args.all_scan == "gather" else
                             (1 + int(w.backward)) * (max(1, (world - 1).bit_length()) - 1))) * args.steps,
            "clocks": sampler.summary()}
    return line


def bench_e2e(args, w, x, device, world):
    """Same metric through the public entry points with host buffers: per step, pinned host ->
    device copies of the inputs (q, k, v, log_g, and dO for fwd+bwd), the headline's calls (the
    training pair for fwd+bwd), and device -> host copies of the
    results (o and S_final; dq, dk, dv, dlog_g and dS0 for fwd+bwd).  Steps are pipelined over
    three streams with two sets of device buffers, as a serving loop would run them: step i's
    inputs are copied in while step i-1 computes and step i-2's results are copied out (PCIe
    moves both directions at once).  Every step copies all of its inputs in and all of its
    results out inside the timed region."""
    from sequence_linear_attention_chunked_b200 import la_seg
    names = ("q", "k", "v", "log_g") + (("dO",) if w.backward else ())
    host = {n: x[n].cpu().pin_memory() for n in names}
    dt = la_seg.LA_F32 if w.dtype == "f32" else la_seg.LA_BF16
    f32 = dict(dtype=torch.float32, device=device)
    mkws = la_seg.train_workspace if w.backward else la_seg.workspace
    ws = [mkws(w.B, w.H, w.L, w.dk, w.dv, w.P, w.chunk, dt, False, device) for _ in range(2)]
    wsb = ([la_seg.train_workspace(w.B, w.H, w.L, w.dk, w.dv, w.P, w.chunk, dt, True, device)
            for _ in range(2)] if w.backward else [None, None])
    NS = la_seg.lib().la_seg_train_saved_states(w.B, w.H, w.L, w.dk, w.dv, w.P, w.chunk, dt)
    bufs = []
    for _ in range(2):  # two sets of device inputs and outputs
        d = {n: torch.empty_like(x[n]) for n in names}
        o_dev = torch.empty((w.B, w.H, w.L, w.dv), dtype=w.torch_dtype, device=device)
        Sf = torch.empty((w.B, w.H, w.dk, w.dv), **f32)
        Sr = torch.empty((w.B, w.H, NS, w.dk, w.dv), **f32) if w.backward else None
        outs = [o_dev, Sf]
        grads = None
        if w.backward:
            grads = [torch.empty_like(x["q"]), torch.empty_like(x["k"]), torch.empty_like(x["v"]),
                     torch.empty_like(x["log_g"]), torch.empty_like(Sf)]
            outs += grads
        bufs.append(dict(inp=d, o=o_dev, Sf=Sf, Sr=Sr, grads=grads, outs=outs,
                         host_out=[torch.empty_like(t, device="cpu").pin_memory() for t in outs]))
    steps = max(3, min(args.steps, 20))
    P = la_seg._ptr
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of a buffer set copied in
    ev_comp = [torch.cuda.Event() for _ in range(2)]   # step done reading inputs, outputs written
    ev_out = [torch.cuda.Event() for _ in range(2)]    # outputs of a buffer set copied out
    used = [False, False]

    def one(i):
        k = i % 2
        bf = bufs[k]
        with torch.cuda.stream(s_in):
            if used[k]:
                s_in.wait_event(ev_comp[k])  # the step two back has read these inputs
            for n in names:
                bf["inp"][n].copy_(host[n], non_blocking=True)
            ev_in[k].record(s_in)
        s_comp.wait_event(ev_in[k])
        if used[k]:
            s_comp.wait_event(ev_out[k])  # the step two back's results are copied out
        st = la_seg._stream(s_comp)
        d = bf["inp"]
        fwd = la_seg.lib().la_seg_train_forward if w.backward else la_seg.lib().la_seg_forward
        la_seg._check(fwd(
            P(d["q"]), P(d["k"]), P(d["v"]), P(d["log_g"]), None, w.B, w.H, w.L, w.dk, w.dv,
            w.P, w.chunk, dt, P(bf["o"]), P(bf["Sf"]), P(bf["Sr"]), 0, P(ws[k]), ws[k].numel(), st),
            "forward")
        if w.backward:
            g = bf["grads"]
            la_seg._check(la_seg.lib().la_seg_train_backward(
                P(d["q"]), P(d["k"]), P(d["v"]), P(d["log_g"]), None, P(bf["Sr"]), P(d["dO"]),
                None, w.B, w.H, w.L, w.dk, w.dv, w.P, w.chunk, dt, P(g[0]), P(g[1]), P(g[2]),
                P(g[3]), P(g[4]), P(wsb[k]), wsb[k].numel(), st), "la_seg_backward")
        ev_comp[k].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[k])
            for dv_, h in zip(bf["outs"], bf["host_out"]):
                h.copy_(dv_, non_blocking=True)
            ev_out[k].record(s_out)
        used[k] = True

    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(steps):
        one(i)
    s_out.wait_event(ev_comp[(steps - 1) % 2])
    e1.record(s_out)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(e0.elapsed_time(e1), world, device)
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = sum(v.numel() * v.element_size() for v in bufs[0]["host_out"])
    api = "la_seg_train_forward + la_seg_train_backward" if w.backward else "la_seg_forward"
    return {"value": round(job_throughput(w.B * w.L, world, steps, ms), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "api": f"{api} (C ABI) with pinned host buffers, steps pipelined over copy-in, "
                   "compute and copy-out streams"}


# ----------------------------------------------------------------------------- oracle arm
def cpu_sample(w: Workload, budget_s: float, steps: int = 0, warmup: int = 0):
    """Times the fp64 oracle on bounded samples of the workload: all B*H heads over the first
    n tokens, n a power of two <= L chosen from a calibration run.  With steps = 0 one sample
    is repeated for about budget_s seconds; otherwise `warmup` untimed and `steps` timed
    samples are run, n sized so that they take about budget_s in total."""
    import oracle

    def run(n):
        xs = make_inputs(w.with_(L=n), "cpu")
        t0 = time.perf_counter()
        oracle.forward(xs["q"], xs["k"], xs["v"], xs["log_g"])
        if w.backward:
            oracle.backward(xs["q"], xs["k"], xs["v"], xs["log_g"], xs["dO"])
        return time.perf_counter() - t0

    cal_n = min(w.L, 256)
    per_token = run(cal_n) / cal_n
    per_sample = budget_s / max(1, steps + warmup) if steps else min(budget_s, 4.0)
    n = cal_n
    while n * 2 <= w.L and per_token * n * 2 <= per_sample:
        n *= 2
    cores = oracle.num_threads()
    if steps:
        for _ in range(warmup):
            run(n)
        el = sum(run(n) for _ in range(steps))
        reps = steps
    else:
        reps, el = 0, 0.0
        while el < budget_s:
            el += run(n)
            reps += 1
    value = w.B * n * reps / el
    return {"value": round(value, 1), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 token-by-token oracle{' fwd+bwd' if w.backward else ''}, all "
                      f"{w.B * w.H} heads x first {n} tokens of {w.name}, {reps} timed samples, "
                      f"{el:.1f} s; tokens/s = B*n*samples/seconds",
            "seconds": round(el, 2)}


def bench_reference(args, w):
    cb = cpu_sample(w, args.cpu_seconds * 6, steps=args.steps, warmup=args.warmup)
    return {"metric": METRIC, "value": cb["value"], "unit": "tokens/s", "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "ms_per_step": round(cb["seconds"] * 1e3 / args.steps, 3),
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": w.describe(), "B": w.B, "H": w.H, "L": w.L, "d": w.dk, "P": w.P,
                       "chunk": w.chunk},
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="C4", choices=sorted(WORKLOADS),
                    help="C4 (fwd+bwd, every step of the path) by default; C0-C3 forward only")
    ap.add_argument("--schedule", default="auto",
                    choices=["auto", "two", "three", "single", "overlap"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--configs", default="C1,C2,C3",
                    help="forward workloads timed after the headline into the line's 'configs' "
                         "('none' to skip)")
    ap.add_argument("--config-steps", type=int, default=10)
    ap.add_argument("--mode", choices=["auto", "replicas", "sp"], default="auto",
                    help="N > 1: sequence parallel across the ranks (sp, the default) or "
                         "independent replicas")
    ap.add_argument("--all-scan", choices=["gather", "tree"], default="gather")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle cpu_baseline leg")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = WORKLOADS[args.workload]

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(bench_reference(args, w)), flush=True)
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    mode = args.mode if args.mode != "auto" else ("sp" if world > 1 else "replicas")
    if mode == "sp" and world == 1:  # the orchestration's collectives on a one-rank group
        import socket
        with socket.socket() as sock:
            sock.bind(("127.0.0.1", 0))
            port = sock.getsockname()[1]
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                                world_size=1, device_id=device)
    try:
        line = bench_sp(args, rank, world, device) if mode == "sp" else bench_ours(args, rank, world, device)
        if rank == 0 and world == 1 and not args.no_cpu:
            line["cpu_baseline"] = cpu_sample(w, args.cpu_seconds)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
