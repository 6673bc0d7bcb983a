#!/usr/bin/env python
"""Benchmark of the one-pass masked attention layer (fwd + bwd) on B200.

One step = the whole hot path over one batch of synthetic conversations:
opr_build_layout -> opr_rope(q), opr_rope(k) -> opr_attn_fwd -> opr_attn_bwd
(row terms, dQ and dK/dV kernels) -> opr_rope(inverse) on dq and dk.

Default workload: the Qwen-3-32B-like fwd+bwd configuration (64 q / 8 kv
heads, head_dim 128, 16 turns per conversation, h~U[64,512], t~U[512,2048],
r~U[128,1024], packed to 65536 tokens), the largest configuration that fits
one GPU.  The line also carries the Qwen-3-8B-like fwd+bwd and Qwen-3-4B-like
forward workloads and the depth sweep (one conversation of 2..16 turns) as
extra keys, each against the same kernels run N-pass.

Metric: useful TFLOP/s = 4 d P Hq (1 + 2.5) / step time, P the visible (q, k)
pairs per head; plus conversation tokens/s (h + t + r per turn, no
duplication) against the same kernels run N-pass.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config C]
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "1-pass masked attn fwd+bwd useful TFLOP/s; conv tokens/s vs N-pass"
UNIT = "TFLOP/s"
DEFAULT_CONFIG = 4
L2_FLUSH_BYTES = 512 << 20
# layout (8), rope of q and k and the fp16 copy of v (3), fwd, bwd (max |dO|, row terms,
# v cast, dq, dkdv), inverse rope x2
KERNELS_PER_STEP = 8 + 3 + 1 + 5 + 2


def kernels_per_step(w) -> int:
    """Library kernels one step launches: one more (the GQA partial sum) when the dK/dV stage
    splits its long columns by q head, which include/opr.h states for a grid below 4 x 148 CTAs
    with GQA and the recommended workspace (which reserves the partials while tiles x Hq <= 4736)."""
    tiles = w.n_seqs * ((w.max_seqlen + 127) // 128)
    split = w.hq > w.hkv and tiles * w.hkv < 4 * 148 and tiles * w.hq <= 4 * 148 * 8
    return KERNELS_PER_STEP + (1 if split else 0)
ORACLE_SAMPLE_TOKENS = 3000  # one-pass tokens of the oracle's sample (cpu_baseline and the reference arm)

# DRAM bytes (read + write) per launch of a kernel, from one ncu capture of
# dram__bytes_read.sum and dram__bytes_write.sum at full size (the capture is
# summarised under profiles/).  A figure holds only for the kernel sources it
# was taken on: the sources' hash is recorded with it and checked at run time.
MEASURED_TRAFFIC = {
    "bwd_dkdv": {
        "config_index": 4,
        "bytes": 23265346560 + 512066560,
        "sources": ["attn_bwd.cu", "attn_common.cuh", "sm100.cuh", "layout.cu", "opr_internal.cuh"],
        "sha256": "2d56eddae8ae839a614b7c25bf15a93698298f9d3b609a247da58566ccbfb24a",
        "capture": "ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum --clock-control none "
                   "-k regex:attn_ -s 9 -c 3 --csv python bench.py --steps 1 --warmup 3 --no-extra --no-e2e "
                   "--no-cpu-baseline --no-npass",
    },
}


def measured_traffic(kernel: str, config_index: int, turns, seed=None):
    """Bytes per launch recorded for this kernel and workload (the default seeded batch), or None
    when absent, stale or measured on another batch."""
    import hashlib

    rec = MEASURED_TRAFFIC.get(kernel)
    if rec is None or rec["config_index"] != config_index or turns is not None or seed is not None:
        return None
    h = hashlib.sha256()
    for f in rec["sources"]:
        with open(os.path.join(ROOT, "block_sparse_masked_segment_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return rec["bytes"] if h.hexdigest() == rec["sha256"] else None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["bf16_tflops"], d.get("bf16_tflops_sustained"), d["hbm_gbs"], "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock and throttle samples every 200 ms while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 8:
                self.samples.append(f)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(s[0]) for s in self.samples if s[0].replace(".", "").isdigit()]
        mx = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in self.samples for i in range(4) if s[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.samples),
                "sm_mhz_min": min(sm) if sm else None}

    def rejected(self) -> bool:
        """A slowdown that invalidates the timing (power capping alone does not)."""
        return any(r in self.summary()["reasons"] for r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"))


# ------------------------------------------------------------------ our path
class Runner:
    """Buffers and calls of one step of the hot path for one workload.

    Two device buffer sets (inputs and gradients) let the end-to-end timing
    overlap one step's host copies with its neighbours' compute; the kernel
    timing uses set 0 with its inputs resident.
    """

    def __init__(self, w: synth.Workload, seed: int, device, forward_only: bool = False):
        import torch

        import block_sparse_masked_segment_b200 as opr
        from block_sparse_masked_segment_b200.pipeline import visible_pairs_closed_form

        self.torch, self.opr, self.w, self.dev = torch, opr, w, device
        self.forward_only = forward_only
        rng = np.random.default_rng(seed)
        n = w.total_tokens
        bf = torch.bfloat16
        host = lambda x: torch.from_numpy(x).to(bf).pin_memory()  # noqa: E731
        self.h_q = host(synth.gaussian(rng, (n, w.hq, w.d)))
        self.h_k = host(synth.gaussian(rng, (n, w.hkv, w.d)))
        self.h_v = host(synth.gaussian(rng, (n, w.hkv, w.d)))
        self.h_do = host(synth.gaussian(rng, (n, w.hq, w.d)))
        self.h_lens = [torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).pin_memory()
                       for a in (w.turn_lens.reshape(-1), w.conv_turn_ptr, w.seq_conv_ptr)]
        self.sets = []
        for _ in range(2):
            self.sets.append({
                "q": self.h_q.to(device), "k": self.h_k.to(device), "v": self.h_v.to(device),
                "do": self.h_do.to(device), "lens": [t.to(device) for t in self.h_lens],
                "grads": (torch.empty((n, w.hq, w.d), dtype=torch.float32, device=device),
                          torch.empty((n, w.hkv, w.d), dtype=torch.float32, device=device),
                          torch.empty((n, w.hkv, w.d), dtype=torch.float32, device=device))})
        self.q_rot = torch.empty(self.h_q.shape, dtype=torch.float16, device=device)
        self.k_rot = torch.empty(self.h_k.shape, dtype=torch.float16, device=device)
        self.v16 = torch.empty(self.h_v.shape, dtype=torch.float16, device=device)
        self.h_grads = tuple(torch.empty(g.shape, dtype=g.dtype).pin_memory() for g in self.sets[0]["grads"])
        self.bwd_ws = torch.empty(max(opr.opr_attn_bwd_workspace_bytes(w.n_seqs, w.max_seqlen, w.hq, w.d), 256),
                                  dtype=torch.uint8, device=device)
        self.total, self.max_seqlen = n, w.max_seqlen
        self.pairs = visible_pairs_closed_form(w.turn_lens, w.conv_turn_ptr)
        self.conv_tokens = w.conversation_tokens()
        self.names = ["layout", "rope", "attn_fwd", "bwd_row_terms", "bwd_dq", "bwd_dkdv", "rope_inv"]
        self.streams = None

    def flops(self):
        d, hq, P = self.w.d, self.w.hq, self.pairs
        return {"useful_fwd": 4.0 * d * P * hq, "useful_bwd": 10.0 * d * P * hq,
                "attn_fwd": 4.0 * d * P * hq, "bwd_dq": 6.0 * d * P * hq, "bwd_dkdv": 8.0 * d * P * hq}

    def step(self, events=None, s: int = 0):
        """One pass of the hot path on buffer set `s`; `events` = CUDA events recorded between calls."""
        opr, torch = self.opr, self.torch
        b = self.sets[s]
        rec = (lambda i: events[i].record()) if events is not None else (lambda i: None)
        rec(0)
        lay = opr.opr_build_layout(*b["lens"], total_tokens=self.total, max_seqlen=self.max_seqlen, device=self.dev,
                                   block_map=False)  # the attention calls use the layout's internal block map
        rec(1)
        # rotated q, k and the fp16 copy of v (P V in fp16), in the attention order
        am = lay.attn_pos
        opr.opr_rope(b["q"], lay.pos_id, self.w.base, out=self.q_rot, dev_status=lay.dev_status, row_map=am)
        opr.opr_rope(b["k"], lay.pos_id, self.w.base, out=self.k_rot, dev_status=lay.dev_status, row_map=am)
        opr.opr_rope(b["v"], None, self.w.base, out=self.v16, dev_status=lay.dev_status, row_map=am)
        rec(2)
        o, lse = opr.opr_attn_fwd(self.q_rot, self.k_rot, self.v16, lay, out_dtype=torch.bfloat16)
        rec(3)
        if self.forward_only:
            for i in (4, 5, 6, 7):
                rec(i)
            self.layout = lay
            return lay
        args = (self.q_rot, self.k_rot, b["v"], o, b["do"], lse, lay)
        kw = dict(workspace=self.bwd_ws, out=b["grads"])
        opr.opr_attn_bwd(*args, stages=opr.BWD_ROW_TERMS, **kw)
        rec(4)
        opr.opr_attn_bwd(*args, stages=opr.BWD_DQ, **kw)
        rec(5)
        opr.opr_attn_bwd(*args, stages=opr.BWD_DKDV, **kw)
        rec(6)
        # gradients w.r.t. the unrotated q and k
        opr.opr_rope(b["grads"][0], lay.pos_id, self.w.base, inverse=True)
        opr.opr_rope(b["grads"][1], lay.pos_id, self.w.base, inverse=True)
        rec(7)
        self.layout = lay
        return lay

    def copy_in(self, s: int):
        """Pinned host -> device copy of one step's inputs into buffer set `s`."""
        b = self.sets[s]
        for dst, src in zip(b["lens"], self.h_lens):
            dst.copy_(src, non_blocking=True)
        for key, src in (("q", self.h_q), ("k", self.h_k), ("v", self.h_v), ("do", self.h_do)):
            b[key].copy_(src, non_blocking=True)

    def copy_out(self, s: int):
        """Device -> pinned host copy of one step's dq, dk, dv from buffer set `s`."""
        for dst, src in zip(self.h_grads, self.sets[s]["grads"]):
            dst.copy_(src, non_blocking=True)

    def pipelined(self, n: int, start=None, end=None):
        """n end-to-end steps with the copies of step i+1 (in) and i-1 (out) overlapping step i.

        Three streams: host->device copies, compute, device->host copies; events
        order each step's compute after its inputs have landed and after the
        buffer set it reuses has been copied out.
        """
        torch = self.torch
        if self.streams is None:
            self.streams = tuple(torch.cuda.Stream(device=self.dev) for _ in range(3))
        h2d, comp, d2h = self.streams
        cur = torch.cuda.current_stream(self.dev)
        for st in self.streams:
            st.wait_stream(cur)
        in_ready = [torch.cuda.Event() for _ in range(n)]
        comp_done = [torch.cuda.Event() for _ in range(n)]
        out_done = [torch.cuda.Event() for _ in range(n)]
        if start is not None:
            start.record(h2d)
        for i in range(n + 2):
            if i < n:  # inputs of step i, once step i-2 has finished reading set i % 2
                with torch.cuda.stream(h2d):
                    if i >= 2:
                        h2d.wait_event(comp_done[i - 2])
                    self.copy_in(i % 2)
                    in_ready[i].record(h2d)
            j = i - 1
            if 0 <= j < n:  # compute of step j, once its inputs are in and set j % 2's gradients are out
                with torch.cuda.stream(comp):
                    comp.wait_event(in_ready[j])
                    if j >= 2:
                        comp.wait_event(out_done[j - 2])
                    self.step(s=j % 2)
                    comp_done[j].record(comp)
            k = i - 2
            if 0 <= k < n:  # results of step k
                with torch.cuda.stream(d2h):
                    d2h.wait_event(comp_done[k])
                    self.copy_out(k % 2)
                    out_done[k].record(d2h)
        if end is not None:
            end.record(d2h)
        for st in self.streams:
            cur.wait_stream(st)

    def h2d_bytes(self):
        return sum(t.numel() * t.element_size() for t in (self.h_q, self.h_k, self.h_v, self.h_do, *self.h_lens))

    def d2h_bytes(self):
        return sum(t.numel() * t.element_size() for t in self.h_grads)


# ------------------------------------------------------------------ ranks
class Ranks:
    """Rank plumbing of a weak-scaling run (one process per GPU).

    Every rank times its own batch between barriers; the job's time is the
    maximum over ranks and its work the sum over ranks.  The two reductions
    run on timing scalars only: the data path has no collective.
    """

    def __init__(self, world: int, device):
        import torch
        import torch.distributed as dist

        self.world, self.device, self._torch, self._dist = world, device, torch, dist

    def barrier(self):
        if self.world > 1:
            self._dist.barrier()

    def _reduce(self, x: float, op) -> float:
        if self.world == 1:
            return x
        t = self._torch.tensor([x], dtype=self._torch.float64, device=self.device)
        self._dist.all_reduce(t, op=op)
        return float(t.item())

    def max(self, x: float) -> float:
        return self._reduce(x, self._dist.ReduceOp.MAX)

    def sum(self, x: float) -> float:
        return self._reduce(x, self._dist.ReduceOp.SUM)


def rank_workload(config: int, rank: int, turns: int | None = None, seed: int | None = None) -> synth.Workload:
    """This rank's batch: the configuration's shape and length mix, drawn from a rank-specific seed
    (base seed 1000 + config unless given)."""
    base = 1000 + config if seed is None else seed
    return synth.make_workload(config, seed=base + 7919 * rank, n_turns=turns)


def time_runner(r: Runner, steps: int, warmup: int, flush, barrier):
    torch = r.torch
    for _ in range(warmup):
        r.step()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(steps)]
    barrier()
    torch.cuda.synchronize()
    for i in range(steps):
        flush()
        r.step(ev[i])
    torch.cuda.synchronize()
    barrier()
    per = {name: [] for name in r.names}
    totals = []
    for e in ev:
        t = [e[j].elapsed_time(e[j + 1]) for j in range(7)]
        for name, x in zip(r.names, t):
            per[name].append(x)
        totals.append(e[0].elapsed_time(e[7]))
    status = r.opr.read_status(r.layout.dev_status)
    if status:
        raise RuntimeError(f"device status after timing: {status}")
    return sum(totals), per


def time_e2e(r: Runner, steps: int, warmup: int, barrier):
    """End to end through host buffers: every step copies its inputs in and its gradients out.

    The copies of neighbouring steps overlap the compute (pipelined); the timed
    region runs from before the first copy in to after the last copy out.  The
    inputs (1.3 GB at the default size) exceed L2, so no flush is needed.
    """
    torch = r.torch
    r.pipelined(warmup)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    r.pipelined(steps, a, b)
    torch.cuda.synchronize()
    barrier()
    status = r.opr.read_status(r.layout.dev_status)
    if status:
        raise RuntimeError(f"device status after end-to-end timing: {status}")
    return a.elapsed_time(b)


# ------------------------------------------------------------------ token duplication
def time_duplication(w: synth.Workload, device, hbm_gbs: float, hidden: int = 4096, reps: int = 5):
    """The step before the attention layer at this workload's size: the one-pass map, a gather of
    bf16 hidden rows (width `hidden`) into the one-pass stream and the fp32 fold of their gradient.
    HBM-bound; bytes are each launch's algorithmic reads plus writes."""
    import torch

    import block_sparse_masked_segment_b200 as opr

    src, copies = opr.opr_duplication_index(w.turn_lens, w.conv_turn_ptr, device=device)
    total, n_orig = src.numel(), copies.shape[0]
    x = torch.randn(n_orig, hidden, device=device).to(torch.bfloat16)
    y = torch.empty(total, hidden, device=device, dtype=torch.bfloat16)
    dy = torch.randn(total, hidden, device=device)
    dx = torch.empty(n_orig, hidden, device=device)

    def timed(fn):
        for _ in range(2):
            fn()
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    t_map = timed(lambda: opr.opr_duplication_index(w.turn_lens, w.conv_turn_ptr, total, n_orig, device=device))
    t_gather = timed(lambda: opr.opr_gather_rows(x, src, out=y))
    t_fold = timed(lambda: opr.opr_fold_rows(dy, copies, out=dx))
    gather_bytes = 2 * total * hidden * 2
    fold_bytes = total * hidden * 4 + n_orig * hidden * 4
    status = opr.read_status(src._inputs[2])
    if status:
        raise RuntimeError(f"device status after duplication timing: {status}")
    return {
        "tokens": {"one_pass": total, "original": n_orig, "hidden": hidden},
        "index_ms": t_map,
        "gather_ms": t_gather, "gather_gbs": gather_bytes / (t_gather * 1e-3) / 1e9,
        "gather_frac_hbm": gather_bytes / (t_gather * 1e-3) / 1e9 / hbm_gbs,
        "fold_ms": t_fold, "fold_gbs": fold_bytes / (t_fold * 1e-3) / 1e9,
        "fold_frac_hbm": fold_bytes / (t_fold * 1e-3) / 1e9 / hbm_gbs,
    }


def time_loss_side(w: synth.Workload, device, hbm_gbs: float, vocab: int = 151936, max_rows: int = 4096, reps: int = 5):
    """The step after the attention layer: the loss-row map of this workload and the fused
    cross-entropy (loss and gradient) over up to max_rows of its loss rows with bf16 logits of
    the Qwen-3 vocabulary.  HBM-bound: two reads and one write of the logits."""
    import torch

    import block_sparse_masked_segment_b200 as opr

    def timed(fn):
        for _ in range(2):
            fn()
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    rows, targets = opr.opr_loss_rows(w.turn_lens, device=device)
    t_rows = timed(lambda: opr.opr_loss_rows(w.turn_lens, device=device))
    n = min(rows.numel(), max_rows)
    logits = (torch.randn(n, vocab, device=device) * 3).to(torch.bfloat16)
    tid = torch.randint(0, vocab, (n,), device=device, dtype=torch.int32)
    t_ce = timed(lambda: opr.opr_cross_entropy(logits, tid, grad_scale=1.0 / n))
    loss, _ = opr.opr_cross_entropy(logits, tid)
    torch.cuda.synchronize()
    status = opr.read_status(rows._inputs[1]) + opr.read_status(loss._status)
    if status:
        raise RuntimeError(f"device status after loss-side timing: {status}")
    bytes_ = 3 * n * vocab * 2
    return {"loss_rows": int(rows.numel()), "loss_rows_ms": t_rows, "ce_rows": n, "vocab": vocab,
            "ce_ms": t_ce, "ce_gbs": bytes_ / (t_ce * 1e-3) / 1e9, "ce_frac_hbm": bytes_ / (t_ce * 1e-3) / 1e9 / hbm_gbs}


def kpass_workload(w: synth.Workload, K: int, device) -> synth.Workload:
    """The K-pass arrangement of w, built on the GPU by opr_kpass (plan and token map)."""
    import torch

    import block_sparse_masked_segment_b200 as opr

    kp = opr.opr_kpass(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr, K, device=device)
    torch.cuda.synchronize()
    status = opr.read_status(kp.dev_status)
    if status:
        raise RuntimeError(f"device status after opr_kpass: {status}")
    return synth.Workload(turn_lens=kp.turn_lens.cpu().numpy(), conv_turn_ptr=kp.conv_turn_ptr.cpu().numpy(),
                          seq_conv_ptr=kp.seq_conv_ptr.cpu().numpy(), hq=w.hq, hkv=w.hkv, d=w.d, base=w.base,
                          name=f"{w.name} [K={K}]")


# ------------------------------------------------------------------ oracle timing
def oracle_sample(w: synth.Workload, target_tokens: int):
    """The first conversation of the workload, cut after the turn that reaches
    `target_tokens` one-pass tokens, with one GQA group (Hq/Hkv q heads, 1 kv head)."""
    t0, t1 = int(w.conv_turn_ptr[0]), int(w.conv_turn_ptr[1])
    turns, n = [], 0
    for t in range(t0, t1):
        h, tt, r = (int(x) for x in w.turn_lens[t])
        turns.append((h, tt, r))
        n += h + tt + 2 * r
        if n >= target_tokens:
            break
    g = w.hq // w.hkv
    sub = synth.make_custom_workload([[turns]], hq=g, hkv=1, d=w.d, base=w.base)
    return sub


def run_oracle_once(sub: synth.Workload, seed: int):
    from block_sparse_masked_segment_b200.pipeline import visible_pairs_closed_form
    from oracle import opr_oracle as orc

    rng = np.random.default_rng(seed)
    n = sub.total_tokens
    q, k, v, do = (synth.gaussian(rng, (n, h, sub.d)) for h in (sub.hq, sub.hkv, sub.hkv, sub.hq))
    lay = orc.build_layout(sub.turn_lens, sub.conv_turn_ptr, sub.seq_conv_ptr)
    t = time.perf_counter()
    o, lse = orc.forward(q, k, v, lay, sub.base)
    orc.backward(q, k, v, o, do, lse, lay, sub.base)
    dt = time.perf_counter() - t
    pairs = visible_pairs_closed_form(sub.turn_lens, sub.conv_turn_ptr)
    return dt, 14.0 * sub.d * pairs * sub.hq, sub.conversation_tokens()


def cpu_baseline(w: synth.Workload, seed: int, target_tokens=ORACLE_SAMPLE_TOKENS):
    sub = oracle_sample(w, target_tokens)
    dt, flops, conv_tok = run_oracle_once(sub, seed)
    cores = len(os.sched_getaffinity(0))
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": (f"fp64 numpy oracle, dense fwd+bwd of the first conversation's first {sub.n_turns} turns "
                       f"({sub.total_tokens} one-pass tokens), one GQA group ({sub.hq} q heads, 1 kv head), "
                       f"d={sub.d}; {dt:.1f} s; useful FLOPs as on the GPU"),
            "seconds": dt, "conv_tokens_per_s": conv_tok / dt}


def run_reference(args, cfg_index):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = synth.make_workload(cfg_index)
    sub = oracle_sample(w, ORACLE_SAMPLE_TOKENS)
    for i in range(args.warmup):
        run_oracle_once(sub, 17 + i)
    t0 = time.perf_counter()
    flops = tok = 0.0
    for i in range(args.steps):
        dt, f, ct = run_oracle_once(sub, 100 + i)
        flops += f
        tok += ct
    total = time.perf_counter() - t0
    value = flops / total / 1e12
    cores = len(os.sched_getaffinity(0))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "sample_tokens": sub.total_tokens, "sample_turns": sub.n_turns,
                   "heads": f"{sub.hq}q/1kv"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"dense fp64 fwd+bwd, first {sub.n_turns} turns of conversation 0 "
                                   f"({sub.total_tokens} tokens), one GQA group"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "conv_tokens_per_s": tok / total,
    }
    emit(line, args.jsonl)


def emit(line: dict, jsonl: str | None) -> None:
    """Print the benchmark's one JSON line; with --jsonl, also append it to that file."""
    text = json.dumps(line)
    print(text, flush=True)
    if jsonl:
        with open(jsonl, "a") as fh:
            fh.write(text + "\n")


# ------------------------------------------------------------------ other workloads
def measure_workload(w: synth.Workload, device, steps: int, warmup: int, flush, forward_only: bool = False,
                     compare: bool = True):
    """One workload on this GPU: kernel times and useful TFLOP/s of one-pass steps, and (compare)
    conversation tokens/s against the same kernels run N-pass and K-pass (K = 2)."""
    import torch

    nobar = lambda: None  # noqa: E731
    r = Runner(w, seed=11, device=device, forward_only=forward_only)
    ms, per = time_runner(r, steps, warmup, flush, nobar)
    fl = r.flops()
    useful = fl["useful_fwd"] + (0.0 if forward_only else fl["useful_bwd"])
    out = {"workload": w.name, "tokens_per_step": w.total_tokens, "conv_tokens_per_step": w.conversation_tokens(),
           "pairs_per_head": r.pairs, "ms_per_step": ms / steps,
           "useful_tflops": useful * steps / (ms * 1e-3) / 1e12,
           "kernel_ms": {k: statistics.mean(v) for k, v in per.items()},
           "pass": "forward only" if forward_only else "forward + backward"}
    bf16_peak = peaks()[0]
    out["fraction_of_bf16_peak"] = out["useful_tflops"] / bf16_peak
    k_fwd = statistics.mean(per["attn_fwd"])
    out["attn_fwd_tflops"] = fl["attn_fwd"] / (k_fwd * 1e-3) / 1e12
    conv_tps = w.conversation_tokens() * steps / (ms * 1e-3)
    out["conv_tokens_per_s"] = conv_tps
    del r
    if compare:
        for name, build in (("npass", lambda: synth.npass_workload(w)[0]), ("kpass2", lambda: kpass_workload(w, 2, device))):
            torch.cuda.empty_cache()
            ow = build()
            ro = Runner(ow, seed=11, device=device, forward_only=forward_only)
            o_ms, _ = time_runner(ro, steps, warmup, flush, nobar)
            o_tps = w.conversation_tokens() * steps / (o_ms * 1e-3)
            out[name] = {"tokens_per_step": ow.total_tokens, "ms_per_step": o_ms / steps, "conv_tokens_per_s": o_tps,
                         "one_pass_vs": conv_tps / o_tps}
            del ro
    torch.cuda.empty_cache()
    return out


def other_workloads(device, steps: int, warmup: int, flush):
    """The other workloads of the line: the Qwen-3-8B-like fwd+bwd batch, the Qwen-3-4B-like forward
    batch, and the depth sweep (one conversation of N turns, fwd+bwd), each one-pass against N-pass."""
    res = {"qwen3-8b-like fwd+bwd (2 x 32K)": measure_workload(synth.make_workload(2), device, steps, warmup, flush),
           "qwen3-4b-like fwd (16K)": measure_workload(synth.make_workload(1), device, steps, warmup, flush,
                                                      forward_only=True)}
    sweep = {}
    for n in synth.DEPTH_SWEEP_TURNS:
        sweep[str(n)] = measure_workload(synth.make_workload(3, n_turns=n), device, steps, warmup, flush)
    res["depth sweep (h128 t512 r256, fwd+bwd)"] = sweep
    return res


# ------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=DEFAULT_CONFIG)
    ap.add_argument("--turns", type=int, default=None, help="turns per conversation (depth sweep)")
    ap.add_argument("--no-npass", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads (8B-like, 4B-like, depth sweep)")
    ap.add_argument("--seed", type=int, default=None, help="base seed of the synthetic batch (default 1000 + config)")
    ap.add_argument("--jsonl", default=None, help="also append the JSON line to this file")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        run_reference(args, args.config)
        return

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=device)
    ranks = Ranks(world, device)
    barrier, max_over_ranks, sum_over_ranks = ranks.barrier, ranks.max, ranks.sum

    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    flush = lambda: flush_buf.zero_()  # noqa: E731

    # every rank runs its own batch of the same shape (weak scaling, no data-path collective)
    w = rank_workload(args.config, rank, args.turns, args.seed)
    r = Runner(w, seed=11 + rank, device=device)
    pairs = r.pairs
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else local
    with ClockSampler(gpu_index) as clocks:
        total_ms, per = time_runner(r, args.steps, args.warmup, flush, barrier)
    remeasured = False
    # a slowdown during the timed region on any rank: every rank measures once more
    if max_over_ranks(1.0 if clocks.rejected() else 0.0) > 0:
        remeasured = True
        with ClockSampler(gpu_index) as clocks:
            total_ms, per = time_runner(r, args.steps, args.warmup, flush, barrier)
    total_ms = max_over_ranks(total_ms)
    fl = r.flops()
    useful = fl["useful_fwd"] + fl["useful_bwd"]
    all_useful = sum_over_ranks(useful * args.steps)
    value = all_useful / (total_ms * 1e-3) / 1e12
    conv_tps = sum_over_ranks(r.conv_tokens * args.steps) / (total_ms * 1e-3)
    mean = {k: statistics.mean(v) for k, v in per.items()}

    e2e = None
    if not args.no_e2e:
        e2e_ms = max_over_ranks(time_e2e(r, args.steps, args.warmup, barrier))
        e2e = {"value": all_useful / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": r.h2d_bytes(), "d2h_bytes_per_step": r.d2h_bytes(),
               "ms_per_step": e2e_ms / args.steps,
               "mode": "pinned host buffers; copies of steps i-1, i+1 overlap step i on separate streams; "
                       "inputs larger than L2, no flush"}

    _, _, hbm, _ = peaks()
    duplication = time_duplication(w, device, hbm)
    loss_side = time_loss_side(w, device, hbm)

    # K-pass (K = 2) on the same conversations and kernels: speed and tokens against one-pass
    kw = kpass_workload(w, 2, device)
    rk = Runner(kw, seed=11 + rank, device=device)
    k_ms, _ = time_runner(rk, args.steps, args.warmup, flush, barrier)
    k_ms = max_over_ranks(k_ms)
    k_conv_tps = sum_over_ranks(w.conversation_tokens() * args.steps) / (k_ms * 1e-3)
    kpass = {"K": 2, "tokens_per_step": kw.total_tokens, "tokens_vs_one_pass": kw.total_tokens / w.total_tokens,
             "ms_per_step": k_ms / args.steps, "conv_tokens_per_s": k_conv_tps,
             "one_pass_vs_kpass": conv_tps / k_conv_tps}
    del rk
    torch.cuda.empty_cache()

    npass = None
    if not args.no_npass:
        nw, _ = synth.npass_workload(w)
        del r
        torch.cuda.empty_cache()
        rn = Runner(nw, seed=11 + rank, device=device)
        n_ms, n_per = time_runner(rn, args.steps, args.warmup, flush, barrier)
        n_ms = max_over_ranks(n_ms)
        n_conv_tps = sum_over_ranks(w.conversation_tokens() * args.steps) / (n_ms * 1e-3)
        npass = {"conv_tokens_per_s": n_conv_tps, "ms_per_step": n_ms / args.steps,
                 "tokens_per_step": nw.total_tokens, "pairs_per_head": rn.pairs,
                 "kernel_ms": {k: statistics.mean(v) for k, v in n_per.items()},
                 "one_pass_speedup": conv_tps / n_conv_tps}
        kpass["kpass_vs_npass"] = k_conv_tps / n_conv_tps

    # roofline of the dominant tensor-core kernel, timed live with CUDA events
    bf16_peak, bf16_sust, hbm, peak_src = peaks()
    dom = max(("attn_fwd", "bwd_dq", "bwd_dkdv"), key=lambda k: mean[k])
    achieved = fl[dom] / (mean[dom] * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": bf16_peak, "unit": "TFLOP/s",
                "frac": achieved / bf16_peak, "traffic": measured_traffic(dom, args.config, args.turns, args.seed),
                "traffic_unit": "bytes per launch (ncu dram read + write)",
                "peak_source": f"{peak_src} bf16_tflops (burst); sustained {bf16_sust}",
                "frac_of_sustained": achieved / bf16_sust if bf16_sust else None,
                "algorithmic_flops": fl[dom]}

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return
    extra = None
    if world == 1 and not args.no_extra and args.turns is None:
        r = None  # the main workload's buffers are no longer needed
        torch.cuda.empty_cache()
        extra = other_workloads(device, args.steps, args.warmup, flush)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, seed=5)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "config_index": args.config, "sequences": w.n_seqs,
                   "conversations": w.n_convs, "turns": w.n_turns, "tokens_per_step": w.total_tokens,
                   "max_seqlen": w.max_seqlen, "conv_tokens_per_step": w.conversation_tokens(),
                   "hq": w.hq, "hkv": w.hkv, "head_dim": w.d, "pairs_per_head": pairs,
                   "parallelism": f"dp{world} (independent batches per GPU)",
                   "l2": "512 MiB buffer zeroed before every step, outside the step's events",
                   "outputs": "O bf16, LSE fp32, dq/dk/dv fp32"},
        "useful_tflop_per_step": useful / 1e12,
        "fraction_of_bf16_peak": value / bf16_peak,
        "conv_tokens_per_s": conv_tps,
        "kernel_ms": mean,
        "roofline": roofline,
        "e2e": e2e,
        "npass": npass,
        "next_rows": {"token_duplication": duplication, "kpass": kpass, "loss_side": loss_side},
        "other_workloads": extra,
        "gpu_launches": kernels_per_step(w) * args.steps,
        "clocks": dict(clocks.summary(), remeasured=remeasured),
        "cpu_baseline": cpu,
    }
    emit(line, args.jsonl)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
