"""Benchmark of the GDN / KDA token mixers on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

With no --workload the line's top level is gdn_prefill and its "workloads" object
holds kda_prefill, decode_gdn, decode_kda and kda_long, each timed in the same run
with its own steps, roofline, clocks, end-to-end figure and oracle baseline.

Workloads (synthetic inputs, recipe in synth/):
  gdn_prefill  GDN chunked prefill, B=1 H=32 T=4096 d=128 bf16       (default)
  kda_prefill  KDA chunked prefill, same shapes, per-channel gates
  decode_gdn   256 sequences x 32 heads, d=128, 512 one-token steps, GDN gates
  decode_kda   same with KDA gates
  kda_long     KDA prefill with a carried state, B=4 H=32 T=65536 d=128
  verify_gdn   multi-token verify (K=4) for 256 sequences x 32 heads, GDN / KDA gates
  verify_kda
  gdn_varlen   64 prompts packed with per-sequence state slots, GDN / KDA gates
  kda_varlen
  gdn_backward the gradients of the gdn_prefill / kda_prefill shapes (fp32 arithmetic)
  kda_backward
  gdn_prefill_prologue, kda_prefill_prologue, decode_gdn_prologue: the same calls with
               the fused prologue (raw q, k normalised and the gates formed in-kernel)

One step is one pass of the workload: one prefill (or verify, packed prefill,
gradient) call, or 512 decode calls.
`value` is whole-job tokens/s (a token = one position of one sequence, all H
heads) with inputs resident in HBM; `e2e` is the same through the public API
with pinned host buffers copied in and results copied out inside the timed
region.  Under torchrun each rank runs its own replica of the workload (the
(sequence, head) chains are independent, so nothing is exchanged): weak
scaling, time = max over ranks.
"""

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import (WORKLOADS, device_inputs, slice_inputs, slice_seed, tokens,  # noqa: E402
                   varlen_lengths)

METRIC = "GDN/KDA prefill tokens/s and decode tokens/s at 1 B200; % of roofline"
L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------------------
# algorithmic work per workload
# ----------------------------------------------------------------------------------------

def algorithmic(w):
    """(bytes, flops) of one pass of workload w, counted from the definition:
    every input read once, every output written once; flops of the chunked form
    at C=64 (2C(3 d_k + 2 d_v) + 6 d_k d_v per token-head, excluding the
    triangular solve and the gate exponentials).  Decode counts the state bytes
    (read + write) only, which is 99% of its traffic."""
    esz = 2 if w.dtype == "bf16" else 4
    th = tokens(w) * w.H
    state = w.B * w.H * w.dv * w.dk * 4
    if w.decode:
        return 2 * state * w.T, th * 6 * w.dk * w.dv
    if w.verify:
        # state read once, one full snapshot written per token, plus the token inputs
        # and outputs (small next to the state)
        a_bytes = 4 * (w.dk if w.mixer == "kda" else 1)
        per_th = esz * (2 * w.dk + w.dv) + a_bytes + 4 + esz * w.dv
        return (1 + w.T) * state + th * per_th, th * 6 * w.dk * w.dv
    a_bytes = 4 * (w.dk if w.mixer == "kda" else 1)
    if w.backward:
        # inputs q, k, v, alpha, beta and dL/do read once; dq, dk, dv, dalpha, dbeta
        # written once (fp32); dL/dS_T read and ds0 written.  Flops of the token-level
        # reverse: the forward recurrence (5 d_k d_v) plus the reverse step (16 d_k d_v).
        per_th = esz * (2 * w.dk + 2 * w.dv) + a_bytes + 4 + 4 * (2 * w.dk + w.dv) + a_bytes + 4
        return th * per_th + 2 * state, th * 21 * w.dk * w.dv
    per_th = esz * (2 * w.dk + w.dv) + a_bytes + 4 + esz * w.dv
    # the final states are written; initial states read when the workload has them
    nbytes = th * per_th + state + (state if w.state == "randn" else 0)
    C = 64
    flops = th * (2 * C * (3 * w.dk + 2 * w.dv) + 6 * w.dk * w.dv)
    return nbytes, flops


def alu_peak_tflops(peaks):
    """fp32 CUDA-core peak of a B200 from its unit counts and clock: 148 SMs x 128 fp32
    lanes x 2 flops per fused multiply-add x the maximum SM clock."""
    mhz = peaks.get("sm_max_mhz") or 1965.0
    return 148 * 128 * 2 * mhz * 1e6 / 1e12


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        out = {k: float(d[k]) for k in FALLBACK_PEAKS}
        out["sm_max_mhz"] = float(d.get("sm_max_mhz", 1965.0))
        return out, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def carry_kernel():
    """The state carry a two-kernel prefill runs: the chained one unless GDR_CARRY picks
    another (the library's rule, restated here to name the kernel in the report)."""
    pick = os.environ.get("GDR_CARRY", "")[:1]
    return {"r": "row_carry_kernel", "s": "sliced_carry_kernel"}.get(pick, "chain_carry_kernel")


def load_traffic(kernel_key):
    """DRAM bytes per call from the committed ncu summary, if it was taken on the
    current source of the kernels (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d.get(kernel_key)
        if not e:
            return None
        if e.get("source_sha") != source_sha(e.get("source", "")):
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


def source_sha(rel):
    """First 16 hex digits of the sha256 of a source file, or of several files'
    contents concatenated (rel a list)."""
    import hashlib
    rels = rel if isinstance(rel, list) else [rel]
    h = hashlib.sha256()
    for r in rels:
        p = os.path.join(ROOT, r)
        if not r or not os.path.exists(p):
            return None
        h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


# ----------------------------------------------------------------------------------------
# distributed plumbing (also exercised on CPU with gloo by the tests)
# ----------------------------------------------------------------------------------------

def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def dist_init(world, backend):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return world > 1


def barrier(active, device=None):
    if active:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(x, active, device):
    """Maximum of a float over all ranks (identity on one rank)."""
    if not active:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(tokens_per_rank, max_ms, world):
    """Whole-job tokens/s: the units all ranks processed over the slowest rank's time."""
    return tokens_per_rank * world / (max_ms / 1e3)


# ----------------------------------------------------------------------------------------
# clocks
# ----------------------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        # the raw samples (one CSV per rank); GDR_CLOCKS_DIR keeps them somewhere chosen
        self.path = os.path.join(os.environ.get("GDR_CLOCKS_DIR") or tempfile.gettempdir(),
                                 f"gdr_clocks_rank{index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------------------

class PrefillRunner:
    """One prefill call per step; enough input sets are rotated that every step
    reads inputs that are not L2-resident (sets total > 3x L2)."""

    def __init__(self, w, dev, seed):
        import gated_delta_rule_79_b200 as g
        self.g, self.w, self.dev = g, w, dev
        self.fn = g.kda_prefill if w.mixer == "kda" else g.gdn_prefill
        one = device_inputs(w, dev, seed=seed)
        set_bytes = sum(t.numel() * t.element_size() for t in one.values() if t is not None)
        set_bytes += w.B * w.T * w.H * w.dv * 2
        nsets = max(1, math.ceil(3 * L2_BYTES / set_bytes))
        self.sets = [one] + [device_inputs(w, dev, seed=seed + 1 + i) for i in range(nsets - 1)]
        self.o = [torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.bfloat16, device=dev)
                  for _ in self.sets]
        self.s = [torch.empty((w.B, w.H, w.dv, w.dk), dtype=torch.float32, device=dev)
                  for _ in self.sets]
        self.ws, _ = g.prefill_workspace(w.B, w.T, w.H, w.dk, w.dv, w.mixer == "kda", dev)
        self.path = g.prefill_path(w.dk, w.dv, w.torch_dtype, w.mixer == "kda")
        # the tensor-core path with a full-size workspace runs a per-chunk prep kernel,
        # then the state carry; the others run one kernel per call
        if self.path == "tensor-core":
            self.kernels = [f"{w.mixer}_chunk_prep_kernel", carry_kernel()]
            self.kernel_key = f"prefill_two-kernel:{w.name}"
        else:
            self.kernels = ["prefill_simt_kernel"]
            self.kernel_key = f"prefill_{self.path}:{w.name}"
        self.launches_per_step = len(self.kernels)
        self.l2_note = f"{len(self.sets)} rotating input sets of {set_bytes / 2**20:.0f} MiB (> 3x L2)"

    def step(self, i):
        x = self.sets[i % len(self.sets)]
        self.fn(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["s0"],
                o=self.o[i % len(self.sets)], s_final=self.s[i % len(self.sets)],
                workspace=self.ws, prologue=self.w.prologue)


class DecodeRunner:
    """512 decode calls per step over a 0.5 GB state (larger than L2)."""

    def __init__(self, w, dev, seed):
        import gated_delta_rule_79_b200 as g
        self.g, self.w, self.dev = g, w, dev
        self.fn = g.kda_decode if w.mixer == "kda" else g.gdn_decode
        self.x = device_inputs(w, dev, seed=seed)
        self.state = self.x["s0"]
        self.o = torch.empty((w.B, w.H, w.dv), dtype=torch.bfloat16, device=dev)
        self.launches_per_step = w.T
        self.kernels = ["decode_kernel"]
        self.kernel_key = f"decode:{w.name}"
        self.path = "decode (CUDA cores, fp32 state)"
        self.l2_note = f"state of {self.state.numel() * 4 / 2**20:.0f} MiB > L2"

    def step(self, i):
        x = self.x
        for t in range(self.w.T):
            self.fn(x["q"][t], x["k"][t], x["v"][t], x["alpha"][t], x["beta"][t], self.state,
                    o=self.o, prologue=self.w.prologue)


class VerifyRunner:
    """One multi-token verify call per step (K tokens for every sequence and head,
    all K snapshots written); the 0.5 GB state and the snapshots exceed L2."""

    def __init__(self, w, dev, seed):
        import gated_delta_rule_79_b200 as g
        self.g, self.w, self.dev = g, w, dev
        self.fn = g.kda_verify if w.mixer == "kda" else g.gdn_verify
        self.x = device_inputs(w, dev, seed=seed)
        self.snaps = torch.empty((w.T, w.B, w.H, w.dv, w.dk), dtype=torch.float32, device=dev)
        self.o = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.bfloat16, device=dev)
        self.launches_per_step = 1
        self.kernels = ["verify_kernel"]
        self.kernel_key = f"verify:{w.name}"
        self.path = "verify (CUDA cores, fp32 state, K snapshots)"
        self.l2_note = (f"state of {self.x['s0'].numel() * 4 / 2**20:.0f} MiB and "
                        f"{self.snaps.numel() * 4 / 2**20:.0f} MiB of snapshots > L2")

    def step(self, i):
        x = self.x
        self.fn(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["s0"], snapshots=self.snaps,
                o=self.o)


class VarlenRunner:
    """One packed prefill call per step: B prompts of varlen_lengths(w) tokens, each
    from and back into its own slot of a state pool (inputs > 3x L2)."""

    def __init__(self, w, dev, seed):
        import gated_delta_rule_79_b200 as g
        self.g, self.w, self.dev = g, w, dev
        self.fn = g.kda_prefill_varlen if w.mixer == "kda" else g.gdn_prefill_varlen
        lens = varlen_lengths(w)
        total = sum(lens)
        x = device_inputs(w.with_(B=1, T=total, varlen=False), dev, seed=seed)
        self.x = {k: (v[0] if k != "s0" else None) for k, v in x.items()}
        gen = torch.Generator(device=dev).manual_seed(seed + 1)
        self.pool = 0.02 * torch.randn((w.B, w.H, w.dv, w.dk), generator=gen, device=dev)
        self.cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32, device=dev)
        self.o = torch.empty((total, w.H, w.dv), dtype=torch.bfloat16, device=dev)
        need = g.lib.gdr_prefill_varlen_workspace_bytes(w.B, total, w.H, w.dk, w.dv,
                                                        int(w.mixer == "kda"))
        self.ws = torch.zeros(need, dtype=torch.uint8, device=dev)
        self.kernels = ["varlen index + " + f"{w.mixer}_chunk_prep_kernel",
                        carry_kernel()]
        self.launches_per_step = 3
        self.kernel_key = f"prefill_two-kernel:{w.name}"
        self.path = "tensor-core"
        in_bytes = sum(t.numel() * t.element_size() for t in self.x.values() if t is not None)
        self.l2_note = (f"{len(lens)} prompts, {total} tokens, {in_bytes / 2**20:.0f} MiB of "
                        f"inputs (> 3x L2)")

    def step(self, i):
        x = self.x
        self.fn(x["q"], x["k"], x["v"], x["alpha"], x["beta"], self.cu, self.pool, o=self.o,
                workspace=self.ws)


class BackwardRunner:
    """One gradient call per step (dq, dk, dv, dalpha, dbeta, ds0 of the whole
    workload); two rotating input sets (each above L2)."""

    def __init__(self, w, dev, seed):
        import gated_delta_rule_79_b200 as g
        self.g, self.w, self.dev = g, w, dev
        self.fn = g.kda_backward if w.mixer == "kda" else g.gdn_backward
        self.sets = []
        for i in range(2):
            x = device_inputs(w, dev, seed=seed + i)
            gen = torch.Generator(device=dev).manual_seed(seed + 50 + i)
            x["do"] = torch.randn((w.B, w.T, w.H, w.dv), generator=gen, device=dev).to(
                w.torch_dtype)
            x["dsf"] = torch.randn((w.B, w.H, w.dv, w.dk), generator=gen, device=dev)
            self.sets.append(x)
        need = g.backward_workspace_bytes(w.B, w.T, w.H, w.dk, w.dv, w.mixer == "kda")
        self.ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
        self.kernels = ["gdr_backward_kernel"]
        self.kernel_key = f"backward:{w.name}"
        self.launches_per_step = 1
        self.path = "backward (CUDA cores, fp32)"
        set_bytes = sum(t.numel() * t.element_size() for t in self.sets[0].values()
                        if t is not None)
        self.l2_note = f"2 rotating input sets of {set_bytes / 2**20:.0f} MiB (> L2)"

    def step(self, i):
        x = self.sets[i % 2]
        self.fn(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["s0"], x["do"], x["dsf"],
                workspace=self.ws)


def time_device(runner, steps, warmup, dev, active, soak_s=0.5):
    """Warm up, then time exactly `steps` steps with CUDA events on the launching
    stream, bracketed by a barrier and a synchronize on both sides.  Also records
    each step's own event pair (the kernel-duration evidence for the roofline) and,
    for prefill, the library's per-kernel events on the same stream (the mean
    duration of each kernel of a call)."""
    stream = torch.cuda.current_stream(dev)
    for i in range(warmup):
        runner.step(i)
    torch.cuda.synchronize(dev)
    # Soak: keep running the same steps (untimed) for about half a second so that
    # the clock sampler sees the GPU under this load right before the timed region.
    t_end = time.perf_counter() + soak_s
    i = warmup
    while time.perf_counter() < t_end:
        runner.step(i)
        i += 1
        torch.cuda.synchronize(dev)
    barrier(active, dev)
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    per_kernel = not (runner.w.decode or runner.w.verify or runner.w.backward)
    if per_kernel:
        runner.g.timing_start()
    t0.record(stream)
    for i in range(steps):
        ev[i][0].record(stream)
        runner.step(warmup + i)
        ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    kernel_ms = runner.g.timing_stop()[0] if per_kernel else None
    barrier(active, dev)
    total_ms = t0.elapsed_time(t1)
    per = [a.elapsed_time(b) for a, b in ev]
    return total_ms, per, kernel_ms


def time_e2e(w, dev, steps, warmup, seed):
    """The public API with pinned host buffers: every step copies the step's
    inputs host->device, runs the path and copies the results back."""
    import gated_delta_rule_79_b200 as g
    stream = torch.cuda.current_stream(dev)
    x = device_inputs(w, dev, seed=seed + 100)
    host = {k: (v.cpu().pin_memory() if v is not None else None) for k, v in x.items()}
    if w.decode:
        return _e2e_decode_overlapped(w, dev, steps, warmup, x, host)
    if w.varlen:
        fn = g.kda_prefill_varlen if w.mixer == "kda" else g.gdn_prefill_varlen
        lens = varlen_lengths(w)
        total = sum(lens)
        xd = device_inputs(w.with_(B=1, T=total, varlen=False), dev, seed=seed + 100)
        keys = ("q", "k", "v", "alpha", "beta")
        host = {k: xd[k][0].cpu().pin_memory() for k in keys}
        dbuf = {k: torch.empty_like(xd[k][0]) for k in keys}
        pool = 0.02 * torch.randn((w.B, w.H, w.dv, w.dk), device=dev)
        cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32, device=dev)
        o = torch.empty((total, w.H, w.dv), dtype=torch.bfloat16, device=dev)
        o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        need = g.lib.gdr_prefill_varlen_workspace_bytes(w.B, total, w.H, w.dk, w.dv,
                                                        int(w.mixer == "kda"))
        ws = torch.zeros(need, dtype=torch.uint8, device=dev)
        h2d = sum(host[k].numel() * host[k].element_size() for k in keys)
        d2h = o.numel() * 2

        def step():
            for key in keys:
                dbuf[key].copy_(host[key], non_blocking=True)
            fn(dbuf["q"], dbuf["k"], dbuf["v"], dbuf["alpha"], dbuf["beta"], cu, pool, o=o,
               workspace=ws)
            o_host.copy_(o, non_blocking=True)
    elif w.backward:
        fn = g.kda_backward if w.mixer == "kda" else g.gdn_backward
        keys = ("q", "k", "v", "alpha", "beta")
        gen = torch.Generator(device=dev).manual_seed(seed + 150)
        x["do"] = torch.randn((w.B, w.T, w.H, w.dv), generator=gen, device=dev).to(w.torch_dtype)
        x["dsf"] = torch.randn((w.B, w.H, w.dv, w.dk), generator=gen, device=dev)
        keys = keys + ("do", "dsf")
        host = {k: x[k].cpu().pin_memory() for k in keys}
        dbuf = {k: torch.empty_like(x[k]) for k in keys}
        need = g.backward_workspace_bytes(w.B, w.T, w.H, w.dk, w.dv, w.mixer == "kda")
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
        out_host = None
        h2d = sum(host[k].numel() * host[k].element_size() for k in keys)
        shapes = [(w.B, w.T, w.H, w.dk), (w.B, w.T, w.H, w.dk), (w.B, w.T, w.H, w.dv),
                  tuple(x["alpha"].shape), (w.B, w.T, w.H), (w.B, w.H, w.dv, w.dk)]
        out_host = [torch.empty(sh, dtype=torch.float32).pin_memory() for sh in shapes]
        d2h = sum(t.numel() * 4 for t in out_host)

        def step():
            for key in keys:
                dbuf[key].copy_(host[key], non_blocking=True)
            grads = fn(dbuf["q"], dbuf["k"], dbuf["v"], dbuf["alpha"], dbuf["beta"], None,
                       dbuf["do"], dbuf["dsf"], workspace=ws)
            for hbuf, gr in zip(out_host, grads):
                hbuf.copy_(gr, non_blocking=True)
    elif w.verify:
        fn = g.kda_verify if w.mixer == "kda" else g.gdn_verify
        keys = ("q", "k", "v", "alpha", "beta")
        dbuf = {k: torch.empty_like(x[k]) for k in keys}
        state = x["s0"]
        snaps = torch.empty((w.T, w.B, w.H, w.dv, w.dk), dtype=torch.float32, device=dev)
        o = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.bfloat16, device=dev)
        o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        h2d = sum(host[k].numel() * host[k].element_size() for k in keys)
        d2h = o.numel() * 2

        def step():
            for key in keys:
                dbuf[key].copy_(host[key], non_blocking=True)
            fn(dbuf["q"], dbuf["k"], dbuf["v"], dbuf["alpha"], dbuf["beta"], state,
               snapshots=snaps, o=o)
            o_host.copy_(o, non_blocking=True)
    else:
        return _e2e_prefill_overlapped(w, dev, steps, warmup, x, host)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b) / steps
    return {"value": tokens(w) / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h)}


def _e2e_decode_overlapped(w, dev, steps, warmup, x, host):
    """Decode through the public API with pinned host buffers: every one of the w.T
    decode calls of a step copies its token's q, k, v, gates and beta host->device and
    its outputs device->host.  Two device buffer sets; the copies of token t+1 run on a
    copy stream while the kernel of token t runs, and token t's outputs go back on a
    third stream."""
    import gated_delta_rule_79_b200 as g
    fn = g.kda_decode if w.mixer == "kda" else g.gdn_decode
    comp = torch.cuda.current_stream(dev)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    keys = ("q", "k", "v", "alpha", "beta")
    state = x["s0"]
    bufs = [{k: torch.empty_like(x[k][0]) for k in keys} for _ in range(2)]
    outs = [torch.empty((w.B, w.H, w.dv), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    o_host = torch.empty((w.T, w.B, w.H, w.dv), dtype=torch.bfloat16).pin_memory()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    h2d = sum(host[k][0].numel() * host[k][0].element_size() for k in keys) * w.T
    d2h = o_host.numel() * 2
    count = [0]

    def call(t):
        i = count[0]
        count[0] += 1
        b = i % 2
        if i >= 2:
            up.wait_event(ev_done[b])          # call i-2 has read this input set
        with torch.cuda.stream(up):
            for k in keys:
                bufs[b][k].copy_(host[k][t], non_blocking=True)
            ev_in[b].record(up)
        comp.wait_event(ev_in[b])
        if i >= 2:
            comp.wait_event(ev_out[b])         # call i-2's outputs have been copied out
        d = bufs[b]
        fn(d["q"], d["k"], d["v"], d["alpha"], d["beta"], state, o=outs[b], prologue=w.prologue)
        ev_done[b].record(comp)
        down.wait_event(ev_done[b])
        with torch.cuda.stream(down):
            o_host[t].copy_(outs[b], non_blocking=True)
            ev_out[b].record(down)

    def run(n):
        for _ in range(n):
            for t in range(w.T):
                call(t)
        for b in range(2):
            comp.wait_event(ev_out[b])

    run(warmup)
    torch.cuda.synchronize(dev)
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(comp)
    up.wait_event(a)
    down.wait_event(a)
    run(steps)
    e.record(comp)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(e) / steps
    return {"value": tokens(w) / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h),
            "copies": "overlapped: host->device of token t+1 and device->host of token t-1 "
                      "beside the kernel of token t, on three streams"}


def _e2e_prefill_overlapped(w, dev, steps, warmup, x, host):
    """Prefill through the public API with pinned host buffers, the copies overlapped with
    the computation: two device buffer sets; step i's inputs go host->device on one copy
    stream while step i-1 computes, and step i-2's outputs go device->host on another.
    Every step copies all of its inputs in and all of its outputs (o and the final state)
    out inside the timed region, which runs from an event before the first copy to one
    after the last copy out."""
    import gated_delta_rule_79_b200 as g
    fn = g.kda_prefill if w.mixer == "kda" else g.gdn_prefill
    comp = torch.cuda.current_stream(dev)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    keys = [k for k, v in x.items() if v is not None]
    sets = [{k: torch.empty_like(x[k]) for k in keys} for _ in range(2)]
    outs = [(torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.bfloat16, device=dev),
             torch.empty((w.B, w.H, w.dv, w.dk), dtype=torch.float32, device=dev))
            for _ in range(2)]
    o_host = torch.empty(outs[0][0].shape, dtype=torch.bfloat16).pin_memory()
    s_host = torch.empty(outs[0][1].shape, dtype=torch.float32).pin_memory()
    ws, _ = g.prefill_workspace(w.B, w.T, w.H, w.dk, w.dv, w.mixer == "kda", dev, stream=comp)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    h2d = sum(sets[0][k].numel() * sets[0][k].element_size() for k in keys)
    d2h = outs[0][0].numel() * 2 + outs[0][1].numel() * 4

    def step(i):
        b = i % 2
        if i >= 2:
            up.wait_event(ev_done[b])          # step i-2 has read this input set
        with torch.cuda.stream(up):
            for k in keys:
                sets[b][k].copy_(host[k], non_blocking=True)
            ev_in[b].record(up)
        comp.wait_event(ev_in[b])
        if i >= 2:
            comp.wait_event(ev_out[b])         # step i-2's outputs have been copied out
        d = sets[b]
        fn(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d.get("s0"), o=outs[b][0],
           s_final=outs[b][1], workspace=ws, prologue=w.prologue)
        ev_done[b].record(comp)
        down.wait_event(ev_done[b])
        with torch.cuda.stream(down):
            o_host.copy_(outs[b][0], non_blocking=True)
            s_host.copy_(outs[b][1], non_blocking=True)
            ev_out[b].record(down)

    def run(first, n):
        for i in range(first, first + n):
            step(i)
        for b in range(2):
            comp.wait_event(ev_out[b])

    run(0, warmup)
    torch.cuda.synchronize(dev)
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(comp)
    up.wait_event(a)
    down.wait_event(a)
    run(warmup, steps)
    e.record(comp)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(e) / steps
    return {"value": tokens(w) / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h),
            "copies": "overlapped: host->device of step i, compute of step i-1 and "
                      "device->host of step i-2 on three streams"}


# ----------------------------------------------------------------------------------------
# the oracle as CPU baseline / reference arm
# ----------------------------------------------------------------------------------------

def _oracle_slice(args):
    """Run the oracle over one (batch, head) chain for the first `t_sample` tokens."""
    name, b, h, t_sample = args
    import numpy as np  # noqa: F401
    from oracle import gated_delta_rule, decode_step, verify_steps
    w = WORKLOADS[name]
    if w.verify:
        # K tokens per chain are too few to time: run t_sample chains of the K tokens
        t = time.perf_counter()
        for i in range(t_sample):
            x = slice_inputs(w, (b + i) % w.B, h)
            verify_steps(*[x[k][None, :, None].double().numpy()
                           for k in ("q", "k", "v", "alpha", "beta")],
                         x["s0"][None, None].double().numpy())
        return time.perf_counter() - t
    x = slice_inputs(w.with_(T=t_sample), b, h)
    if w.prologue:
        from oracle import apply_prologue
        qk = apply_prologue(x["q"].double().numpy(), x["k"].double().numpy(),
                            x["alpha"].double().numpy(), l2norm=bool(w.prologue & 1),
                            gate_logit=bool(w.prologue & 2), bf16=w.dtype == "bf16")
        x = dict(x, q=torch.from_numpy(qk[0]), k=torch.from_numpy(qk[1]),
                 alpha=torch.from_numpy(qk[2]))
    col = lambda key: x[key][None, :, None].double().numpy()  # noqa: E731
    s0 = None if x["s0"] is None else x["s0"][None, None].double().numpy()
    if w.backward:
        from oracle import gated_delta_rule_backward
        g = torch.Generator().manual_seed(slice_seed(7, b, h))
        do = torch.randn((1, t_sample, 1, w.dv), generator=g).double().numpy()
        dsf = torch.randn((1, 1, w.dv, w.dk), generator=g).double().numpy()
        t = time.perf_counter()
        gated_delta_rule_backward(col("q"), col("k"), col("v"), col("alpha"), col("beta"), s0,
                                  do, dsf)
        return time.perf_counter() - t
    t = time.perf_counter()
    if w.decode:
        st = s0
        for i in range(t_sample):
            _, st = decode_step(*[x[k][i][None, None].double().numpy()
                                  for k in ("q", "k", "v", "alpha", "beta")], st)
    else:
        gated_delta_rule(col("q"), col("k"), col("v"), col("alpha"), col("beta"), s0)
    return time.perf_counter() - t


_THREAD_VARS = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS",
                "NUMEXPR_NUM_THREADS")


def _single_thread_worker():
    torch.set_num_threads(1)


class OracleTimer:
    """Times the oracle on the host cores over a bounded sample of workload w: a
    spawn pool with one process per core, each running whole (batch, head) chains
    over the first t_sample tokens, t_sample calibrated so that one timed pass
    takes about `budget_s` seconds."""

    def __init__(self, w, budget_s):
        import multiprocessing as mp
        self.w = w
        self.cores = min(len(os.sched_getaffinity(0)), w.B * w.H)
        if w.verify:
            # t_sample counts chains of K tokens per process
            per_chain = _oracle_slice((w.name, 0, 0, 4)) / 4
            self.t_sample = max(1, int(budget_s / max(per_chain, 1e-9)))
            self.tokens_per_unit = w.T
            what = f"{self.t_sample} chains of {w.T} tokens"
        else:
            t_cal = min(w.T, 64)
            per_token_head = _oracle_slice((w.name, 0, 0, t_cal)) / t_cal
            self.t_sample = max(1, min(w.T, int(budget_s / max(per_token_head, 1e-9))))
            if w.backward:
                # the backward oracle keeps every state of its sample in memory
                self.t_sample = min(self.t_sample, 512)
            self.tokens_per_unit = 1
            what = f"{self.t_sample} tokens"
        self.chains = [(w.name, i // w.H, i % w.H, self.t_sample) for i in range(self.cores)]
        # one thread per worker process (numpy's BLAS and torch would otherwise start a
        # pool of their own in every worker and oversubscribe the cores)
        saved = {k: os.environ.get(k) for k in _THREAD_VARS}
        os.environ.update({k: "1" for k in _THREAD_VARS})
        try:
            self.pool = mp.get_context("spawn").Pool(processes=self.cores,
                                                     initializer=_single_thread_worker)
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
        self.pool.map(_oracle_slice, [(w.name, 0, 0, 1)] * self.cores)   # start the workers
        self.sample = (f"{self.cores} processes x {what} of {w.name} per pass, fp64 numpy "
                       f"oracle, one single-threaded spawn process per core; tokens/s = "
                       f"token-heads/s / H")

    def tokens_per_pass(self):
        """Tokens (token-heads / H) one sampled pass processes."""
        return self.cores * self.t_sample * self.tokens_per_unit / self.w.H

    def rate(self):
        return self.timed_pass()[0]

    def timed_pass(self):
        """One sampled pass: (tokens/s, wall seconds)."""
        t0 = time.perf_counter()
        self.pool.map(_oracle_slice, self.chains)
        wall = time.perf_counter() - t0
        return self.tokens_per_pass() / wall, wall

    def close(self):
        self.pool.close()
        self.pool.join()


# ----------------------------------------------------------------------------------------

DEFAULT_WORKLOAD = "gdn_prefill"
# The other configurations the default run times (each with its own roofline, clocks and
# end-to-end figure), so that one invocation covers every bf16 configuration of the path.
DEFAULT_EXTRA = ("kda_prefill", "decode_gdn", "decode_kda", "kda_long")


def default_steps(w):
    return 5 if (w.decode or w.name == "kda_long") else 20 if w.verify else 50


def run_reference(w, steps, warmup, n_gpus):
    """The reference arm: the fp64 oracle on the host cores.  One step is one bounded
    sample pass of the workload (a fixed number of whole (batch, head) chains over a
    token prefix), timed by the wall clock; ms_per_step is that pass's measured time."""
    ot = OracleTimer(w, budget_s=min(10.0, 120.0 / max(1, steps + warmup)))
    for _ in range(warmup):
        ot.timed_pass()
    passes = [ot.timed_pass() for _ in range(steps)]
    ot.close()
    v = statistics.median(r for r, _ in passes)
    wall_ms = statistics.median(t for _, t in passes) * 1e3
    return {"metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": n_gpus,
            "steps": steps, "warmup": warmup, "ms_per_step": wall_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "impl": "reference",
            "step": "one bounded sample pass of the workload on the host cores (not a whole "
                    "call): ms_per_step is its measured wall time",
            "tokens_per_step": ot.tokens_per_pass(),
            "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk,
                       "dv": w.dv, "in_dtype": w.dtype},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": ot.cores,
                             "kind": "oracle", "sample": ot.sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def run_ours(w, steps, warmup, dev, rank, world, active, peaks, peak_kind, e2e=True,
             cpu_budget=12.0):
    """Time workload w on this rank's GPU; returns its JSON record (rank 0's view)."""
    runner = (DecodeRunner if w.decode else VerifyRunner if w.verify
              else VarlenRunner if w.varlen else BackwardRunner if w.backward
              else PrefillRunner)(w, dev, seed=1000 * rank)
    clocks = ClockSampler(dev.index)
    clocks.start()
    total_ms, per, kernel_ms = time_device(runner, steps, warmup, dev, active)
    clk = clocks.stop()
    max_ms = max_over_ranks(total_ms, active, dev)
    ntok = tokens(w)
    value = aggregate(ntok * steps, max_ms, world)
    nbytes, flops = algorithmic(w)
    kern_ms = statistics.mean(per)
    if w.decode:
        # per-step event pairs bracket 512 launches; the kernel's own duration is
        # that over the launches (launch gaps included, so this is conservative)
        launch_ms = kern_ms / w.T
        bytes_launch = nbytes / w.T
        flops_launch = flops / w.T
    else:
        launch_ms, bytes_launch, flops_launch = kern_ms, nbytes, flops
    hbm = bytes_launch / (launch_ms / 1e3) / 1e9
    tflops = flops_launch / (launch_ms / 1e3) / 1e12
    traffic = load_traffic(runner.kernel_key)
    roofline = {"bound": "hbm", "achieved": hbm, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": hbm / peaks["hbm_gbs"], "traffic": traffic,
                "peak_source": peak_kind, "algorithmic_bytes_per_launch": bytes_launch,
                "launch_ms": launch_ms}
    if kernel_ms:
        # one "launch" of the roofline is one call of the path; its kernels, timed
        # with events on the launching stream over the same timed steps:
        tot = sum(kernel_ms)
        roofline["launch"] = "one prefill call (" + " + ".join(runner.kernels) + ")"
        roofline["kernels"] = [{"name": n, "ms": m, "share": m / tot if tot else None}
                               for n, m in zip(runner.kernels, kernel_ms)]
        dom = max(range(len(kernel_ms)), key=lambda i: kernel_ms[i])
        roofline["dominant"] = runner.kernels[dom] if dom < len(runner.kernels) else None
    if w.backward:
        # fp32 arithmetic on the CUDA cores bounds the gradient pass (its HBM time is a
        # tenth of the fp32 time), so the roofline is the fp32 CUDA-core peak
        alu = alu_peak_tflops(peaks)
        roofline = {"bound": "alu", "achieved": tflops, "peak": alu, "unit": "TFLOP/s",
                    "frac": tflops / alu, "traffic": traffic,
                    "peak_source": "unit counts: 148 SMs x 128 fp32 lanes x 2 x max SM clock",
                    "algorithmic_flops_per_launch": flops_launch, "launch_ms": launch_ms,
                    "hbm": {"achieved": hbm, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": hbm / peaks["hbm_gbs"],
                            "algorithmic_bytes_per_launch": bytes_launch}}
    extra = {}
    if not (w.decode or w.verify or w.backward):
        extra["roofline_tensor"] = {
            "bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "frac": tflops / peaks["bf16_tflops"],
            "frac_of_sustained": tflops / peaks["bf16_tflops_sustained"],
            "algorithmic_flops_per_launch": flops_launch, "peak_source": peak_kind}
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": steps, "warmup": warmup, "ms_per_step": max_ms / steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if runner.path == "tensor-core" else "f32",
            "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk, "dv": w.dv,
                       "tokens_per_step": ntok, "in_dtype": w.dtype,
                       "out_dtype": "f32" if w.backward else "bf16",
                       "chunk": 64, "prologue": w.prologue,
                       "kernel": runner.path, "l2": runner.l2_note,
                       "clocks_window": "0.5 s soak of the same steps, then the timed region",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
            "roofline": roofline, **extra,
            "gpu_launches": runner.launches_per_step * steps,
            "clocks": clk}
    del runner
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    if e2e:
        big = w.name == "kda_long"
        line["e2e"] = time_e2e(w, dev, steps=max(1, min(steps, 3 if big else 10)),
                               warmup=1 if big else 2, seed=rank)
        if world > 1:
            line["e2e"]["value"] *= world
        torch.cuda.synchronize(dev)
        torch.cuda.empty_cache()
    if rank == 0 and cpu_budget and world == 1:
        ot = OracleTimer(w, budget_s=cpu_budget)
        rate = ot.rate()
        ot.close()
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": ot.cores,
                                "kind": "oracle", "sample": ot.sample}
    return line


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--workload", default=None, choices=sorted(WORKLOADS),
                    help=f"one workload alone (default: {DEFAULT_WORKLOAD}, with "
                         f"{', '.join(DEFAULT_EXTRA)} under 'workloads')")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    a = ap.parse_args()
    w = WORKLOADS[a.workload or DEFAULT_WORKLOAD]
    if w.name == "gdn_seq_f32":
        raise SystemExit("gdn_seq_f32 is a parity case, not a bench line")
    steps = a.steps if a.steps is not None else default_steps(w)
    warmup = max(3, a.warmup if a.warmup is not None else 5)
    rank, world, local = dist_env()

    if a.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(w, steps, warmup, a.gpus)), flush=True)
        return 0

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (there is no CPU path)")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    active = dist_init(world, "nccl")
    peaks, peak_kind = load_peaks()
    cpu = None if a.no_cpu_baseline else 12.0
    line = run_ours(w, steps, warmup, dev, rank, world, active, peaks, peak_kind,
                    e2e=not a.no_e2e, cpu_budget=cpu)
    if a.workload is None:
        # the other configurations, each on its own clock record
        subs = {}
        for name in DEFAULT_EXTRA:
            wx = WORKLOADS[name]
            sx = a.steps if a.steps is not None else default_steps(wx)
            sub = run_ours(wx, sx, warmup, dev, rank, world, active, peaks, peak_kind,
                           e2e=not a.no_e2e, cpu_budget=None if cpu is None else 5.0)
            for key in ("metric", "n_gpus", "higher_is_better", "scaling", "vs_baseline",
                        "data"):
                sub.pop(key, None)
            subs[name] = sub
        line["workloads"] = subs
    if rank == 0:
        print(json.dumps(line), flush=True)
    if active:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
