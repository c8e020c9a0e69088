#!/usr/bin/env python
"""Benchmark: paged decode attention on B200 (K/V GB/s, fraction of HBM peak).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

One step is one pass of the whole hot path over the workload: the row write
(tf_kv_put_rows: each stream's new rows into their pages) followed by the
attention call (tf_paged_attn_decode / _verify / _prompt), all inputs resident
in HBM.  The default workload is batched decode: 12 streams at 40,960
positions, 8 KV / 32 query heads (GQA 4), head dim 128, pages of 512 in a
shuffled pool 1.2x the pages needed (TensorFold #1620's ``--parallel 12
--context 40960`` cells).

value  = algorithmic K/V bytes per step (visible positions x KV heads x
         head_dim x 2 bytes x {K, V}) / device time per step, whole job.
e2e    = the same metric through the public API with host buffers: every
         step's query and new rows copied from pinned host memory and its
         output copied back, inside the timed region, on copy streams that
         overlap the neighbouring steps' kernels (two sets of device
         buffers, as a serving loop runs).
roofline = the attention call (partial + merge kernels) alone, its K/V bytes
         over its CUDA-event time, against the measured HBM copy bandwidth.
cpu_baseline = the fp64 CPU oracle timed on the host on a bounded sample.

With N > 1 (torchrun), every rank runs its own replica of the workload on
its own GPU (the streams are independent; there is no exchange step):
weak scaling, value = all ranks' bytes / the slowest rank's time.
--impl reference times the oracle (rank 0 only) on per-step samples.

The default run also times the draft-verify workload (4 streams at 131,072
positions, 4 KV / 32 query heads, 8-row windows) the same way and reports its
verify tokens/s (window rows per second) under "verify", and likewise the head
dim 512 verify workload ("hd512"), the 9,216-token chunked prompt ("prompt",
causal TFLOP/s) and the shape variants ("variants": GQA 12, GQA 16 at head dim
512, head dim 256); --no-verify skips them all.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention K/V GB/s (fraction of HBM peak) and verify tokens/sec"
FALLBACK_HBM_GBS = 6650.0


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def recorded_traffic(workload):
    """DRAM bytes per launch of the workload's dominant kernel, from the ncu capture
    summarised in profiles/traffic.json -- or None when the kernel's sources have
    changed since that capture (the hash no longer matches) or there is none."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[workload]
        h = hashlib.sha256()
        for name in rec["files"]:
            with open(os.path.join(ROOT, name), "rb") as f:
                h.update(f.read())
        if h.hexdigest()[:16] != rec["source_hash"]:
            return None
        return int(rec["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def kv_bytes(lens, hkv, d):
    return int(np.sum(np.asarray(lens, dtype=np.int64))) * hkv * d * 2 * 2

PROMPT_METRIC = "chunked prompt attention causal TFLOP/s (fraction of bf16 tensor peak)"
FALLBACK_TENSOR_TFLOPS = 1400.0


def tensor_peak():
    """Dense bf16 tensor peak: the sustained figure, for kernels timed inside a
    long run of back-to-back steps."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured (sustained)"
    except (OSError, KeyError, ValueError):
        return FALLBACK_TENSOR_TFLOPS, "fallback (sustained)"


def throughput(wl, ms, world=1):
    """The workload's headline unit: causal TFLOP/s for a chunked prompt (tensor
    bound), K/V GB/s otherwise (HBM bound)."""
    if wl.w.prompt_len:
        return world * wl.flops_per_step / (ms * 1e-3) / 1e12, "TFLOP/s"
    return world * wl.bytes_per_step / (ms * 1e-3) / 1e9, "GB/s"


NOMINAL_HBM_GBS = 8000.0        # B200 HBM3e, vendor figure (DGX)
NOMINAL_TENSOR_TFLOPS = 2250.0  # B200 dense bf16, vendor figure


def roofline(wl, attn_ms):
    """The attention calls (partial + merge kernels) of one step against the bound
    that limits them."""
    achieved, unit = throughput(wl, attn_ms)
    if wl.w.prompt_len:
        peak, src = tensor_peak()
        bound = "tensor"
    else:
        peak, src = hbm_peak()
        bound = "hbm"
    nominal = NOMINAL_TENSOR_TFLOPS if wl.w.prompt_len else NOMINAL_HBM_GBS
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": achieved / peak, "traffic": recorded_traffic(wl.name),
            "kernel": "attention calls (partial + merge)", "peak_source": src,
            "peak_nominal": nominal, "frac_nominal": achieved / nominal}


def measure_other(name, args, barrier, dist, world, local):
    import torch
    wl = Workload(name, f"cuda:{local}")
    total, attn = time_steps(wl, args.steps, args.warmup, barrier)
    wl.check_flags()
    step = total / args.steps
    if dist is not None:
        t = torch.tensor([step, attn], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        step, attn = t.tolist()
    value, unit = throughput(wl, step, world)
    out = {"workload": name, "value": value, "unit": unit, "ms_per_step": step, "attn_ms": attn,
           "roofline": roofline(wl, attn),
           "rows_per_s": world * wl.rows_per_step / (step * 1e-3),
           "gpu_launches": 3 * len(wl.parts()) * args.steps, "config": workload_config(name)}
    if 1 < wl.w.rows <= 8:
        out["verify_tokens_per_s"] = out["rows_per_s"]
    del wl
    return out


def measure_state_copy(args, barrier, dist, world, local, name="decode_12x40k"):
    """The page-walking state copy (tf_kv_copy_state) of a workload's state (by
    default the decode workload's: 12 streams x 40,960 positions x 8 KV heads
    at head dim 128), from its shuffled pages to another shuffled set of pages
    in a second pool.  Bytes are read + write (the measured copy peak counts
    the same way)."""
    import torch
    import synth
    wl = Workload(name, f"cuda:{local}")
    tf, w = wl.tf, wl.w
    w2 = dataclasses.replace(w, seed=w.seed + 1000)
    t2, n2, _ = synth.page_table(w2, wl.lens_np)
    dst_table = torch.from_numpy(t2).to(wl.k_pool.device)
    shape = (n2, w.n_kv_heads, w.page_size, w.head_dim)
    dk = torch.empty(shape, dtype=torch.bfloat16, device=wl.k_pool.device)
    dv = torch.empty(shape, dtype=torch.bfloat16, device=wl.k_pool.device)
    status = torch.zeros(1, dtype=torch.int32, device=wl.k_pool.device)

    def copy():
        tf.tf_kv_copy_state(wl.k_pool, wl.v_pool, wl.table, wl.lens, dk, dv, dst_table,
                            wl.max_len, status=status)
    for _ in range(args.warmup):
        copy()
    torch.cuda.synchronize()
    barrier()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for e0, e1 in ev:
        e0.record()
        copy()
        e1.record()
    torch.cuda.synchronize()
    barrier()
    ms = sum(e0.elapsed_time(e1) for e0, e1 in ev) / args.steps
    if dist is not None:
        t = torch.tensor([ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = t.item()
    if int(status.item()) != 0:
        raise RuntimeError(f"state copy status {int(status.item()):#x}")
    # after timing, a sample: K and V of the first, middle and last page of the
    # first and the last stream (the used slots of a partial last page only)
    # hold the source's bytes
    P = w.page_size
    ok = True
    for s in sorted({0, len(wl.lens_np) - 1}):
        n = int(wl.lens_np[s])
        n_pages_s = (n + P - 1) // P
        for i in sorted({0, n_pages_s // 2, n_pages_s - 1}):
            used = min(P, n - i * P)
            src_pg, dst_pg = int(wl.table[s, i]), int(t2[s, i])
            ok = ok and torch.equal(dk[dst_pg, :, :used], wl.k_pool[src_pg, :, :used])
            ok = ok and torch.equal(dv[dst_pg, :, :used], wl.v_pool[src_pg, :, :used])
    moved = 2 * kv_bytes(wl.lens_np, w.n_kv_heads, w.head_dim)      # read + write
    gbs = world * moved / (ms * 1e-3) / 1e9
    peak, src = hbm_peak()
    label = "state_copy_" + name.split("_", 1)[1] if "_" in name else "state_copy_" + name
    out = {"workload": label, "value": gbs, "unit": "GB/s", "ms_per_step": ms,
           "roofline": {"bound": "hbm", "achieved": gbs / world, "peak": peak, "unit": "GB/s",
                        "frac": gbs / world / peak, "traffic": None, "kernel": "kv_copy_kernel",
                        "peak_source": src},
           "check": "K and V of 3 pages of the first and last stream equal" if ok else "MISMATCH",
           "gpu_launches": args.steps,
           "config": {"workload": label, "streams": len(wl.lens_np), "context": int(wl.lens_np.max()),
                      "kv_heads": w.n_kv_heads, "head_dim": w.head_dim, "page_size": w.page_size,
                      "bytes": "K+V read and written", "parallelism": "replicas",
                      "l2": f"inputs {moved / 2e9:.2f} GB > 126 MB L2"}}
    del wl, dk, dv
    torch.cuda.empty_cache()
    return out


# --------------------------------------------------------------------------
# clocks during the timed region
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid):
        self.uuid = gpu_uuid
        self.proc = None
        self.lines = []
        self.t_marks = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.uuid}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self):
        self.t_marks.append(time.time())

    def stop(self):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        for t, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((t, float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        if len(self.t_marks) >= 2:
            inside = [r for r in rows if self.t_marks[0] - 0.15 <= r[0] <= self.t_marks[-1] + 0.15]
            rows = inside or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_max_mhz": max(r[2] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------
# the workload on the device
class Workload:
    """One workload resident on the device.  A step is ``parts()``: (row write,
    attention call) pairs -- one pair for decode and verify, one per chunk for
    a chunked prompt (the chunk's rows written, then attended causally)."""

    def __init__(self, name, device):
        import torch
        import synth
        import verify_paged_gqa_b200 as tf
        self.torch, self.tf = torch, tf
        w = synth.WORKLOADS[name]
        self.w = w
        self.name = name
        W = w.rows
        if w.prompt_len:
            assert w.prompt_len % W == 0
            self.lens_np = np.array([w.prompt_len], dtype=np.int32)
        else:
            self.lens_np = synth.stream_lens(w)
        table, n_pages, _ = synth.page_table(w, self.lens_np)
        self.n_pages = n_pages
        S = len(self.lens_np)
        shape = (n_pages, w.n_kv_heads, w.page_size, w.head_dim)
        self.k_pool = torch.full(shape, float("nan"), dtype=torch.bfloat16, device=device)
        self.v_pool = torch.full(shape, float("nan"), dtype=torch.bfloat16, device=device)
        self.table = torch.from_numpy(table).to(device)
        self.lens = torch.from_numpy(self.lens_np).to(device)
        self.max_len = int(self.lens_np.max())
        d, Hq, Hkv = w.head_dim, w.n_q_heads, w.n_kv_heads
        if w.prompt_len:
            L = w.prompt_len
            k, v = synth.kv_rows_torch(w, 0, L, device)
            self.k_new, self.v_new = k[None].contiguous(), v[None].contiguous()   # [1][L][Hkv][d]
            self.q = synth.q_rows_torch(w, 1, L, device=device)                  # [1][L][Hq][d]
            self.chunk_lens = [torch.tensor([W * (c + 1)], dtype=torch.int32, device=device)
                               for c in range(L // W)]
            self.bytes_per_step = sum(kv_bytes([W * (c + 1)], Hkv, d) for c in range(L // W))
            self.flops_per_step = 4 * d * Hq * L * (L + 1) // 2       # causal pairs only
            self.rows_per_step = L
        else:
            new_k, new_v = [], []
            for s in range(S):
                n = int(self.lens_np[s])
                k, v = synth.kv_rows_torch(w, s, n, device)
                tf.tf_kv_put_rows(self.k_pool, self.v_pool, self.table[s:s + 1], self.lens[s:s + 1],
                                  k[None], v[None], max_len=n)
                new_k.append(k[n - W:])
                new_v.append(v[n - W:])
                del k, v
            self.k_new = torch.stack(new_k).contiguous()          # [S][W][Hkv][d]
            self.v_new = torch.stack(new_v).contiguous()
            self.q = synth.q_rows_torch(w, S, W, device=device)     # [S][W][Hq][d]
            self.chunk_lens = None
            self.bytes_per_step = kv_bytes(self.lens_np, Hkv, d)
            self.tree_np = synth.workload_tree(w)
            if self.tree_np is None:
                seen = [int(n) - W + r + 1 for n in self.lens_np for r in range(W)]
            else:   # the positions before the window plus the window rows each mask names
                seen = [int(n) - W + bin(int(self.tree_np[s, r]) & ((1 << W) - 1)).count("1")
                        for s, n in enumerate(self.lens_np) for r in range(W)]
            self.flops_per_step = 4 * d * Hq * sum(seen)
            self.rows_per_step = S * W
        self.out = torch.empty(self.q.shape, dtype=torch.float32, device=device)
        self.bytes_in_l2 = kv_bytes(self.lens_np, Hkv, d) < L2_BYTES
        nbytes = tf.tf_paged_attn_workspace_bytes(self.k_pool, self.v_pool, self.table, self.lens,
                                                  Hq, W, self.max_len)
        self.ws = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        self.attn_fn = (tf.tf_paged_attn_decode if W == 1 else
                        tf.tf_paged_attn_verify if W <= 8 else tf.tf_paged_attn_prompt)
        if not w.prompt_len and self.tree_np is not None:
            self.tree = torch.from_numpy(self.tree_np).to(device)
            self.attn_fn = lambda kp, vp, tb, ln, q, sc, out, ws, ml: tf.tf_paged_attn_verify_tree(
                kp, vp, tb, ln, q, self.tree, sc, out, ws, ml)
        torch.cuda.synchronize()

    def parts(self, k_new=None, v_new=None, q=None, out=None):
        """The step's (row write, attention) pairs, optionally on other input and
        output buffers."""
        k_new = self.k_new if k_new is None else k_new
        v_new = self.v_new if v_new is None else v_new
        q = self.q if q is None else q
        out = self.out if out is None else out
        tf, w = self.tf, self.w
        if self.chunk_lens is None:
            return [(lambda: tf.tf_kv_put_rows(self.k_pool, self.v_pool, self.table, self.lens,
                                               k_new, v_new, max_len=self.max_len),
                     lambda: self.attn_fn(self.k_pool, self.v_pool, self.table, self.lens, q,
                                          w.scale, out, self.ws, self.max_len))]
        W = w.rows
        pairs = []
        for c, lens_c in enumerate(self.chunk_lens):
            sl = slice(c * W, (c + 1) * W)
            pairs.append((
                lambda sl=sl, lens_c=lens_c: tf.tf_kv_put_rows(
                    self.k_pool, self.v_pool, self.table, lens_c, k_new[:, sl], v_new[:, sl],
                    max_len=self.max_len),
                lambda sl=sl, lens_c=lens_c: self.attn_fn(
                    self.k_pool, self.v_pool, self.table, lens_c, q[:, sl], w.scale,
                    out[:, sl], self.ws, self.max_len)))
        return pairs

    def step(self):
        for put, att in self.parts():
            put()
            att()

    def check_flags(self):
        torch = self.torch
        site = int(self.ws[4:8].view(torch.int32).item())   # which wait gave up, if any
        self.ws[4:8].zero_()
        flags = self.tf.tf_workspace_status(self.ws)
        if flags:
            raise RuntimeError(f"device status word set: {flags:#x} (wait sites {site:#x})")


L2_BYTES = 126 * 2**20


def time_steps(wl, steps, warmup, barrier, sampler=None, blocks=10):
    """Device time of ``steps`` steps, and the mean per step of the attention
    calls alone.

    The steps run back to back with nothing between their kernels, as in a
    serving loop (the attention kernels are programmatic dependents of the
    kernel before them): CUDA events on the launching stream bracket runs of
    steps, not calls.  The attention calls' own time comes from as many
    steps that run only the attention calls (the row writes already put the
    rows in place), also back to back; an event between a row write and the
    call after it would keep that call from starting early.  The two kinds
    alternate in ``blocks`` runs each, so both see the same clocks as the
    power cap settles.  A workload whose K/V fits in L2 gets L2 flushed (a
    256 MB write) before every step of either kind, outside that step's
    events."""
    torch = wl.torch
    parts = wl.parts()
    flush = None
    if wl.bytes_in_l2:
        flush = torch.empty(256 * 2**20, dtype=torch.uint8, device=wl.k_pool.device)
    for _ in range(warmup):
        wl.step()
    torch.cuda.synchronize()
    barrier()
    stream = torch.cuda.current_stream()
    mk = lambda: torch.cuda.Event(enable_timing=True)
    blocks = max(1, min(blocks, steps))
    bounds = [steps * k // blocks for k in range(blocks + 1)]
    full = lambda: [(put(), att()) for put, att in parts]
    attn_only = lambda: [att() for _, att in parts]
    runs = {0: [], 1: []}   # 0: whole steps, 1: attention calls; lists of (start, end) events

    def run(kind, n, i0):
        body = full if kind == 0 else attn_only
        if flush is None:
            ev = (mk(), mk())
            ev[0].record(stream)
            for _ in range(n):
                body()
            ev[1].record(stream)
            runs[kind].append(ev)
        else:
            for i in range(i0, i0 + n):
                flush.fill_(i & 255)
                ev = (mk(), mk())
                ev[0].record(stream)
                body()
                ev[1].record(stream)
                runs[kind].append(ev)

    if sampler:
        sampler.mark()
    for k in range(blocks):
        n = bounds[k + 1] - bounds[k]
        run(0, n, bounds[k])
        run(1, n, bounds[k])
    torch.cuda.synchronize()
    if sampler:
        sampler.mark()
    barrier()
    total_ms = sum(a.elapsed_time(b) for a, b in runs[0])
    attn_ms = sum(a.elapsed_time(b) for a, b in runs[1]) / steps
    return total_ms, attn_ms


def time_e2e(wl, steps, warmup, barrier):
    """The same steps through the public API from pinned host buffers, run as a
    serving loop runs them: every step copies its query and new rows in from
    pinned host memory and its output back, but on copy streams of their own
    and into two sets of device buffers, so step k + 1's inputs cross PCIe
    while step k computes, and step k's output crosses back while step k + 1
    computes.  Every copy of every step lies inside the timed region (events
    on the compute stream bracket all three streams)."""
    torch = wl.torch
    q_h = wl.q.cpu().pin_memory()
    k_h = wl.k_new.cpu().pin_memory()
    v_h = wl.v_new.cpu().pin_memory()
    out_h = [torch.empty(wl.out.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    bufs = [(torch.empty_like(wl.q), torch.empty_like(wl.k_new), torch.empty_like(wl.v_new),
             torch.empty_like(wl.out)) for _ in range(2)]
    parts = [wl.parts(k_d, v_d, q_d, out=o_d) for q_d, k_d, v_d, o_d in bufs]
    comp = torch.cuda.current_stream()
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_ready = [ev(), ev()]    # set b's inputs landed
    computed = [ev(), ev()]    # the step on set b computed (its inputs are free again)
    out_back = [ev(), ev()]    # set b's output copied back (its output buffer is free again)

    def one(k):
        b = k & 1
        q_d, k_d, v_d, o_d = bufs[b]
        with torch.cuda.stream(h2d_s):
            if k >= 2:
                h2d_s.wait_event(computed[b])
            q_d.copy_(q_h, non_blocking=True)
            k_d.copy_(k_h, non_blocking=True)
            v_d.copy_(v_h, non_blocking=True)
            in_ready[b].record(h2d_s)
        comp.wait_event(in_ready[b])
        if k >= 2:
            comp.wait_event(out_back[b])
        for put, att in parts[b]:
            put()
            att()
        computed[b].record(comp)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(computed[b])
            out_h[b].copy_(o_d, non_blocking=True)
            out_back[b].record(d2h_s)

    def run(n):
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(comp)
        h2d_s.wait_event(start)
        d2h_s.wait_event(start)
        for k in range(n):
            one(k)
        comp.wait_event(out_back[(n - 1) & 1])
        end.record(comp)
        return start, end

    run(warmup)
    torch.cuda.synchronize()
    barrier()
    start, end = run(steps)
    torch.cuda.synchronize()
    barrier()
    h2d = (q_h.numel() * q_h.element_size() + k_h.numel() * k_h.element_size()
           + v_h.numel() * v_h.element_size())
    d2h = out_h[0].numel() * out_h[0].element_size()
    return start.elapsed_time(end), h2d, d2h


# --------------------------------------------------------------------------
# the oracle on the host (CPU baseline and the reference arm)
_ORACLE_INPUTS = {}


def _oracle_inputs(wl_name, device_kv=None):
    """Stream 0 of the workload as host bf16 bits (drawn once per process)."""
    import synth
    if wl_name not in _ORACLE_INPUTS:
        w = synth.WORKLOADS[wl_name]
        n0 = int(synth.stream_lens(w)[0])
        if device_kv is not None:
            k, v = synth.to_bits(device_kv[0]), synth.to_bits(device_kv[1])
        else:
            k, v = synth.kv_rows(w, 0, n0)
        q = synth.q_rows(synth.dataclasses.replace(w, n_streams=1), w.rows)
        _ORACLE_INPUTS[wl_name] = (q, [k], [v])
    return _ORACLE_INPUTS[wl_name]


def oracle_sample(wl_name, n_units, threads, device_kv=None):
    """Time the fp64 oracle on ``n_units`` (stream 0, row r, query head h) units of the
    workload; returns (seconds, attributed K/V bytes, description)."""
    import oracle
    import synth
    w = synth.WORKLOADS[wl_name]
    lens = synth.stream_lens(w)
    n0 = int(lens[0])
    q, k_lin, v_lin = _oracle_inputs(wl_name, device_kv)
    Hq = w.n_q_heads
    base = [(0, r, h) for r in range(w.rows) for h in range(Hq)]
    units = np.array([base[k % len(base)] for k in range(n_units)], dtype=np.int32)
    t0 = time.perf_counter()
    oracle.attend(q, k_lin, v_lin, lens[:1], w.rows, w.group, w.scale, units=units,
                  threads=threads)
    dt = time.perf_counter() - t0
    visible = [n0 - w.rows + int(r) + 1 for _, r, _ in units]
    if w.prompt_len:
        # causal flops of the sampled rows (q.k and p.v: 4 d per visible position)
        work = sum(4 * w.head_dim * n for n in visible) / 1e12
    else:
        per_unit = w.head_dim * 2 * 2 / w.group      # one query head's share of a K/V row
        work = sum(n * per_unit for n in visible) / 1e9
    desc = (f"{len(units)} (stream, row, query head) output rows of stream 0 at {n0} positions "
            f"(the stream's {len(base)} rows, repeated), fp64, {threads} threads")
    return dt, work, desc


def cpu_baseline(wl_name, device_kv, budget_s=12.0):
    threads = os.cpu_count() or 1
    dt1, _, _ = oracle_sample(wl_name, threads, threads, device_kv)
    n = int(max(threads, budget_s / max(dt1, 1e-3) * threads))
    dt, work, desc = oracle_sample(wl_name, n, threads, device_kv)
    return {"value": work / dt, "unit": oracle_unit(wl_name), "cores": threads, "kind": "oracle",
            "sample": desc, "seconds": round(dt, 3)}


def oracle_unit(wl_name):
    import synth
    return "TFLOP/s" if synth.WORKLOADS[wl_name].prompt_len else "GB/s"


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import synth
    w = synth.WORKLOADS[args.workload]
    threads = os.cpu_count() or 1
    budget = 150.0
    per_step = budget / max(1, args.steps + args.warmup)
    dt1, _, _ = oracle_sample(args.workload, threads, threads)
    n_units = int(max(1, per_step / max(dt1, 1e-3) * threads))
    for _ in range(args.warmup):
        oracle_sample(args.workload, n_units, threads)
    secs, work = 0.0, 0.0
    desc = ""
    for _ in range(args.steps):
        dt, wk, desc = oracle_sample(args.workload, n_units, threads)
        secs += dt
        work += wk
    value = work / secs
    unit = oracle_unit(args.workload)
    line = {"impl": "reference", "metric": METRIC if unit == "GB/s" else PROMPT_METRIC,
            "value": value, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(args.workload),
            "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(name):
    import synth
    w = synth.WORKLOADS[name]
    lens = synth.stream_lens(w)
    cfg = {"workload": name, "streams": len(lens), "context": int(lens.max()),
           "kv_heads": w.n_kv_heads, "q_heads": w.n_q_heads, "head_dim": w.head_dim,
           "page_size": w.page_size, "rows": w.rows, "parallelism": "replicas",
           "l2": f"inputs {kv_bytes(lens, w.n_kv_heads, w.head_dim) / 1e9:.2f} GB > 126 MB L2"}
    if w.tree:
        cfg["window"] = "seeded random draft tree per stream (row r sees its ancestors and itself)"
    if w.prompt_len:
        cfg["chunks"] = w.prompt_len // w.rows
        cfg["l2"] = (f"K/V {kv_bytes(lens, w.n_kv_heads, w.head_dim) / 1e6:.1f} MB < 126 MB L2: "
                     "L2 flushed (256 MB write) between timed steps, outside the step's events")
    return cfg


def summary(line):
    """The headline figures of every workload the run measured, compact, so that
    they close the JSON line: per workload its value per step, the attention
    calls' fraction of the measured peak ("frac") and of the vendor's nominal
    peak ("frac_nominal"), and verify tokens/s where the workload has windows."""
    def one(d):
        r = d["roofline"]
        s = {"value": round(d["value"], 1), "unit": d["unit"],
             "ms_per_step": round(d["ms_per_step"], 4), "attn_ms": round(d.get("attn_ms", 0.0), 4),
             "attn_achieved": round(r["achieved"], 1), "frac": round(r["frac"], 3),
             "frac_nominal": round(r["frac_nominal"], 3)}
        if "verify_tokens_per_s" in d:
            s["verify_tokens_per_s"] = round(d["verify_tokens_per_s"])
        return s
    out = {line["config"]["workload"]: one(line)}
    for key in ("verify", "hd512", "prompt"):
        if key in line:
            out[line[key]["workload"]] = one(line[key])
    for v in line.get("variants", []):
        out[v["workload"]] = {"value": round(v["value"], 1), "frac": round(v["roofline"]["frac"], 3),
                              "frac_nominal": round(v["roofline"]["frac_nominal"], 3)}
    if "state_copy" in line:
        out[line["state_copy"]["workload"]] = {"value": round(line["state_copy"]["value"], 1),
                                               "frac": round(line["state_copy"]["roofline"]["frac"], 3),
                                               "check": "MISMATCH" if line["state_copy"]["check"] == "MISMATCH" else "ok"}
    out["peaks"] = {"hbm_gbs": hbm_peak()[0], "bf16_tflops_sustained": tensor_peak()[0],
                    "hbm_nominal_gbs": NOMINAL_HBM_GBS, "bf16_nominal_tflops": NOMINAL_TENSOR_TFLOPS}
    return out


# --------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="decode_12x40k")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-verify", action="store_true", help="skip the verify-workload measurement")
    ap.add_argument("--state-copy", action="store_true",
                    help="time only the state copy (tf_kv_copy_state) of --workload's state")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    def barrier():
        if dist is not None:
            dist.barrier()

    if args.state_copy:
        out = measure_state_copy(args, barrier, dist, world, local, name=args.workload)
        if rank == 0:
            print(json.dumps(out), flush=True)
        if dist is not None:
            dist.destroy_process_group()
        return 0

    wl = Workload(args.workload, f"cuda:{local}")
    uuid = str(torch.cuda.get_device_properties(local).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    sampler.start()
    total_ms, attn_ms = time_steps(wl, args.steps, args.warmup, barrier, sampler)
    sampler.stop()
    wl.check_flags()
    e2e_ms, h2d, d2h = time_e2e(wl, args.steps, args.warmup, barrier)
    wl.check_flags()
    n_parts = len(wl.parts())

    ms_step = total_ms / args.steps
    e2e_step = e2e_ms / args.steps
    if dist is not None:
        t = torch.tensor([ms_step, e2e_step, attn_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_step, e2e_step, attn_ms = t.tolist()
    value, unit = throughput(wl, ms_step, world)
    e2e_value, _ = throughput(wl, e2e_step, world)
    line = {
        "metric": METRIC if not wl.w.prompt_len else PROMPT_METRIC,
        "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(args.workload),
        "roofline": roofline(wl, attn_ms),
        "e2e": {"value": e2e_value, "unit": unit, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": 3 * n_parts * args.steps,
        "clocks": sampler.summary(),
        "rows_per_s": world * wl.rows_per_step / (ms_step * 1e-3),
        "attn_ms": attn_ms,
    }
    del wl
    torch.cuda.empty_cache()

    # the metric's second half (verify tokens/s) and the other workloads, each
    # timed the same way on its own
    if args.workload == "decode_12x40k" and not args.no_verify:
        for name, key in (("verify_4x131k", "verify"), ("hd512_verify", "hd512"),
                          ("prompt_9216", "prompt")):
            line[key] = measure_other(name, args, barrier, dist, world, local)
            torch.cuda.empty_cache()
        # the shape variants the pages mention (GQA 12, GQA 16 at head dim 512,
        # head dim 256), each timed the same way
        line["variants"] = []
        for name in ("gqa12_verify", "gqa16_hd512_decode", "hd256_verify", "tree_verify_4x131k",
                     "decode_12x40k_p37", "decode_64x2k"):
            line["variants"].append(measure_other(name, args, barrier, dist, world, local))
            torch.cuda.empty_cache()
        line["state_copy"] = measure_state_copy(args, barrier, dist, world, local)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import synth
        w0 = synth.WORKLOADS[args.workload]
        n0 = int(synth.stream_lens(w0)[0])
        k, v = synth.kv_rows_torch(w0, 0, n0, f"cuda:{local}")
        line["cpu_baseline"] = cpu_baseline(args.workload, (k, v))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    # last key of the line: the headline figures of every workload measured
    line["summary"] = summary(line)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
