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
e2e    = the same metric through the public API with host buffers: the
         step's query and new rows copied from pinned host memory, the
         output copied back, inside the timed region.
roofline = the attention call (partial + merge kernels) alone, its K/V bytes
         over its CUDA-event time, against the measured HBM copy bandwidth.
cpu_baseline = the fp64 CPU oracle timed on the host on a bounded sample.

With N > 1 (torchrun), every rank runs its own replica of the workload on
its own GPU (the streams are independent; there is no exchange step):
weak scaling, value = all ranks' bytes / the slowest rank's time.
--impl reference times the oracle (rank 0 only) on per-step samples.

The default run also times the draft-verify workload (4 streams at 131,072
positions, 4 KV / 32 query heads, 8-row windows) the same way and reports its
verify tokens/s (window rows per second) under "verify" (--no-verify skips).
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
    def __init__(self, name, device):
        import torch
        import synth
        import verify_paged_gqa_b200 as tf
        self.torch, self.tf = torch, tf
        w = synth.WORKLOADS[name]
        self.w = w
        self.name = name
        self.lens_np = synth.stream_lens(w)
        table, n_pages, _ = synth.page_table(w, self.lens_np)
        self.n_pages = n_pages
        S, W = len(self.lens_np), w.rows
        shape = (n_pages, w.n_kv_heads, w.page_size, w.head_dim)
        self.k_pool = torch.full(shape, float("nan"), dtype=torch.bfloat16, device=device)
        self.v_pool = torch.full(shape, float("nan"), dtype=torch.bfloat16, device=device)
        self.table = torch.from_numpy(table).to(device)
        self.lens = torch.from_numpy(self.lens_np).to(device)
        self.max_len = int(self.lens_np.max())
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
        self.out = torch.empty(self.q.shape, dtype=torch.float32, device=device)
        nbytes = tf.tf_paged_attn_workspace_bytes(self.k_pool, self.v_pool, self.table, self.lens,
                                                  w.n_q_heads, W, self.max_len)
        self.ws = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        self.attn_fn = (tf.tf_paged_attn_decode if W == 1 else
                        tf.tf_paged_attn_verify if W <= 8 else tf.tf_paged_attn_prompt)
        self.bytes_per_step = kv_bytes(self.lens_np, w.n_kv_heads, w.head_dim)
        self.rows_per_step = S * W
        torch.cuda.synchronize()

    def put(self, k_new=None, v_new=None):
        self.tf.tf_kv_put_rows(self.k_pool, self.v_pool, self.table, self.lens,
                               self.k_new if k_new is None else k_new,
                               self.v_new if v_new is None else v_new, max_len=self.max_len)

    def attend(self, q=None):
        self.attn_fn(self.k_pool, self.v_pool, self.table, self.lens,
                     self.q if q is None else q, self.w.scale, self.out, self.ws, self.max_len)

    def step(self):
        self.put()
        self.attend()

    def check_flags(self):
        torch = self.torch
        site = int(self.ws[4:8].view(torch.int32).item())   # which wait gave up, if any
        self.ws[4:8].zero_()
        flags = self.tf.tf_workspace_status(self.ws)
        if flags:
            raise RuntimeError(f"device status word set: {flags:#x} (wait sites {site:#x})")


def time_steps(wl, steps, warmup, barrier, sampler=None):
    torch = wl.torch
    for _ in range(warmup):
        wl.step()
    torch.cuda.synchronize()
    barrier()
    stream = torch.cuda.current_stream()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    if sampler:
        sampler.mark()
    start.record(stream)
    for i in range(steps):
        wl.put()
        ev[i][0].record(stream)
        wl.attend()
        ev[i][1].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    if sampler:
        sampler.mark()
    barrier()
    total_ms = start.elapsed_time(end)
    attn_ms = [a.elapsed_time(b) for a, b in ev]
    return total_ms, statistics.mean(attn_ms)


def time_e2e(wl, steps, warmup, barrier):
    """Same steps through the public API from pinned host buffers (copies inside)."""
    torch = wl.torch
    q_h = wl.q.cpu().pin_memory()
    k_h = wl.k_new.cpu().pin_memory()
    v_h = wl.v_new.cpu().pin_memory()
    out_h = torch.empty(wl.out.shape, dtype=torch.float32).pin_memory()
    q_d, k_d, v_d = torch.empty_like(wl.q), torch.empty_like(wl.k_new), torch.empty_like(wl.v_new)

    def one():
        q_d.copy_(q_h, non_blocking=True)
        k_d.copy_(k_h, non_blocking=True)
        v_d.copy_(v_h, non_blocking=True)
        wl.put(k_d, v_d)
        wl.attend(q_d)
        out_h.copy_(wl.out, non_blocking=True)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    barrier()
    stream = torch.cuda.current_stream()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        one()
    end.record(stream)
    torch.cuda.synchronize()
    barrier()
    h2d = (q_h.numel() * q_h.element_size() + k_h.numel() * k_h.element_size()
           + v_h.numel() * v_h.element_size())
    d2h = out_h.numel() * out_h.element_size()
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
    per_unit = w.head_dim * 2 * 2 / w.group          # one query head's share of a K/V row
    nbytes = sum((n0 - w.rows + int(r) + 1) * per_unit for _, r, _ in units)
    desc = (f"{len(units)} (stream, row, query head) output rows of stream 0 at {n0} positions "
            f"(the stream's {len(base)} rows, repeated), fp64, {threads} threads")
    return dt, nbytes, desc


def cpu_baseline(wl_name, device_kv, budget_s=12.0):
    threads = os.cpu_count() or 1
    dt1, _, _ = oracle_sample(wl_name, threads, threads, device_kv)
    n = int(max(threads, budget_s / max(dt1, 1e-3) * threads))
    dt, nbytes, desc = oracle_sample(wl_name, n, threads, device_kv)
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": desc, "seconds": round(dt, 3)}


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
    secs, nbytes = 0.0, 0.0
    desc = ""
    for _ in range(args.steps):
        dt, nb, desc = oracle_sample(args.workload, n_units, threads)
        secs += dt
        nbytes += nb
    value = nbytes / secs / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(args.workload),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(name):
    import synth
    w = synth.WORKLOADS[name]
    lens = synth.stream_lens(w)
    return {"workload": name, "streams": len(lens), "context": int(lens.max()),
            "kv_heads": w.n_kv_heads, "q_heads": w.n_q_heads, "head_dim": w.head_dim,
            "page_size": w.page_size, "rows": w.rows, "parallelism": "replicas",
            "l2": f"inputs {kv_bytes(lens, w.n_kv_heads, w.head_dim) / 1e9:.2f} GB > 126 MB L2"}


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

    wl = Workload(args.workload, f"cuda:{local}")
    uuid = str(torch.cuda.get_device_properties(local).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    sampler.start()
    total_ms, attn_ms = time_steps(wl, args.steps, args.warmup, barrier, sampler)
    sampler.stop()
    wl.check_flags()
    e2e_ms, h2d, d2h = time_e2e(wl, args.steps, args.warmup, barrier)
    wl.check_flags()
    bytes_per_step, rows_per_step = wl.bytes_per_step, wl.rows_per_step

    # the metric's second half: verify tokens/s on the draft-verify workload
    secondary = None
    if args.workload == "decode_12x40k" and not args.no_verify:
        del wl
        torch.cuda.empty_cache()
        vw = Workload("verify_4x131k", f"cuda:{local}")
        v_total, v_attn = time_steps(vw, args.steps, args.warmup, barrier)
        vw.check_flags()
        v_step = v_total / args.steps
        if dist is not None:
            t = torch.tensor([v_step, v_attn], device="cuda")
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            v_step, v_attn = t.tolist()
        v_ach = vw.bytes_per_step / (v_attn * 1e-3) / 1e9
        peak_v, _ = hbm_peak()
        secondary = {"workload": "verify_4x131k", "verify_tokens_per_s": world * vw.rows_per_step / (v_step * 1e-3),
                     "kv_gbs": world * vw.bytes_per_step / (v_step * 1e-3) / 1e9, "ms_per_step": v_step,
                     "attn_ms": v_attn, "roofline_frac": v_ach / peak_v,
                     "traffic": recorded_traffic("verify_4x131k"),
                     "gpu_launches": 3 * args.steps, "config": workload_config("verify_4x131k")}
        del vw
        torch.cuda.empty_cache()

    ms_step = total_ms / args.steps
    e2e_step = e2e_ms / args.steps
    if dist is not None:
        t = torch.tensor([ms_step, e2e_step, attn_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_step, e2e_step, attn_ms = t.tolist()
    value = world * bytes_per_step / (ms_step * 1e-3) / 1e9
    e2e_value = world * bytes_per_step / (e2e_step * 1e-3) / 1e9
    peak, src = hbm_peak()
    achieved = bytes_per_step / (attn_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(args.workload),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": recorded_traffic(args.workload),
                     "kernel": "attention call (partial + merge)", "peak_source": src},
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": 3 * args.steps,
        "clocks": sampler.summary(),
        "rows_per_s": world * rows_per_step / (ms_step * 1e-3),
        "attn_ms": attn_ms,
    }
    if secondary is not None:
        line["verify"] = secondary
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import synth
        w0 = synth.WORKLOADS[args.workload]
        n0 = int(synth.stream_lens(w0)[0])
        k, v = synth.kv_rows_torch(w0, 0, n0, f"cuda:{local}")
        line["cpu_baseline"] = cpu_baseline(args.workload, (k, v))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
