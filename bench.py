"""Benchmark of the DSA forward hot path on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode_128k_paged]

A step is one pass of all three stages (indexer -> top-k -> sparse MLA) over
one batch of the workload: for the default 128K paged decode workload, 16
sequences x 2 query rows with contexts drawn from [98304, 131072], one
dsa_decode_step call; for the prefill workloads (--workload prefill_8k or
prefill_64k), one dsa_forward call over the whole causal sequence.  The metric
is query-tokens/s of one DSA layer.  The per-stage breakdown comes from an
untimed pass: events the library records between its launches (decode), or
the three stage calls over the whole batch (prefill).

Under torchrun each rank runs its own batch (different seed, same shapes):
weak scaling, no collective on the data path; the barrier and the max over
ranks of the device time are the only cross-rank steps.

`--impl reference` times the float64 CPU oracle (the only reference this
method has) on a bounded sample of the same workload.

`--op cache_append` measures the write that precedes the three stages
instead: the workload's new tokens (a decode step's 32; all 65,536 of the 64K
prefill, the default for this op) quantised to FP8 and written into the paged
caches by one dsa_cache_append call.  Its metric is appended tokens/s.

`--op output_projection` measures the two GEMMs after the path (u = W_UV o
per head, y = W_out u) for the workload's query rows (32 in decode, 65,536 in
the 64K prefill) with H = 128, d_c = 512, d_v = 128, d_model = 7168: one
dsa_output_projection call per step.  Its metric is rows/s.

`--op warmup` measures a warm-up step of the indexer on the 8-16K decode batch
(default): indexer scores, KL to a seeded teacher with its gradient, and the
backward to q_I, w and k_I (dsa_indexer_scores, dsa_indexer_kl,
dsa_indexer_backward).  Its metric is query-rows/s.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DSA layer query-tokens/s at 128K decode & 64K prefill; % of roofline"
UNIT = "query-tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=None,
                    help="decode_128k_paged (path default) or prefill_64k (cache_append default)")
    ap.add_argument("--op", default="path",
                    choices=["path", "cache_append", "output_projection", "warmup"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=4, help="oracle rows per CPU-baseline sample")
    ap.add_argument("--n-seqs", type=int, default=None, help="smaller batch (profiling captures)")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the 64K prefill measurement that the default decode run adds")
    return ap.parse_args()


def dist_info():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def rank_config(cfg, rank: int):
    """The batch of one rank: same shapes, its own seed (weak scaling)."""
    return cfg.replace(seed=cfg.seed + 1000 * rank)


def max_over_ranks(value: float, world: int, device=None) -> float:
    """MAX of a per-rank device time over all ranks (the only data-free collective)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(world: int, rows_per_rank: int, steps: int, total_ms: float) -> float:
    """Whole-job query-tokens/s: all ranks' rows over the slowest rank's time."""
    return world * rows_per_rank * steps / (total_ms / 1e3)


def path_config(cfg, rows_per_gpu: int, world: int) -> dict:
    """The `config` object of a path line; both arms print the same one."""
    return {"workload": workload_desc(cfg), "rows_per_gpu": int(rows_per_gpu),
            "l2": "flushed before every step (256 MiB write, untimed)",
            "parallelism": f"{world} independent ranks (weak scaling)"}


def workload_desc(cfg) -> str:
    if cfg.prefill:
        head = f"prefill L={cfg.seq_len}"
    else:
        head = (f"decode {cfg.n_seqs} seqs x {cfg.rows_per_seq} rows, ctx U[{cfg.ctx_lo},{cfg.ctx_hi}]"
                + (", 64-token pages, shuffled block table" if cfg.paged else ", contiguous cache"))
    return (f"{cfg.name}: {head}; indexer H_I={cfg.h_idx} d_I={cfg.d_idx} "
            f"{'e4m3+per-token fp32 scales' if cfg.fp8 else 'fp32'}; top-k={cfg.topk}; "
            f"MLA H={cfg.n_heads} d_c={cfg.d_c} d_r={cfg.d_r} {'bf16' if cfg.bf16 else 'fp32'}")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- peaks
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_traffic(kernel: str, workload: str, alg_bytes: int):
    """DRAM bytes per launch of `kernel` on this launch's work, from a committed
    ncu capture: the captured launch's DRAM bytes scaled by the ratio of
    algorithmic bytes (the capture may be of a smaller batch of the same
    workload, where traffic grows with the keys processed).  None when any
    source of the kernel changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(f"{kernel}@{workload}")
    if not d:
        return None
    h = hashlib.sha256()
    for s in d["sources"]:
        src = os.path.join(ROOT, s)
        if not os.path.exists(src):
            return None
        h.update(open(src, "rb").read())
    if h.hexdigest() != d["sha256"]:
        return None
    return d["dram_bytes"] * alg_bytes / d["algorithmic_bytes"]


# ----------------------------------------------------------------------------- oracle arm
def oracle_rows_per_s(inp, rows, reps=1):
    from oracle import dsa_ref as R
    t0 = time.perf_counter()
    for _ in range(reps):
        R.dsa_forward_rows(inp, rows)
    dt = time.perf_counter() - t0
    return reps * len(rows) / dt, dt


def sample_rows(inp, n):
    import numpy as np
    T = len(inp["row_seq"])
    return sorted(set(np.linspace(0, T - 1, n).astype(int).tolist()))


def run_reference(args):
    rank, world, _ = dist_info()
    if rank != 0:
        return 0
    from long_context_sparse_04_b200 import inputs as I
    cfg = I.CONFIGS[args.workload]
    inp = I.generate(cfg, with_q=True)
    rows = sample_rows(inp, 1)
    cores = len(os.sched_getaffinity(0))
    for _ in range(args.warmup):
        oracle_rows_per_s(inp, rows[:1])
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_rows_per_s(inp, rows)
    dt = time.perf_counter() - t0
    value = args.steps * len(rows) / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": path_config(cfg, len(inp["row_seq"]), world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{len(rows)} of {len(inp['row_seq'])} query rows per step "
                                   f"(all three stages, float64 NumPy)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- our arm
def algorithmic(cfg, inp, stage):
    """Algorithmic bytes / FLOPs of one launch of a stage on this batch."""
    import numpy as np
    klen = inp["row_klen"].astype(np.int64)
    seqs = inp["row_seq"]
    T = len(klen)
    if stage == "indexer":
        # keys of each sequence read once for all its rows: 128 B e4m3 + 4 B scale per key
        per_seq = {}
        for s, k in zip(seqs, klen):
            per_seq[int(s)] = max(per_seq.get(int(s), 0), int(k))
        by = sum(per_seq.values()) * (cfg.d_idx + 4)
        fl = 2 * cfg.h_idx * cfg.d_idx * int(klen.sum())
        return {"bytes": by, "flops": fl}
    if stage == "topk":
        return {"bytes": int(klen.sum()) * 4 + T * cfg.topk * 4, "flops": 0}
    sel = np.minimum(klen, cfg.topk)
    by = int(sel.sum()) * cfg.d_qk * 2 + T * cfg.n_heads * (cfg.d_qk + cfg.d_c) * 2
    fl = int(sel.sum()) * 2 * cfg.n_heads * (cfg.d_qk + cfg.d_c)
    return {"bytes": by, "flops": fl}


def measure_e2e_pipelined(N, torch, wl, out, lse, dev, stream, world, T, steps, warmup):
    """End to end over `steps` decode steps through the C ABI, each step's
    inputs copied in from pinned host memory and its outputs copied back, the
    way a serving loop overlaps them: step i computes on the main stream while
    step i+1's inputs copy in on one stream and step i-1's outputs copy out on
    another (two sets of device buffers).  Timed from the first input copy to
    the last output copy.  No L2 flush between steps: a step reads ~311 MB of
    caches, more than the 126 MB L2."""
    from long_context_sparse_04_b200.workload import _vp
    keys = [k for k in ("q_idx", "q_scale", "w", "q", "row_klen") if getattr(wl, k) is not None]
    host_in = {k: getattr(wl, k).cpu().pin_memory() for k in keys}
    dev_in = [{k: torch.empty_like(getattr(wl, k)) for k in keys} for _ in range(2)]
    dev_out = [(torch.empty_like(out), torch.empty_like(lse)) for _ in range(2)]
    host_out = [(torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                 torch.empty(lse.shape, dtype=lse.dtype).pin_memory()) for _ in range(2)]
    rows = [N.dsa_rows(num_rows=wl.rows.num_rows, row_seq=wl.rows.row_seq,
                       row_klen=_vp(dev_in[b]["row_klen"]), max_klen=wl.rows.max_klen,
                       q_group=wl.rows.q_group) for b in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out[0])
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=False)
    in_ready, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    saved = {k: getattr(wl, k) for k in keys}, wl.rows

    def enqueue(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(comp_done[b])        # step i-2 has read this input set
            for k in keys:
                dev_in[b][k].copy_(host_in[k], non_blocking=True)
            in_ready[b].record(s_in)
        stream.wait_event(in_ready[b])
        if i >= 2:
            stream.wait_event(out_done[b])           # step i-2's outputs are copied out
        for k in keys:
            setattr(wl, k, dev_in[b][k])
        wl.rows = rows[b]
        wl.decode_step(out=dev_out[b][0], lse=dev_out[b][1])
        comp_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[b])
            host_out[b][0].copy_(dev_out[b][0], non_blocking=True)
            host_out[b][1].copy_(dev_out[b][1], non_blocking=True)
            out_done[b].record(s_out)

    try:
        for i in range(max(warmup, 2)):
            enqueue(i)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for i in range(steps):
            enqueue(i)
        e1.record(s_out)
        torch.cuda.synchronize(dev)
        tot = max_over_ranks(e0.elapsed_time(e1), world, dev)
        # the last step's outputs read back equal the device outputs
        assert torch.equal(host_out[(steps - 1) % 2][1], dev_out[(steps - 1) % 2][1].cpu())
    finally:
        for k, v in saved[0].items():
            setattr(wl, k, v)
        wl.rows = saved[1]
    return {"value": throughput(world, T, steps, tot), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "overlap": "step i runs while step i+1's inputs copy in and step i-1's outputs copy out",
            "l2": "not flushed between steps (each reads ~311 MB of caches, above the 126 MB L2)"}


def measure_path(args, cfg, dev, rank: int, world: int, steps: int, warmup: int,
                 want_e2e: bool, want_cpu: bool) -> dict:
    """Time `steps` passes of the whole path over one batch of `cfg` on `dev`:
    device time per step (max over ranks), per-stage breakdown, roofline of the
    dominant stage, and optionally the end-to-end and host-oracle figures."""
    import torch

    from long_context_sparse_04_b200 import _native as N
    from long_context_sparse_04_b200 import inputs as I
    from long_context_sparse_04_b200.workload import DeviceWorkload

    cfg_r = rank_config(cfg, rank)
    inp = I.generate(cfg_r, threads=max(4, min(32, len(os.sched_getaffinity(0)))))
    wl = DeviceWorkload(inp, device=dev)
    T = wl.T
    stream = torch.cuda.current_stream(dev)

    # L2 flush buffer (larger than the 126 MB L2), written before every timed step
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for e in ev:                 # torch creates the CUDA event on its first record
        e.record(stream)
    torch.cuda.synchronize(dev)
    step_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    out = torch.empty((T, wl.H, wl.d_c), dtype=wl.out_dtype(), device=dev)
    lse = torch.empty((T, wl.H), dtype=torch.float32, device=dev)
    prefill = bool(cfg.prefill)
    op = N.DSA_OP_FORWARD if prefill else N.DSA_OP_DECODE_STEP
    idx_out = torch.empty((T, wl.topk), dtype=torch.int32, device=dev) if prefill else None

    def step():
        # one pass of the whole hot path over the batch: the fused decode call,
        # or the chunked prefill forward
        if prefill:
            wl.forward(out=out, lse=lse, idx=idx_out)
        else:
            wl.decode_step(out=out, lse=lse)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(max(warmup, 0)):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    st = wl.status(op)
    ran = wl.kernels_ran(op)
    assert st == (0, -1), f"device status {st}"

    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    clocks.start()
    # keep the GPU busy with identical untimed steps for ~1.5 s so the clock
    # samples (10 Hz) are taken under this load; the timed steps follow at once
    t_end = time.perf_counter() + 1.5
    while time.perf_counter() < t_end:
        for _ in range(20 if not prefill else 1):
            flush.zero_()
            step()
        torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    # timed steps: one event pair around each call (events between the
    # kernels of a call would cut their programmatic overlap)
    step_ms = []
    for _ in range(steps):
        flush.zero_()
        step_ev[0].record(stream)
        step()
        step_ev[1].record(stream)
        torch.cuda.synchronize(dev)
        step_ms.append(step_ev[0].elapsed_time(step_ev[1]))
    barrier()
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    # per-stage breakdown (untimed for the headline)
    stage_ms = {"indexer": [], "topk": [], "mla": []}
    if prefill:
        # the three stage calls over the whole batch (the forward runs them
        # per 512-row chunk)
        scores = torch.empty((T, wl.ld), dtype=torch.float32, device=dev)
        for _ in range(steps):
            flush.zero_()
            ev[0].record(stream)
            wl.indexer(scores)
            ev[1].record(stream)
            wl.topk_(scores, idx_out)
            ev[2].record(stream)
            wl.mla(idx_out, out, lse)
            ev[3].record(stream)
            torch.cuda.synchronize(dev)
            stage_ms["indexer"].append(ev[0].elapsed_time(ev[1]))
            stage_ms["topk"].append(ev[1].elapsed_time(ev[2]))
            stage_ms["mla"].append(ev[2].elapsed_time(ev[3]))
        del scores
    else:
        # the library records events between its launches
        N.dsa_set_stage_events([e.cuda_event for e in ev])
        for _ in range(steps):
            flush.zero_()
            wl.decode_step(out=out, lse=lse)
            torch.cuda.synchronize(dev)
            stage_ms["indexer"].append(ev[0].elapsed_time(ev[1]))
            stage_ms["topk"].append(ev[1].elapsed_time(ev[2]))
            stage_ms["mla"].append(ev[2].elapsed_time(ev[3]))
        N.dsa_set_stage_events([])
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    ms_per_step = total_ms / steps
    value = throughput(world, T, steps, total_ms)
    launches_per_step = path_launches(N, ran, T, prefill)

    # ---- end to end through the C ABI from pinned host buffers
    e2e = None
    if want_e2e and not prefill:
        e2e = measure_e2e_pipelined(N, torch, wl, out, lse, dev, stream, world, T, steps, warmup)
    elif want_e2e:
        host_in = {k: getattr(wl, k).cpu().pin_memory() for k in ("q_idx", "q_scale", "w", "q", "row_klen")
                   if getattr(wl, k) is not None}
        host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        host_lse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in host_in.values())
        d2h = host_out.numel() * host_out.element_size() + host_lse.numel() * host_lse.element_size()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        tot = 0.0
        for i in range(warmup + steps):
            flush.zero_()
            e0.record(stream)
            for k, v in host_in.items():
                getattr(wl, k).copy_(v, non_blocking=True)
            step()
            host_out.copy_(out, non_blocking=True)
            host_lse.copy_(lse, non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            if i >= warmup:
                tot += e0.elapsed_time(e1)
        tot = max_over_ranks(tot, world, dev)
        e2e = {"value": throughput(world, T, steps, tot), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}

    # ---- roofline of the dominant kernel
    peaks, peak_kind = measured_peaks()
    avg = {k: statistics.mean(v) for k, v in stage_ms.items()}
    dom = max(avg, key=avg.get)
    alg = algorithmic(cfg_r, inp, dom)
    mla_tc = bool(ran & N.DSA_KERNEL_MLA_TC)
    idx_tc = bool(ran & N.DSA_KERNEL_INDEXER_TC)
    simt = (dom == "mla" and not mla_tc) or (dom == "indexer" and not idx_tc)
    if simt:
        # CUDA-core fp32 kernels: 148 SMs x 128 fp32 lanes x 2 FLOP (FMA) at
        # the maximum SM clock
        bound = "alu"
        achieved = alg["flops"] / (avg[dom] / 1e3) / 1e12
        peak = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
        unit = "TFLOP/s"
        peak_kind = "derived (SM count x fp32 lanes x 2 x max SM clock)"
    elif dom == "mla":
        bound = "tensor"
        achieved = alg["flops"] / (avg[dom] / 1e3) / 1e12
        peak = peaks.get("bf16_tflops")
        unit = "TFLOP/s"
    elif dom == "indexer" and prefill:
        # FP8 contraction: no measured fp8 peak; the nominal fp8/bf16 ratio (2)
        # times the measured bf16 peak
        bound = "tensor"
        achieved = alg["flops"] / (avg[dom] / 1e3) / 1e12
        peak = 2.0 * peaks.get("bf16_tflops") if peaks.get("bf16_tflops") else None
        unit = "TFLOP/s"
        peak_kind = peak_kind + " (bf16 x 2, the nominal fp8/bf16 ratio)"
    else:
        bound = "hbm"
        achieved = alg["bytes"] / (avg[dom] / 1e3) / 1e9
        peak = peaks.get("hbm_gbs")
        unit = "GB/s"
    kname = {"indexer": "indexer_tc_kernel" if idx_tc else "indexer_simt_kernel", "topk": "topk_kernel",
             "mla": "mla_tc_kernel" if mla_tc else "mla_simt_kernel"}[dom]
    roof = {"kernel": kname, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": achieved / peak if peak else None, "peak_source": peak_kind,
            "traffic": kernel_traffic(kname, cfg.name, alg["bytes"]),
            "algorithmic_per_launch": alg["bytes"] if bound == "hbm" else alg["flops"]}
    stages = {}
    for k in avg:
        a = algorithmic(cfg_r, inp, k)
        s = avg[k] / 1e3
        stages[k] = {"us": 1e3 * avg[k], "hbm_gbs": a["bytes"] / s / 1e9,
                     "tflops": a["flops"] / s / 1e12}

    cpu = None
    if want_cpu and rank == 0 and world == 1:
        # bounded sample: about 10-20 s of oracle work on the host cores
        _, t1 = oracle_rows_per_s(inp, sample_rows(inp, 1))
        n = int(max(1, min(T, 12.0 / max(t1, 1e-3))))
        reps = int(max(1, min(8, 12.0 / max(t1 * n, 1e-3))))
        rows = sample_rows(inp, n)
        v, dt = oracle_rows_per_s(inp, rows, reps)
        cpu = {"value": v, "unit": UNIT, "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
               "sample": f"{len(rows)} of {T} query rows of one batch x {reps}, all three "
                         f"stages, float64 NumPy, {dt:.1f} s"}
    del wl, inp, out, lse, idx_out, flush
    torch.cuda.empty_cache()
    return {"T": T, "value": value, "ms_per_step": ms_per_step, "steps": steps, "warmup": warmup,
            "stages": stages, "roofline": roof, "e2e": e2e, "cpu_baseline": cpu,
            "gpu_launches": launches_per_step * steps, "clocks": clk}


def path_launches(N, ran: int, T: int, prefill: bool) -> int:
    """Kernels of this library one step launches: indexer, top-k and attention
    (the split-K combine runs inside the attention kernel)."""
    if prefill:   # three kernels per 512-row chunk
        return 3 * ((T + 511) // 512)
    return 3


def run_ours(args):
    import torch
    rank, world, local = dist_info()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)

    from long_context_sparse_04_b200 import build
    build.build()
    from long_context_sparse_04_b200 import inputs as I

    cfg = I.CONFIGS[args.workload]
    if args.n_seqs:
        cfg = cfg.replace(n_seqs=args.n_seqs)
    m = measure_path(args, cfg, dev, rank, world, args.steps, args.warmup,
                     want_e2e=not args.no_e2e, want_cpu=not args.no_cpu_baseline)
    # The metric names both halves: the 128K decode step is the headline value
    # and the 64K causal prefill is measured in the same run (one GPU only: a
    # 64K workload holds ~11 GB of inputs per rank), a few steps of one
    # dsa_forward over all 65,536 rows each.
    pre = None
    if (world == 1 and args.workload == "decode_128k_paged" and not args.n_seqs
            and not args.no_prefill):
        p = measure_path(args, I.CONFIGS["prefill_64k"], dev, rank, world, 3, 3,
                         want_e2e=False, want_cpu=False)
        pre = {"workload": workload_desc(I.CONFIGS["prefill_64k"]), "value": p["value"],
               "unit": UNIT, "ms_per_step": p["ms_per_step"], "steps": p["steps"],
               "warmup": p["warmup"], "stages": p["stages"], "roofline": p["roofline"],
               "gpu_launches": p["gpu_launches"], "clocks": p["clocks"]}

    if rank == 0:
        line = {
            "metric": METRIC, "value": m["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp8e4m3+bf16 (fp32 accumulate)",
            "data": "synthetic",
            "config": path_config(cfg, m["T"], world),
            "stages": m["stages"], "roofline": m["roofline"], "cpu_baseline": m["cpu_baseline"],
            "e2e": m["e2e"],
            "gpu_launches": m["gpu_launches"],
            "clocks": m["clocks"],
        }
        if pre is not None:
            line["prefill_64k"] = pre
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------- cache append
APPEND_METRIC = "cache-append tokens/s (fused FP8 quantise + paged cache write)"
APPEND_UNIT = "tokens/s"


def append_bytes_per_token(cfg) -> int:
    """Algorithmic bytes of one appended token: the fp32 key, the latent row,
    its (seq, pos) and one block-table (or seq_start) entry read; the codes,
    the scale and the latent row written."""
    lat = cfg.d_qk * (2 if cfg.bf16 else 4)
    key_in = 4 * cfg.d_idx
    key_out = cfg.d_idx + 4 if cfg.fp8 else 4 * cfg.d_idx
    return key_in + lat + 8 + 4 + key_out + lat


def append_inputs(cfg):
    from long_context_sparse_04_b200 import inputs as I
    tok_seq, tok_pos = I.new_tokens(cfg)
    k_new, lat_new = I.token_keys(cfg, tok_seq, tok_pos)
    return tok_seq, tok_pos, k_new, lat_new


def oracle_append_tokens_per_s(inp, cfg, toks, n):
    from oracle import dsa_ref as R
    tok_seq, tok_pos, k_new, lat_new = toks
    c = inp["cache"]
    num_seqs = c["block_table"].shape[0] if c["block_table"] is not None else len(c["seq_start"])
    t0 = time.perf_counter()
    R.cache_append(inp, num_seqs, tok_seq[:n], tok_pos[:n], k_new[:n], lat_new[:n])
    dt = time.perf_counter() - t0
    return n / dt, dt


def run_append_reference(args, cfg):
    from long_context_sparse_04_b200 import inputs as I
    inp = I.generate(cfg, with_q=False, rows=[])       # the caches only
    toks = append_inputs(cfg)
    n_tok = len(toks[0])
    n = min(n_tok, 500)
    for _ in range(args.warmup):
        oracle_append_tokens_per_s(inp, cfg, toks, min(n, 16))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_append_tokens_per_s(inp, cfg, toks, n)
    dt = time.perf_counter() - t0
    value = args.steps * n / dt
    line = {
        "impl": "reference", "metric": APPEND_METRIC, "value": value, "unit": APPEND_UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 -> e4m3", "data": "synthetic",
        "config": {"workload": workload_desc(cfg), "tokens_per_step": n_tok},
        "cpu_baseline": {"value": value, "unit": APPEND_UNIT, "cores": len(os.sched_getaffinity(0)),
                         "kind": "oracle", "sample": f"{n} of {n_tok} tokens per step (NumPy)"},
        "e2e": {"value": value, "unit": APPEND_UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_append(args):
    """One dsa_cache_append of the workload's new tokens per step."""
    import numpy as np
    import torch
    rank, world, local = dist_info()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    from long_context_sparse_04_b200 import build
    build.build()
    from long_context_sparse_04_b200 import _native as N
    from long_context_sparse_04_b200 import inputs as I
    from long_context_sparse_04_b200.workload import DeviceWorkload, to_device

    cfg = I.CONFIGS[args.workload]
    if args.n_seqs:
        cfg = cfg.replace(n_seqs=args.n_seqs)
    cfg_r = rank_config(cfg, rank)
    inp = I.generate(cfg_r, with_q=False, rows=[])     # the caches only
    wl = DeviceWorkload(inp, device=dev)
    toks = append_inputs(cfg_r)
    n_tok = len(toks[0])
    d_in = [to_device(np.ascontiguousarray(toks[0], np.int32), dev),
            to_device(np.ascontiguousarray(toks[1], np.int32), dev),
            to_device(np.ascontiguousarray(toks[2], np.float32), dev), to_device(toks[3], dev)]
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def step():
        wl.append(*d_in)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(max(args.warmup, 0)):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    st = wl.status(N.DSA_OP_CACHE_APPEND)
    assert st == (0, -1), f"device status {st}"
    assert wl.kernels_ran(N.DSA_OP_CACHE_APPEND) & N.DSA_KERNEL_CACHE_APPEND

    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    clocks.start()
    t_end = time.perf_counter() + 1.5
    while time.perf_counter() < t_end:
        for _ in range(20):
            flush.zero_()
            step()
        torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    ms = []
    for _ in range(args.steps):
        flush.zero_()
        e0.record(stream)
        step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms.append(e0.elapsed_time(e1))
    barrier()
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    total_ms = max_over_ranks(sum(ms), world, dev)
    value = throughput(world, n_tok, args.steps, total_ms)

    e2e = None
    if not args.no_e2e:
        host = [x.cpu().pin_memory() for x in d_in]
        ws, ws_n = wl.workspace(N.DSA_OP_CACHE_APPEND)
        host_st = torch.empty(8, dtype=torch.uint8).pin_memory()
        h2d = sum(x.numel() * x.element_size() for x in host)
        tot = 0.0
        for i in range(args.warmup + args.steps):
            flush.zero_()
            e0.record(stream)
            for d, h in zip(d_in, host):
                d.copy_(h, non_blocking=True)
            step()
            host_st.copy_(ws[:8], non_blocking=True)   # the status word: the step's result
            e1.record(stream)
            torch.cuda.synchronize(dev)
            if i >= args.warmup:
                tot += e0.elapsed_time(e1)
        tot = max_over_ranks(tot, world, dev)
        e2e = {"value": throughput(world, n_tok, args.steps, tot), "unit": APPEND_UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": 8}

    peaks, peak_kind = measured_peaks()
    avg_s = statistics.mean(ms) / 1e3
    alg = append_bytes_per_token(cfg_r) * n_tok
    achieved = alg / avg_s / 1e9
    peak = peaks.get("hbm_gbs")
    roof = {"kernel": "cache_append_kernel", "bound": "hbm", "achieved": achieved, "peak": peak,
            "unit": "GB/s", "frac": achieved / peak if peak else None, "peak_source": peak_kind,
            "traffic": kernel_traffic("cache_append_kernel", args.workload, alg),
            "algorithmic_per_launch": alg}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        _, t1 = oracle_append_tokens_per_s(inp, cfg_r, toks, min(n_tok, 16))
        n = int(max(1, min(n_tok, 16 * 10.0 / max(t1, 1e-4))))
        v, dt = oracle_append_tokens_per_s(inp, cfg_r, toks, n)
        cpu = {"value": v, "unit": APPEND_UNIT, "cores": len(os.sched_getaffinity(0)),
               "kind": "oracle", "sample": f"{n} of {n_tok} tokens of one step, NumPy, {dt:.1f} s"}

    if rank == 0:
        line = {
            "metric": APPEND_METRIC, "value": value, "unit": APPEND_UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32 -> e4m3 (+ bf16 copy)", "data": "synthetic",
            "config": {"workload": workload_desc(cfg), "tokens_per_step": n_tok,
                       "l2": "flushed before every step (256 MiB write, untimed)",
                       "parallelism": f"{world} independent ranks (weak scaling)"},
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------- output projection
PROJ_METRIC = "output-projection rows/s (u = W_UV o per head, y = W_out u)"
PROJ_UNIT = "rows/s"


def proj_algorithmic(cfg, T):
    """FLOPs and minimum HBM bytes of one dsa_output_projection call: both
    weight matrices read once, o read, u written and read back, y written."""
    H, d_c, d_v, dm = cfg.n_heads, cfg.d_c, cfg.d_v, cfg.d_model
    flops = 2 * T * H * d_v * (d_c + dm)
    by = 2 * (H * d_v * d_c + dm * H * d_v) + 2 * T * (H * d_c + 2 * H * d_v + dm)
    return flops, by


def oracle_proj_rows_per_s(o_bits, w_uv, w_out, rows):
    from oracle import dsa_ref as R
    wu, wo = R.bf16_decode(w_uv), R.bf16_decode(w_out)
    t0 = time.perf_counter()
    for t in rows:
        R.output_projection_row(R.bf16_decode(o_bits[t]), wu, wo)
    dt = time.perf_counter() - t0
    return len(rows) / dt, dt


def run_out_proj(args):
    import ctypes
    import numpy as np
    import torch
    rank, world, local = dist_info()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    from long_context_sparse_04_b200 import build
    build.build()
    from long_context_sparse_04_b200 import _native as N
    from long_context_sparse_04_b200 import inputs as I
    from long_context_sparse_04_b200.workload import to_device

    cfg = rank_config(I.CONFIGS[args.workload], rank)
    T = cfg.n_rows
    w_uv_h, w_out_h = I.out_proj_weights(cfg)
    blk = min(T, 1024)
    o_blk = I.latent_out_rows(cfg, range(blk))
    o = to_device(o_blk, dev).repeat((T + blk - 1) // blk, 1, 1)[:T].contiguous()
    w_uv, w_out = to_device(w_uv_h, dev), to_device(w_out_h, dev)
    u = torch.empty((T, cfg.n_heads, cfg.d_v), dtype=torch.bfloat16, device=dev)
    y = torch.empty((T, cfg.d_model), dtype=torch.bfloat16, device=dev)
    dims = N.dsa_proj_dims(n_heads=cfg.n_heads, d_c=cfg.d_c, d_v=cfg.d_v, d_model=cfg.d_model)
    nbytes = N.dsa_output_projection_ws_size(dims, T)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = ctypes.c_void_p(stream.cuda_stream)
    vp = lambda x: ctypes.c_void_p(x.data_ptr())
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def step():
        N.dsa_output_projection(dims, T, vp(o), vp(w_uv), vp(w_out), vp(u), vp(y), vp(ws), nbytes, sp)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(max(args.warmup, 0)):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    st = N.dsa_read_device_status(vp(ws), sp)
    assert st == (0, -1), f"device status {st}"
    ran = N.dsa_read_kernel_trace(vp(ws), sp)
    assert ran & N.DSA_KERNEL_OUT_PROJ

    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    clocks.start()
    t_end = time.perf_counter() + 1.5
    while time.perf_counter() < t_end:
        for _ in range(20 if T < 4096 else 1):
            flush.zero_()
            step()
        torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    ms = []
    for _ in range(args.steps):
        flush.zero_()
        e0.record(stream)
        step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms.append(e0.elapsed_time(e1))
    barrier()
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    total_ms = max_over_ranks(sum(ms), world, dev)
    value = throughput(world, T, args.steps, total_ms)
    launches = 2 + (1 if ran & N.DSA_KERNEL_OUT_PROJ_REDUCE else 0)

    e2e = None
    if not args.no_e2e and T * cfg.n_heads * cfg.d_c * 2 <= (1 << 30):
        host_o = o.cpu().pin_memory()
        host_y = torch.empty(y.shape, dtype=y.dtype).pin_memory()
        tot = 0.0
        for i in range(args.warmup + args.steps):
            flush.zero_()
            e0.record(stream)
            o.copy_(host_o, non_blocking=True)
            step()
            host_y.copy_(y, non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            if i >= args.warmup:
                tot += e0.elapsed_time(e1)
        tot = max_over_ranks(tot, world, dev)
        e2e = {"value": throughput(world, T, args.steps, tot), "unit": PROJ_UNIT,
               "h2d_bytes_per_step": host_o.numel() * 2, "d2h_bytes_per_step": host_y.numel() * 2}

    peaks, peak_kind = measured_peaks()
    avg_s = statistics.mean(ms) / 1e3
    flops, by = proj_algorithmic(cfg, T)
    if T >= 4096:      # the products are tensor-bound at prefill batch sizes
        roof = {"kernel": "out_proj_kernel (both launches)", "bound": "tensor",
                "achieved": flops / avg_s / 1e12, "peak": peaks.get("bf16_tflops"), "unit": "TFLOP/s",
                "algorithmic_per_launch": flops}
    else:              # decode: the weights' HBM stream
        roof = {"kernel": "out_proj_kernel (both launches)", "bound": "hbm",
                "achieved": by / avg_s / 1e9, "peak": peaks.get("hbm_gbs"), "unit": "GB/s",
                "algorithmic_per_launch": by}
    roof["frac"] = roof["achieved"] / roof["peak"] if roof["peak"] else None
    roof["peak_source"] = peak_kind
    roof["traffic"] = kernel_traffic("out_proj_kernel", args.workload, by)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        _, t1 = oracle_proj_rows_per_s(o_blk, w_uv_h, w_out_h, [0])
        n = int(max(1, min(blk, 10.0 / max(t1, 1e-3))))
        v, dt = oracle_proj_rows_per_s(o_blk, w_uv_h, w_out_h, list(range(n)))
        cpu = {"value": v, "unit": PROJ_UNIT, "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
               "sample": f"{n} of {T} rows, float64 NumPy, {dt:.1f} s"}

    if rank == 0:
        line = {
            "metric": PROJ_METRIC, "value": value, "unit": PROJ_UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 (fp32 accumulate)", "data": "synthetic",
            "config": {"workload": f"{cfg.name}: {T} rows, H={cfg.n_heads} d_c={cfg.d_c} "
                                   f"d_v={cfg.d_v} d_model={cfg.d_model}; o is a seeded "
                                   f"{blk}-row block repeated down the rows",
                       "l2": "flushed before every step (256 MiB write, untimed)",
                       "parallelism": f"{world} independent ranks (weak scaling)"},
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches * args.steps, "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------- indexer warm-up
WARMUP_METRIC = "indexer warm-up query-rows/s (scores, KL to the teacher, backward to q_I, w, k_I)"
WARMUP_UNIT = "query-rows/s"


def warmup_teacher(cfg, inp, ld):
    """Seeded stand-in for the dense-attention teacher of every row: positive
    weights with some exact zeros, summing to 1 over the row's visible keys."""
    import numpy as np
    klen = inp["row_klen"].astype(int)
    p = np.zeros((len(klen), ld), np.float32)
    for t, n in enumerate(klen):
        r = np.random.default_rng([cfg.seed, 90, t])
        x = r.random(n) ** 3
        x[r.random(n) < 0.1] = 0.0
        x[0] = max(x[0], 1e-3)
        p[t, :n] = x / x.sum()
    return p


def warmup_flops(inp):
    """Algorithmic FLOPs of the warm-up backward, all fp32 fma on the CUDA cores:
    per visible (row, key) pair the 64 x 128 dot products twice (for dq and dw,
    and again for dk; the few whose sign the fp32 sum cannot settle are redone
    in fp64) and the dq and dk contractions (64 x 128 each)."""
    pairs = int(inp["row_klen"].astype("int64").sum())
    h, d = int(inp["h_idx"]), int(inp["d_idx"])
    return {"fp32": 4 * 2 * h * d * pairs, "pairs": pairs}


def run_warmup(args):
    import numpy as np
    import torch
    rank, world, local = dist_info()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    from long_context_sparse_04_b200 import build
    build.build()
    from long_context_sparse_04_b200 import _native as N
    from long_context_sparse_04_b200 import inputs as I
    from long_context_sparse_04_b200.workload import DeviceWorkload, _vp

    cfg = rank_config(I.CONFIGS[args.workload], rank)
    inp = I.generate(cfg, with_q=False, threads=max(4, min(32, len(os.sched_getaffinity(0)))))
    wl = DeviceWorkload(inp, device=dev)
    T, ld = wl.T, wl.ld
    p = torch.from_numpy(warmup_teacher(cfg, inp, ld)).to(dev)
    scores = torch.empty((T, ld), dtype=torch.float32, device=dev)
    grad = torch.empty((T, ld), dtype=torch.float32, device=dev)
    loss = torch.empty(T, dtype=torch.float32, device=dev)
    H_I, d_I = wl.dims.n_idx_heads, wl.dims.d_idx
    dq = torch.empty((T, H_I, d_I), dtype=torch.float32, device=dev)
    dw = torch.empty((T, H_I), dtype=torch.float32, device=dev)
    dk = torch.zeros((int(inp["k_idx"].shape[0]), d_I), dtype=torch.float32, device=dev)
    n_kl = N.dsa_workspace_size(wl.dims, wl.rows, N.DSA_OP_INDEXER_KL)
    ws_kl = torch.zeros(n_kl, dtype=torch.uint8, device=dev)
    n_bw = N.dsa_workspace_size(wl.dims, wl.rows, N.DSA_OP_INDEXER_BACKWARD)
    ws_bw = torch.zeros(n_bw, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]

    def step():
        # one warm-up step over the batch: indexer scores, KL + dL/dI, backward
        wl.indexer(scores)
        ev[1].record(stream)
        N.dsa_indexer_kl(wl.rows, _vp(scores), ld, _vp(p), ld, _vp(grad), ld, _vp(loss), _vp(ws_kl),
                         n_kl, wl.stream)
        N.dsa_indexer_backward(wl.dims, wl.rows, wl.cache, _vp(wl.q_idx), _vp(wl.q_scale), _vp(wl.w),
                               _vp(grad), ld, _vp(dq), _vp(dw), _vp(dk), _vp(ws_bw), n_bw, wl.stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(max(args.warmup, 0)):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    for ws in (ws_kl, ws_bw):
        st = N.dsa_read_device_status(_vp(ws), wl.stream)
        assert st == (0, -1), f"device status {st}"
    assert N.dsa_read_kernel_trace(_vp(ws_bw), wl.stream) & N.DSA_KERNEL_WARMUP

    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    clocks.start()
    t_end = time.perf_counter() + 1.5
    while time.perf_counter() < t_end:
        flush.zero_()
        step()
        torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    ms, ms_bwd = [], []
    for _ in range(args.steps):
        flush.zero_()
        ev[0].record(stream)
        step()
        ev[2].record(stream)
        torch.cuda.synchronize(dev)
        ms.append(ev[0].elapsed_time(ev[2]))
        ms_bwd.append(ev[1].elapsed_time(ev[2]))
    barrier()
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    total_ms = max_over_ranks(sum(ms), world, dev)
    value = throughput(world, T, args.steps, total_ms)

    peaks, peak_kind = measured_peaks()
    fl = warmup_flops(inp)
    t_bwd = statistics.mean(ms_bwd) / 1e3
    clock = peaks.get("sm_max_mhz", 1965.0) * 1e6
    fp32_peak = 148 * 128 * 2 * clock / 1e12
    roof = {"kernel": "indexer_kl_kernel + indexer_bwd_{dq,reduce,dk}_kernel", "bound": "alu",
            "achieved": fl["fp32"] / t_bwd / 1e12, "peak": fp32_peak, "unit": "TFLOP/s",
            "frac": fl["fp32"] / t_bwd / 1e12 / fp32_peak,
            "peak_source": "derived (148 SMs x 128 fp32 FMA lanes x 2 x max SM clock): fp32 fma "
                           "dot products and contractions",
            "traffic": None, "algorithmic_per_launch": fl["fp32"]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, dt, n = oracle_warmup_rows_per_s(inp, p.cpu().numpy(), 10.0)
        cpu = {"value": v, "unit": WARMUP_UNIT, "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
               "sample": f"{n} of {T} rows (scores, KL, backward), float64 NumPy, {dt:.1f} s"}

    if rank == 0:
        line = {
            "metric": WARMUP_METRIC, "value": value, "unit": WARMUP_UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8e4m3 scores; fp32 dots with an exact (fp64) sign check, fp32 gradients", "data": "synthetic",
            "config": {"workload": workload_desc(cfg) + "; teacher: seeded positive weights per row",
                       "rows_per_gpu": T, "pairs": fl["pairs"],
                       "l2": "flushed before every step (256 MiB write, untimed)",
                       "parallelism": f"{world} independent ranks (weak scaling)"},
            "stages": {"backward_ms": 1e3 * t_bwd, "scores_ms": statistics.mean(ms) - 1e3 * t_bwd},
            "roofline": roof, "cpu_baseline": cpu, "e2e": None,
            "gpu_launches": 5 * args.steps, "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def oracle_warmup_rows_per_s(inp, p, budget_s):
    """The oracle's warm-up step (scores, KL, backward) on rows of the batch,
    for about budget_s seconds."""
    import numpy as np
    from oracle import dsa_ref as R
    T = len(inp["row_klen"])
    t0 = time.perf_counter()
    n = 0
    for t in np.linspace(0, T - 1, T).astype(int):
        klen = int(inp["row_klen"][t])
        rows = R.physical_rows(int(inp["row_seq"][t]), np.arange(klen), inp["cache"])
        kd, qd = R.dequant_keys(inp, rows), R.dequant_queries(inp, t)
        w = np.asarray(inp["w"][t], dtype=np.float32).astype(np.float64)
        sc = R.indexer_row(qd, w, kd)
        _, g = R.indexer_kl_row(p[t, :klen].astype(np.float64), sc)
        R.indexer_backward_row(qd, w, kd, g)
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return n / dt, dt, n


def run_warmup_reference(args, cfg):
    from long_context_sparse_04_b200 import inputs as I
    inp = I.generate(cfg, with_q=False)
    ld = ((int(inp["row_klen"].max()) + 127) // 128) * 128
    p = warmup_teacher(cfg, inp, ld)
    for _ in range(args.warmup):
        oracle_warmup_rows_per_s(inp, p, 0.0)
    t0 = time.perf_counter()
    n = 0
    for _ in range(args.steps):
        _, _, k = oracle_warmup_rows_per_s(inp, p, 0.0)
        n += k
    dt = time.perf_counter() - t0
    value = n / dt
    line = {
        "impl": "reference", "metric": WARMUP_METRIC, "value": value, "unit": WARMUP_UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(cfg) + "; teacher: seeded positive weights per row",
                   "rows_per_gpu": len(inp["row_klen"]), "pairs": warmup_flops(inp)["pairs"],
                   "l2": "flushed before every step (256 MiB write, untimed)",
                   "parallelism": f"{args.gpus} independent ranks (weak scaling)"},
        "cpu_baseline": {"value": value, "unit": WARMUP_UNIT, "cores": len(os.sched_getaffinity(0)),
                         "kind": "oracle", "sample": "1 row per step (scores, KL, backward), float64"},
        "e2e": {"value": value, "unit": WARMUP_UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_out_proj_reference(args, cfg):
    from long_context_sparse_04_b200 import inputs as I
    T = cfg.n_rows
    w_uv, w_out = I.out_proj_weights(cfg)
    o = I.latent_out_rows(cfg, range(min(T, 4)))
    for _ in range(args.warmup):
        oracle_proj_rows_per_s(o, w_uv, w_out, [0])
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_proj_rows_per_s(o, w_uv, w_out, list(range(len(o))))
    dt = time.perf_counter() - t0
    value = args.steps * len(o) / dt
    line = {
        "impl": "reference", "metric": PROJ_METRIC, "value": value, "unit": PROJ_UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{cfg.name}: {T} rows, H={cfg.n_heads} d_c={cfg.d_c} "
                               f"d_v={cfg.d_v} d_model={cfg.d_model}"},
        "cpu_baseline": {"value": value, "unit": PROJ_UNIT, "cores": len(os.sched_getaffinity(0)),
                         "kind": "oracle", "sample": f"{len(o)} of {T} rows per step (float64 NumPy)"},
        "e2e": {"value": value, "unit": PROJ_UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.workload is None:
        args.workload = {"cache_append": "prefill_64k", "output_projection": "prefill_64k",
                         "warmup": "decode_16k"}.get(args.op, "decode_128k_paged")
    if args.op == "warmup":
        if args.impl == "reference":
            rank, _, _ = dist_info()
            if rank != 0:
                return 0
            from long_context_sparse_04_b200 import inputs as I
            return run_warmup_reference(args, I.CONFIGS[args.workload])
        return run_warmup(args)
    if args.op == "output_projection":
        if args.impl == "reference":
            rank, _, _ = dist_info()
            if rank != 0:
                return 0
            from long_context_sparse_04_b200 import inputs as I
            return run_out_proj_reference(args, I.CONFIGS[args.workload])
        return run_out_proj(args)
    if args.op == "cache_append":
        if args.impl == "reference":
            rank, _, _ = dist_info()
            if rank != 0:
                return 0
            from long_context_sparse_04_b200 import inputs as I
            return run_append_reference(args, I.CONFIGS[args.workload])
        return run_append(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
