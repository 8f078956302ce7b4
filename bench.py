#!/usr/bin/env python
"""Benchmark of the CSA2 decode step on B200.

One step = one csa2_decode_stack call: the append of this step's keys and Main
KV rows (FP4 quantiser), the Full layer's indexer scan over the whole visible
context with its block top-P pool and own top-K, the Reindex layers' pool
rescoring and top-K, and attention for every layer (sparse FP4 Main KV, plus
the FP8 sliding window where the workload has one).

Default workload: the million-token configuration (4 sequences x 1,048,576
cached positions, 1 query token each, 1 Full + 3 Reindex + 16 Reuse layers).
Metric: decode query tokens per second through the layer stack; the indexer
scan's HBM GB/s is reported as the roofline of the dominant kernel.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: one process per GPU (torchrun); sequences are independent, so each
rank decodes its own batch of the workload (weak scaling, no collective on the
data path); the time is the max over ranks.  The reference arm times the CPU
oracle (there is no reference implementation to run).
"""
from __future__ import annotations

import argparse
import ctypes
import json
import math
import os
import signal
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA2 decode query-tokens/s per layer stack at 1M ctx; indexer-scan HBM GB/s"
UNIT = "qtok/s"


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=4, help="workload number (1..6; 6 = chunked prefill)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the oracle sample")
    return ap.parse_args()


def source_digest(text: str) -> str:
    """First 16 hex digits of the SHA-256 of a C/CUDA source with its comments
    removed and its whitespace collapsed: the code the compiler sees, so that an
    edit of a comment leaves it unchanged."""
    import hashlib
    import re
    code = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    code = re.sub(r"//[^\n]*", " ", code)
    code = " ".join(code.split())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def _profiled_traffic(kernel_src: str, summary: str):
    """DRAM bytes per launch (read + write) from a committed ncu summary, valid
    only while the kernel's code is the one the counters were taken on (the
    summary records its source_digest)."""
    import re
    try:
        with open(os.path.join(ROOT, kernel_src), encoding="utf-8") as f:
            h = source_digest(f.read())
        with open(os.path.join(ROOT, summary)) as f:
            txt = f.read()
        src = re.search(r"source_digest:\s*([0-9a-f]{16})", txt)
        tr = re.search(r"traffic_bytes_per_launch:\s*([0-9]+)", txt)
        if src and tr and src.group(1) == h:
            return int(tr.group(1))
    except OSError:
        pass
    return None


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def algorithmic_flops(w) -> dict:
    """Multiply-adds x 2 the method needs per decode step: the scan's and the
    rescoring's q.k over every visible (resp. pooled) position and indexer
    head, and attention's Q K^T and P V over the selected and window rows."""
    import numpy as np

    c = w.cfg
    n_sel = sum(1 for m in w.modes if m in "FR")
    vis = w.tok_pos.astype(np.int64) + 1
    pool = np.minimum(np.minimum((vis + 7) // 8, c.P) * 8, vis)
    rows = np.minimum(vis, c.K) + (np.minimum(vis, c.window) if c.swa else 0)
    return {"scan": int(vis.sum()) * c.H_I * c.d_I * 2,
            "rescore": int(pool.sum()) * n_sel * c.H_I * c.d_I * 2,
            "attend": int(rows.sum()) * len(w.modes) * c.Hq * c.D * 4}


def cache_bytes(w) -> int:
    """bytes of the FP4 caches the step reads from (indexer K and Main KV)"""
    c = w.cfg
    return int(w.n_rows) * (c.d_I // 2 + c.d_I // 32 + c.D // 2 + c.D // 32)


L2_BYTES = 126 * 2**20  # B200 L2


def l2_policy(w, l2_bytes: int = L2_BYTES) -> bool:
    """True when the L2 must be flushed between timed steps: the step's
    inputs are not at least twice the L2 (otherwise the inputs themselves
    evict it, and a flush by writing would add its dirty write-backs to the
    first kernel of the step)"""
    return cache_bytes(w) < 2 * l2_bytes


def _workload_desc(cfg, w, flush: bool):
    return {
        "workload": f"{cfg.name}: B={cfg.B}, L={'x'.join(str(int(x)) for x in sorted(set(w.lens.tolist())))[:60]}"
                    f", T={w.T}, H_I={cfg.H_I}, d_I={cfg.d_I}, P={cfg.P}, K={cfg.K}, Hq={cfg.Hq}, D={cfg.D}, "
                    f"layers={''.join(w.modes)}{', paged' if cfg.paged else ''}{', swa' if cfg.swa else ''}",
        "sum_context": int(w.lens.sum()),
        "query_tokens_per_step": int(w.T),
        "layers": len(w.modes),
        "q_dtype": cfg.q_dtype,
        "out_dtype": cfg.out_dtype,
        "l2": (f"flushed (256 MiB write) before every timed step; caches {cache_bytes(w) / 1e9:.2f} GB"
               if flush else f"inputs larger than L2: caches {cache_bytes(w) / 1e9:.2f} GB read every step, "
                             f"no flush between steps"),
    }


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.3)
        self.proc.send_signal(signal.SIGTERM)
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) < 9:
                    continue
                try:
                    sm.append(float(f[1]))
                    mx.append(float(f[2]))
                except ValueError:
                    continue
                for n, v in zip(names, f[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
            os.remove(self.path)
        except Exception:
            pass
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- oracle sample
class Ranks:
    """One process per GPU (torchrun): rank/world from the environment, and the
    few host-side reductions the benchmark needs (NCCL on GPUs, gloo on CPU).
    Every rank takes the same collective steps in the same order."""

    def __init__(self, device: str = "cuda", timeout_s: int = 120):
        import datetime

        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.device = device
        self.dist = None
        if self.world > 1:
            import torch.distributed as dist

            dist.init_process_group("nccl" if device == "cuda" else "gloo",
                                    timeout=datetime.timedelta(seconds=timeout_s))
            self.dist = dist

    def _reduce(self, x: float, op) -> float:
        if self.dist is None:
            return float(x)
        import torch

        t = torch.tensor([float(x)], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=op)
        return float(t.item())

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def allmax(self, x: float) -> float:
        return self._reduce(x, None if self.dist is None else self.dist.ReduceOp.MAX)

    def allsum(self, x: float) -> float:
        return self._reduce(x, None if self.dist is None else self.dist.ReduceOp.SUM)

    def close(self):
        if self.dist is not None:
            self.dist.barrier()
            self.dist.destroy_process_group()
            self.dist = None


def whole_job_rate(tokens_all_ranks: float, steps: int, max_ms: float) -> float:
    """query tokens per second of the whole job: every rank's tokens over the
    slowest rank's time"""
    return tokens_all_ranks * steps / (max_ms / 1000.0)


def oracle_sample(cfg_id: int, seconds: float, seed_offset: int = 0):
    """Times the CPU oracle on a bounded sample of the workload: whole query
    tokens (all layers of the stack), as many as fit in `seconds` (>= 1).
    Input preparation (regenerating and quantising the cached keys) is not
    timed, as the GPU timing excludes the cache fill."""
    import numpy as np

    import oracle
    from synth.workloads import BLOCK, CONFIGS, make_workload
    cfg = CONFIGS[cfg_id]
    w = make_workload(cfg.with_(seed=cfg.seed + seed_offset))
    c = cfg
    timed, toks = 0.0, 0
    tok = 0
    keys = {}  # (sequence, visible length) -> quantised keys, reused when the sample cycles
    while toks == 0 or timed < seconds:
        b, p = int(w.tok_seq[tok]), int(w.tok_pos[tok])
        if (b, p) not in keys:
            kx = w.kidx.rows_f32(b, 0, p + 1)
            keys[(b, p)] = oracle.quantize_fp4(kx)[:2]
            del kx
        kc, ks = keys[(b, p)]
        qs = {l: w.iq_f32(l, tok) for l, m in enumerate(w.modes) if m in "FR"}
        ws = {l: w.iw_f32(l, tok).astype(np.float64) for l in qs}
        qm = {l: w.qmain_f64(l, tok) for l in range(len(w.modes))}
        sw = {}
        if c.swa:
            for l in range(len(w.modes)):
                codes, sc = w.swa_rows_e4m3(l, tok)
                sw[l] = (codes, sc)
        t0 = time.perf_counter()
        idx = None
        pool = None
        for l, m in enumerate(w.modes):
            if m in "FR":
                qc, qsc, _ = oracle.quantize_fp4(qs[l])
                q = oracle.dequant_fp4(qc, qsc)
                if m == "F":
                    r = oracle.full_select(q, ws[l], kc, ks, p, c.P, c.K, BLOCK)
                    pool, idx = r.pool, r.idx
                else:
                    idx, _, _ = oracle.reindex_select(q, ws[l], kc, ks, p, pool, c.K, BLOCK)
                rows_x = w.kv.select_rows_f32(b, idx)
                vc, vs, _ = oracle.quantize_fp4(rows_x)
                kv_rows = oracle.dequant_fp4(vc, vs)
            swr = None
            if c.swa:
                codes, sc = sw[l]
                swr = oracle.e4m3_decode_array(codes) * sc.astype(np.float64)[:, None]
            oracle.attend_rows(qm[l], kv_rows, swr, 1.0 / math.sqrt(c.D))
        timed += time.perf_counter() - t0
        toks += 1
        tok = (tok + 1) % w.T
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return toks / timed, toks, timed, cores


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from synth.workloads import CONFIGS, make_workload
    cfg = CONFIGS[args.config]
    w = make_workload(cfg)
    # the whole --steps run stays within a few minutes: at most ~150 s of samples
    per_step = max(1.0, min(args.cpu_seconds, 6.0, 150.0 / max(1, args.steps)))
    for _ in range(args.warmup):
        oracle_sample(args.config, 0.0)
    vals, times = [], []
    for _ in range(args.steps):
        v, toks, t, cores = oracle_sample(args.config, per_step)
        vals.append(v)
        times.append(t / toks)
    value = sum(1.0 / t for t in times) / len(times)
    sample = f"whole query tokens of {cfg.name} through all {len(w.modes)} layers, >= 1 per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * sum(times) / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": _workload_desc(cfg, w, l2_policy(w)),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU arm
def run_ours(args):
    import numpy as np
    import torch

    import csa2_fp4_sparse_b200 as C
    from synth.gpu import DeviceWorkload
    from synth.workloads import CONFIGS, algorithmic_bytes, make_workload

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    R = Ranks("cuda")
    world, rank = R.world, R.rank
    barrier, allmax = R.barrier, R.allmax

    cfg = CONFIGS[args.config]
    cfg = cfg.with_(seed=cfg.seed + 1000 * rank)
    w = make_workload(cfg)
    dw = DeviceWorkload(w)
    dw.fill_caches(include_new=False)
    desc = dw.stack_desc(append=True, copies=False)
    ws = dw.stack_workspace(desc)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    need_flush = l2_policy(w)

    def flush():
        if need_flush:
            flush_buf.zero_()

    def step():
        rc = C.csa2_decode_stack(ctypes.byref(desc), ws.data_ptr(), ws.numel(), sp)
        if rc != 0:
            raise RuntimeError(f"csa2_decode_stack: {rc} {C.csa2_last_error()}")

    for _ in range(args.warmup):
        flush()
        step()
    st = C.csa2_get_status(sp)
    assert st == 0, f"device status {st}"
    # measured tensor peaks of the two MMA kinds the step uses (outside the
    # timed region): block-scaled FP4 (indexer) and fp16 (attention)
    probe = {"fp4_tflops": C.csa2_tensor_peak(1, 8192, sp), "f16_tflops": C.csa2_tensor_peak(0, 8192, sp)}

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.4)
    barrier()
    torch.cuda.synchronize()
    n0 = C.csa2_launch_count()
    for k in range(args.steps):
        flush()
        ev[k][0].record(stream)
        step()
        ev[k][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    n_launch = C.csa2_launch_count() - n0
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = allmax(sum(step_ms))
    tokens_all = R.allsum(w.T)  # ranks decode different seeded batches
    st = C.csa2_get_status(sp)
    assert st == 0, f"device status {st}"
    value = whole_job_rate(tokens_all, args.steps, total_ms)
    q = np.percentile(np.asarray(step_ms), [10, 50, 90])

    # the same steps with an L2 flush (256 MiB write) before each: secondary,
    # for comparison only (the flush's dirty lines are written back during the
    # step's first kernel)
    ev_w = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for k in range(args.steps):
        flush_buf.zero_()
        ev_w[k][0].record(stream)
        step()
        ev_w[k][1].record(stream)
    torch.cuda.synchronize()
    flushed_ms = allmax(sum(a.elapsed_time(b) for a, b in ev_w)) / args.steps

    # per-kernel times (second pass, profiler on; same steps)
    C.csa2_profiler_read()
    C.csa2_profiler_enable(1)
    for _ in range(args.steps):
        flush()
        step()
    torch.cuda.synchronize()
    kstats = C.csa2_profiler_read()
    C.csa2_profiler_enable(0)
    ab = algorithmic_bytes(w)
    peak_hbm, peak_bf16, peak_kind = _peaks()
    scan_name = next((n for n in kstats if n.startswith("scan")), None)
    roof = None
    kernels = {}
    tot_prof = sum(v[1] for v in kstats.values())
    fl = algorithmic_flops(w)
    # per kernel: algorithmic bytes (HBM) and tensor FLOPs per step over its time
    # per step; FP4 MMAs against the FP4 peak measured by the probe above
    # (tensor_frac; tensor_frac_bf16x4: against the measured bf16 peak x 4, the
    # nominal 9 / 2.25 PFLOP/s ratio), fp16 MMAs against the measured bf16 peak
    fp4_peak = probe["fp4_tflops"]
    per_kernel = {"scan": (ab["scan"], fl["scan"], fp4_peak), "rescore": (ab["rescore"], fl["rescore"], fp4_peak),
                  "attend": (ab["attend"] + ab["swa"], fl["attend"], peak_bf16)}
    for n, (cnt, ms) in sorted(kstats.items(), key=lambda kv: -kv[1][1]):
        kernels[n] = {"launches_per_step": cnt / args.steps, "us_per_step": 1000.0 * ms / args.steps,
                      "share": ms / tot_prof if tot_prof else None}
        key = next((k for k in per_kernel if n.startswith(k)), None)
        if key and ms > 0:
            b, f, tpeak = per_kernel[key]
            sec = ms / args.steps / 1000.0
            kernels[n].update({"hbm_gbs": b / sec / 1e9, "hbm_frac": b / sec / 1e9 / peak_hbm,
                               "tensor_tflops": f / sec / 1e12, "tensor_frac": f / sec / 1e12 / tpeak})
            if key != "attend":
                kernels[n]["tensor_frac_bf16x4"] = f / sec / 1e12 / (4.0 * peak_bf16)
    if scan_name:
        cnt, ms = kstats[scan_name]
        avg_s = ms / cnt / 1000.0
        traffic = None
        if args.config == 4:  # the profiled workload
            traffic = _profiled_traffic("csa2_fp4_sparse_b200/csrc/scan_tc.cu", "profiles/scan_tc_ctx1m.md")
        # the scan's bound: HBM while its FP4 work per byte read stays below the
        # ridge (FP4 peak / HBM peak), the FP4 tensor pipe above it (many query
        # tokens per sequence, as in chunked prefill)
        if fl["scan"] / max(ab["scan"], 1) > fp4_peak * 1e12 / (peak_hbm * 1e9):
            achieved = fl["scan"] / avg_s / 1e12
            roof = {"kernel": scan_name, "bound": "tensor", "achieved": achieved, "peak": fp4_peak,
                    "unit": "TFLOP/s", "frac": achieved / fp4_peak, "peak_source": "FP4 MMA probe",
                    "traffic": traffic, "algorithmic_flops_per_launch": fl["scan"],
                    "algorithmic_bytes_per_launch": ab["scan"], "avg_launch_us": avg_s * 1e6}
        else:
            achieved = ab["scan"] / avg_s / 1e9
            roof = {"kernel": scan_name, "bound": "hbm", "achieved": achieved, "peak": peak_hbm, "unit": "GB/s",
                    "frac": achieved / peak_hbm, "peak_source": peak_kind, "traffic": traffic,
                    "algorithmic_bytes_per_launch": ab["scan"], "avg_launch_us": avg_s * 1e6}

    # end to end through the public call with host buffers (pinned)
    e2e = None
    try:
        e2e = _e2e(args, C, dw, desc, ws, stream, flush, w)
        err = ""
    except Exception as ex:  # reported, not hidden
        e2e, err = None, str(ex)[:200]
    # every rank reduces, failed or not (same collective steps on all ranks)
    e2e_ms = allmax(e2e["ms_per_step"] * args.steps if e2e else float("inf"))
    if e2e and math.isfinite(e2e_ms):
        e2e["value"] = whole_job_rate(tokens_all, args.steps, e2e_ms)
        e2e["ms_per_step"] = e2e_ms / args.steps
    else:
        e2e = {"value": None, "unit": UNIT, "error": err or "a rank failed"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, toks, t, cores = oracle_sample(args.config, args.cpu_seconds)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{toks} whole query token(s) of {cfg.name} through all {len(w.modes)} layers "
                         f"({t:.1f} s of CPU time; cache fill excluded)"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp4", "data": "synthetic",
            "config": _workload_desc(cfg, w, need_flush), "parallelism": f"replicas x{world}",
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": int(n_launch),
            "clocks": clk, "kernels": kernels,
            "tensor_peaks": dict(probe, bf16_measured_tflops=peak_bf16, source=peak_kind),
            "scan_gbs": (ab["scan"] / (roof["avg_launch_us"] * 1e-6) / 1e9) if roof else None,
            "algorithmic_bytes_per_step": ab,
            "step_ms_min_max": [min(step_ms), max(step_ms)],
            "step_ms_p10_p50_p90": [float(x) for x in q],
            "flushed_ms_per_step": flushed_ms,
        }
        print(json.dumps(line), flush=True)
    R.close()


def _e2e(args, C, dw, desc, ws, stream, flush, w):
    """Same step through the public call, with every per-step input copied in
    from pinned host memory and every output read back, inside the timing.
    The indexer's inputs (selector queries and head weights, the new tokens)
    go in on the step's stream; the Main queries, read only by attention, go in
    on a second stream while the indexer kernels run, and the stack's attention
    waits for them (attend_wait_event).  All layers' outputs come back in one
    transfer."""
    import torch
    h_idx = dw.inputs_index.cpu().pin_memory()
    h_q = dw.inputs_main_q.cpu().pin_memory()
    h_out = torch.empty(dw.out_all.shape, dtype=dw.out_all.dtype).pin_memory()
    bi = h_idx.numel() + h_q.numel()
    bo = h_out.numel() * h_out.element_size()
    s2 = torch.cuda.Stream()
    started, q_ready = torch.cuda.Event(), torch.cuda.Event()
    q_ready.record(s2)  # creates the event
    d2 = type(desc)()
    ctypes.memmove(ctypes.byref(d2), ctypes.byref(desc), ctypes.sizeof(desc))
    d2.attend_wait_event = q_ready.cuda_event
    sp = stream.cuda_stream
    n_w = max(3, args.warmup)  # untimed: the first transfers of fresh pinned buffers cost extra
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_w + args.steps)]
    torch.cuda.synchronize()
    for k in range(n_w + args.steps):
        flush()
        ev[k][0].record(stream)
        started.record(stream)  # the previous step (and its reads of the queries) is done
        s2.wait_event(started)
        with torch.cuda.stream(s2):
            dw.inputs_main_q.copy_(h_q, non_blocking=True)
            q_ready.record(s2)
        dw.inputs_index.copy_(h_idx, non_blocking=True)
        rc = C.csa2_decode_stack(ctypes.byref(d2), ws.data_ptr(), ws.numel(), sp)
        if rc != 0:
            raise RuntimeError(C.csa2_last_error())
        h_out.copy_(dw.out_all, non_blocking=True)
        ev[k][1].record(stream)
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in ev[n_w:])
    return {"value": w.T * args.steps / (ms / 1000.0), "unit": UNIT, "h2d_bytes_per_step": bi,
            "d2h_bytes_per_step": bo, "ms_per_step": ms / args.steps}


def main():
    args = _args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
