#!/usr/bin/env python
"""Benchmark of the AdaCluster clustered sparse attention call (ac_forward).

One step = one ac_forward call over the whole workload (Q clustering, K
clustering, critical-cluster selection, cluster sort + gather, block-sparse
attention) on the Wan-2.1-shaped workload: 40 heads x 75,600 tokens x d=128,
bf16, 250 query / 500 key clusters, 10 k-means iterations, top-p 0.9.

Prints one JSON line (rank 0).  Besides the headline workload the line carries
`per_config` (every workload of the suite: ms per call, stages, roofline and
the SDPA comparator) and `top_p_sweep` (the headline workload at top-p 0.8,
0.9 and 0.95).  --impl reference times the CPU oracle on bounded samples of the
same workload instead.  Under torchrun every rank runs its own independent
call (heads and calls share nothing), so scaling is weak and value = calls over
all ranks / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from clustered_sparse_attention_head_b200 import workloads as W  # noqa: E402

DEFAULT_WORKLOAD = "wan21-n75600-h40-d128"
METRIC = "clustered sparse-attn calls/s & achieved TFLOPS at 75.6K tokens vs dense attn"
# dram__bytes_read.sum + dram__bytes_write.sum of one attention launch (ncu) on
# the default workload cut to 8 heads; None whenever the kernel changes, until
# it is captured again
ATTN_TRAFFIC_8H = 0.655e9
L2_BYTES = 126 * 2 ** 20
# the CPU oracle's bounded sample: one head clustered and selected in full,
# attention for SAMPLE_ROWS query rows; heads 0..SAMPLE_HEADS-1 in turn
SAMPLE_ROWS = 128
SAMPLE_HEADS = 4
TOP_P_SWEEP = (0.8, 0.9, 0.95)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=W.ORDER)
    ap.add_argument("--top-p", type=float, default=None)
    ap.add_argument("--heads", type=int, default=None, help="fewer heads (profiling captures only)")
    ap.add_argument("--kq", type=int, default=None, help="another query cluster count (selection timings)")
    ap.add_argument("--kk", type=int, default=None, help="another key cluster count (selection timings)")
    ap.add_argument("--select-mode", default=None, choices=sorted(SELECT_MODES),
                    help="time the main call with one of the selection options instead of the top-p cut")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="skip the per-workload and top-p sweep keys")
    ap.add_argument("--per-config-calls", type=int, default=3, help="timed calls per workload in per_config")
    ap.add_argument("--denoise-steps", type=int, default=0,
                    help="also run the multi-step driver (ac_forward_step) over this many drifting steps")
    ap.add_argument("--drift", type=float, default=0.02, help="per-element drift per denoising step")
    ap.add_argument("--text-keys", action="store_true",
                    help="attend every query to the workload's text keys (a dense strip), not clustered")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time (all ranks call this in the same order)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def calls_per_second(ms_max: float, world: int) -> float:
    """Whole-job throughput: every rank completes one call per step, and the
    job's step takes as long as its slowest rank."""
    return world * 1000.0 / ms_max


def gen_inputs(w, heads=None):
    """Seeded inputs, all heads (threads: numpy releases the GIL in bulk draws)."""
    from concurrent.futures import ThreadPoolExecutor
    hs = list(range(w.heads)) if heads is None else heads
    with ThreadPoolExecutor(max_workers=min(16, len(hs))) as ex:
        res = list(ex.map(lambda h: W.head_inputs(w, h), hs))
    return res


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            out, _ = self.p.communicate(timeout=5)
        except Exception:
            self.p.kill()
            out = ""
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ cpu baseline
def oracle_sample(w, hi, rows_sample: int = SAMPLE_ROWS):
    """Time the oracle on one head: full Q and K clustering and selection, and
    attention for `rows_sample` query rows.  Returns (seconds one whole call
    would take at this rate: x heads, x n / rows_sample rows; wall seconds)."""
    import oracle
    oracle.build()
    spec = oracle.HeadSpec(kq=w.kq, kk=w.kk, iters=w.iters, top_p=w.top_p, adaptive_q=w.adaptive_q,
                           adaptive_k=w.adaptive_k, tau_rule=w.tau_rule, tau_value=w.tau_value, nmax_q=w.nmax_q,
                           nmax_k=w.nmax_k)
    t0 = time.perf_counter()
    rq, qmn = oracle.cluster_q(hi.q, spec)
    rk = oracle.cluster_k(hi.k, spec)
    dense = int(rq.dense or rk.dense)
    if dense:
        sel, cnt = np.zeros((rq.nclusters, max(rk.nclusters, 1)), np.int32), np.zeros(rq.nclusters, np.int32)
    else:
        sel, cnt = oracle.select(rq.cent, qmn, rq.count, rk.cent, rk.count, spec.top_p)
    t1 = time.perf_counter()
    rows = np.linspace(0, w.n - 1, rows_sample).astype(np.int32)
    oracle.attention_rows(hi.q, hi.k, hi.v, rq.assign, rk.assign, rk.nclusters, sel, cnt, dense, rows)
    t2 = time.perf_counter()
    per_call = w.heads * ((t1 - t0) + (t2 - t1) * w.n / rows_sample)
    return per_call, t2 - t0


def omp_threads():
    v = os.environ.get("OMP_NUM_THREADS")
    return int(v) if v and v.isdigit() else (os.cpu_count() or 1)


def sample_text(w, heads_used, walls):
    return (f"per sample: one head (heads 0-{heads_used - 1} of {w.heads} in turn) with Q and K clustering and "
            f"selection in full and attention for {SAMPLE_ROWS} of {w.n} query rows; the mean extrapolated "
            f"x{w.heads} heads and x{w.n}/{SAMPLE_ROWS} rows to one call; {len(walls)} samples, "
            f"{sum(walls):.1f} s wall time measured")


def cpu_baseline_obj(w, his):
    """The oracle on bounded samples of the workload (the same samples as the
    reference arm's steps), extrapolated to calls/s."""
    per, walls = zip(*(oracle_sample(w, hi) for hi in his))
    per_call = statistics.mean(per)
    return {"value": 1.0 / per_call, "unit": "calls/s", "cores": omp_threads(), "kind": "oracle",
            "extrapolated": True, "samples_timed": len(walls), "wall_s": sum(walls),
            "scale_per_sample": w.heads * w.n / SAMPLE_ROWS,
            "sample": sample_text(w, len(his), walls)}


def config_of(w, world, text_keys=0):
    """The `config` object of the JSON line, the same for both arms."""
    tb = tensor_bytes(w)
    l2 = (f"inputs larger than L2 ({tb / 1e6:.0f} MB per tensor), no flush" if tb > L2_BYTES else
          f"L2 flushed between timed calls (a {2 * L2_BYTES >> 20} MiB write; {tb / 1e6:.1f} MB per tensor)")
    return {"workload": w.name, "heads": w.heads, "n": w.n, "d": w.d, "kq": w.kq, "kk": w.kk, "iters": w.iters,
            "top_p": w.top_p, "text_keys": text_keys, "parallelism": f"dp{world} (independent calls)", "l2": l2}


def tensor_bytes(w):
    return w.heads * w.n * w.d * (2 if w.dtype == "bf16" else 4)


# -------------------------------------------------------------- reference
def run_reference(a, w):
    """The CPU oracle as the reference arm.  A step is one bounded sample (one
    head, SAMPLE_ROWS attention rows), so steps x ms_per_step is the measured
    wall time; value is the samples' mean extrapolated to whole calls."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    his = [W.head_inputs(w, h) for h in range(min(SAMPLE_HEADS, w.heads))]
    per, walls = [], []
    for i in range(a.warmup + a.steps):
        per_call, wall = oracle_sample(w, his[i % len(his)])
        if i >= a.warmup:
            per.append(per_call)
            walls.append(wall)
    v = 1.0 / statistics.mean(per)
    ms_step = 1e3 * statistics.mean(walls)
    line = {"metric": METRIC, "value": v, "unit": "calls/s", "n_gpus": 0, "steps": a.steps, "warmup": a.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "impl": "reference", "config": config_of(w, 1),
            "extrapolated": True,
            "step": f"one bounded sample ({SAMPLE_ROWS} attention rows of one head); value extrapolates the samples "
                    f"to whole calls (x{w.heads * w.n / SAMPLE_ROWS:.0f} per sample)",
            "cpu_baseline": {"value": v, "unit": "calls/s", "cores": omp_threads(), "kind": "oracle",
                             "extrapolated": True, "samples_timed": len(walls), "wall_s": sum(walls),
                             "scale_per_sample": w.heads * w.n / SAMPLE_ROWS,
                             "sample": sample_text(w, len(his), walls)},
            "e2e": {"value": v, "unit": "calls/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------- ours
def main():
    a = parse()
    w = W.WORKLOADS[a.workload]
    from dataclasses import replace
    if a.top_p is not None:
        w = replace(w, top_p=a.top_p)
    if a.heads is not None:
        w = replace(w, heads=a.heads)
    if a.kq is not None:
        w = replace(w, kq=a.kq)
    if a.kk is not None:
        w = replace(w, kk=a.kk)
    if a.impl == "reference":
        return run_reference(a, w)

    rank, world, local = dist_env()
    # the oracle sample needs no GPU; run it before CUDA starts
    hs = gen_inputs(w)
    cpu_base = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu_base = cpu_baseline_obj(w, hs[:min(SAMPLE_HEADS, len(hs))])

    import torch
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    from clustered_sparse_attention_head_b200 import _abi
    from clustered_sparse_attention_head_b200.api import AdaCluster, Config

    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    q_h = torch.from_numpy(np.stack([h.q for h in hs])).to(tdt)
    k_h = torch.from_numpy(np.stack([h.k for h in hs])).to(tdt)
    v_h = torch.from_numpy(np.stack([h.v for h in hs])).to(tdt)
    del hs
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    # two contexts: `ac_t` with the default flags is the one timed (the library
    # replays its cached CUDA graph of the call when a call repeats the buffers);
    # `ac` records per-stage events, which keeps it launch by launch, and gives
    # the stage breakdown, the statistics and a launch-by-launch timing
    def main_cfg():
        cfg = Config.from_workload(w)
        if a.text_keys:
            cfg.text_keys = w.text
        for key, val in SELECT_MODES.get(a.select_mode, {}).items():
            setattr(cfg, key, val)
        return cfg
    ac_t = AdaCluster(main_cfg(), device=dev)
    cfg = main_cfg()
    cfg.flags = _abi.AC_FLAG_PROFILE
    ac = AdaCluster(cfg, device=dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize(dev)

    # warm-up (both contexts), then one call with statistics (pairs, dense heads)
    for _ in range(max(a.warmup, 3) - 1):
        ac_t.ac_forward(q, k, v, out=out)
        ac.ac_forward(q, k, v, out=out)
    _, st = ac.ac_forward(q, k, v, out=out, stats=True)
    for c_ in (ac, ac_t):
        status = c_.get_status()
        if status != 0:
            raise RuntimeError(f"device status {status}: {_abi.status_string(status)}")
    ac.profile_read()
    ac_t.profile_read()

    # timed region: inputs larger than L2 need no flush; smaller ones get an L2
    # flush before every call, outside the events that time the call
    sampler = ClockSampler(local)
    flush = None if tensor_bytes(w) > L2_BYTES else torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    barrier()
    sampler.start()
    ms = time_calls(lambda: ac_t.ac_forward(q, k, v, out=out), a.steps, stream, flush)
    barrier()
    clocks = sampler.stop()
    prof_t = ac_t.profile_read()
    status = ac_t.get_status()
    if status != 0:
        raise RuntimeError(f"device status {status}: {_abi.status_string(status)}")
    # the same calls launch by launch, with per-stage events
    ms_lbl = time_calls(lambda: ac.ac_forward(q, k, v, out=out), a.steps, stream, flush)
    t_lbl = max_over_ranks(ms_lbl, world, dev)
    prof = ac.profile_read()
    status = ac.get_status()
    if status != 0:
        raise RuntimeError(f"device status {status}: {_abi.status_string(status)}")
    t_max = max_over_ranks(ms, world, dev)
    calls_per_s = calls_per_second(t_max, world)
    flops = 4.0 * w.d * st["pairs"]
    tflops_call = flops / (ms * 1e-3) / 1e12
    attn_ms = prof["ms_attn_kernel"]
    tflops_attn = flops / (attn_ms * 1e-3) / 1e12

    # end to end through the same call with host buffers (pinned), copies timed.
    # Pipelined as a serving loop would run it: step s+1's inputs are copied in
    # (own stream, second device buffer set) while step s computes, and step s's
    # output is copied out (own stream) while step s+1 computes.  Every step's
    # copies lie inside the timed region.
    e2e = None
    if not a.no_e2e:
        qp, kp, vp = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
        op = torch.empty_like(qp).pin_memory()
        qs, ks, vs, outs = [q, torch.empty_like(q)], [k, torch.empty_like(k)], [v, torch.empty_like(v)], \
            [out, torch.empty_like(out)]
        h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()
        in_ready, in_free, out_ready, out_free = [ev(), ev()], [ev(), ev()], [ev(), ev()], [ev(), ev()]

        def run_steps(n):
            for i in range(n):
                b = i % 2
                with torch.cuda.stream(h2d):
                    if i >= 2:
                        h2d.wait_event(in_free[b])
                    qs[b].copy_(qp, non_blocking=True)
                    ks[b].copy_(kp, non_blocking=True)
                    vs[b].copy_(vp, non_blocking=True)
                    in_ready[b].record(h2d)
                stream.wait_event(in_ready[b])
                if i >= 2:
                    stream.wait_event(out_free[b])
                ac_t.ac_forward(qs[b], ks[b], vs[b], out=outs[b], stream=stream)
                in_free[b].record(stream)
                out_ready[b].record(stream)
                with torch.cuda.stream(d2h):
                    d2h.wait_event(out_ready[b])
                    op.copy_(outs[b], non_blocking=True)
                    out_free[b].record(d2h)
            stream.wait_stream(d2h)

        run_steps(4)  # each buffer set twice: both graphs captured before the timed steps
        torch.cuda.synchronize(dev)
        barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        h2d.wait_event(s0)
        n_e2e = max(2, a.steps)
        run_steps(n_e2e)
        s1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        ms_e2e = max_over_ranks(s0.elapsed_time(s1) / n_e2e, world, dev)
        nb = q.numel() * q.element_size()
        e2e = {"value": calls_per_second(ms_e2e, world), "unit": "calls/s", "h2d_bytes_per_step": 3 * nb,
               "d2h_bytes_per_step": nb, "ms_per_step": ms_e2e, "steps": n_e2e,
               "pipelined": "step s+1 inputs copied in and step s output copied out during compute "
                            "(two copy streams, two device buffer sets)"}
        del qs[1], ks[1], vs[1], outs[1]
        ac.profile_read()

    # dense comparator: torch SDPA at the same shape (40 heads x 75.6K x 128)
    dense = None
    if not a.no_dense and rank == 0:
        dms = sdpa_ms(q, k, v, stream, flush)
        dense = {"impl": "torch.nn.functional.scaled_dot_product_attention", "ms": dms,
                 "tflops": w.dense_flops() / (dms * 1e-3) / 1e12, "speedup_of_clustered_call": dms / ms}
        # the library's own dense path (Algorithm 3's dense branch): every head flagged
        # dense, so the attention kernel takes all N keys of each head
        cq, ck = ac.ac_cluster_q(q), ac.ac_cluster_k(k)
        dflag = torch.ones(w.heads, dtype=torch.uint8, device=dev)
        sel0 = torch.zeros(w.heads, ac.kq_cap, ac.kk_cap, dtype=torch.int32, device=dev)
        cnt0 = torch.zeros(w.heads, ac.kq_cap, dtype=torch.int32, device=dev)
        args = (q, k, v, cq["assign"], ck["assign"], sel0, cnt0)
        ac.ac_sparse_attn(*args, dense_flag=dflag, out=out)
        oms = time_calls(lambda: ac.ac_sparse_attn(*args, dense_flag=dflag, out=out), 3, stream, flush)
        del cq, ck, sel0, cnt0, args
        dense["own_dense"] = {"impl": "ac_sparse_attn with every head dense (gathered copy + attn3_kernel)",
                              "ms": oms, "tflops": w.dense_flops() / (oms * 1e-3) / 1e12}

    launches_timed = int(prof_t["launches"]) if e2e is None else launches_per_call(ac_t, q, k, v, out) * a.steps
    denoise = None
    if rank == 0 and a.denoise_steps > 0:
        denoise = denoise_steps(ac, q, k, v, out, a.denoise_steps, a.drift, stream)
    qs = ks = vs = outs = None

    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        pass
    peak = peaks.get("bf16_tflops_sustained") or 1390.6
    peak_src = "measured (MEASURED_PEAKS.json bf16_tflops_sustained)" if peaks else "fallback"
    # DRAM bytes of one attention launch, from an ncu capture of this kernel
    # version on the Wan-shaped workload cut to 8 heads, scaled by heads; only
    # for that workload (None until such a capture exists)
    traffic = None
    if w.name == DEFAULT_WORKLOAD and w.top_p == 0.9 and ATTN_TRAFFIC_8H and not a.select_mode:
        traffic = ATTN_TRAFFIC_8H * w.heads / 8
    roof = {"kernel": "attn3_kernel (block-sparse attention, tcgen05)", "bound": "tensor", "achieved": tflops_attn,
            "peak": peak, "unit": "TFLOP/s", "frac": tflops_attn / peak, "traffic": traffic,
            "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum, 8-head capture scaled by heads"
            if traffic else None,
            "peak_source": peak_src, "ms_per_launch": attn_ms,
            "flops_per_launch": flops, "flops_rule": "4 * d * computed (query, key) pairs"}

    extra = {}
    if rank == 0:
        extra["launch_by_launch"] = {
            "ms_per_call": t_lbl, "calls_per_s": calls_per_second(t_lbl, world),
            "how": "the same calls with AC_FLAG_PROFILE (per-stage events), which ac_forward never replays "
                   "from its cached CUDA graph"}
    if rank == 0 and not a.no_per_config and world == 1:
        # every workload gets its own context
        extra["top_p_sweep"] = top_p_sweep(w, q, k, v, out, dev, stream, a.per_config_calls, peak,
                                           dense["ms"] if dense else None)
        extra["select_modes"] = select_modes(w, q, k, v, out, dev, stream, a.per_config_calls, peak)
        del q, k, v, out
        ac.close()
        ac_t.close()
        torch.cuda.empty_cache()
        extra["per_config"] = per_config(dev, stream, a.per_config_calls, peak)

    if rank == 0:
        line = {"metric": METRIC, "value": calls_per_s, "unit": "calls/s", "n_gpus": world, "steps": a.steps,
                "warmup": max(a.warmup, 3), "ms_per_step": t_max, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
                "config": dict(config_of(w, world, cfg.text_keys),
                               **({"select_mode": {a.select_mode: SELECT_MODES[a.select_mode]}} if a.select_mode else {})),
                "tflops_effective_call": tflops_call, "tflops_effective_attn": tflops_attn,
                "pairs": st["pairs"], "density": st["pairs"] / (w.heads * float(w.n) ** 2),
                "dense_heads": st["dense_heads"],
                "stage_ms": {k2: prof[k2] for k2 in ("ms_cluster_q", "ms_cluster_k", "ms_select", "ms_prep",
                                                     "ms_attn_kernel", "ms_total")},
                "roofline": roof, "dense_attention": dense,
                "cpu_baseline": cpu_base, "e2e": e2e,
                "gpu_launches": launches_timed, "clocks": clocks}
        line.update(extra)
        if denoise is not None:
            line["denoise_steps"] = denoise
        print(json.dumps(line), flush=True)
    ac.close()
    ac_t.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def time_calls(fn, n, stream, flush=None):
    """Mean ms of n calls of fn, CUDA events on the launching stream.  With a
    flush buffer, L2 is overwritten before every call, outside the timing."""
    import torch
    if flush is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1) / n
    evs = []
    for _ in range(n):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        evs.append((e0, e1))
    evs[-1][1].synchronize()
    return sum(x.elapsed_time(y) for x, y in evs) / n


def sdpa_ms(q, k, v, stream, flush, calls=3):
    import torch.nn.functional as F
    qd, kd, vd = (t.unsqueeze(0) for t in (q, k, v))
    F.scaled_dot_product_attention(qd, kd, vd)
    return time_calls(lambda: F.scaled_dot_product_attention(qd, kd, vd), calls, stream, flush)


def measure(w, q, k, v, out, dev, stream, calls, peak, text_keys=0, over=None):
    """One workload through ac_forward: ms per call (CUDA events, L2 flushed
    first when an input tensor fits in L2) with the default flags (so a repeated
    call replays the library's cached CUDA graph where the counts are fixed),
    the same launch by launch with per-stage events (the stage breakdown), the
    computed pairs and the attention kernel's rate against the peak."""
    import torch
    from clustered_sparse_attention_head_b200 import _abi
    from clustered_sparse_attention_head_b200.api import AdaCluster, Config

    def make(flags):
        cfg = Config.from_workload(w)
        cfg.flags = flags
        cfg.text_keys = text_keys
        for key, val in (over or {}).items():
            setattr(cfg, key, val)
        return AdaCluster(cfg, device=dev)
    ac_t, ac = make(0), make(_abi.AC_FLAG_PROFILE)
    flush = None if tensor_bytes(w) > L2_BYTES else torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(2):  # the second call on these buffers captures the library's graph
        ac_t.ac_forward(q, k, v, out=out)
    ac.ac_forward(q, k, v, out=out)
    _, st = ac.ac_forward(q, k, v, out=out, stats=True)
    if ac.get_status() != 0 or ac_t.get_status() != 0:
        raise RuntimeError(f"{w.name}: device status {ac.get_status()} / {ac_t.get_status()}")
    ac.profile_read()
    ac_t.profile_read()
    ms = time_calls(lambda: ac_t.ac_forward(q, k, v, out=out), calls, stream, flush)
    launches = ac_t.profile_read()["launches"]
    ms_lbl = time_calls(lambda: ac.ac_forward(q, k, v, out=out), calls, stream, flush)
    prof = ac.profile_read()
    status = max(ac.get_status(), ac_t.get_status())
    ac.close()
    ac_t.close()
    if status != 0:
        raise RuntimeError(f"{w.name}: device status {status}")
    flops = 4.0 * w.d * st["pairs"]
    attn = prof["ms_attn_kernel"]
    r = {"ms_per_call": ms, "calls_per_s": 1e3 / ms, "ms_per_call_launch_by_launch": ms_lbl,
         "pairs": st["pairs"], "pairs_computed": st["pairs_computed"],
         "density": st["pairs"] / (w.heads * float(w.n) ** 2), "dense_heads": st["dense_heads"],
         "stages_q": st["max_stages_q"], "stages_k": st["max_stages_k"],
         "stage_ms": {k2: prof[k2] for k2 in ("ms_cluster_q", "ms_cluster_k", "ms_select", "ms_prep",
                                              "ms_attn_kernel", "ms_total")},
         "launches_per_call": int(launches) // max(calls, 1),
         "tflops_effective_call": flops / (ms * 1e-3) / 1e12,
         "tflops_effective_attn": flops / (attn * 1e-3) / 1e12 if attn > 0 else None,
         "roofline_frac_attn": flops / (attn * 1e-3) / 1e12 / peak if attn > 0 else None,
         "l2": config_of(w, 1)["l2"]}
    return r, flush


def top_p_sweep(w, q, k, v, out, dev, stream, calls, peak, sdpa):
    """The headline workload at each top-p of TOP_P_SWEEP (same inputs)."""
    from dataclasses import replace
    rows = []
    for tp in TOP_P_SWEEP:
        r, _ = measure(replace(w, top_p=tp), q, k, v, out, dev, stream, calls, peak)
        r["top_p"] = tp
        if sdpa:
            r["sdpa_ms"] = sdpa
            r["speedup_vs_sdpa"] = sdpa / r["ms_per_call"]
        rows.append(r)
    return rows


SELECT_MODES = {
    "quest_top_p": dict(score_mode=1),
    "centroid_top_k64": dict(top_k=64),
    "per_query_top_k64": dict(top_k=64, per_query=True),
}


def select_modes(w, q, k, v, out, dev, stream, calls, peak):
    """The selection options on the headline workload: the Quest score with the
    top-p cut, argtopk per query cluster, argtopk per query row."""
    res = {}
    for name, over in SELECT_MODES.items():
        r, _ = measure(w, q, k, v, out, dev, stream, calls, peak, over=over)
        r["options"] = over
        res[name] = r
    return res


def per_config(dev, stream, calls, peak):
    """Every workload of the suite at full size, with the SDPA comparator."""
    import torch
    res = {}
    for name in W.ORDER:
        w = W.WORKLOADS[name]
        hs = gen_inputs(w)
        tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        q, k, v = (torch.from_numpy(np.stack([getattr(h, a) for h in hs])).to(dev).to(tdt) for a in "qkv")
        del hs
        out = torch.empty_like(q)
        r, flush = measure(w, q, k, v, out, dev, stream, calls, peak)
        d = sdpa_ms(q, k, v, stream, flush)
        r["sdpa_ms"] = d
        r["sdpa_tflops"] = w.dense_flops() / (d * 1e-3) / 1e12
        r["speedup_vs_sdpa"] = d / r["ms_per_call"]
        res[name] = r
        del q, k, v, out, flush
        torch.cuda.empty_cache()
    return res


def denoise_steps(ac, q, k, v, out, steps, drift, stream):
    """The multi-step driver on inputs that drift by drift * N(0, 1) per element
    and step (seeded, drawn on the device before each step's timed call): step
    0 clusters as configured, later steps keep its counts and warm-start
    k-means.  Per step: call time (CUDA events) and the k-means rounds run."""
    import torch
    state = ac.step_state()
    gen = torch.Generator(device=q.device)
    gen.manual_seed(1234)
    qs, ks, vs = q.clone(), k.clone(), v.clone()
    rows = []
    for s in range(steps):
        if s > 0:
            for t in (qs, ks, vs):
                t.copy_((t.float() + drift * torch.randn(t.shape, generator=gen, device=t.device)).to(t.dtype))
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        _, st = ac.ac_forward_step(s, qs, ks, vs, state, out=out, stats=True)
        e1.record(stream)
        torch.cuda.synchronize()
        rows.append({"step": s, "ms": e0.elapsed_time(e1), "ms_cluster_q": st["ms_cluster_q"],
                     "ms_cluster_k": st["ms_cluster_k"], "rounds_q": st["kmeans_rounds_q"],
                     "rounds_k": st["kmeans_rounds_k"]})
    status = ac.get_status()
    if status != 0:
        raise RuntimeError(f"device status {status}")
    return {"drift": drift, "steps": rows}


def launches_per_call(ac, q, k, v, out):
    ac.profile_read()
    ac.ac_forward(q, k, v, out=out)
    return int(ac.profile_read()["launches"])


if __name__ == "__main__":
    sys.exit(main())
