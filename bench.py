#!/usr/bin/env python
"""Throughput of the batch-invariant MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]
                    [--workload NAME] [--T TOKENS] [--no-cpu-baseline] [--no-sweeps]

One step is one full layer forward (RMSNorm, router GEMM, top-k with the
expert histogram, offsets + stable scatter, row gather, gate/up + SwiGLU GEMM,
down GEMM, fixed-order combine + residual + RMSNorm) over one batch of the
DeepSeek-V3-shaped workload (T=8192 tokens, D=7168, 256 experts top-8 sigmoid
scores with a selection bias, normalised over the chosen 8, routed scale 2.5,
SwiGLU clamp 10, I=2048, one shared expert of 2048) with seeded synthetic
inputs and random weights of that architecture.  The L2 cache is flushed (a
512 MiB write) before every timed step; each step is timed with CUDA events
on the launching stream.  N > 1 (torchrun, one rank per GPU) runs independent
replicas on disjoint token batches: the layer shards by token with no data
exchange, so scaling is weak and `value` = all ranks' tokens / the slowest
rank's time.

Printed by rank 0 as one JSON line: tokens/s; the roofline of the dominant
kernel (the gate/up + SwiGLU grouped GEMM, tensor-bound) against the measured
peak (and, as `frac_of_nominal`, against the nominal dense bf16 peak); the
end-to-end number through the public API with pinned host buffers (copies in
and out every step, pipelined across steps by HostPipeline); SM clocks sampled
during the timed region; the fine-grained workload (T=4096, D=2048, 64 experts
top-6) as a sub-object; the decode sweep (T = 1, 8, 64, 128, 512 on the
fine-grained weights, HBM-bound) as a sub-object; and the fp64 CPU oracle
timed on a bounded sample (`cpu_baseline`) with the GPU's outputs on that
sample compared against it (`parity`).

--workload picks another headline workload (fine_grained, skew_zipf,
skew_hash, fine_grained_situ, latent_situ, fine_grained_fp8, latent_situ_fp8,
tiny, tiny_fp8, or skew_epilogue for the 8-partial reduce + residual +
RMSNorm); --T overrides its batch size; --no-sweeps drops the two
sub-objects.  `--impl reference` times only the oracle.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/sec at 1 B200; % bf16 TC peak (prefill) / % HBM BW (decode)"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "v3_shaped"
GATEUP_STAGE = 5
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic_gemm_gateup.json")
GEMM_SOURCES = [os.path.join(ROOT, "deterministic_expert_b200", "csrc", n)
                for n in ("grouped_gemm.cu", "common.cuh", "moe_internal.h")]
# Nominal B200 figures (dense bf16 tensor peak; HBM3e bandwidth as the
# spec target states it), reported beside the measured-peak fractions.
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 8000.0
L2_NOTE = "flushed before every step (512 MiB write, untimed)"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="b200", choices=["b200", "reference"])
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--T", type=int, default=None, help="override the workload's batch size")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-sweeps", action="store_true", help="skip the fine-grained and decode sub-objects")
    a = p.parse_args()
    a.warmup = max(a.warmup, 3)
    return a


def workload(a):
    from synth import workloads as W
    cfg = W.CONFIGS[a.workload]
    return cfg.with_T(a.T) if a.T else cfg


def describe(cfg):
    from synth import workloads as W
    return {"workload": W.pretty(cfg), "T": cfg.T, "D": cfg.D, "E": cfg.E, "k": cfg.k, "I": cfg.I,
            "n_shared": cfg.n_shared, "I_shared": cfg.I_shared,
            "router": {0: "softmax", 1: "sigmoid+bias", 2: "hash"}[cfg.router],
            "renormalize": bool(cfg.renormalize),
            "activation": "SiTU-GLU" if cfg.activation == 1 else "SwiGLU", "latent": cfg.latent,
            "expert_weights": {0: "bf16", 1: "FP4 values as E4M3 (E4M3 x E4M3 GEMMs)",
                               2: "FP4 packed E2M1 + UE8M0 block scales (block-scaled E2M1 x E4M3 GEMMs)"}[
                                   cfg.weight_format]}


def bench_config(cfg, world):
    """The `config` object both arms print for a workload."""
    return {**describe(cfg), "l2": L2_NOTE, "parallelism": f"replicas x{world} (token-sharded, no collective)"}


def peaks():
    """Measured peaks (MEASURED_PEAKS.json) or the machine's fallback figures."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"tc": d["bf16_tflops"], "tc_sustained": d.get("bf16_tflops_sustained"), "hbm": d["hbm_gbs"],
                "kind": "measured"}
    return {"tc": 1590.0, "tc_sustained": 1400.0, "hbm": 6650.0, "kind": "fallback"}


def host_threads():
    """Threads the oracle's BLAS uses, and the host's usable cores."""
    from threadpoolctl import threadpool_info
    blas = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return blas, len(os.sched_getaffinity(0))


def gemm_source_hash():
    h = hashlib.sha256()
    for p in GEMM_SOURCES:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def ncu_traffic(cfg):
    """DRAM bytes per launch of the gate/up GEMM from the committed ncu summary,
    or None when the kernel source changed since the counters were taken."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f)
    sha = gemm_source_hash()
    for e in d.get("entries", []):
        if e.get("source_sha256") == sha and e.get("T") == cfg.T and e.get("workload") == cfg.name:
            return e.get("dram_bytes_per_launch")
    return None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    def __init__(self, index):
        self.file = tempfile.NamedTemporaryFile(prefix="clocks", suffix=".csv", delete=False)
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(index), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.close()
        rows = []
        with open(self.file.name) as f:
            for line in f:
                parts = [s.strip() for s in line.split(",")]
                if len(parts) >= 8:
                    rows.append(parts)
        os.unlink(self.file.name)
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = max(float(r[1]) for r in rows if r[1].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------------ oracle
class TimedWeights:
    """The workload's host weights (fp64 arrays of the bf16 values, regenerated
    from the seeded generator) with the time spent regenerating experts
    recorded, so the oracle can be timed without its input generation."""

    def __init__(self, cfg, cache_experts):
        import oracle as O
        from synth import device as SD
        self.base = SD.HostWeights(cfg, cache_experts=cache_experts)
        self.gen_s = 0.0
        for n in ("w_router", "router_bias", "g_in", "g_out", "w_proj_down", "w_proj_up"):
            setattr(self, n, getattr(self.base, n, None))
        # FP4 experts: the oracle's own FP4 quantisation of the master weights (part of its work).
        self.view = O.FP4Weights(self) if cfg.weight_format else self

    def _timed(self, fn, i):
        t0 = time.perf_counter()
        out = fn(i)
        self.gen_s += time.perf_counter() - t0
        return out

    def routed(self, e):
        return self._timed(self.base.routed, e)

    def shared(self, s):
        return self._timed(self.base.shared, s)


def _cache_for(cfg, budget_bytes=8 << 30):
    """Experts kept in fp64 at once: all of them when they fit the budget."""
    from synth import workloads as W
    per = 3 * (cfg.latent or cfg.D) * cfg.I * 8
    return max(2, min(cfg.E + cfg.n_shared, budget_bytes // per)), per * cfg.E <= budget_bytes


def oracle_run(cfg, rows, tw, x_all=None):
    """The oracle on rows of the workload's batch; returns (ref, oracle seconds
    without weight regeneration)."""
    import numpy as np

    import oracle as O
    from synth import device as SD
    from synth import workloads as W
    x = SD.host_rows(cfg, "x", rows, T=cfg.T)
    r = SD.host_rows(cfg, "residual", rows, T=cfg.T)
    ids = W.host_token_ids(cfg, cfg.T)[np.asarray(rows)]
    g0 = tw.gen_s
    t0 = time.perf_counter()
    ref = O.moe_layer(cfg, tw.view, x, r, ids)
    return ref, (time.perf_counter() - t0) - (tw.gen_s - g0)


def oracle_sample(cfg, budget_s=12.0, wall_s=90.0):
    """Time the fp64 oracle (as it stands) on consecutive chunks of the
    workload's tokens until about budget_s of oracle time (or wall_s of wall
    time, weight regeneration included) has passed.  Expert weights are
    regenerated on the host from the seeded generator; that time is not
    counted.  Returns (cpu_baseline dict, [(rows, ref), ...])."""
    import numpy as np
    cache, all_fit = _cache_for(cfg)
    tw = TimedWeights(cfg, cache)
    chunk = 256 if all_fit else 16
    tokens, spent, chunks, refs = 0, 0.0, 0, []
    w0 = time.perf_counter()
    while spent < budget_s and tokens < cfg.T and time.perf_counter() - w0 < wall_s:
        rows = np.arange(tokens, min(cfg.T, tokens + chunk))
        ref, dt = oracle_run(cfg, rows, tw)
        spent += dt
        tokens += len(rows)
        chunks += 1
        refs.append((rows, ref))
    blas, ncpu = host_threads()
    return ({"value": round(tokens / spent, 2), "unit": UNIT, "cores": blas, "host_cores": ncpu,
             "kind": "oracle",
             "sample": f"tokens 0..{tokens - 1} of the {cfg.T}-token batch ({chunks} chunks of {chunk}), full "
                       f"layer in fp64, {spent:.1f} s of oracle time; regenerating the expert weights on the "
                       f"host ({tw.gen_s:.1f} s) not timed"}, refs)


def parity_readout(refs, out_norm, out_residual, idx):
    """The GPU's outputs on the oracle sample's tokens against the oracle
    (tokens routed differently are counted, not value-compared here; the
    test suite classifies and value-checks them)."""
    import numpy as np
    import torch
    gi = idx.cpu().numpy()
    on = out_norm.to(torch.float32).cpu().numpy().astype(np.float64)
    orr = out_residual.to(torch.float32).cpu().numpy().astype(np.float64)
    alike, differ, emax, esum, n = 0, 0, 0.0, 0.0, 0
    for rows, ref in refs:
        same = np.all(gi[rows] == ref["idx"], axis=1)
        alike += int(same.sum())
        differ += int((~same).sum())
        for g, o in ((on[rows][same], ref["out_norm"][same]), (orr[rows][same], ref["out_residual"][same])):
            e = np.abs(g - o) / np.maximum(1.0, np.abs(o))
            if e.size:
                emax = max(emax, float(e.max()))
                esum += float(e.sum())
                n += e.size
    return {"tokens": alike + differ, "routed_like_oracle": alike, "routed_differently": differ,
            "max_rel_err": round(emax, 6), "mean_rel_err": round(esum / max(n, 1), 7),
            "tolerance": {"max": 2e-2, "mean": 4e-3}}


def run_reference(a):
    """--impl reference: the oracle on the same workload, rank 0 only.  Every
    step times the oracle on the same bounded sample of the batch (its first
    tokens), as every GPU step runs the same batch; the weights of the experts
    it touches are regenerated once, untimed."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(a.gpus)))
    if rank != 0:
        return
    import numpy as np
    cfg = workload(a)
    cache, all_fit = _cache_for(cfg)
    n = 128 if all_fit else 2
    rows = np.arange(min(n, cfg.T))
    tw = TimedWeights(cfg, max(cache, cfg.k * n + cfg.n_shared + 1))
    times = []
    for step in range(a.warmup + a.steps):
        _, dt = oracle_run(cfg, rows, tw)
        if step >= a.warmup:
            times.append(dt)
    secs = sum(times)
    value = len(rows) * len(times) / secs
    blas, ncpu = host_threads()
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * secs / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded counter-based generator; random weights of the workload's shape)",
        "config": bench_config(cfg, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas, "host_cores": ncpu, "kind": "oracle",
                         "sample": f"each step: tokens 0..{len(rows) - 1} of the {cfg.T}-token batch, full layer "
                                   f"in fp64; expert weight regeneration ({tw.gen_s:.1f} s) not timed"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def epilogue_oracle_sample(budget_s, chunk=256):
    """The oracle's fixed-order reduce + residual + RMSNorm on consecutive
    256-row chunks of the epilogue workload until ``budget_s`` has passed."""
    import numpy as np

    import oracle as O
    from synth import device as SD
    from synth import workloads as W
    P, T, D = W.EPILOGUE_P, W.EPILOGUE_T, W.EPILOGUE_D
    g = np.ones(D)
    secs, rows = 0.0, 0
    r0 = 0
    while secs < budget_s:
        n = min(chunk, T - r0)
        parts = np.stack([SD.f64(W.host_partial(p, T, D, start=r0 * D, count=n * D)).reshape(n, D)
                          for p in range(P)])
        res = SD.f64(W.host_bf16(W.C5, "residual", start=r0 * D, count=n * D)).reshape(n, D)
        t0 = time.perf_counter()
        O.reduce_partials(parts, res, g, W.C5.eps)
        secs += time.perf_counter() - t0
        rows += n
        r0 = (r0 + n) % T
    cores, ncpu = host_threads()
    return {"value": round(rows / secs, 1), "unit": UNIT, "cores": cores, "host_cores": ncpu, "kind": "oracle",
            "sample": f"{rows} rows of the {T}-row epilogue in {chunk}-row chunks, fp32 fixed-order sum, fp64 norm"}


def run_reference_epilogue(a):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from synth import workloads as W
    budget = max(2.0, 60.0 / max(1, a.steps + a.warmup))
    vals = [epilogue_oracle_sample(budget) for _ in range(a.warmup + a.steps)][a.warmup:]
    value = sum(v["value"] for v in vals) / len(vals)
    cpu = dict(vals[-1], value=round(value, 1))
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": a.gpus,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(1e3 * W.EPILOGUE_T / value, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded counter-based generator)",
        "config": {"workload": f"skewed workload epilogue: {W.EPILOGUE_P} partial buffers "
                               f"[T={W.EPILOGUE_T}, D={W.EPILOGUE_D}]"},
        "cpu_baseline": cpu,
        "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# --------------------------------------------------------------- b200 arm
def run_epilogue(a):
    """--workload skew_epilogue: the 8-partial fixed-order reduce + residual +
    RMSNorm of the skewed workload (8 bf16 buffers of [16384, 4096] N(0,1)/8),
    HBM-bound; reported as tokens/s with its share of the measured HBM copy
    bandwidth (algorithmic bytes (P + 3) * T * D * 2 per launch).  With N > 1
    ranks (N dividing 8) the same job runs tensor parallel: the partials are
    spread over the ranks and every rank reduces T / N rows over NVLink
    (strong scaling, share of the measured peer-copy bandwidth)."""
    import torch
    import torch.distributed as dist

    import deterministic_expert_b200 as moe
    from synth import device as SD
    from synth import workloads as W
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    P, T, D = W.EPILOGUE_P, W.EPILOGUE_T, W.EPILOGUE_D
    res = SD.device_bf16(W.C5, "residual", T=T, device=dev)
    g = SD.device_bf16(W.C5, "g_out", device=dev)
    stream = torch.cuda.current_stream()
    # N > 1 (N dividing 8): tensor parallel, as in the Fireworks parity post
    # (Trap 1, one reduction order on every rank).  Rank r holds
    # partials r*8/N .. (r+1)*8/N - 1 in exported peer memory; each step is one
    # TPAllReduceNorm call (device barrier, one kernel reducing this rank's rows
    # over every rank's partials and storing them to every rank, barrier).
    tp = None
    if world > 1 and P % world == 0:
        tp = moe.TPAllReduceNorm(T, D, per_rank=P // world, device=dev)
        for j in range(P // world):
            SD.fill_partial(tp.partial[j], rank * (P // world) + j)
        step = lambda: tp(res, g, stream=stream)  # noqa: E731
    else:
        parts = SD.device_partials(P, T, D, device=dev)
        on = torch.empty((T, D), dtype=torch.bfloat16, device=dev)
        orr = torch.empty_like(on)
        step = lambda: moe.reduce_partials(parts, res, g, on, orr, stream=stream)  # noqa: E731
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    for _ in range(a.warmup):
        flush.fill_(1)
        step()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(a.steps)]
    clocks = ClockSampler(local) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for e0, e1 in evs:
        flush.fill_(1)
        e0.record(stream)
        step()
        e1.record(stream)
    torch.cuda.synchronize()
    if tp is not None:
        tp.check()   # raises if a device barrier wait gave up
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if clocks else None
    ms = torch.tensor([sum(e0.elapsed_time(e1) for e0, e1 in evs)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(ms, op=dist.ReduceOp.MAX)
    ms_per_step = float(ms.item()) / a.steps
    e2e = None
    if rank == 0 and tp is None:
        # End to end: partials and residual from pinned host memory, both outputs back.
        hp = [torch.empty((T, D), dtype=torch.bfloat16, pin_memory=True) for _ in range(P)]
        for h, d in zip(hp, parts):
            h.copy_(d)
        hr = torch.empty((T, D), dtype=torch.bfloat16, pin_memory=True)
        hr.copy_(res)
        hon = torch.empty_like(hr, pin_memory=True)
        hor = torch.empty_like(hr, pin_memory=True)
        n_e2e = 3
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_e2e):
            for h, d in zip(hp, parts):
                d.copy_(h, non_blocking=True)
            res.copy_(hr, non_blocking=True)
            moe.reduce_partials(parts, res, g, on, orr, stream=stream)
            hon.copy_(on, non_blocking=True)
            hor.copy_(orr, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e = {"value": round(n_e2e * T / (e0.elapsed_time(e1) / 1e3), 1), "unit": UNIT,
               "h2d_bytes_per_step": (P + 1) * T * D * 2, "d2h_bytes_per_step": 2 * T * D * 2}
    cpu = None if (rank != 0 or a.no_cpu_baseline) else epilogue_oracle_sample(budget_s=12.0)
    if rank == 0:
        pk = peaks()
        hbm_peak, peak_kind = pk["hbm"], pk["kind"]
        wl = (f"skewed workload epilogue: {P} partial buffers [T={T}, D={D}] bf16 "
              f"N(0,1)/8, fixed r0..r{P - 1} order + residual + RMSNorm")
        if tp is None:
            nbytes = (P + 3) * T * D * 2
            gbs = nbytes / (ms_per_step / 1e3) / 1e9
            value, scaling = world * T / (ms_per_step / 1e3), "weak"
            roof = {"bound": "hbm", "kernel": "reduce_partials", "achieved": round(gbs, 1),
                    "peak": hbm_peak, "unit": "GB/s", "frac": round(gbs / hbm_peak, 4), "traffic": None,
                    "peak_source": f"{peak_kind} HBM copy", "bytes_per_launch": nbytes}
        else:
            # One T-row job split across the ranks.  Bytes that cross this
            # rank's NVLink per step: the other ranks' partials for its rows
            # in, its normalised rows for the other ranks out (both outputs).
            rows = tp.rows
            link = ((P - P // world) * rows * D * 2) + 2 * (world - 1) * rows * D * 2
            gbs = link / (ms_per_step / 1e3) / 1e9
            value, scaling = T / (ms_per_step / 1e3), "strong"
            wl = f"tensor parallel over {world} ranks ({P // world} partials each, {rows} rows reduced per rank): " + wl
            roof = {"bound": "nvlink", "kernel": "reduce_partials (row slice, peer loads and stores)",
                    "achieved": round(gbs, 1), "peak": 770.0, "unit": "GB/s", "frac": round(gbs / 770.0, 4),
                    "traffic": None, "peak_source": "measured peer copy per direction (profiling recipe)",
                    "bytes_per_launch": link}
        print(json.dumps({
            "metric": METRIC, "value": round(value, 1), "unit": UNIT,
            "n_gpus": world, "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": scaling, "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded counter-based generator)",
            "config": {"workload": wl, "l2": "flushed before every step (512 MiB write, untimed)"},
            "roofline": roof,
            "gpu_launches": a.steps * (1 if tp is None else 3), "clocks": clk, "e2e": e2e,
            "cpu_baseline": cpu}), flush=True)
    if world > 1:
        dist.barrier()
        if tp is not None:
            tp.close()
        dist.destroy_process_group()


def timed_steps(layer, x, r, on, orr, ws, ids, steps, flush, stream, cnt=None, profile=None):
    """Run `steps` layer forwards, L2 flushed before each, each bracketed by a
    CUDA event pair on the launching stream; returns the per-step ms and, with
    ``profile`` (stage indices), the per-stage average ms over the steps."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    if profile is not None:
        layer.profile_enable(profile)
    for e0, e1 in evs:
        flush.fill_(1)
        e0.record(stream)
        layer.forward(x, r, on, orr, ws, token_ids=ids, out_counts=cnt, stream=stream)
        e1.record(stream)
    torch.cuda.synchronize()
    stage = None
    if profile is not None:
        ms, n = layer.profile_read()
        layer.profile_enable([])
        stage = [ms[i] / n[i] if n[i] else None for i in range(len(ms))]
    return [e0.elapsed_time(e1) for e0, e1 in evs], stage


def gemm_roofline(cfg, gate_ms, pk, traffic):
    from synth import workloads as W
    tc = pk["tc"] * (2.0 if cfg.weight_format else 1.0)
    nominal = NOMINAL_BF16_TFLOPS * (2.0 if cfg.weight_format else 1.0)
    fl = W.moe_flops(cfg)["gateup"]
    achieved = fl / (gate_ms / 1e3) / 1e12
    src = f"{pk['kind']} bf16 (burst)"
    if cfg.weight_format:
        # E4M3 x E4M3 and block-scaled E2M1 x E4M3 run at the FP8 rate: the bf16 peak times the
        # nominal dense ratio of the two formats (4.5 / 2.25 PFLOP/s).
        src += " x 2, nominal FP8 / bf16 ratio"
    return {"bound": "tensor", "kernel": "gemm_gateup_swiglu", "achieved": round(achieved, 1), "peak": tc,
            "unit": "TFLOP/s", "frac": round(achieved / tc, 4), "traffic": traffic, "peak_source": src,
            "frac_of_nominal": round(achieved / nominal, 4), "nominal_peak": nominal,
            "flops_per_launch": fl, "avg_launch_ms": round(gate_ms, 4)}


def layer_numbers(cfg, T, ms, distinct, pk):
    from synth import workloads as W
    tc = pk["tc"] * (2.0 if cfg.weight_format else 1.0)
    nominal = NOMINAL_BF16_TFLOPS * (2.0 if cfg.weight_format else 1.0)
    fl = W.moe_flops(cfg, T)["total"]
    tf = fl / (ms / 1e3) / 1e12
    nbytes = W.layer_bytes(cfg, T, distinct)
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"tflops": round(tf, 1), "frac_of_tc_peak": round(tf / tc, 4), "frac_of_nominal_tc": round(tf / nominal, 4),
            "flops_per_step": fl, "distinct_experts": distinct, "algorithmic_bytes": nbytes,
            "hbm_gbs": round(gbs, 1), "frac_of_hbm": round(gbs / pk["hbm"], 4),
            "frac_of_nominal_hbm": round(gbs / NOMINAL_HBM_GBS, 4)}


def fine_grained_object(a, dev, flush, stream, pk, cfg=None, w=None):
    """The fine-grained workload (T=4096, D=2048, 64 experts top-6 softmax
    renormalised, I=1408, 2 shared) timed as the headline is; with cfg / w the
    same shapes in another weight format (the given weights)."""
    import torch

    import deterministic_expert_b200 as moe
    from synth import device as SD
    from synth import workloads as W
    cfg = W.C2 if cfg is None else cfg
    if w is None:
        w = SD.device_weights(cfg, device=dev)
    x, r, _ = SD.device_inputs(cfg, device=dev)
    layer = moe.MoELayer(SD.layer_config(cfg, cfg.T), w)
    ws = torch.empty(layer.workspace_size(cfg.T), dtype=torch.uint8, device=dev)
    on, orr = torch.empty_like(x), torch.empty_like(x)
    cnt = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    timed_steps(layer, x, r, on, orr, ws, None, a.warmup, flush, stream)
    ms_steps, stage = timed_steps(layer, x, r, on, orr, ws, None, a.steps, flush, stream, cnt=cnt,
                                  profile=[GATEUP_STAGE])
    if layer.device_error(ws) != moe.MOE_OK:
        raise RuntimeError("device wait timed out (fine-grained)")
    ms = sum(ms_steps) / len(ms_steps)
    out = {"workload": W.pretty(cfg), "ms_per_step": round(ms, 4), "value": round(cfg.T / (ms / 1e3), 1),
           "unit": UNIT, "steps": a.steps,
           "layer": layer_numbers(cfg, cfg.T, ms, int((cnt > 0).sum().item()), pk),
           "roofline": gemm_roofline(cfg, stage[GATEUP_STAGE], pk, ncu_traffic(cfg)),
           "gpu_launches": a.steps * layer.launch_count(cfg.T)}
    layer.close()
    return out, w


def decode_object(a, dev, flush, stream, pk, w, cfg=None):
    """The decode sweep: batches of T = 1, 8, 64, 128, 512 tokens (the first T
    rows of an 8192-row input) on the fine-grained weights (bf16, or their FP4
    storage form with cfg = the fine_grained_fp4 workload); HBM-bound, so the
    figure is algorithmic bytes (the weights of the experts actually routed to,
    shared and router weights, activations) over the time per forward."""
    import torch

    import deterministic_expert_b200 as moe
    from synth import device as SD
    from synth import workloads as W
    cfg = W.C2 if cfg is None else cfg
    xa, ra, _ = SD.device_inputs(cfg, T=W.C4_SOURCE_T, device=dev)
    tmax = max(W.C4_T)
    layer = moe.MoELayer(SD.layer_config(cfg, tmax), w)
    ws = torch.empty(layer.workspace_size(tmax), dtype=torch.uint8, device=dev)
    cnt = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    rows = []
    launches = 0
    for T in W.C4_T:
        x, r = xa[:T].contiguous(), ra[:T].contiguous()
        on, orr = torch.empty_like(x), torch.empty_like(x)
        timed_steps(layer, x, r, on, orr, ws, None, a.warmup, flush, stream)
        ms_steps, _ = timed_steps(layer, x, r, on, orr, ws, None, a.steps, flush, stream, cnt=cnt)
        ms = sum(ms_steps) / len(ms_steps)
        distinct = int((cnt > 0).sum().item())
        nb = W.layer_bytes(cfg, T, distinct)
        gbs = nb / (ms / 1e3) / 1e9
        rows.append({"T": T, "us_per_forward": round(ms * 1e3, 2), "tokens_per_s": round(T / (ms / 1e3), 1),
                     "distinct_experts": distinct, "algorithmic_bytes": nb, "hbm_gbs": round(gbs, 1),
                     "frac_of_hbm": round(gbs / pk["hbm"], 4), "frac_of_nominal_hbm": round(gbs / NOMINAL_HBM_GBS, 4)})
        launches += a.steps * layer.launch_count(T)
    if layer.device_error(ws) != moe.MOE_OK:
        raise RuntimeError("device wait timed out (decode)")
    layer.close()
    return {"weights": W.pretty(cfg), "source_batch": f"first T rows of a {W.C4_SOURCE_T}-row input",
            "bound": "hbm", "peak_gbs": pk["hbm"], "nominal_gbs": NOMINAL_HBM_GBS, "steps": a.steps,
            "sweep": rows, "gpu_launches": launches}


def ep_waves_object(a, dev, flush, stream, w, world=8, T_rank=512, waves=(1, 2, 4)):
    """Expert parallelism over ``world`` virtual ranks on this one device
    (VirtualEP, fine-grained weights, T_rank tokens per rank): the step time
    with the four phases in one stream (waves = 1) and with the experts in
    waves, the sends of wave w + 1 on a second stream beside the GEMMs of wave
    w.  Every wave count must give the same bits.  On one device the sends are
    copies inside HBM, a small share of the step, so this measures what the
    wave split costs (more, smaller GEMM launches), not what it hides on links."""
    import torch

    import deterministic_expert_b200 as moe
    from synth import device as SD
    from synth import workloads as W
    cfg = W.C2.with_T(world * T_rank)
    x, r, _ = SD.device_inputs(cfg, device=dev)
    ep = moe.VirtualEP(SD.layer_config(cfg, T_rank), w, world, device=dev)
    xs = [x[q * T_rank:(q + 1) * T_rank].contiguous() for q in range(world)]
    rs = [r[q * T_rank:(q + 1) * T_rank].contiguous() for q in range(world)]
    rows, ref = [], None
    with torch.cuda.stream(stream):
        for n in waves:
            times = []
            for i in range(a.warmup + a.steps):
                flush.fill_(i & 0xFF)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                outs = ep.forward(xs, rs, stream=stream, waves=n)
                e1.record(stream)
                torch.cuda.synchronize()
                if i >= a.warmup:
                    times.append(e0.elapsed_time(e1))
            got = torch.cat([o[0] for o in outs]).view(torch.int16)
            ref = got.clone() if ref is None else ref
            ms = sum(times) / len(times)
            rows.append({"waves": n, "ms_per_step": round(ms, 4), "tokens_per_s": round(world * T_rank / (ms / 1e3), 1),
                         "bits_equal_one_wave": bool(torch.equal(got, ref))})
    if ep.device_errors() != [moe.MOE_OK] * world:
        raise RuntimeError("device error (virtual expert parallelism)")
    return {"workload": f"{W.pretty(cfg)}; {world} virtual expert-parallel ranks of {T_rank} tokens on one device",
            "steps": a.steps, "sweep": rows}


def main():
    a = parse()
    if a.impl == "reference":
        if a.workload == "skew_epilogue":
            run_reference_epilogue(a)
        else:
            run_reference(a)
        return
    if a.workload == "skew_epilogue":
        run_epilogue(a)
        return
    import torch
    import torch.distributed as dist

    import deterministic_expert_b200 as moe
    from synth import device as SD
    from synth import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != a.gpus:
        a.gpus = world
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    cfg = workload(a)
    T = cfg.T
    stream = torch.cuda.current_stream()
    pk = peaks()

    w = SD.device_weights(cfg, device=dev)
    if cfg.weight_format == 1:
        # FP4 expert weights: the library's quantiser turns the bf16 master
        # weights into their E4M3 codes once, before anything is timed.
        w = moe.quantize_expert_weights(w)
        torch.cuda.synchronize()
    elif cfg.weight_format == 2:
        # ... or into their storage form (packed E2M1 codes and block exponents).
        w = moe.pack_expert_weights_fp4(w)
        torch.cuda.synchronize()
    # Each rank takes its own T rows of a world*T-row batch (disjoint tokens).
    xa, ra, ida = SD.device_inputs(cfg, T=T * world, device=dev)
    x, r, ids = (xa[rank * T:(rank + 1) * T].contiguous(), ra[rank * T:(rank + 1) * T].contiguous(),
                 ida[rank * T:(rank + 1) * T].contiguous())
    del xa, ra, ida
    layer = moe.MoELayer(SD.layer_config(cfg, T_max=T), w)
    ws = torch.empty(layer.workspace_size(T), dtype=torch.uint8, device=dev)
    on = torch.empty((T, cfg.D), dtype=torch.bfloat16, device=dev)
    orr = torch.empty_like(on)
    cnt = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    use_ids = ids if cfg.router == W.ROUTER_HASH else None

    timed_steps(layer, x, r, on, orr, ws, use_ids, a.warmup, flush, stream)
    if layer.device_error(ws) != moe.MOE_OK:
        raise RuntimeError("device wait timed out during warm-up")

    # ------------------------------------------------ timed region (value)
    clocks = ClockSampler(local) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ms_steps, stage = timed_steps(layer, x, r, on, orr, ws, use_ids, a.steps, flush, stream, cnt=cnt,
                                  profile=[GATEUP_STAGE])
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if clocks else None
    if layer.device_error(ws) != moe.MOE_OK:
        raise RuntimeError("device wait timed out in the timed region")
    ms_total = torch.tensor([sum(ms_steps)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(ms_total, op=dist.ReduceOp.MAX)
    ms_per_step = float(ms_total.item()) / a.steps
    value = world * T / (ms_per_step / 1e3)
    distinct = int((cnt > 0).sum().item())
    gate_ms = stage[GATEUP_STAGE]

    # --------------------------------------------- per-stage breakdown (untimed)
    _, all_stage = timed_steps(layer, x, r, on, orr, ws, use_ids, 3, flush, stream, profile=list(range(moe.NUM_STAGES)))
    stage_avg = {moe.STAGE_NAMES[i]: round(v * 1e3, 2) if v else None for i, v in enumerate(all_stage)}
    # The GPU's outputs (and routing) of the batch, for the parity readout.
    layer.forward(x, r, on, orr, ws, token_ids=use_ids, out_topk_idx=idx, stream=stream)
    torch.cuda.synchronize()

    # ------------------------------------------------------- e2e (host buffers)
    # Through the public API: HostPipeline copies every step's inputs in from
    # pinned host memory and both outputs back, overlapping the copies of
    # neighbouring steps with each step's forward.
    hx, hr = x.cpu().pin_memory(), r.cpu().pin_memory()
    hid = ids.cpu().pin_memory() if use_ids is not None else None
    hon = [torch.empty(on.shape, dtype=on.dtype).pin_memory() for _ in range(2)]
    hor = [torch.empty(on.shape, dtype=on.dtype).pin_memory() for _ in range(2)]
    pipe = moe.HostPipeline(layer, T, device=dev)
    h2d = hx.numel() * 2 + hr.numel() * 2 + (hid.numel() * 4 if hid is not None else 0)
    d2h = 2 * on.numel() * 2

    def e2e(n):
        pipe.run([hx] * n, [hr] * n, [hon[i & 1] for i in range(n)], [hor[i & 1] for i in range(n)],
                 token_ids=None if hid is None else [hid] * n)

    e2e(a.warmup)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    e2e(a.steps)
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    if layer.device_error(pipe.ws) != moe.MOE_OK:
        raise RuntimeError("device wait timed out (end to end)")
    e2e_ms = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(e2e_ms, op=dist.ReduceOp.MAX)
    e2e_value = world * T * a.steps / (float(e2e_ms.item()) / 1e3)
    e2e_bits = torch.equal(hon[(a.steps - 1) & 1].view(torch.int16), on.cpu().view(torch.int16))
    del pipe

    sub = {}
    if not a.no_sweeps and cfg.name == DEFAULT_WORKLOAD and not a.T:
        fg, w2 = fine_grained_object(a, dev, flush, stream, pk)
        sub["fine_grained"] = fg
        sub["decode"] = decode_object(a, dev, flush, stream, pk, w2)
        # The same sweep with the FP4 experts in their storage form (half a
        # byte per weight plus block exponents, block-scaled E2M1 x E4M3 GEMMs).
        w4 = moe.pack_expert_weights_fp4(w2)
        sub["decode_fp4"] = decode_object(a, dev, flush, stream, pk, w4, cfg=W.C2P)
        # The prefill-sized batch with the FP4 storage form (block-scaled GEMMs).
        sub["fine_grained_fp4"], _ = fine_grained_object(a, dev, flush, stream, pk, cfg=W.C2P, w=w4)
        del w4
        sub["ep_waves"] = ep_waves_object(a, dev, flush, stream, w2)
        del w2

    if rank == 0:
        cpu = par = None
        if world == 1 and not a.no_cpu_baseline:
            cpu, refs = oracle_sample(cfg)
            par = parity_readout(refs, on, orr, idx)
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": {0: "bf16", 1: "e4m3", 2: "e2m1 x e4m3"}[cfg.weight_format],
            "data": "synthetic (seeded counter-based generator; random weights of the workload's shape)",
            "config": bench_config(cfg, world),
            "roofline": gemm_roofline(cfg, gate_ms, pk, ncu_traffic(cfg)),
            "layer": layer_numbers(cfg, T, ms_per_step, distinct, pk),
            "stage_us": stage_avg,
            "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "api": "HostPipeline (copy-in, compute and copy-out streams, "
                                                       "two buffer sets, steps overlapped)",
                    "outputs_bit_equal_to_device_forward": bool(e2e_bits)},
            "gpu_launches": a.steps * layer.launch_count(T),
            "clocks": clk,
            **sub,
            "cpu_baseline": cpu,
            "parity": par,
        }
        print(json.dumps(line), flush=True)
    layer.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
