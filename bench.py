#!/usr/bin/env python
"""Throughput of the batch-invariant MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]
                    [--workload NAME] [--T TOKENS] [--no-cpu-baseline]

--workload picks another workload (v3_shaped, skew_zipf, skew_hash,
fine_grained_situ, latent_situ, fine_grained_fp8, latent_situ_fp8, tiny, tiny_fp8,
or skew_epilogue for the 8-partial
reduce + residual + RMSNorm); --T overrides the batch size (the decode sweep
is --T 1, 8, 64, 128, 512 on the fine-grained weights).

One step is one full layer forward (all eight kernels: RMSNorm, router GEMM,
top-k with the expert histogram, offsets + stable scatter, row gather,
gate/up + SwiGLU GEMM, down GEMM, fixed-order combine + residual + RMSNorm) over one batch of the
fine-grained workload (T=4096 tokens, D=2048, 64 experts top-6 softmax
renormalised, I=1408, 2 shared experts of 1408) with seeded synthetic inputs
and random weights of that architecture.  The L2 cache is flushed (a 512 MiB
write) before every timed step; each step is timed with CUDA events on the
launching stream.  N > 1 (torchrun, one rank per GPU) runs independent
replicas on disjoint token batches: the layer shards by token with no data
exchange, so scaling is weak and `value` = all ranks' tokens / the slowest
rank's time.

Printed by rank 0 as one JSON line: tokens/s, the roofline of the dominant
kernel (the gate/up + SwiGLU grouped GEMM, tensor-bound), the end-to-end
number through the public API with host buffers, SM clocks sampled during the
timed region, and the fp64 CPU oracle timed on a bounded sample
(`cpu_baseline`).  `--impl reference` times only that oracle.
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
GATEUP_STAGE = 5
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic_gemm_gateup.json")
GEMM_SOURCES = [os.path.join(ROOT, "deterministic_expert_b200", "csrc", n)
                for n in ("grouped_gemm.cu", "common.cuh", "moe_internal.h")]


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="b200", choices=["b200", "reference"])
    p.add_argument("--workload", default="fine_grained")
    p.add_argument("--T", type=int, default=None, help="override the workload's batch size")
    p.add_argument("--no-cpu-baseline", action="store_true")
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
            "expert_weights": "FP4 values as E4M3 (E4M3 x E4M3 GEMMs)" if cfg.weight_format else "bf16"}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d["bf16_tflops"], d["hbm_gbs"], "measured"
    return 1590.0, 6650.0, "fallback"


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
def oracle_sample(cfg, budget_s=12.0, chunk=256):
    """Time the fp64 oracle (as it stands) on chunks of the workload's tokens
    until about budget_s of CPU work has run.  Weight generation is not timed."""
    import numpy as np
    from threadpoolctl import threadpool_info

    import oracle as O
    from synth import device as SD
    hw = SD.HostWeights(cfg)
    if cfg.weight_format:
        hw = O.FP4Weights(hw)   # the oracle's own FP4 quantisation of the master weights
    for e in range(cfg.E):
        hw.routed(e)
    for s in range(cfg.n_shared):
        hw.shared(s)
    from synth import workloads as W
    tokens, spent, chunks = 0, 0.0, 0
    while spent < budget_s and tokens < cfg.T:
        rows = np.arange(tokens, min(cfg.T, tokens + chunk))
        x = SD.host_rows(cfg, "x", rows, T=cfg.T)
        r = SD.host_rows(cfg, "residual", rows, T=cfg.T)
        ids = W.host_token_ids(cfg, cfg.T)[rows]
        t0 = time.perf_counter()
        O.moe_layer(cfg, hw, x, r, ids)
        spent += time.perf_counter() - t0
        tokens += len(rows)
        chunks += 1
    cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return {"value": tokens / spent, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{tokens} of {cfg.T} tokens ({chunks} chunks of {chunk}), full layer in fp64, "
                      f"{spent:.1f} s of oracle time; weight generation not timed"}


def run_reference(a):
    """--impl reference: the oracle on the same workload, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg = workload(a)
    import numpy as np
    from threadpoolctl import threadpool_info

    import oracle as O
    from synth import device as SD
    from synth import workloads as W
    hw = SD.HostWeights(cfg)
    if cfg.weight_format:
        hw = O.FP4Weights(hw)   # the oracle's own FP4 quantisation of the master weights
    for e in range(cfg.E):
        hw.routed(e)
    for s in range(cfg.n_shared):
        hw.shared(s)
    chunk = 128
    ids_all = W.host_token_ids(cfg, cfg.T)
    times = []
    for step in range(a.warmup + a.steps):
        r0 = (step * chunk) % cfg.T
        rows = np.arange(r0, min(cfg.T, r0 + chunk))
        x = SD.host_rows(cfg, "x", rows, T=cfg.T)
        r = SD.host_rows(cfg, "residual", rows, T=cfg.T)
        t0 = time.perf_counter()
        O.moe_layer(cfg, hw, x, r, ids_all[rows])
        dt = time.perf_counter() - t0
        if step >= a.warmup:
            times.append((dt, len(rows)))
    secs = sum(t for t, _ in times)
    toks = sum(n for _, n in times)
    value = toks / secs
    cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": a.gpus,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * secs / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded counter-based generator; random weights of the workload's shape)",
        "config": describe(cfg),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: {chunk} tokens of the {cfg.T}-token batch, full layer in fp64"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def epilogue_oracle_sample(budget_s, chunk=256):
    """The oracle's fixed-order reduce + residual + RMSNorm on consecutive
    256-row chunks of the epilogue workload until ``budget_s`` has passed."""
    import numpy as np
    from threadpoolctl import threadpool_info

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
    cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return {"value": round(rows / secs, 1), "unit": UNIT, "cores": cores, "kind": "oracle",
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
        _, hbm_peak, peak_kind = peaks()
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
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    cfg = workload(a)
    T = cfg.T
    stream = torch.cuda.current_stream()

    w = SD.device_weights(cfg, device=dev)
    if cfg.weight_format:
        # FP4 expert weights: the library's quantiser turns the bf16 master
        # weights into their E4M3 codes once, before anything is timed.
        w = moe.quantize_expert_weights(w)
        torch.cuda.synchronize()
    # Each rank takes its own T rows of a world*T-row batch (disjoint tokens).
    xa, ra, ida = SD.device_inputs(cfg, T=T * world, device=dev)
    x, r, ids = (xa[rank * T:(rank + 1) * T].contiguous(), ra[rank * T:(rank + 1) * T].contiguous(),
                 ida[rank * T:(rank + 1) * T].contiguous())
    del xa, ra, ida
    lc = SD.layer_config(cfg, T_max=T)
    layer = moe.MoELayer(lc, w)
    ws = torch.empty(layer.workspace_size(T), dtype=torch.uint8, device=dev)
    on = torch.empty((T, cfg.D), dtype=torch.bfloat16, device=dev)
    orr = torch.empty_like(on)
    cnt = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    use_ids = ids if cfg.router == W.ROUTER_HASH else None

    def step(timed_events=None):
        flush.fill_(1)
        if timed_events:
            timed_events[0].record(stream)
        layer.forward(x, r, on, orr, ws, token_ids=use_ids, out_counts=cnt, stream=stream)
        if timed_events:
            timed_events[1].record(stream)

    for _ in range(a.warmup):
        step()
    torch.cuda.synchronize()
    if layer.device_error(ws) != moe.MOE_OK:
        raise RuntimeError("device wait timed out during warm-up")

    # ------------------------------------------------ timed region (value)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(a.steps)]
    clocks = ClockSampler(local) if rank == 0 else None
    layer.profile_enable([GATEUP_STAGE])
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(a.steps):
        step(evs[i])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if clocks else None
    ms_steps = [e0.elapsed_time(e1) for e0, e1 in evs]
    stage_ms, stage_n = layer.profile_read()
    layer.profile_enable([])
    if layer.device_error(ws) != moe.MOE_OK:
        raise RuntimeError("device wait timed out in the timed region")
    ms_total = torch.tensor([sum(ms_steps)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(ms_total, op=dist.ReduceOp.MAX)
    ms_per_step = float(ms_total.item()) / a.steps
    value = world * T / (ms_per_step / 1e3)
    distinct = int((cnt > 0).sum().item())

    # --------------------------------------------- per-stage breakdown (untimed)
    layer.profile_enable(None)
    for _ in range(3):
        step()
    all_ms, all_n = layer.profile_read()
    layer.profile_enable([])
    stage_avg = {moe.STAGE_NAMES[i]: round(all_ms[i] / all_n[i] * 1e3, 2) if all_n[i] else None
                 for i in range(moe.NUM_STAGES)}

    # ------------------------------------------------------- e2e (host buffers)
    xh, rh = x.cpu().pin_memory(), r.cpu().pin_memory()
    idh = ids.cpu().pin_memory()
    onh = torch.empty(on.shape, dtype=on.dtype).pin_memory()
    orh = torch.empty_like(onh).pin_memory()
    h2d = xh.numel() * 2 + rh.numel() * 2 + (idh.numel() * 4 if use_ids is not None else 0)
    d2h = onh.numel() * 2 + orh.numel() * 2

    def e2e_step(ev=None):
        flush.fill_(1)
        if ev:
            ev[0].record(stream)
        x.copy_(xh, non_blocking=True)
        r.copy_(rh, non_blocking=True)
        if use_ids is not None:
            ids.copy_(idh, non_blocking=True)
        layer.forward(x, r, on, orr, ws, token_ids=use_ids, stream=stream)
        onh.copy_(on, non_blocking=True)
        orh.copy_(orr, non_blocking=True)
        if ev:
            ev[1].record(stream)

    for _ in range(a.warmup):
        e2e_step()
    ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(a.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(a.steps):
        e2e_step(ev2[i])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e2e_ms = torch.tensor([sum(e0.elapsed_time(e1) for e0, e1 in ev2)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(e2e_ms, op=dist.ReduceOp.MAX)
    e2e_value = world * T / (float(e2e_ms.item()) / a.steps / 1e3)

    if rank == 0:
        tc_peak, hbm_peak, peak_kind = peaks()
        peak_src = f"{peak_kind} bf16 (burst)"
        if cfg.weight_format:
            # E4M3 x E4M3: the measured bf16 peak times the nominal dense ratio
            # of the two formats (4.5 / 2.25 PFLOP/s).
            tc_peak, peak_src = 2.0 * tc_peak, f"{peak_kind} bf16 (burst) x 2, nominal E4M3 / bf16 ratio"
        fl = W.moe_flops(cfg)
        gate_ms = stage_ms[GATEUP_STAGE] / max(stage_n[GATEUP_STAGE], 1)
        achieved = fl["gateup"] / (gate_ms / 1e3) / 1e12
        traffic = ncu_traffic(cfg)
        roof = {"bound": "tensor", "kernel": "gemm_gateup_swiglu", "achieved": round(achieved, 1),
                "peak": tc_peak, "unit": "TFLOP/s", "frac": round(achieved / tc_peak, 4),
                "traffic": traffic, "peak_source": peak_src,
                "flops_per_launch": fl["gateup"], "avg_launch_ms": round(gate_ms, 4)}
        layer_tflops = fl["total"] / (ms_per_step / 1e3) / 1e12
        cpu = None
        if world == 1 and not a.no_cpu_baseline:
            cpu = oracle_sample(cfg)
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3" if cfg.weight_format else "bf16",
            "data": "synthetic (seeded counter-based generator; random weights of the workload's shape)",
            "config": {**describe(cfg), "l2": "flushed before every step (512 MiB write, untimed)",
                       "parallelism": f"replicas x{world} (token-sharded, no collective)"},
            "roofline": roof,
            "layer": {"tflops": round(layer_tflops, 1), "frac_of_tc_peak": round(layer_tflops / tc_peak, 4),
                      "flops_per_step": fl["total"], "distinct_experts": distinct,
                      "algorithmic_bytes": W.layer_bytes(cfg, T, distinct),
                      "hbm_gbs": round(W.layer_bytes(cfg, T, distinct) / (ms_per_step / 1e3) / 1e9, 1),
                      "frac_of_hbm": round(W.layer_bytes(cfg, T, distinct) / (ms_per_step / 1e3) / 1e9
                                           / hbm_peak, 4)},
            "stage_us": stage_avg,
            "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": a.steps * layer.launch_count(T),
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    layer.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
