"""Bitwise batch invariance on the GPU (the GPU against itself; no oracle).

The Meituan parity article ("逐 token logprob 一致") asks for bit-pattern
comparison, one configuration axis at a time: here the batch is split into
chunks, permuted, and re-run, and every output bit must match the full-batch
run.  The decode sweep checks that a token's output is the same bits whether
it runs alone, in a batch of 8 .. 512, or inside the 8192-row batch.
"""
import dataclasses

import numpy as np
import pytest

from gpu_util import Run
from synth import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


@pytest.mark.parametrize("name,splits", [("tiny", 7), ("fine_grained", 4), ("skew_hash", 3),
                                         ("fine_grained_situ", 5), ("latent_situ", 4),
                                         ("tiny_fp8", 6), ("fine_grained_fp8", 4), ("latent_situ_fp8", 3)])
def test_splits_permutation_repeats(torch_cuda, name, splits):
    torch = torch_cuda
    cfg = W.CONFIGS[name]
    if name == "skew_hash":
        cfg = dataclasses.replace(cfg, T=4096)
    run = Run(cfg)
    x, r, ids = run.inputs()
    perm = torch.from_numpy(W.token_permutation(cfg.T).astype(np.int32)).cuda()
    ws = torch.empty(run.layer.invariance_workspace_size(cfg.T), dtype=torch.uint8, device="cuda")
    mism = run.layer.check_invariance(x, r, ws, token_ids=ids, n_splits=splits, perm=perm, repeats=2)
    assert mism == 0


def test_decode_sweep_matches_full_batch(torch_cuda):
    """Each decode batch (first T rows, and a random subset of T rows, of the
    8192-row input) must reproduce those rows of the 8192-row run bit for bit."""
    torch = torch_cuda
    cfg = W.C2.with_T(W.C4_SOURCE_T)
    run = Run(cfg, T_max=W.C4_SOURCE_T)
    x, r, ids = run.inputs()
    full = run.forward(x, r, ids)
    for T in W.C4_T:
        for rows in (np.arange(T), W.decode_subset(T)):
            ri = torch.from_numpy(rows).cuda()
            out = run.forward(x[ri].contiguous(), r[ri].contiguous(), ids[ri].contiguous())
            for key in ("out_norm", "out_residual", "idx", "w"):
                a = out[key].view(torch.int16) if out[key].dtype == torch.bfloat16 else out[key]
                b = full[key][ri]
                b = b.view(torch.int16) if b.dtype == torch.bfloat16 else b
                assert torch.equal(a, b), (T, key)


def test_repeat_runs_same_bits_v3_shape_small(torch_cuda):
    torch = torch_cuda
    cfg = dataclasses.replace(W.C3, T=512)
    run = Run(cfg)
    x, r, ids = run.inputs()
    ws = torch.empty(run.layer.invariance_workspace_size(cfg.T), dtype=torch.uint8, device="cuda")
    perm = torch.from_numpy(W.token_permutation(cfg.T, salt=3).astype(np.int32)).cuda()
    assert run.layer.check_invariance(x, r, ws, token_ids=ids, n_splits=5, perm=perm, repeats=1) == 0


def test_fp8_decode_sweep_matches_full_batch(torch_cuda):
    """FP4 expert weights: every decode batch reproduces its rows of the
    8192-row run bit for bit (the per-row E4M3 scales are row-local)."""
    torch = torch_cuda
    cfg = W.C2F.with_T(W.C4_SOURCE_T)
    run = Run(cfg, T_max=W.C4_SOURCE_T)
    x, r, ids = run.inputs()
    full = run.forward(x, r, ids)
    for T in W.C4_T:
        rows = W.decode_subset(T)
        ri = torch.from_numpy(rows).cuda()
        out = run.forward(x[ri].contiguous(), r[ri].contiguous(), ids[ri].contiguous())
        for key in ("out_norm", "out_residual"):
            assert torch.equal(out[key].view(torch.int16), full[key][ri].view(torch.int16)), (T, key)


@pytest.mark.parametrize("name,chunks", [("fine_grained", 1), ("fine_grained", 3), ("skew_hash", 2)])
def test_host_pipeline_matches_single_calls(torch_cuda, name, chunks):
    """End-to-end forwards through HostPipeline (pinned host batches copied in,
    outputs copied out, neighbouring steps overlapped on three streams, each
    batch optionally split into row blocks) give the bits of one device
    forward per batch."""
    import deterministic_expert_b200 as moe
    torch = torch_cuda
    cfg = W.CONFIGS[name]
    T = 1024
    run = Run(cfg.with_T(T), T_max=T)
    xa, ra, ida = run.inputs(3 * T)
    batches = [(xa[i * T:(i + 1) * T].contiguous(), ra[i * T:(i + 1) * T].contiguous(),
                ida[i * T:(i + 1) * T].contiguous()) for i in range(3)]
    want = [run.forward(*b) for b in batches]
    pipe = moe.HostPipeline(run.layer, T, chunks=chunks)
    hx = [b[0].cpu().pin_memory() for b in batches]
    hr = [b[1].cpu().pin_memory() for b in batches]
    hid = [b[2].cpu().pin_memory() for b in batches]
    hon = [torch.full((T, cfg.D), float("nan"), dtype=torch.bfloat16).pin_memory() for _ in range(3)]
    hor = [torch.full((T, cfg.D), float("nan"), dtype=torch.bfloat16).pin_memory() for _ in range(3)]
    # Five steps over the three batches: buffer sets are reused across steps.
    order = [0, 1, 2, 1, 0]
    outs_n = [hon[i] for i in order]
    outs_r = [hor[i] for i in order]
    pipe.run([hx[i] for i in order], [hr[i] for i in order], outs_n, outs_r,
             token_ids=[hid[i] for i in order] if cfg.router == W.ROUTER_HASH else None)
    torch.cuda.synchronize()
    assert run.layer.device_error(pipe.ws) == 0
    for i in range(3):
        assert torch.equal(hon[i].view(torch.int16), want[i]["out_norm"].cpu().view(torch.int16)), i
        assert torch.equal(hor[i].view(torch.int16), want[i]["out_residual"].cpu().view(torch.int16)), i


def test_v3_full_batch_with_wide_tiles_matches_splits(torch_cuda):
    """The V3-shaped batch (T=8192: about 256 rows per expert, so the GEMMs run
    wide tiles for experts with 257-320 rows) against four 2048-token splits
    (64 rows per expert: no wide tiles) and a permuted order: the same bits."""
    torch = torch_cuda
    cfg = W.C3
    run = Run(cfg)
    x, r, ids = run.inputs()
    perm = torch.from_numpy(W.token_permutation(cfg.T, salt=7).astype(np.int32)).cuda()
    ws = torch.empty(run.layer.invariance_workspace_size(cfg.T), dtype=torch.uint8, device="cuda")
    assert run.layer.check_invariance(x, r, ws, token_ids=ids, n_splits=4, perm=perm, repeats=1) == 0
