"""The no-allocation forward (moe_layer_forward_noalloc) against the regular one.

Some callers cannot allocate device memory (a plugin enqueue path that must
not allocate, a process whose allocator already holds the free memory, a
latency-critical path that cannot take cudaMalloc's synchronisation); for
them the library keeps its scratch in a static 32 MiB device array.  Two calls
in a row, with different batches, must match the workspace entry point within
the layer's output tolerance (they run the same kernels, so the bits agree),
and a batch too large for the static array must be refused with
MOE_EWORKSPACE.  This file is collected last; it also passes on its own.
"""
import numpy as np
import pytest

from gpu_util import TOL_MAX, TOL_MEAN, Run, np64, rel_err
from synth import workloads as W

pytestmark = pytest.mark.gpu


def test_noalloc_forward_matches_workspace_forward():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import deterministic_expert_b200 as moe

    cfg = W.C2.with_T(512)
    run = Run(cfg, T_max=512)
    xa, ra, ida = run.inputs(512)
    for rows in (np.arange(64), np.arange(100, 137)):   # two calls in a row, different batches
        ri = torch.from_numpy(rows).cuda()
        x, r, ids = xa[ri].contiguous(), ra[ri].contiguous(), ida[ri].contiguous()
        want = run.forward(x, r, ids)                   # the workspace entry point
        T = len(rows)
        on = torch.full((T, cfg.D), float("nan"), dtype=torch.bfloat16, device="cuda")
        orr = torch.full_like(on, float("nan"))
        idx = torch.full((T, cfg.k), -1, dtype=torch.int32, device="cuda")
        moe.forward_noalloc(run.layer, x, r, on, orr, out_topk_idx=idx)
        torch.cuda.synchronize()
        assert run.layer.device_error(None) == moe.MOE_OK   # the static scratch's error word
        assert torch.equal(idx, want["idx"])
        for got, ref in ((on, want["out_norm"]), (orr, want["out_residual"])):
            assert torch.equal(got.view(torch.int16), ref.view(torch.int16))

    # A batch whose workspace exceeds the static array is refused.
    x, r = xa.contiguous(), ra.contiguous()
    on = torch.empty((512, cfg.D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoEError) as err:
        moe.forward_noalloc(run.layer, x, r, on, torch.empty_like(on))
    assert err.value.status == moe.MOE_EWORKSPACE
    assert run.layer.workspace_size(512) > (32 << 20)
