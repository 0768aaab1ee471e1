"""The bounds-checked build (libmoe_checked.so, MOE_CHECK_BOUNDS): every index a
kernel computes from device data is tested against its buffer before use.

Each test runs in a child process started with MOE_LIBRARY=checked (the
binding then loads the checked library), so the parent's regular library is
untouched.  Clean runs (bf16, E4M3 and FP4 layers; an expert-parallel step in
one pass and in waves) must report no index error and give the bits of the
regular build's contract (oracle parity, EP == single device); a corrupted
per-expert count handed between expert-parallel phases must be reported as
MOE_EINDEX with every out-of-range row skipped (the send kernel writes only
rows inside the receive buffers)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CLEAN = r"""
import dataclasses, numpy as np, torch
import deterministic_expert_b200 as moe
assert moe.LIB_PATH.endswith("libmoe_checked.so"), moe.LIB_PATH
import sys; sys.path.insert(0, "tests")
from gpu_util import Run, verify
from synth import device as SD, workloads as W
for cfg in (W.C1, W.C1F, dataclasses.replace(W.C1, T=129, n_shared=0), W.C1P, dataclasses.replace(W.C1P, T=300)):
    run = Run(cfg)
    out = run.forward(*run.inputs())          # asserts device_error == 0
    verify(run, out)
cfg = W.C1.with_T(300)
w = SD.device_weights(cfg)
x, r, ids = SD.device_inputs(cfg, T=300)
ep = moe.VirtualEP(SD.layer_config(cfg, 100), w, 4)
Ts = [100, 0, 77, 100]
cut = np.concatenate([[0], np.cumsum(Ts)])
outs = ep.forward([x[cut[q]:cut[q + 1]] for q in range(4)], [r[cut[q]:cut[q + 1]] for q in range(4)])
torch.cuda.synchronize()
assert ep.device_errors() == [0, 0, 0, 0], ep.device_errors()
single = moe.MoELayer(SD.layer_config(cfg, 277), w)
ws = torch.empty(single.workspace_size(277), dtype=torch.uint8, device="cuda")
on = torch.empty((277, cfg.D), dtype=torch.bfloat16, device="cuda"); orr = torch.empty_like(on)
single.forward(x[:277].contiguous(), r[:277].contiguous(), on, orr, ws)
torch.cuda.synchronize()
got = torch.cat([o[0] for o in outs])
assert torch.equal(got.view(torch.int16), on.view(torch.int16))
# The same step in two waves of experts (wave-limited send and expert phases).
outs = ep.forward([x[cut[q]:cut[q + 1]] for q in range(4)], [r[cut[q]:cut[q + 1]] for q in range(4)], waves=2)
torch.cuda.synchronize()
assert ep.device_errors() == [0, 0, 0, 0], ep.device_errors()
got = torch.cat([o[0] for o in outs])
assert torch.equal(got.view(torch.int16), on.view(torch.int16))
print("CLEAN-OK")
"""

BAD_COUNTS = r"""
import numpy as np, torch
import deterministic_expert_b200 as moe
assert moe.LIB_PATH.endswith("libmoe_checked.so"), moe.LIB_PATH
from synth import device as SD, workloads as W
cfg = W.C1.with_T(200)
w = SD.device_weights(cfg)
x, r, ids = SD.device_inputs(cfg, T=200)
ep = moe.VirtualEP(SD.layer_config(cfg, 50), w, 4)
xs = [x[50 * q:50 * (q + 1)].contiguous() for q in range(4)]
for q, rk in enumerate(ep.ranks):
    rk.route(xs[q], None, moe._ptr(ep.xbuf[q]))
torch.cuda.synchronize()
# Rank 1 publishes impossible counts (its board is the first E int32 of its
# exchange buffer): 200 rows for every expert, where a rank has 100 (token,
# slot) rows in all.  The destination rows computed from them run past each
# owner's 400-row receive buffer, to row 487 at most on this routing (about
# 380 expected from the other ranks' counts); every row stays inside the
# owner's own exchange allocation (receive rows, their return addresses, then
# the 100 KB of slot rows), so a send path whose check went missing would
# overwrite memory this process owns instead of faulting the GPU.
exch = ep.xbuf[1].numel()
rows_in_alloc = exch // (cfg.D * 2)
assert rows_in_alloc > 487 + 8, rows_in_alloc
ep.xbuf[1][:4 * cfg.E].view(torch.int32).fill_(200)
for q, rk in enumerate(ep.ranks):
    rk.send(50, ep.peers)
torch.cuda.synchronize()                      # no CUDA error: the bad rows were skipped
errs = ep.device_errors()
assert moe.MOE_EINDEX in errs, errs
assert all(e in (0, moe.MOE_EINDEX) for e in errs), errs
print("BAD-COUNTS-CAUGHT", errs)
"""


def _child(code):
    env = dict(os.environ, MOE_LIBRARY="checked", PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
    return subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=600)


def test_checked_build_clean_runs():
    p = _child(CLEAN)
    assert p.returncode == 0 and "CLEAN-OK" in p.stdout, p.stdout[-2000:] + p.stderr[-4000:]


def test_checked_build_reports_bad_expert_counts():
    p = _child(BAD_COUNTS)
    assert p.returncode == 0 and "BAD-COUNTS-CAUGHT" in p.stdout, p.stdout[-2000:] + p.stderr[-4000:]
