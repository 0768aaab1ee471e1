"""Expert parallelism on one device: ``world`` virtual ranks (each with its own
block of routed experts, workspace and exchange buffer) run the four phases
in stream order, and every rank's outputs must equal, bit for bit, the
single-device layer's rows for the same tokens (the DeepSeek V4 infra notes,
§6.1 dispatch / compute / combine; the Fireworks parity post, Trap 3: the slot
sum happens in fp32 on the token's own rank, so moving rows between ranks
changes no bit).  The per-rank batches are ragged, including a rank with a
single token."""
import dataclasses

import numpy as np
import pytest

from synth import device as SD
from synth import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


CASES = {
    "tiny_w2": (W.C1, 2, [37, 100]),
    "tiny_w4": (W.C1, 4, [1, 64, 129, 30]),
    "tiny_w8": (W.C1, 8, [5, 17, 33, 1, 64, 2, 90, 11]),
    "tiny_w4_empty_rank": (W.C1, 4, [40, 0, 70, 25]),
    "tiny_fp8_w4": (W.C1F, 4, [50, 7, 200, 64]),
    "hash_w2": (dataclasses.replace(W.C1, router=W.ROUTER_HASH, k=3, name="hash_small"), 2, [77, 120]),
    "situ_w2": (dataclasses.replace(W.C1, activation=1, name="tiny_situ"), 2, [90, 40]),
    "fine_grained_w4": (W.C2, 4, [512, 300, 1, 1024]),
    "fine_grained_fp8_w2": (W.C2F, 2, [700, 333]),
    "tiny_fp4_w4": (W.C1P, 4, [50, 7, 200, 64]),
}


# Wave scheduling (§6.1 "MegaMoE": experts in waves, the next wave's rows in
# flight while the current wave computes): the same batches split into n
# waves, sends and GEMMs on two streams, must still give the single-device bits.
WAVE_CASES = {
    "tiny_w2_waves2": (W.C1, 2, [37, 100], 2),
    "tiny_w2_one_expert_per_wave": (W.C1, 2, [129, 64], 4),
    "tiny_w4_empty_rank_waves2": (W.C1, 4, [40, 0, 70, 25], 2),
    "tiny_fp8_w2_uneven_waves": (W.C1F, 2, [50, 200], 3),
    "tiny_fp4_w2_waves2": (W.C1P, 2, [50, 200], 2),
    "hash_w2_waves2": (dataclasses.replace(W.C1, router=W.ROUTER_HASH, k=3, name="hash_small"), 2, [77, 120], 2),
    "fine_grained_w4_waves4": (W.C2, 4, [512, 300, 1, 1024], 4),
    "fine_grained_w8_waves8": (W.C2, 8, [256, 100, 1, 512, 64, 300, 7, 128], 8),
    "fine_grained_fp8_w2_waves2": (W.C2F, 2, [700, 333], 2),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_virtual_ep_matches_single_device(torch_cuda, case):
    base, world, Ts = CASES[case]
    _check_against_single_device(torch_cuda, base, world, Ts, waves=1)


@pytest.mark.parametrize("case", sorted(WAVE_CASES))
def test_virtual_ep_waves_match_single_device(torch_cuda, case):
    base, world, Ts, waves = WAVE_CASES[case]
    _check_against_single_device(torch_cuda, base, world, Ts, waves=waves)


def test_virtual_ep_rejects_bad_wave_counts(torch_cuda):
    import deterministic_expert_b200 as moe
    cfg = W.C1.with_T(64)
    ep = moe.VirtualEP(SD.layer_config(cfg, 32), SD.device_weights(cfg), 2)
    x, r, _ = SD.device_inputs(cfg, T=64)
    for waves in (0, cfg.E // 2 + 1):
        with pytest.raises(ValueError):
            ep.forward([x[:32].contiguous(), x[32:].contiguous()], [r[:32].contiguous(), r[32:].contiguous()],
                       waves=waves)
    # The C ABI refuses a wave outside [0, n) and n outside [1, E / world].
    rk = ep.ranks[0]
    for wave, n in ((1, 1), (-1, 2), (0, cfg.E // 2 + 1), (0, 0)):
        with pytest.raises(moe.MoEError):
            rk.send(32, ep.peers, wave=wave, n_waves=n)
        with pytest.raises(moe.MoEError):
            rk.experts(32, ep.peers, wave=wave, n_waves=n)


def _check_against_single_device(torch, base, world, Ts, waves):
    import deterministic_expert_b200 as moe
    T = sum(Ts)
    cfg = base.with_T(T)
    weights = SD.device_weights(cfg)
    if cfg.weight_format == 1:
        weights = moe.quantize_expert_weights(weights)
    elif cfg.weight_format == 2:
        weights = moe.pack_expert_weights_fp4(weights)
    x, r, ids = SD.device_inputs(cfg, T=T)
    # The single-device layer over all T tokens.
    single = moe.MoELayer(SD.layer_config(cfg, T), weights)
    ws = torch.empty(single.workspace_size(T), dtype=torch.uint8, device="cuda")
    on = torch.empty((T, cfg.D), dtype=torch.bfloat16, device="cuda")
    orr = torch.empty_like(on)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    tw = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
    single.forward(x, r, on, orr, ws, token_ids=ids, out_topk_idx=idx, out_topk_w=tw)
    # The same tokens over `world` ranks, rank q holding the next Ts[q] of them.
    ep = moe.VirtualEP(SD.layer_config(cfg, max(Ts)), weights, world)
    cut = np.concatenate([[0], np.cumsum(Ts)])
    sl = [slice(int(cut[q]), int(cut[q + 1])) for q in range(world)]
    outs = ep.forward([x[s].contiguous() for s in sl], [r[s].contiguous() for s in sl],
                      [ids[s].contiguous() for s in sl], waves=waves)
    torch.cuda.synchronize()
    assert ep.device_errors() == [0] * world
    assert single.device_error(ws) == 0
    for q, s in enumerate(sl):
        e_on, e_orr, e_idx, e_w = outs[q]
        assert torch.equal(e_idx, idx[s]), q
        assert torch.equal(e_w.view(torch.int32), tw[s].view(torch.int32)), q
        assert torch.equal(e_on.view(torch.int16), on[s].view(torch.int16)), q
        assert torch.equal(e_orr.view(torch.int16), orr[s].view(torch.int16)), q


def test_virtual_ep_repeat_steps(torch_cuda):
    """Three steps through the same exchange buffers with different batches
    give each step's single-device bits (buffers are fully rewritten)."""
    torch = torch_cuda
    import deterministic_expert_b200 as moe
    cfg = W.C1.with_T(400)
    weights = SD.device_weights(cfg)
    x, r, ids = SD.device_inputs(cfg, T=400)
    single = moe.MoELayer(SD.layer_config(cfg, 400), weights)
    ep = moe.VirtualEP(SD.layer_config(cfg, 200), weights, 2)
    for a0, a1, b1 in ((0, 100, 300), (50, 250, 400), (10, 11, 12)):
        T = b1 - a0
        ws = torch.empty(single.workspace_size(T), dtype=torch.uint8, device="cuda")
        on = torch.empty((T, cfg.D), dtype=torch.bfloat16, device="cuda")
        orr = torch.empty_like(on)
        single.forward(x[a0:b1].contiguous(), r[a0:b1].contiguous(), on, orr, ws)
        outs = ep.forward([x[a0:a1].contiguous(), x[a1:b1].contiguous()],
                          [r[a0:a1].contiguous(), r[a1:b1].contiguous()])
        torch.cuda.synchronize()
        got = torch.cat([outs[0][0], outs[1][0]])
        assert torch.equal(got.view(torch.int16), on.view(torch.int16)), (a0, a1, b1)
