"""Host-side pieces of expert parallelism (no GPU): the expert blocks of each
rank and the weight shards, and, on two gloo ranks, that the blocks of all
ranks tile the experts exactly once."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import deterministic_expert_b200 as moe


def test_expert_ranges_tile_the_experts():
    for E, world in ((8, 2), (64, 4), (256, 8), (128, 1)):
        seen = []
        for r in range(world):
            e0, e1 = moe.expert_range(E, world, r)
            assert e1 - e0 == E // world
            seen.extend(range(e0, e1))
        assert seen == list(range(E))
    with pytest.raises(ValueError):
        moe.expert_range(10, 4, 0)


def test_shard_expert_weights_views():
    E, I, D = 8, 4, 6
    w = {n: torch.arange(E * I * D, dtype=torch.float32).reshape(E, I, D) for n in ("w_gate", "w_up")}
    w["w_down"] = torch.arange(E * D * I, dtype=torch.float32).reshape(E, D, I)
    w["w_router"] = torch.ones(E, D)
    s = moe.shard_expert_weights(w, 4, 3)
    assert torch.equal(s["w_gate"], w["w_gate"][6:8]) and s["w_gate"].is_contiguous()
    assert torch.equal(s["w_down"], w["w_down"][6:8])
    assert s["w_router"] is w["w_router"]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    e0, e1 = moe.expert_range(64, world, rank)
    owned = torch.zeros(64, dtype=torch.int64)
    owned[e0:e1] = 1
    dist.all_reduce(owned)
    q.put(owned.tolist())
    dist.destroy_process_group()


def test_expert_blocks_over_gloo_ranks():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(60)
        assert p.exitcode == 0
    for _ in range(2):
        assert q.get(timeout=5) == [1] * 64
