"""The multi-GPU path on CPU: token-sharded replicas with world_size 2 (gloo).

`bench.py --gpus N` gives rank r the rows [r*T, (r+1)*T) of an N*T-row batch,
runs the layer with no data exchange, and reduces only the step time (max over
ranks).  Here two gloo ranks run the oracle on their shards; the gathered
outputs must equal the single-process run on all rows bit for bit (every row
depends only on itself and the weights), and the timing reduction must take
the slowest rank.
"""
import dataclasses
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from synth import device as SD
from synth import workloads as W

CFG = dataclasses.replace(W.C1, T=48)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _shard(rank, world, T):
    return np.arange(rank * T, (rank + 1) * T)


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    T = CFG.T // world
    rows = _shard(rank, world, T)
    hw = SD.HostWeights(CFG)
    x = SD.host_rows(CFG, "x", rows, T=CFG.T)
    r = SD.host_rows(CFG, "residual", rows, T=CFG.T)
    res = O.moe_layer(CFG, hw, x, r)
    mine = torch.from_numpy(np.concatenate([res["out_norm"], res["out_residual"]], axis=1))
    gathered = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(gathered, mine)
    t = torch.tensor([10.0 + rank], dtype=torch.float64)  # a fake per-rank step time
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    if rank == 0:
        np.save(os.path.join(out_dir, "gathered.npy"), torch.cat(gathered).numpy())
        np.save(os.path.join(out_dir, "tmax.npy"), t.numpy())
    dist.barrier()
    dist.destroy_process_group()


def test_token_sharded_replicas_match_single_process(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    got = np.load(tmp_path / "gathered.npy")
    hw = SD.HostWeights(CFG)
    full = O.moe_layer(CFG, hw, SD.host_rows(CFG, "x", range(CFG.T)),
                       SD.host_rows(CFG, "residual", range(CFG.T)))
    want = np.concatenate([full["out_norm"], full["out_residual"]], axis=1)
    assert np.array_equal(got, want)
    assert float(np.load(tmp_path / "tmax.npy")[0]) == 11.0


def test_shards_are_disjoint_and_cover_the_batch():
    for world in (1, 2, 4, 8):
        T = 4096
        allrows = np.concatenate([_shard(r, world, T) for r in range(world)])
        assert np.array_equal(allrows, np.arange(world * T))
