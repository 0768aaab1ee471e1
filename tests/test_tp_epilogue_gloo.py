"""The tensor-parallel epilogue across ranks, on CPU (gloo, world_size 2).

TPAllReduceNorm gives partial p to rank p // per_rank (partial_order) and rank
r the rows row_slices(T, world)[r]; every rank reduces its rows over all P
partials in the order p = 0 .. P-1, adds the residual and normalises, and the
rows land on every rank.  Here two gloo ranks hold 4 partials each, gather
them in partial_order, reduce their row slice with the oracle's fixed-order
epilogue, and gather the slices: every rank must hold, bit for bit, what one
process gets over all 8 partials and all rows.  (The CUDA kernel the class
launches is the single-GPU one with a row range and several destinations;
its own bits are checked against the oracle by the GPU tests.)
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from deterministic_expert_b200 import partial_order, row_slices
from synth import workloads as W

T, D, PER_RANK, WORLD = 37, 128, 4, 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _partial(p):
    return O.bf16_bits_to_f64(W.host_partial(p, T, D)).reshape(T, D)


def _residual():
    return O.bf16_bits_to_f64(W.normal_bf16(W.k_("residual"), 0, T * D, 1.0)).reshape(T, D)


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    order = partial_order(world, PER_RANK)
    mine = torch.from_numpy(np.stack([_partial(p) for p, (r, _) in enumerate(order) if r == rank]))
    gathered = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(gathered, mine)
    parts = np.stack([gathered[r][j].numpy() for r, j in order])     # p = 0 .. P-1
    row0, rows = row_slices(T, world)[rank]
    g = np.ones(D)
    on, orr, _ = O.reduce_partials(parts[:, row0:row0 + rows], _residual()[row0:row0 + rows], g, 1e-6)
    out = np.zeros((2, T, D))
    out[0, row0:row0 + rows], out[1, row0:row0 + rows] = on, orr
    t = torch.from_numpy(out)
    dist.all_reduce(t)   # each row is non-zero on exactly one rank
    np.save(os.path.join(out_dir, f"rank{rank}.npy"), t.numpy())
    dist.barrier()
    dist.destroy_process_group()


def test_tp_epilogue_ranks_match_single_process(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(WORLD, port, str(tmp_path)), nprocs=WORLD, start_method="spawn")
    P = WORLD * PER_RANK
    parts = np.stack([_partial(p) for p in range(P)])
    on, orr, _ = O.reduce_partials(parts, _residual(), np.ones(D), 1e-6)
    for r in range(WORLD):
        got = np.load(os.path.join(tmp_path, f"rank{r}.npy"))
        assert np.array_equal(got[0], on) and np.array_equal(got[1], orr)


def test_partial_order_and_row_slices():
    assert partial_order(4, 2) == [(0, 0), (0, 1), (1, 0), (1, 1), (2, 0), (2, 1), (3, 0), (3, 1)]
    for T_, w in [(37, 2), (8, 8), (5, 8), (16384, 8), (1, 1)]:
        s = row_slices(T_, w)
        assert len(s) == w and s[0][0] == 0
        assert all(a[0] + a[1] == b[0] for a, b in zip(s, s[1:]))
        assert s[-1][0] + s[-1][1] == T_ and max(n for _, n in s) - min(n for _, n in s) <= 1
