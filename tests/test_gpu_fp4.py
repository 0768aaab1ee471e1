"""FP4 expert weights in their storage form (DeepSeek V4 infra notes, §6.2 FP4
QAT: FP4 (E2M1) weights with one scale per block, dequantised losslessly to
FP8, FP8 x FP8 GEMMs).  The weights live in HBM as packed E2M1 codes (half a
byte each) with their block exponents; the expert GEMMs hand the codes to the
tensor core's block-scaled E2M1 x E4M3 MMA with the exponents as UE8M0 block
scales.  Every code times its scale is an E4M3 value, so the products are
those of the E4M3 weights.

* The packed quantiser writes, code for code and exponent for exponent, the
  oracle's FP4 storage form (pack_fp4 of quantize_weights_fp4).
* A layer with packed weights gives, bit for bit, the outputs of the same layer
  with the E4M3 weights of the same master weights (whose GEMMs use every shape
  of tile: 256-row, 128-row and operand-swapped; SwiGLU and SiTU-GLU; a latent
  width; hash routing; no shared expert).
* It matches the oracle within the layer tolerances, and its decode batches
  reproduce their rows of the 8192-row batch bit for bit.
"""
import dataclasses

import numpy as np
import pytest

import oracle as O
from gpu_util import Run, verify
from synth import workloads as W
from test_gpu_fp8 import _edge_weights

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _oracle_storage(master):
    """The oracle's storage form of master weights [rows, K]: packed codes and
    the exponent words laid out [K / 128, rows] (four int8 a word, block 4c in
    the lowest byte)."""
    q, s = O.quantize_weights_fp4(master)
    packed, s8 = O.pack_fp4(q, s)
    rows, nb = s8.shape
    words = s8.astype(np.uint8).reshape(rows, nb // 4, 4).astype(np.uint32)
    words = words[..., 0] | (words[..., 1] << 8) | (words[..., 2] << 16) | (words[..., 3] << 24)
    return packed, words.T.astype(np.uint32)


def test_packed_quantiser_bit_exact(torch_cuda):
    torch = torch_cuda
    import deterministic_expert_b200 as moe
    wh = _edge_weights(torch)
    rnd = (torch.randn((96, 384), generator=torch.Generator().manual_seed(5)) * 0.02).to(torch.bfloat16)
    for m in (wh, rnd):
        w = m.cuda()
        K = w.shape[1]
        p = torch.full((w.shape[0], K // 2), 0xAB, dtype=torch.uint8, device="cuda")
        x = torch.full((K // 128, w.shape[0]), -1, dtype=torch.int32, device="cuda")
        moe.quantize_weights_fp4_packed(w, p, x)
        torch.cuda.synchronize()
        want_p, want_x = _oracle_storage(m.to(torch.float64).numpy())
        assert np.array_equal(p.cpu().numpy(), want_p)
        assert np.array_equal(x.cpu().numpy().view(np.uint32), want_x)
        # The storage form decodes to the E4M3 values the E4M3 quantiser writes.
        q8 = torch.empty(w.shape, dtype=torch.uint8, device="cuda")
        moe.quantize_weights_fp4(w, q8)
        torch.cuda.synchronize()
        s = want_x.T.view(np.uint8).reshape(w.shape[0], -1).view(np.int8)
        assert np.array_equal(O.e4m3_bits(O.unpack_fp4(want_p, s)), q8.cpu().numpy())


VARIANTS = {
    "tiny": dataclasses.replace(W.C1P, T=300),
    "tiny_T1": dataclasses.replace(W.C1P, T=1),
    "fine_grained_512": W.C2P.with_T(512),
    "fine_grained_4096": W.C2P,
    "latent_situ_512": W.C6P.with_T(512),
    "situ": dataclasses.replace(W.C1P, T=300, activation=1, name="tiny_fp4_situ"),
    "hash": dataclasses.replace(W.C1P, T=300, router=W.ROUTER_HASH, k=3, name="tiny_fp4_hash"),
    "no_shared": dataclasses.replace(W.C1P, T=300, n_shared=0, name="tiny_fp4_noshared"),
}


@pytest.mark.parametrize("name", sorted(VARIANTS))
def test_packed_layer_bit_equal_to_e4m3_layer(torch_cuda, name):
    torch = torch_cuda
    cfg = VARIANTS[name]
    packed = Run(cfg)
    e4m3 = Run(dataclasses.replace(cfg, weight_format=1))
    x, r, ids = packed.inputs()
    a = packed.forward(x, r, ids)
    b = e4m3.forward(x, r, ids)
    for key in ("idx", "w", "counts"):
        assert torch.equal(a[key], b[key]), key
    for key in ("out_norm", "out_residual"):
        assert torch.equal(a[key].view(torch.int16), b[key].view(torch.int16)), key


@pytest.mark.parametrize("name", ["tiny", "fine_grained_512"])
def test_packed_layer_oracle_parity(torch_cuda, name):
    run = Run(VARIANTS[name])
    verify(run, run.forward(*run.inputs()))


def test_packed_decode_sweep_matches_full_batch(torch_cuda):
    torch = torch_cuda
    cfg = W.C2P.with_T(W.C4_SOURCE_T)
    run = Run(cfg, T_max=W.C4_SOURCE_T)
    x, r, ids = run.inputs()
    full = run.forward(x, r, ids)
    for T in W.C4_T:
        ri = torch.from_numpy(W.decode_subset(T)).cuda()
        out = run.forward(x[ri].contiguous(), r[ri].contiguous(), ids[ri].contiguous())
        for key in ("out_norm", "out_residual"):
            assert torch.equal(out[key].view(torch.int16), full[key][ri].view(torch.int16)), (T, key)


def test_packed_splits_permutation_repeats(torch_cuda):
    torch = torch_cuda
    cfg = W.C2P
    run = Run(cfg)
    x, r, ids = run.inputs()
    perm = torch.from_numpy(W.token_permutation(cfg.T).astype(np.int32)).cuda()
    ws = torch.empty(run.layer.invariance_workspace_size(cfg.T), dtype=torch.uint8, device="cuda")
    assert run.layer.check_invariance(x, r, ws, token_ids=ids, n_splits=5, perm=perm, repeats=2) == 0
