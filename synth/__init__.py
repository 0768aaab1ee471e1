"""Seeded synthetic inputs shared by the tests, the oracle harness and the benchmark.

This package draws random numbers and nothing else: it holds none of the MoE
layer's arithmetic.  Two twins implement one counter-based generator from its
published definition (SplitMix64 output function + Irwin-Hall n=12 normal; see
``gen_host.c``): a host library used to regenerate any slice of a tensor for
the oracle, and a device library (``gen_device.cu``) that fills large tensors
in place on the GPU.  They agree bit for bit, which a GPU test checks.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
HOST_SO = os.path.join(_HERE, "libsynth_host.so")
DEVICE_SO = os.path.join(_HERE, "libsynth_dev.so")

_host = None
_dev = None


def build_host(force: bool = False) -> str:
    """Compile the host twin with gcc (OpenMP, no FMA contraction)."""
    src = os.path.join(_HERE, "gen_host.c")
    if force or not os.path.exists(HOST_SO) or os.path.getmtime(HOST_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                               "-o", HOST_SO, src])
    return HOST_SO


def build_device(force: bool = False) -> str:
    """Compile the device twin for sm_100a with nvcc."""
    src = os.path.join(_HERE, "gen_device.cu")
    if force or not os.path.exists(DEVICE_SO) or os.path.getmtime(DEVICE_SO) < os.path.getmtime(src):
        subprocess.check_call(["nvcc", "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
                               "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
                               "-o", DEVICE_SO, src])
    return DEVICE_SO


def _h():
    global _host
    if _host is None:
        lib = ctypes.CDLL(build_host())
        u64, f32, vp = ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p
        lib.syn_key.restype = u64
        lib.syn_key.argtypes = [u64, u64]
        lib.syn_draw.restype = u64
        lib.syn_draw.argtypes = [u64, u64]
        lib.syn_normal_bf16.argtypes = [u64, u64, u64, f32, vp]
        lib.syn_normal_f32.argtypes = [u64, u64, u64, f32, vp]
        lib.syn_normal_bf16_as_f64.argtypes = [u64, u64, u64, f32, vp]
        lib.syn_uniform_int.argtypes = [u64, u64, u64, ctypes.c_uint32, vp]
        lib.syn_splitmix64_sequence.argtypes = [u64, u64, vp]
        _host = lib
    return _host


def _d():
    global _dev
    if _dev is None:
        if not os.path.exists(DEVICE_SO):
            raise RuntimeError(f"{DEVICE_SO} is missing: run __graft_entry__.build() first")
        lib = ctypes.CDLL(DEVICE_SO)
        u64, f32, vp = ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p
        lib.syn_dev_normal_bf16.argtypes = [u64, u64, u64, f32, vp, vp]
        lib.syn_dev_normal_f32.argtypes = [u64, u64, u64, f32, vp, vp]
        lib.syn_dev_uniform_int.argtypes = [u64, u64, u64, ctypes.c_uint32, vp, vp]
        _dev = lib
    return _dev


# ---------------------------------------------------------------- host twin
def key(seed: int, stream: int) -> int:
    return int(_h().syn_key(seed, stream))


def splitmix64_sequence(seed: int, count: int) -> np.ndarray:
    out = np.empty(count, np.uint64)
    _h().syn_splitmix64_sequence(seed, count, out.ctypes.data)
    return out


def normal_bf16(k: int, start: int, count: int, sigma: float) -> np.ndarray:
    """bf16 bit patterns (uint16) of elements start..start+count-1."""
    out = np.empty(count, np.uint16)
    _h().syn_normal_bf16(k, start, count, sigma, out.ctypes.data)
    return out


def normal_f32(k: int, start: int, count: int, sigma: float) -> np.ndarray:
    out = np.empty(count, np.float32)
    _h().syn_normal_f32(k, start, count, sigma, out.ctypes.data)
    return out


def normal_bf16_as_f64(k: int, start: int, count: int, sigma: float) -> np.ndarray:
    """The draws of normal_bf16, each bf16 value widened exactly to float64."""
    out = np.empty(count, np.float64)
    if count:
        _h().syn_normal_bf16_as_f64(k, start, count, sigma, out.ctypes.data)
    return out


def uniform_int(k: int, start: int, count: int, n: int) -> np.ndarray:
    out = np.empty(count, np.int32)
    _h().syn_uniform_int(k, start, count, n, out.ctypes.data)
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32 (a storage format change)."""
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


# -------------------------------------------------------------- device twin
def dev_normal_bf16(k: int, start: int, count: int, sigma: float, ptr: int, stream: int = 0) -> None:
    rc = _d().syn_dev_normal_bf16(k, start, count, sigma, ptr, stream)
    if rc:
        raise RuntimeError(f"syn_dev_normal_bf16 launch failed: cudaError {rc}")


def dev_normal_f32(k: int, start: int, count: int, sigma: float, ptr: int, stream: int = 0) -> None:
    rc = _d().syn_dev_normal_f32(k, start, count, sigma, ptr, stream)
    if rc:
        raise RuntimeError(f"syn_dev_normal_f32 launch failed: cudaError {rc}")


def dev_uniform_int(k: int, start: int, count: int, n: int, ptr: int, stream: int = 0) -> None:
    rc = _d().syn_dev_uniform_int(k, start, count, n, ptr, stream)
    if rc:
        raise RuntimeError(f"syn_dev_uniform_int launch failed: cudaError {rc}")
