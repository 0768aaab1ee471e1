"""Batch-invariant MoE layer forward for B200 (sm_100a): Python binding of libmoe.so.

This module only marshals arguments: every step of the layer runs in the CUDA
kernels of ``libmoe.so`` (built from ``csrc/`` by ``__graft_entry__.build()``).
There is no fallback: importing the binding without the built library, or
calling it without a CUDA device, raises.

PyTorch supplies device memory and streams; tensors are passed to the C ABI
as raw pointers (bf16 tensors as their bit patterns).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
# MOE_LIBRARY=checked loads the build with device-side index checks
# (MOE_CHECK_BOUNDS: an out-of-range index skips its access and the forward
# reports MOE_EINDEX); anything else loads the regular build.
LIB_PATH = os.path.join(_HERE, "libmoe_checked.so" if os.environ.get("MOE_LIBRARY") == "checked" else "libmoe.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "moe.h")

MOE_OK, MOE_EINVAL, MOE_ETOOBIG, MOE_EWORKSPACE, MOE_EUNSUPPORTED, MOE_ECUDA, MOE_ETIMEOUT, MOE_EINDEX = (
    0, -1, -2, -3, -4, -5, -6, -7)
ROUTER_SOFTMAX, ROUTER_SIGMOID_BIAS, ROUTER_HASH = 0, 1, 2
ACT_SWIGLU, ACT_SITU_GLU = 0, 1
WEIGHTS_BF16, WEIGHTS_FP8, WEIGHTS_FP4 = 0, 1, 2
NUM_STAGES = 12
STAGE_NAMES = ("rmsnorm_in", "router_gemm", "router_topk", "dispatch", "gather_rows",
               "gemm_gateup_swiglu", "gemm_down", "combine_norm", "latent_down", "latent_combine",
               "latent_up", "quant_h")


EXPERT_WEIGHTS = ("w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down")


class MoEError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


class moe_config(ctypes.Structure):
    _fields_ = [("D", ctypes.c_int), ("E", ctypes.c_int), ("k", ctypes.c_int), ("I", ctypes.c_int),
                ("n_shared", ctypes.c_int), ("I_shared", ctypes.c_int), ("T_max", ctypes.c_int),
                ("router", ctypes.c_int), ("renormalize", ctypes.c_int),
                ("routed_scale", ctypes.c_float), ("gate_clamp_max", ctypes.c_float),
                ("up_clamp", ctypes.c_float), ("eps", ctypes.c_float), ("hash_mult", ctypes.c_uint32),
                ("activation", ctypes.c_int), ("situ_beta_gate", ctypes.c_float),
                ("situ_beta_up", ctypes.c_float), ("latent", ctypes.c_int), ("weight_format", ctypes.c_int),
                ("ep_world", ctypes.c_int), ("ep_rank", ctypes.c_int)]


class moe_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w_router", "router_bias", "w_gate", "w_up", "w_down",
                                               "ws_gate", "ws_up", "ws_down", "g_in", "g_out",
                                               "w_proj_down", "w_proj_up", "w_gate_exp", "w_up_exp",
                                               "w_down_exp", "ws_gate_exp", "ws_up_exp", "ws_down_exp")]


class moe_views(ctypes.Structure):
    _fields_ = [("xn", ctypes.c_void_p), ("logits", ctypes.c_void_p), ("E_pad", ctypes.c_int),
                ("topk_idx", ctypes.c_void_p), ("topk_w", ctypes.c_void_p), ("counts", ctypes.c_void_p),
                ("offsets", ctypes.c_void_p), ("src_token", ctypes.c_void_p),
                ("dest_row", ctypes.c_void_p), ("h_routed", ctypes.c_void_p),
                ("h_shared", ctypes.c_void_p), ("y_slot", ctypes.c_void_p),
                ("y_shared", ctypes.c_void_p), ("z", ctypes.c_void_p), ("agg", ctypes.c_void_p),
                ("y_latent", ctypes.c_void_p), ("xq", ctypes.c_void_p), ("xq_exp", ctypes.c_void_p),
                ("hq_routed", ctypes.c_void_p), ("hq_routed_exp", ctypes.c_void_p),
                ("hq_shared", ctypes.c_void_p), ("hq_shared_exp", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, sz, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
        L.moe_init.argtypes = [ctypes.POINTER(moe_config), ctypes.POINTER(moe_weights), ctypes.POINTER(vp)]
        L.moe_workspace_size.argtypes = [vp, i]
        L.moe_workspace_size.restype = sz
        L.moe_invariance_workspace_size.argtypes = [vp, i]
        L.moe_invariance_workspace_size.restype = sz
        L.moe_layer_forward.argtypes = [vp, i, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_get_device_error.argtypes = [vp, vp, vp]
        L.moe_reduce_partials.argtypes = [i, ctypes.POINTER(vp), vp, vp, vp, vp, i, i, f, vp]
        L.moe_check_invariance.argtypes = [vp, i, vp, vp, vp, i, vp, i, vp, sz,
                                           ctypes.POINTER(ctypes.c_ulonglong), vp]
        L.moe_workspace_views.argtypes = [vp, i, vp, ctypes.POINTER(moe_views)]
        L.moe_profile_enable.argtypes = [vp, i]
        L.moe_profile_read.argtypes = [vp, ctypes.POINTER(f), ctypes.POINTER(i)]
        L.moe_forward_launch_count.argtypes = [vp, i]
        L.moe_selftest_wait_timeout.argtypes = [i, vp]
        L.moe_destroy.argtypes = [vp]
        L.moe_status_string.argtypes = [i]
        L.moe_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


def _check(status: int, what: str) -> None:
    if status != MOE_OK:
        raise MoEError(status, what)


def _ptr(t) -> int | None:
    return None if t is None else int(t.data_ptr())


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _torch_stream(stream, device):
    """The caller's stream as a torch stream (None: the current one; a raw
    cudaStream_t handle is wrapped), for recording and waiting on events."""
    import torch
    if stream is None:
        return torch.cuda.current_stream(device)
    if hasattr(stream, "cuda_stream"):
        return stream
    return torch.cuda.ExternalStream(int(stream), device=device)


@dataclass
class LayerConfig:
    D: int
    E: int
    k: int
    I: int
    n_shared: int = 0
    I_shared: int = 0
    T_max: int = 8192
    router: int = ROUTER_SOFTMAX
    renormalize: int = 0
    routed_scale: float = 1.0
    gate_clamp_max: float = float("inf")
    up_clamp: float = float("inf")
    eps: float = 1e-6
    hash_mult: int = 2654435761
    activation: int = ACT_SWIGLU
    situ_beta_gate: float = 4.0
    situ_beta_up: float = 25.0
    latent: int = 0
    weight_format: int = WEIGHTS_BF16
    ep_world: int = 0
    ep_rank: int = 0

    def to_c(self) -> moe_config:
        return moe_config(self.D, self.E, self.k, self.I, self.n_shared,
                          self.I_shared if self.n_shared else self.I, self.T_max, self.router,
                          self.renormalize, self.routed_scale, self.gate_clamp_max, self.up_clamp,
                          self.eps, self.hash_mult, self.activation, self.situ_beta_gate,
                          self.situ_beta_up, self.latent, self.weight_format, self.ep_world, self.ep_rank)


def _check_weight_sizes(cfg: LayerConfig, weights: dict) -> None:
    """The library reads each weight through a descriptor sized from the
    configuration, so a tensor of another size must be refused here."""
    L = cfg.latent or cfg.D
    S, Is = cfg.n_shared, (cfg.I_shared if cfg.n_shared else cfg.I)
    El = cfg.E // cfg.ep_world if cfg.ep_world > 1 else cfg.E   # routed experts held here
    want = {"w_router": cfg.E * L, "router_bias": cfg.E, "w_gate": El * cfg.I * L,
            "w_up": El * cfg.I * L, "w_down": El * L * cfg.I, "ws_gate": S * Is * cfg.D,
            "ws_up": S * Is * cfg.D, "ws_down": S * cfg.D * Is, "g_in": cfg.D, "g_out": cfg.D,
            "w_proj_down": cfg.latent * cfg.D, "w_proj_up": cfg.D * cfg.latent}
    fp4 = cfg.weight_format == WEIGHTS_FP4
    if fp4:
        # Packed codes: half a byte per weight; one exponent word per row per 128 of K.
        for n in EXPERT_WEIGHTS:
            want[n + "_exp"] = want[n] // 128
            want[n] //= 2
    for name, n in want.items():
        t = weights.get(name)
        if t is None:
            continue
        if not t.is_contiguous() or t.numel() != n:
            raise ValueError(f"weight {name}: expected {n} contiguous elements for this configuration, "
                             f"got {t.numel()} (contiguous={t.is_contiguous()})")
        import torch
        dtype = torch.float32 if name == "router_bias" else torch.bfloat16
        if cfg.weight_format != WEIGHTS_BF16 and name in EXPERT_WEIGHTS:
            dtype = torch.uint8   # E4M3 codes, or packed E2M1 codes
        if name.endswith("_exp"):
            dtype = torch.int32   # four int8 block exponents a word
        if t.dtype != dtype:
            raise ValueError(f"weight {name}: expected {dtype}, got {t.dtype}")


class MoELayer:
    """A handle over caller-owned device weights (torch tensors, bf16 unless
    noted).  ``weights`` maps the moe_weights field names to tensors; the
    tensors must outlive the layer."""

    def __init__(self, cfg: LayerConfig, weights: dict):
        self.cfg = cfg
        _check_weight_sizes(cfg, weights)
        self._keep = dict(weights)
        w = moe_weights(*[_ptr(weights.get(n)) for n, _ in moe_weights._fields_])
        h = ctypes.c_void_p()
        _check(lib().moe_init(ctypes.byref(cfg.to_c()), ctypes.byref(w), ctypes.byref(h)), "moe_init")
        self.handle = h

    def close(self):
        h = getattr(self, "handle", None)
        if h:
            self.handle = None
            lib().moe_destroy(h)

    def __del__(self):
        try:
            self.close()
        except Exception:  # interpreter shutdown: the library may already be unloaded
            pass

    def workspace_size(self, T: int) -> int:
        return int(lib().moe_workspace_size(self.handle, T))

    def invariance_workspace_size(self, T: int) -> int:
        return int(lib().moe_invariance_workspace_size(self.handle, T))

    def forward(self, x, residual, out_norm, out_residual, workspace, token_ids=None,
                out_topk_idx=None, out_topk_w=None, out_counts=None, stream=None) -> None:
        T = int(x.shape[0])
        _check(lib().moe_layer_forward(self.handle, T, _ptr(x), _ptr(residual), _ptr(token_ids),
                                       _ptr(out_norm), _ptr(out_residual), _ptr(out_topk_idx),
                                       _ptr(out_topk_w), _ptr(out_counts), _ptr(workspace),
                                       workspace.numel() * workspace.element_size() if workspace is not None else 0,
                                       _stream(stream)),
               "moe_layer_forward")

    def device_error(self, workspace, stream=None) -> int:
        """moe_get_device_error: read and clear the device error word of the
        last forward on ``workspace`` (None: the no-allocation forward's static
        scratch on the current device)."""
        return int(lib().moe_get_device_error(self.handle, _ptr(workspace), _stream(stream)))

    def check_invariance(self, x, residual, workspace, token_ids=None, n_splits=0, perm=None,
                         repeats=0, stream=None) -> int:
        out = ctypes.c_ulonglong(0)
        _check(lib().moe_check_invariance(self.handle, int(x.shape[0]), _ptr(x), _ptr(residual),
                                          _ptr(token_ids), n_splits, _ptr(perm), repeats,
                                          _ptr(workspace), workspace.numel() * workspace.element_size(),
                                          ctypes.byref(out), _stream(stream)),
               "moe_check_invariance")
        return int(out.value)

    def views(self, T: int, workspace) -> moe_views:
        v = moe_views()
        _check(lib().moe_workspace_views(self.handle, T, _ptr(workspace), ctypes.byref(v)),
               "moe_workspace_views")
        return v

    def profile_enable(self, stages=None) -> None:
        """Time the given stage indices (all when None; [] turns timing off)."""
        stages = range(NUM_STAGES) if stages is None else stages
        mask = 0
        for s_ in stages:
            mask |= 1 << int(s_)
        _check(lib().moe_profile_enable(self.handle, mask), "moe_profile_enable")

    def profile_read(self):
        ms = (ctypes.c_float * NUM_STAGES)()
        n = (ctypes.c_int * NUM_STAGES)()
        _check(lib().moe_profile_read(self.handle, ms, n), "moe_profile_read")
        return list(ms), list(n)

    def launch_count(self, T: int) -> int:
        return int(lib().moe_forward_launch_count(self.handle, T))


class HostPipeline:
    """Layer forwards of batches held in pinned host memory, end to end.

    Each step copies its batch (x, residual and, for hash routing, the token
    ids) from pinned host memory to the device, runs the layer forward, and
    copies out_norm and out_residual back to pinned host memory.  Three streams
    (copy-in, compute, copy-out) and two sets of device buffers let the copy-in
    of step i + 1 and the copy-out of step i - 1 run while step i computes, so
    the steady state costs max(compute, copy-in, copy-out) per step instead of
    their sum.  ``chunks`` > 1 also splits every batch into that many row
    blocks, each its own forward: a row's outputs do not depend on the rest of
    its batch, so the bits are those of one call over the whole batch.

    Only copies and stream ordering happen here; every step of the layer runs
    in the library's kernels."""

    def __init__(self, layer: "MoELayer", T: int, chunks: int = 1, device=None):
        import torch
        self.layer, self.T = layer, int(T)
        self.chunks = max(1, min(int(chunks), self.T))
        cfg = layer.cfg
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.device = dev
        bounds = [self.T * c // self.chunks for c in range(self.chunks + 1)]
        self.blocks = [(bounds[c], bounds[c + 1]) for c in range(self.chunks) if bounds[c + 1] > bounds[c]]
        tmax = max(b - a for a, b in self.blocks)
        mk = lambda: torch.empty((self.T, cfg.D), dtype=torch.bfloat16, device=dev)  # noqa: E731
        self.x = [mk(), mk()]
        self.r = [mk(), mk()]
        self.on = [mk(), mk()]
        self.orr = [mk(), mk()]
        self.ids = [torch.empty(self.T, dtype=torch.int32, device=dev) for _ in range(2)]
        self.ws = torch.empty(max(layer.workspace_size(tmax), 256), dtype=torch.uint8, device=dev)
        self.s_in, self.s_comp, self.s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
        ev = lambda: [torch.cuda.Event(), torch.cuda.Event()]  # noqa: E731
        self.in_done, self.comp_done, self.out_done = ev(), ev(), ev()
        self._used = [False, False]

    def run(self, xs, residuals, outs_norm, outs_residual, token_ids=None) -> None:
        """Forward every batch i: xs[i], residuals[i] (pinned host [T, D] bf16)
        -> outs_norm[i], outs_residual[i] (pinned host [T, D] bf16).
        ``token_ids`` (list of pinned host [T] int32) is required for hash
        routing.  Returns once the work is queued; synchronise the device (or
        ``self.s_out``) before reading the outputs."""
        import torch
        hashr = self.layer.cfg.router == ROUTER_HASH
        if hashr and token_ids is None:
            raise ValueError("hash routing needs token_ids")
        cur = torch.cuda.current_stream(self.device)
        # Work queued on the caller's stream before this call comes first.
        for s in (self.s_in, self.s_comp, self.s_out):
            s.wait_stream(cur)
        for i in range(len(xs)):
            b = i & 1
            if self._used[b]:
                # Buffer set b is free for new inputs once step i - 2 has computed.
                self.s_in.wait_event(self.comp_done[b])
            with torch.cuda.stream(self.s_in):
                self.x[b].copy_(xs[i], non_blocking=True)
                self.r[b].copy_(residuals[i], non_blocking=True)
                if hashr:
                    self.ids[b].copy_(token_ids[i], non_blocking=True)
                self.in_done[b].record(self.s_in)
            self.s_comp.wait_event(self.in_done[b])
            if self._used[b]:
                # ... and its outputs may be overwritten once step i - 2 was copied out.
                self.s_comp.wait_event(self.out_done[b])
            for a, e in self.blocks:
                self.layer.forward(self.x[b][a:e], self.r[b][a:e], self.on[b][a:e], self.orr[b][a:e], self.ws,
                                   token_ids=self.ids[b][a:e] if hashr else None, stream=self.s_comp)
            self.comp_done[b].record(self.s_comp)
            self.s_out.wait_event(self.comp_done[b])
            with torch.cuda.stream(self.s_out):
                outs_norm[i].copy_(self.on[b], non_blocking=True)
                outs_residual[i].copy_(self.orr[b], non_blocking=True)
                self.out_done[b].record(self.s_out)
            self._used[b] = True
        # The caller's stream continues after the last copy-out.
        cur.wait_stream(self.s_out)


def reduce_partials(partials, residual, g, out_norm, out_residual, eps: float = 1e-6,
                    stream=None) -> None:
    """Fixed r0..r7 order partial reduction + residual + RMSNorm (P <= 8 bf16 tensors)."""
    P = len(partials)
    arr = (ctypes.c_void_p * P)(*[_ptr(p) for p in partials])
    T, D = int(residual.shape[0]), int(residual.shape[1])
    _check(lib().moe_reduce_partials(P, arr, _ptr(residual), _ptr(g), _ptr(out_norm),
                                     _ptr(out_residual), T, D, eps, _stream(stream)),
           "moe_reduce_partials")


def quantize_weights_fp4(w, w8, block_exp=None, stream=None) -> None:
    """moe_quantize_weights_fp4: bf16 master weights [..., K] -> E4M3 codes (uint8,
    same shape) of their FP4 values, and optionally the int8 block exponents
    [..., K / 32]."""
    L = lib()
    K = int(w.shape[-1])
    rows = w.numel() // K if K else 0
    if w8.numel() != w.numel() or w8.dtype.itemsize != 1:
        raise ValueError("w8 must be a byte tensor with as many elements as w")
    L.moe_quantize_weights_fp4.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_longlong, ctypes.c_int, ctypes.c_void_p]
    _check(L.moe_quantize_weights_fp4(_ptr(w), _ptr(w8), _ptr(block_exp), rows, K, _stream(stream)),
           "moe_quantize_weights_fp4")




def quantize_expert_weights(weights: dict, stream=None) -> dict:
    """A copy of a moe_weights dict whose expert matrices (bf16 master weights)
    are replaced by their E4M3 codes from quantize_weights_fp4, for a layer
    configured with weight_format=WEIGHTS_FP8.  Other entries are shared."""
    import torch
    out = dict(weights)
    for n in EXPERT_WEIGHTS:
        t = weights.get(n)
        if t is None:
            continue
        q = torch.empty(t.shape, dtype=torch.uint8, device=t.device)
        quantize_weights_fp4(t, q, stream=stream)
        out[n] = q
    return out


def quantize_weights_fp4_packed(w, packed, exps, stream=None) -> None:
    """moe_quantize_weights_fp4_packed: bf16 master weights [..., K] -> their FP4
    storage form: ``packed`` uint8 [..., K / 2] (two E2M1 codes a byte, low nibble
    first) and ``exps`` int32 [K / 128, rows] (four int8 block exponents a word)."""
    L = lib()
    K = int(w.shape[-1])
    rows = w.numel() // K if K else 0
    if packed.numel() * 2 != w.numel() or packed.dtype.itemsize != 1:
        raise ValueError("packed must be a byte tensor with half as many elements as w")
    if exps.numel() * 128 != w.numel() or exps.dtype.itemsize != 4:
        raise ValueError("exps must be a 4-byte tensor with one word per 128 elements of w")
    L.moe_quantize_weights_fp4_packed.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                  ctypes.c_longlong, ctypes.c_int, ctypes.c_void_p]
    _check(L.moe_quantize_weights_fp4_packed(_ptr(w), _ptr(packed), _ptr(exps), rows, K, _stream(stream)),
           "moe_quantize_weights_fp4_packed")


def pack_expert_weights_fp4(weights: dict, stream=None) -> dict:
    """A copy of a moe_weights dict whose expert matrices (bf16 master weights)
    are replaced by their FP4 storage form from quantize_weights_fp4_packed
    (packed codes under the matrix's name, exponent words under name + "_exp"),
    for a layer configured with weight_format=WEIGHTS_FP4.  Other entries are
    shared."""
    import torch
    out = dict(weights)
    for n in EXPERT_WEIGHTS:
        t = weights.get(n)
        if t is None:
            continue
        K = int(t.shape[-1])
        rows = t.numel() // K
        p = torch.empty(t.shape[:-1] + (K // 2,), dtype=torch.uint8, device=t.device)
        x = torch.empty((K // 128, rows), dtype=torch.int32, device=t.device)
        quantize_weights_fp4_packed(t, p, x, stream=stream)
        out[n] = p
        out[n + "_exp"] = x
    return out


def selftest_wait_timeout(limit_us: int, stream=None) -> int:
    return int(lib().moe_selftest_wait_timeout(limit_us, _stream(stream)))


def forward_noalloc(layer: MoELayer, x, residual, out_norm, out_residual, token_ids=None,
                    out_topk_idx=None, out_topk_w=None, out_counts=None, stream=None) -> None:
    """moe_layer_forward_noalloc: the layer forward for decode-sized batches
    without a caller workspace (scratch in a static 32 MiB device array), for
    callers that cannot allocate device memory.  See include/moe.h."""
    L = lib()
    fn = L.moe_layer_forward_noalloc
    vp = ctypes.c_void_p
    fn.argtypes = [vp, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    _check(fn(layer.handle, int(x.shape[0]), _ptr(x), _ptr(residual), _ptr(token_ids),
              _ptr(out_norm), _ptr(out_residual), _ptr(out_topk_idx), _ptr(out_topk_w),
              _ptr(out_counts), _stream(stream)),
           "moe_layer_forward_noalloc")


def reduce_partials_rows(partials, residual, g, out_norms, out_residuals, row0: int, rows: int,
                         eps: float = 1e-6, stream=None) -> None:
    """moe_reduce_partials_rows: rows [row0, row0 + rows) of the partial
    buffers (device pointers, local or peer-mapped, each [T, D] bf16) reduced in
    list order + residual + RMSNorm, stored to every (out_norm, out_residual)
    pair.  ``partials`` / ``out_*`` are tensors or raw device addresses."""
    P, n = len(partials), len(out_norms)
    addr = lambda t: t if isinstance(t, int) else t.data_ptr()  # noqa: E731
    pa = (ctypes.c_void_p * P)(*[addr(p) for p in partials])
    on = (ctypes.c_void_p * n)(*[addr(p) for p in out_norms])
    orr = (ctypes.c_void_p * n)(*[addr(p) for p in out_residuals])
    L = lib()
    fn = L.moe_reduce_partials_rows
    vp = ctypes.c_void_p
    fn.argtypes = [ctypes.c_int, vp, vp, vp, ctypes.c_int, vp, vp, ctypes.c_int, ctypes.c_int,
                   ctypes.c_int, ctypes.c_float, vp]
    D = int(residual.shape[-1])
    _check(fn(P, pa, _ptr(residual), _ptr(g), n, on, orr, row0, rows, D, eps, _stream(stream)),
           "moe_reduce_partials_rows")


def partial_order(world: int, per_rank: int):
    """(rank, index) of partial p = 0 .. world * per_rank - 1: rank-major, so
    partial p lives on rank p // per_rank.  The reduction adds them in this
    order on every rank."""
    return [(p // per_rank, p % per_rank) for p in range(world * per_rank)]


def row_slices(T: int, world: int):
    """Contiguous (row0, rows) of each rank: the first T % world ranks get one
    row more.  Rows are independent, so the partition never changes a bit."""
    base, extra = divmod(T, world)
    out, r0 = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((r0, n))
        r0 += n
    return out


PEER_HANDLE_BYTES = 64


def peer_alloc(nbytes: int):
    """moe_peer_alloc: (device address, IPC handle bytes) of a new zeroed,
    exported allocation on the current device."""
    L = lib()
    ptr = ctypes.c_void_p()
    h = (ctypes.c_ubyte * PEER_HANDLE_BYTES)()
    L.moe_peer_alloc.argtypes = [ctypes.c_size_t, ctypes.POINTER(ctypes.c_void_p), ctypes.c_void_p]
    _check(L.moe_peer_alloc(nbytes, ctypes.byref(ptr), h), "moe_peer_alloc")
    return int(ptr.value), bytes(h)


def peer_open(handle: bytes) -> int:
    """moe_peer_open: map another process's exported allocation; its address."""
    L = lib()
    ptr = ctypes.c_void_p()
    h = (ctypes.c_ubyte * PEER_HANDLE_BYTES).from_buffer_copy(handle)
    L.moe_peer_open.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_void_p)]
    _check(L.moe_peer_open(h, ctypes.byref(ptr)), "moe_peer_open")
    return int(ptr.value)


def peer_close(addr: int) -> None:
    L = lib()
    L.moe_peer_close.argtypes = [ctypes.c_void_p]
    _check(L.moe_peer_close(addr), "moe_peer_close")


def peer_free(addr: int) -> None:
    L = lib()
    L.moe_peer_free.argtypes = [ctypes.c_void_p]
    _check(L.moe_peer_free(addr), "moe_peer_free")


def peer_barrier(flags, rank: int, epoch: int, err, limit_us: int, stream=None) -> None:
    """moe_peer_barrier over len(flags) ranks (flag-array device addresses in
    rank order); a timed-out wait stores 1 to the device int32 tensor ``err``."""
    L = lib()
    arr = (ctypes.c_void_p * len(flags))(*flags)
    L.moe_peer_barrier.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_uint32,
                                   ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    _check(L.moe_peer_barrier(len(flags), rank, arr, epoch, _ptr(err), limit_us, _stream(stream)),
           "moe_peer_barrier")


class _DeviceArray:
    """A device address exposed through __cuda_array_interface__ (int16 words),
    so that torch can view memory this library allocated."""

    def __init__(self, addr: int, n: int):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": "<i2", "data": (addr, False),
                                         "version": 3, "strides": None}


class TPAllReduceNorm:
    """The tensor-parallel epilogue across GPUs (the Fireworks parity post,
    Trap 1 and Trap 2: every rank reduces r_0 + r_1 + ... in the same fixed
    order, then residual + RMSNorm).  Each rank exports one allocation
    (moe_peer_alloc) holding its barrier flags, its ``per_rank`` partial
    buffers [T, D] and its two outputs, and maps every other rank's
    (moe_peer_open; handles travel over the process group).  A call is three
    kernels on the caller's stream: a device barrier, moe_reduce_partials_rows
    on this rank's row slice (all ranks' partials read over NVLink with plain
    loads, the rows stored to every rank's outputs), and a second barrier.
    Every rank ends with the bits the single-GPU moe_reduce_partials gives over
    the same P partials.

    Fill ``partial[j]`` (partial rank * per_rank + j) before the call; read
    ``out_norm`` / ``out_residual`` after it.  A barrier wait that gives up
    after ``barrier_timeout_ms`` records it in a device word: ``check()``
    raises MoEError(MOE_ETIMEOUT) if any did.  ``close()`` (collective)
    releases the memory; the tensors are invalid after it."""

    _ALIGN = 4096

    def __init__(self, T: int, D: int, per_rank: int = 1, group=None, device=None,
                 barrier_timeout_ms: int = 5000):
        import torch
        import torch.distributed as dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if self.world * per_rank > 8:
            raise ValueError("at most 8 partials in all")
        if not 1 <= barrier_timeout_ms <= 60000:
            raise ValueError("barrier_timeout_ms must be in 1 .. 60000")
        self.T, self.D, self.per_rank = T, D, per_rank
        self.limit_us = barrier_timeout_ms * 1000
        up = lambda n: (n + self._ALIGN - 1) // self._ALIGN * self._ALIGN  # noqa: E731
        buf = T * D * 2
        off_part = up(4 * self.world)
        off_norm = off_part + up(per_rank * buf)
        off_res = off_norm + up(buf)
        total = off_res + up(buf)
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        with torch.cuda.device(dev):
            self._base, handle = peer_alloc(total)
        self._opened, self._closed = [], False
        info = [None] * self.world
        dist.all_gather_object(info, (handle, T, D, per_rank), group=group)
        if any(x[1:] != (T, D, per_rank) for x in info):
            raise ValueError(f"ranks disagree on (T, D, per_rank): {[x[1:] for x in info]}")
        bases = []
        with torch.cuda.device(dev):
            for r in range(self.world):
                if r == self.rank:
                    bases.append(self._base)
                else:
                    bases.append(peer_open(info[r][0]))
                    self._opened.append(bases[-1])
        view = lambda addr, n, shape: torch.as_tensor(  # noqa: E731
            _DeviceArray(addr, n), device=dev).view(torch.bfloat16).view(shape)
        self.partial = view(self._base + off_part, per_rank * T * D, (per_rank, T, D))
        self.out_norm = view(self._base + off_norm, T * D, (T, D))
        self.out_residual = view(self._base + off_res, T * D, (T, D))
        self._flags = [b for b in bases]
        self._partials = [bases[r] + off_part + j * buf for r, j in partial_order(self.world, per_rank)]
        self._outs_n = [b + off_norm for b in bases]
        self._outs_r = [b + off_res for b in bases]
        self.row0, self.rows = row_slices(T, self.world)[self.rank]
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self._epoch = 0

    def _barrier(self, stream):
        self._epoch += 1
        peer_barrier(self._flags, self.rank, self._epoch, self.err, self.limit_us, stream)

    def __call__(self, residual, g, eps: float = 1e-6, stream=None):
        # Every rank's partials are written before anyone reads them ...
        self._barrier(stream)
        reduce_partials_rows(self._partials, residual, g, self._outs_n, self._outs_r, self.row0, self.rows,
                             eps, stream)
        # ... and every rank's rows are stored before anyone reads the outputs
        # or rewrites its partials.
        self._barrier(stream)
        return self.out_norm, self.out_residual

    def check(self) -> None:
        """Raise MoEError(MOE_ETIMEOUT) if a barrier wait gave up (synchronises)."""
        e = int(self.err.item())
        self.err.zero_()
        if e:
            raise MoEError(MOE_ETIMEOUT, "TPAllReduceNorm barrier")

    def close(self) -> None:
        """Collective: unmap the peers' memory, then free this rank's."""
        import torch
        import torch.distributed as dist
        if self._closed:
            return
        torch.cuda.synchronize()
        dist.barrier(group=self.group)
        for a in self._opened:
            peer_close(a)
        dist.barrier(group=self.group)
        peer_free(self._base)
        self._closed = True


# ------------------------------------------------------------ expert parallelism
class moe_ep_peers(ctypes.Structure):
    _fields_ = [("xbuf", ctypes.c_void_p * 8)]


def expert_range(E: int, world: int, rank: int):
    """Routed experts [e0, e1) held by ``rank`` of ``world`` (contiguous blocks)."""
    if world < 1 or E % world:
        raise ValueError("the expert count must divide evenly over the ranks")
    n = E // world
    return rank * n, (rank + 1) * n


def shard_expert_weights(weights: dict, world: int, rank: int) -> dict:
    """The moe_weights dict of one expert-parallel rank: its block of routed
    experts (views of the full tensors, first axis = expert), everything else
    whole."""
    out = dict(weights)
    for n in ("w_gate", "w_up", "w_down"):
        t = weights[n]
        E = int(t.shape[0])
        e0, e1 = expert_range(E, world, rank)
        out[n] = t[e0:e1]
        x = weights.get(n + "_exp")
        if x is not None:
            # FP4 exponent words [K / 128, E * rows]: this rank's columns, made contiguous.
            per = x.shape[1] // E
            out[n + "_exp"] = x[:, e0 * per:e1 * per].contiguous()
    return out


def _ep_call(name, *args):
    L = lib()
    fn = getattr(L, name)
    _check(fn(*args), name)


class _EPRank:
    """One expert-parallel rank: its handle, workspace and exchange buffer.
    ``own_copy``: keep a private copy of this rank's expert block (so the full
    weight tensors can be freed) instead of views into them."""

    def __init__(self, cfg: LayerConfig, weights: dict, rank: int, world: int, device, own_copy: bool = False):
        import dataclasses

        import torch
        self.rank = rank
        self.cfg = dataclasses.replace(cfg, ep_world=world, ep_rank=rank)
        shard = shard_expert_weights(weights, world, rank)
        if own_copy:
            shard = {n: (t.clone() if n in ("w_gate", "w_up", "w_down") else t) for n, t in shard.items()}
        self.layer = MoELayer(self.cfg, shard)
        L = lib()
        L.moe_ep_exchange_size.restype = ctypes.c_size_t
        L.moe_ep_exchange_size.argtypes = [ctypes.c_void_p]
        self.xbytes = int(L.moe_ep_exchange_size(self.layer.handle))
        self.ws = torch.empty(max(self.layer.workspace_size(cfg.T_max), 256), dtype=torch.uint8, device=device)
        self.device = device

    def route(self, x, token_ids, xbuf, stream=None):
        # A rank with no tokens still publishes its (zero) counts.
        L = lib()
        L.moe_ep_route.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
        _check(L.moe_ep_route(self.layer.handle, int(x.shape[0]), _ptr(x), _ptr(token_ids), xbuf,
                              _ptr(self.ws), self.ws.numel(), _stream(stream)), "moe_ep_route")

    def send(self, T, peers, stream=None, wave=None, n_waves=1):
        """The whole send (wave None), or the rows of wave ``wave`` of ``n_waves``."""
        L = lib()
        if wave is None:
            L.moe_ep_send.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(moe_ep_peers), ctypes.c_void_p,
                                      ctypes.c_size_t, ctypes.c_void_p]
            _check(L.moe_ep_send(self.layer.handle, T, ctypes.byref(peers), _ptr(self.ws), self.ws.numel(),
                                 _stream(stream)), "moe_ep_send")
            return
        L.moe_ep_send_wave.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(moe_ep_peers), ctypes.c_int,
                                       ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
        _check(L.moe_ep_send_wave(self.layer.handle, T, ctypes.byref(peers), wave, n_waves, _ptr(self.ws),
                                  self.ws.numel(), _stream(stream)), "moe_ep_send_wave")

    def experts(self, T, peers, stream=None, wave=None, n_waves=1):
        """All of the rank's experts (wave None), or those of wave ``wave`` of ``n_waves``."""
        L = lib()
        if wave is None:
            L.moe_ep_experts.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(moe_ep_peers),
                                         ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
            _check(L.moe_ep_experts(self.layer.handle, T, ctypes.byref(peers), _ptr(self.ws), self.ws.numel(),
                                    _stream(stream)), "moe_ep_experts")
            return
        L.moe_ep_experts_wave.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(moe_ep_peers),
                                          ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t,
                                          ctypes.c_void_p]
        _check(L.moe_ep_experts_wave(self.layer.handle, T, ctypes.byref(peers), wave, n_waves, _ptr(self.ws),
                                     self.ws.numel(), _stream(stream)), "moe_ep_experts_wave")

    def combine(self, residual, xbuf, out_norm, out_residual, out_idx=None, out_w=None, stream=None):
        L = lib()
        vp = ctypes.c_void_p
        L.moe_ep_combine.argtypes = [vp, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        _check(L.moe_ep_combine(self.layer.handle, int(residual.shape[0]), _ptr(residual), xbuf, _ptr(out_norm),
                                _ptr(out_residual), _ptr(out_idx), _ptr(out_w), _ptr(self.ws), self.ws.numel(),
                                _stream(stream)), "moe_ep_combine")

    def device_error(self, stream=None) -> int:
        return self.layer.device_error(self.ws, stream)


class VirtualEP:
    """``world`` expert-parallel ranks sharing one device: each rank has its own
    handle (its block of routed experts), workspace and exchange buffer.  With
    ``waves`` = 1 a step runs every rank's route, send, experts and combine in
    the order of one stream.  With ``waves`` = n > 1 (wave scheduling, DeepSeek
    V4 infra notes §6.1 "MegaMoE") the experts are split into n waves: every
    rank's sends run on a communication stream, wave after wave, and every
    rank's expert GEMMs on a compute stream, wave w after the event that closes
    wave w's sends, so the rows of wave w + 1 travel while wave w computes.
    Ordering is by stream order and events only: no kernel waits on another.
    Either way each rank's outputs are bit for bit those of the single-device
    layer on its tokens.  ``weights`` holds all E routed experts."""

    def __init__(self, cfg: LayerConfig, weights: dict, world: int, device="cuda"):
        import torch
        if world < 2 or world > 8:
            raise ValueError("2 .. 8 ranks")
        self.world = world
        self.ranks = [_EPRank(cfg, weights, r, world, device) for r in range(world)]
        self.E_loc = cfg.E // world
        self.xbuf = [torch.zeros(max(rk.xbytes, 256), dtype=torch.uint8, device=device) for rk in self.ranks]
        self.peers = moe_ep_peers()
        for r in range(world):
            self.peers.xbuf[r] = _ptr(self.xbuf[r])
        self._comm = torch.cuda.Stream(device=device)
        self._comp = torch.cuda.Stream(device=device)

    def forward(self, xs, residuals, token_ids=None, stream=None, waves: int = 1):
        """xs, residuals: one [T_r, D] bf16 tensor per rank; returns per rank
        (out_norm, out_residual, topk_idx, topk_w).  ``waves``: 1 .. E / world."""
        import torch
        if waves < 1 or waves > self.E_loc:
            raise ValueError(f"waves must be in 1 .. {self.E_loc}")
        ids = token_ids if token_ids is not None else [None] * self.world
        Ts = [int(x.shape[0]) for x in xs]
        for r, rk in enumerate(self.ranks):
            rk.route(xs[r], ids[r], _ptr(self.xbuf[r]), stream)
        if waves == 1:
            for r, rk in enumerate(self.ranks):
                rk.send(Ts[r], self.peers, stream)
            for r, rk in enumerate(self.ranks):
                rk.experts(Ts[r], self.peers, stream)
        else:
            main = _torch_stream(stream, self.xbuf[0].device)
            routed = torch.cuda.Event()
            routed.record(main)
            self._comm.wait_event(routed)
            self._comp.wait_event(routed)
            for w in range(waves):
                for r, rk in enumerate(self.ranks):
                    rk.send(Ts[r], self.peers, self._comm, wave=w, n_waves=waves)
                sent = torch.cuda.Event()
                sent.record(self._comm)
                self._comp.wait_event(sent)
                for r, rk in enumerate(self.ranks):
                    rk.experts(Ts[r], self.peers, self._comp, wave=w, n_waves=waves)
            main.wait_stream(self._comm)
            main.wait_stream(self._comp)
        outs = []
        for r, rk in enumerate(self.ranks):
            T = int(xs[r].shape[0])
            k = rk.cfg.k
            on = torch.empty_like(residuals[r])
            orr = torch.empty_like(residuals[r])
            idx = torch.empty((T, k), dtype=torch.int32, device=on.device)
            w = torch.empty((T, k), dtype=torch.float32, device=on.device)
            rk.combine(residuals[r], _ptr(self.xbuf[r]), on, orr, idx, w, stream)
            outs.append((on, orr, idx, w))
        return outs

    def device_errors(self):
        return [rk.device_error() for rk in self.ranks]


class EPMoELayer:
    """Expert parallelism across processes, one GPU each (torch.distributed
    group of ``world`` ranks): this rank's handle with its block of routed
    experts, and one exported allocation holding its barrier flags and its
    exchange buffer, mapped by every other rank (moe_peer_open; handles travel
    over the process group).  A step is the four phases on the caller's
    stream with a device barrier (bounded; ``check()`` reports a time-out)
    after route, send and experts.  ``weights`` holds all E routed experts; the
    rank keeps its own copy of its block, so the caller may free the rest.
    ``close()`` (collective) releases the memory."""

    _FLAGS = 4096

    def __init__(self, cfg: LayerConfig, weights: dict, group=None, device=None, barrier_timeout_ms: int = 5000):
        import torch
        import torch.distributed as dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.me = _EPRank(cfg, weights, self.rank, self.world, dev, own_copy=True)
        self.limit_us = barrier_timeout_ms * 1000
        with torch.cuda.device(dev):
            self._base, handle = peer_alloc(self._FLAGS + self.me.xbytes)
        info = [None] * self.world
        dist.all_gather_object(info, (handle, self.me.xbytes), group=group)
        if any(x[1] != self.me.xbytes for x in info):
            raise ValueError("ranks disagree on the exchange buffer size (configurations differ)")
        self._opened, self._closed = [], False
        bases = []
        with torch.cuda.device(dev):
            for r in range(self.world):
                if r == self.rank:
                    bases.append(self._base)
                else:
                    bases.append(peer_open(info[r][0]))
                    self._opened.append(bases[-1])
        self._flags = bases
        self.peers = moe_ep_peers()
        for r in range(self.world):
            self.peers.xbuf[r] = bases[r] + self._FLAGS
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self._epoch = 0
        self._comm = self._comp = None

    def _barrier(self, stream):
        self._epoch += 1
        peer_barrier(self._flags, self.rank, self._epoch, self.err, self.limit_us, stream)

    def forward(self, x, residual, token_ids=None, stream=None, waves: int = 1):
        """One step.  ``waves`` = n > 1: the experts in n waves, every rank's
        send of wave w followed by a barrier on a communication stream, and the
        expert GEMMs of wave w on a compute stream after that barrier, so the
        rows of wave w + 1 cross the links while wave w computes.  Every rank
        must pass the same ``waves``: the barriers' epochs follow the same
        order on every rank (route, the waves' sends, the results)."""
        import torch
        T = int(x.shape[0])
        E_loc = self.me.cfg.E // self.world
        if waves < 1 or waves > E_loc:
            raise ValueError(f"waves must be in 1 .. {E_loc}")
        mine = self.peers.xbuf[self.rank]
        self.me.route(x, token_ids, mine, stream)
        self._barrier(stream)          # every rank's counts are out
        if waves == 1:
            self.me.send(T, self.peers, stream)
            self._barrier(stream)      # every row has reached its owner
            self.me.experts(T, self.peers, stream)
            self._barrier(stream)      # every result row is back home
        else:
            dev = self.err.device
            if self._comm is None:
                self._comm, self._comp = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
            main = _torch_stream(stream, dev)
            routed = torch.cuda.Event()
            routed.record(main)
            self._comm.wait_event(routed)
            self._comp.wait_event(routed)
            for w in range(waves):
                self.me.send(T, self.peers, self._comm, wave=w, n_waves=waves)
                self._barrier(self._comm)      # wave w's rows have reached their owners
                arrived = torch.cuda.Event()
                arrived.record(self._comm)
                self._comp.wait_event(arrived)
                self.me.experts(T, self.peers, self._comp, wave=w, n_waves=waves)
            self._barrier(self._comp)          # every result row is back home
            main.wait_stream(self._comm)
            main.wait_stream(self._comp)
        on, orr = torch.empty_like(residual), torch.empty_like(residual)
        idx = torch.empty((T, self.me.cfg.k), dtype=torch.int32, device=on.device)
        w = torch.empty((T, self.me.cfg.k), dtype=torch.float32, device=on.device)
        self.me.combine(residual, mine, on, orr, idx, w, stream)
        return on, orr, idx, w

    def check(self) -> None:
        """Raise MoEError if a barrier wait gave up or a kernel reported a device
        error (a bounded wait, or an index check in the checked build)."""
        e = int(self.err.item())
        self.err.zero_()
        if e:
            raise MoEError(MOE_ETIMEOUT, "EPMoELayer barrier")
        st = self.me.device_error()
        if st != MOE_OK:
            raise MoEError(st, "EPMoELayer device error")

    def close(self) -> None:
        import torch
        import torch.distributed as dist
        if self._closed:
            return
        torch.cuda.synchronize()
        dist.barrier(group=self.group)
        for a in self._opened:
            peer_close(a)
        dist.barrier(group=self.group)
        peer_free(self._base)
        self._closed = True
