"""The C ABI without a GPU: the library loads, exports every declared entry
point, and rejects bad arguments before touching CUDA."""
import ctypes
import re

import pytest

import deterministic_expert_b200 as moe


def declared_functions():
    with open(moe.HEADER_PATH) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char\*)\s+(moe_\w+)\s*\(", src, flags=re.M)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 14
    lib = moe.lib()
    for n in names:
        assert hasattr(lib, n), n


def test_bounds_checked_build_exports_the_same_symbols():
    """The MOE_CHECK_BOUNDS build (libmoe_checked.so) is the same ABI."""
    import os
    path = os.path.join(os.path.dirname(moe.LIB_PATH), "libmoe_checked.so")
    assert os.path.exists(path), "build libmoe_checked.so with __graft_entry__.build()"
    checked = ctypes.CDLL(path)
    for n in declared_functions():
        assert hasattr(checked, n), n
    checked.moe_status_string.restype = ctypes.c_char_p
    assert b"index" in checked.moe_status_string(moe.MOE_EINDEX)


def test_status_strings():
    assert moe.status_string(0) == "ok"
    assert "timed out" in moe.status_string(moe.MOE_ETIMEOUT)
    assert moe.status_string(12345) == "unknown status"


def _init(**kw):
    base = dict(D=256, E=8, k=2, I=128, n_shared=1, I_shared=128, T_max=64)
    base.update(kw)
    cfg = moe.LayerConfig(**base).to_c()
    fake = 1 << 20  # never dereferenced: validation fails first
    w = moe.moe_weights(*[fake] * 10)
    h = ctypes.c_void_p()
    return moe.lib().moe_init(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)), h


@pytest.mark.parametrize("kw,status", [
    (dict(D=100), moe.MOE_EUNSUPPORTED), (dict(I=96), moe.MOE_EUNSUPPORTED),
    (dict(E=300), moe.MOE_EUNSUPPORTED), (dict(k=9), moe.MOE_EUNSUPPORTED),
    (dict(k=0), moe.MOE_EINVAL), (dict(T_max=0), moe.MOE_EINVAL), (dict(router=7), moe.MOE_EINVAL),
    (dict(n_shared=9), moe.MOE_EUNSUPPORTED), (dict(eps=-1.0), moe.MOE_EINVAL),
    (dict(D=32768), moe.MOE_EUNSUPPORTED), (dict(T_max=1 << 21), moe.MOE_EUNSUPPORTED),
])
def test_init_rejects_bad_configs_without_cuda(kw, status):
    rc, h = _init(**kw)
    assert rc == status and not h.value


def test_init_rejects_missing_weights():
    cfg = moe.LayerConfig(D=256, E=8, k=2, I=128).to_c()
    w = moe.moe_weights()
    h = ctypes.c_void_p()
    assert moe.lib().moe_init(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)) == moe.MOE_EINVAL
    assert moe.lib().moe_init(None, ctypes.byref(w), ctypes.byref(h)) == moe.MOE_EINVAL


def test_calls_reject_null_handles():
    L = moe.lib()
    assert L.moe_workspace_size(None, 4) == 0
    assert L.moe_layer_forward(None, 4, *[None] * 9, 0, None) == moe.MOE_EINVAL
    assert L.moe_destroy(None) == moe.MOE_EINVAL
    assert L.moe_forward_launch_count(None, 1) == -1
    assert L.moe_reduce_partials(0, None, None, None, None, None, 1, 64, 1e-6, None) == moe.MOE_EINVAL
    arr = (ctypes.c_void_p * 1)(1 << 20)
    assert L.moe_reduce_partials(1, arr, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 4, 100, 1e-6, None) \
        == moe.MOE_EUNSUPPORTED
    assert L.moe_selftest_wait_timeout(0, None) == moe.MOE_EINVAL
    assert L.moe_ep_send_wave(None, 4, None, 0, 1, None, 0, None) == moe.MOE_EINVAL
    assert L.moe_ep_experts_wave(None, 4, None, 0, 1, None, 0, None) == moe.MOE_EINVAL


def test_weight_size_mismatch_is_refused():
    """A weight tensor sized for another configuration (e.g. full-width experts
    under a latent configuration) is refused before the library sees it."""
    import torch
    import deterministic_expert_b200 as moe
    cfg = moe.LayerConfig(D=256, E=8, k=2, I=128, latent=64)
    w = {"w_gate": torch.empty(8 * 128 * 256, dtype=torch.bfloat16)}
    with pytest.raises(ValueError):
        moe.MoELayer(cfg, w)
    w = {"router_bias": torch.empty(8, dtype=torch.bfloat16)}
    with pytest.raises(ValueError):
        moe.MoELayer(cfg, w)


def test_weight_format_and_expert_shard_checks():
    """E4M3 expert weights must be byte tensors (bf16 ones are refused, and
    E4M3 bytes under a bf16 configuration too); an expert-parallel rank's
    routed matrices hold E / ep_world experts, the router all E."""
    import torch
    import deterministic_expert_b200 as moe
    D, E, I = 256, 8, 128
    fp8 = moe.LayerConfig(D=D, E=E, k=2, I=I, weight_format=moe.WEIGHTS_FP8)
    with pytest.raises(ValueError):
        moe.MoELayer(fp8, {"w_gate": torch.empty(E * I * D, dtype=torch.bfloat16)})
    bf16 = moe.LayerConfig(D=D, E=E, k=2, I=I)
    with pytest.raises(ValueError):
        moe.MoELayer(bf16, {"w_gate": torch.empty(E * I * D, dtype=torch.uint8)})
    ep = moe.LayerConfig(D=D, E=E, k=2, I=I, ep_world=4, ep_rank=1)
    with pytest.raises(ValueError):   # all 8 experts given to a rank that holds 2
        moe.MoELayer(ep, {"w_gate": torch.empty(E * I * D, dtype=torch.bfloat16)})
    with pytest.raises(ValueError):   # the router is whole on every rank
        moe.MoELayer(ep, {"w_router": torch.empty(2 * D, dtype=torch.bfloat16)})
    # Packed FP4 storage: half a byte per weight, one int32 exponent word per 128.
    fp4 = moe.LayerConfig(D=D, E=E, k=2, I=I, weight_format=moe.WEIGHTS_FP4)
    with pytest.raises(ValueError):   # E4M3 bytes (one per weight) are not the packed form
        moe.MoELayer(fp4, {"w_gate": torch.empty(E * I * D, dtype=torch.uint8)})
    with pytest.raises(ValueError):   # exponent words of the wrong count
        moe.MoELayer(fp4, {"w_gate_exp": torch.empty(E * I * D // 64, dtype=torch.int32)})
    with pytest.raises(ValueError):   # ... or type
        moe.MoELayer(fp4, {"w_gate_exp": torch.empty(E * I * D // 128, dtype=torch.uint8)})


def test_header_is_plain_c_and_links(tmp_path):
    """include/moe.h compiles as C99 and a C program links against libmoe.so
    and calls entry points that need no GPU (status strings, argument
    checks): the boundary is a real C ABI, not a Python-only one."""
    import os
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "moe.h"
int main(void) {
  moe_config cfg;
  moe_weights w;
  moe_handle* h = 0;
  memset(&cfg, 0, sizeof cfg);
  memset(&w, 0, sizeof w);
  if (strcmp(moe_status_string(MOE_OK), "ok") != 0) return 1;
  if (moe_init(&cfg, &w, &h) != MOE_EINVAL || h != 0) return 2;       /* D = 0: refused before CUDA */
  if (moe_workspace_size(0, 16) != 0) return 3;
  if (moe_ep_exchange_size(0) != 0) return 4;
  if (moe_quantize_weights_fp4(0, 0, 0, 1, 32, 0) != MOE_EINVAL) return 5;
  printf("%s\n", moe_status_string(MOE_EINDEX));
  return 0;
}
''')
    lib_dir = os.path.dirname(moe.LIB_PATH)
    inc = os.path.dirname(moe.HEADER_PATH)
    exe = tmp_path / "abi"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", inc, str(src), "-o", str(exe),
                           "-L", lib_dir, "-l:libmoe.so", "-Wl,-rpath," + lib_dir])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, (out.returncode, out.stderr)
    assert "index" in out.stdout


def test_ctypes_structs_match_the_c_layout(tmp_path):
    """The binding's ctypes mirrors of moe_config, moe_weights, moe_views and
    moe_ep_peers have the C structs' size and every field's offset."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    structs = {"moe_config": moe.moe_config, "moe_weights": moe.moe_weights, "moe_views": moe.moe_views,
               "moe_ep_peers": moe.moe_ep_peers}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "moe.h"', "int main(void) {"]
    for cname, ct in structs.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in ct._fields_:
            lines.append(f'  printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    import os
    subprocess.check_call(["gcc", "-std=c99", "-I", os.path.dirname(moe.HEADER_PATH), str(src), "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    got = {tuple(l.split()[:2]): int(l.split()[2]) for l in out if l.strip()}
    for cname, ct in structs.items():
        assert got[(cname, "size")] == ctypes.sizeof(ct), cname
        for fname, _ in ct._fields_:
            assert got[(cname, fname)] == getattr(ct, fname).offset, (cname, fname)


def test_binding_argument_counts_match_the_header():
    """Every ctypes argtypes list in the binding has as many entries as the
    header declares parameters for that entry point."""
    import inspect
    with open(moe.HEADER_PATH) as f:
        hdr = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    decl = {}
    for m in re.finditer(r"^\s*(?:int|size_t|const char\*)\s+(moe_\w+)\s*\(([^;]*?)\)\s*;", hdr, flags=re.M | re.S):
        decl[m.group(1)] = len([p for p in m.group(2).split(",") if p.strip() and p.strip() != "void"])
    src = inspect.getsource(moe)
    # "L.moe_x.argtypes = [...]" and "fn = L.moe_x" followed by "fn.argtypes = [...]"
    found = {}
    for m in re.finditer(r"\.(moe_\w+)\.argtypes\s*=\s*\[|fn = L\.(moe_\w+)\n(?:.*\n){0,3}?\s*fn\.argtypes\s*=\s*\[", src):
        name = m.group(1) or m.group(2)
        i, depth = m.end(), 1
        while depth:
            depth += {"[": 1, "]": -1}.get(src[i], 0)
            i += 1
        body = src[m.end():i - 1]
        found[name] = len([x for x in re.split(r",(?![^\[]*\])", body) if x.strip()])
    assert len(found) >= 25
    for name, n in found.items():
        assert decl.get(name) == n, (name, n, decl.get(name))
