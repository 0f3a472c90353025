"""The C-ABI library loads, exports every function include/ssd.h declares,
and rejects bad arguments before touching the device (CPU only: no call here
reaches a kernel launch)."""
import ctypes
import os
import re

import pytest

from selective_state_space_43_b200 import build as build_mod
from selective_state_space_43_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build_mod.build()
    return ops.lib()


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names.update(re.findall(r"SSD_API\s+[\w\s\*]+?\b(ssd_\w+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("ssd_prefill", "ssd_decode_step", "ssd_prefill_workspace_bytes", "ssd_status_string"):
        assert required in names


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), f"{name} declared in include/ but not exported"


def test_status_strings_and_version(L):
    for code in range(0, 10):
        assert L.ssd_status_string(code) and L.ssd_status_string(code) != b"unknown status"
    assert b"sm_100a" in L.ssd_version()


def dims(**kw):
    base = dict(batch=1, seqlen=4096, nheads=128, headdim=64, d_state=128, ngroups=8, chunk=128)
    base.update(kw)
    return ops.make_dims(**base)


def test_path_and_workspace_queries(L):
    import torch
    d = dims()
    path = ops.prefill_path(d, torch.bfloat16)
    assert path in (1, 2)
    ws = ops.prefill_workspace_bytes(d, torch.bfloat16)
    if path == 1:
        assert ws == 1 * 4096 * 2 * 8 * 128 * 2
    else:
        assert ws == 0
    assert ops.prefill_path(dims(headdim=32), torch.bfloat16) == -2
    assert ops.prefill_path(dims(nheads=12, ngroups=8), torch.bfloat16) == -2
    assert ops.prefill_path(dims(chunk=96), torch.bfloat16) == -2
    assert ops.prefill_path(dims(d_state=48), torch.bfloat16) == -2
    # fp32 activations and small shapes always take the CUDA-core path
    assert ops.prefill_path(dims(d_state=32, chunk=64, nheads=4, ngroups=1), torch.float32) == 2
    # bf16 with P = 64, d_state 64 or 128, chunk 64 or 128 and nheads a multiple of 8: tensor cores
    for N in (64, 128):
        for Q in (64, 128):
            assert ops.prefill_path(dims(d_state=N, chunk=Q), torch.bfloat16) == 1, (N, Q)
            assert ops.prefill_path(dims(d_state=N, chunk=Q), torch.float32) == 2
    assert ops.prefill_path(dims(d_state=32), torch.bfloat16) == 2
    assert ops.prefill_path(dims(d_state=16), torch.bfloat16) == 2
    assert ops.prefill_path(dims(nheads=12, ngroups=4), torch.bfloat16) == 2
    assert ops.prefill_workspace_bytes(dims(headdim=32), torch.bfloat16) == 0


def _fake_params():
    # 16-byte aligned fake addresses: every call below fails validation first
    return ops.SsdParams(0x1000, 0x2000, 0x3000, 0x4000, 0x5000)


def _call_prefill(L, d, dtype=1, params=None, ptrs=None, ws=None, ws_bytes=0):
    p = ptrs or dict(x=0x10000, dt=0x20000, B=0x30000, C=0x40000, z=0x50000, init=None, init_conv=None,
                     y=0x60000, fs=0x70000, cs=0x80000)
    prm = params if params is not None else _fake_params()
    return L.ssd_prefill(ctypes.byref(d), dtype, ctypes.byref(prm) if prm is not False else None,
                         p["x"], p["dt"], p["B"], p["C"], p["z"], p["init"], p["init_conv"], p["y"], p["fs"],
                         p["cs"], ws, ws_bytes, None)


def test_prefill_rejects_bad_arguments_before_launch(L):
    assert L.ssd_prefill(None, 1, None, *([None] * 11), 0, None) == 1
    assert _call_prefill(L, dims(headdim=32)) == 2
    assert _call_prefill(L, dims(d_conv=3) if False else ops.SsdDims(1, 16, 4, 64, 32, 1, 64, 3)) == 2
    assert _call_prefill(L, dims(), dtype=7) == 3
    assert _call_prefill(L, dims(), params=False) == 1
    assert _call_prefill(L, dims(), params=ops.SsdParams(0x1000, 0, 0x3000, 0x4000, 0x5000)) == 1
    assert _call_prefill(L, dims(), params=ops.SsdParams(0x1004, 0x2000, 0x3000, 0x4000, 0x5000)) == 4
    base = dict(x=0x10000, dt=0x20000, B=0x30000, C=0x40000, z=0x50000, init=None, init_conv=None,
                y=0x60000, fs=0x70000, cs=0x80000)
    assert _call_prefill(L, dims(), ptrs={**base, "x": None}) == 1
    assert _call_prefill(L, dims(), ptrs={**base, "fs": None}) == 1
    assert _call_prefill(L, dims(), ptrs={**base, "B": 0x30008}) == 4
    assert _call_prefill(L, dims(), ptrs={**base, "y": base["x"]}) == 5
    assert _call_prefill(L, dims(), ptrs={**base, "init_conv": 0x80000}) == 5
    assert _call_prefill(L, dims(batch=-1)) == 2
    # zero tokens: activations may be NULL, the states may not
    empty = {**base, "x": None, "dt": None, "B": None, "C": None, "z": None, "y": None}
    assert _call_prefill(L, dims(seqlen=0), ptrs={**empty, "fs": None}) == 1
    assert _call_prefill(L, dims(seqlen=0), ptrs={**empty, "cs": None}) == 1
    import torch
    if ops.prefill_path(dims(), torch.bfloat16) == 1:
        assert _call_prefill(L, dims()) == 7                       # no workspace
        assert _call_prefill(L, dims(), ws=0x90000, ws_bytes=16) == 7


def test_decode_rejects_bad_arguments_before_launch(L):
    d = dims(seqlen=1, batch=256)
    prm = _fake_params()
    ok = [0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 0x60000, 0x70000, 0x80000]
    assert L.ssd_decode_step(None, 1, ctypes.byref(prm), *ok, None) == 1
    for i in range(8):
        args = list(ok)
        args[i] = None
        assert L.ssd_decode_step(ctypes.byref(d), 1, ctypes.byref(prm), *args, None) == 1
    args = list(ok)
    args[6] = 0x70004
    assert L.ssd_decode_step(ctypes.byref(d), 1, ctypes.byref(prm), *args, None) == 4
    args = list(ok)
    args[7] = args[0]
    assert L.ssd_decode_step(ctypes.byref(d), 1, ctypes.byref(prm), *args, None) == 5
    bad = dims(nheads=10, ngroups=4)
    assert L.ssd_decode_step(ctypes.byref(bad), 1, ctypes.byref(prm), *ok, None) == 2


def test_timing_hook_requires_both_or_neither(L):
    assert L.ssd_set_timing_events(ctypes.c_void_p(0x10), None) == 1
    assert L.ssd_set_timing_events(None, None) == 0


def _call_varlen(L, d, cu=0x98000, ptrs=None, ws=None, ws_bytes=0, params=None):
    p = ptrs or dict(x=0x10000, dt=0x20000, B=0x30000, C=0x40000, z=0x50000, init=None, init_conv=None,
                     y=0x60000, fs=0x70000, cs=0x80000)
    prm = params if params is not None else _fake_params()
    return L.ssd_prefill_varlen(ctypes.byref(d), 1, ctypes.byref(prm), cu, p["x"], p["dt"], p["B"], p["C"],
                                p["z"], p["init"], p["init_conv"], p["y"], p["fs"], p["cs"], ws, ws_bytes, None)


def test_varlen_rejects_bad_arguments_before_launch(L):
    import torch
    d = dims(batch=32, seqlen=30000)
    assert _call_varlen(L, d, cu=None) == 1                       # offsets required
    assert _call_varlen(L, d, cu=0x98004) == 4                    # int64 offsets: 8-byte aligned
    assert _call_varlen(L, dims(batch=32, seqlen=30000, headdim=32)) == 2
    assert _call_varlen(L, dims(batch=32, seqlen=1 << 31)) == 2   # rows beyond 32-bit tensor-map coordinates
    base = dict(x=0x10000, dt=0x20000, B=0x30000, C=0x40000, z=0x50000, init=None, init_conv=None,
                y=0x60000, fs=0x70000, cs=0x80000)
    assert _call_varlen(L, d, ptrs={**base, "z": None}) == 1
    assert _call_varlen(L, d, ptrs={**base, "y": base["z"]}) == 5
    assert _call_varlen(L, d, ptrs={**base, "cs": 0x80008}) == 4
    if ops.prefill_path(d, torch.bfloat16) == 1:
        need = ops.prefill_varlen_workspace_bytes(d, torch.bfloat16)
        assert need == 30000 * 2 * 8 * 128 * 2                    # post-conv B/C of every row
        assert _call_varlen(L, d) == 7
        assert _call_varlen(L, d, ws=0x90000, ws_bytes=need - 16) == 7
    # fp32 activations take the CUDA-core path, which needs no workspace
    assert ops.prefill_varlen_workspace_bytes(dims(d_state=32, chunk=64, nheads=4, ngroups=1), torch.float32) == 0


def test_strided_prefill_checks_the_row_strides(L):
    d = dims(batch=2, seqlen=300, nheads=16, ngroups=2)
    base = [0x10000, 0x20000, 0x30000, 0x40000, 0x50000, None, None, 0x60000, 0x70000, 0x80000]

    def call(rs):
        return L.ssd_prefill_strided(ctypes.byref(d), 1, ctypes.byref(_fake_params()),
                                     None if rs is None else ctypes.byref(ops.SsdRowStrides(*rs)), *base, None, 0,
                                     None)
    wide = 2 * 1024 + 2 * 256 + 16                      # z | x | B | C | dt per token
    assert call((wide, wide, wide, wide, wide)) == 7    # valid strides: fails only for want of a workspace
    assert call((1000, wide, wide, wide, wide)) == 2    # x rows narrower than H*P
    assert call((wide, wide, 8, wide, wide)) == 2       # dt rows narrower than H
    assert call((wide + 4, wide, wide, wide, wide)) == 4  # not a multiple of 16 bytes
    assert call(None) == 7                              # NULL: contiguous rows, as ssd_prefill


def test_context_parallel_helpers_check_arguments(L):
    d = dims(batch=2, seqlen=300, nheads=16, ngroups=2)
    assert L.ssd_conv_window(None, 1, 0x10000, 0x30000, 0x40000, None, 0x80000, None) == 1
    assert L.ssd_conv_window(ctypes.byref(d), 1, None, 0x30000, 0x40000, None, 0x80000, None) == 1
    assert L.ssd_conv_window(ctypes.byref(d), 1, 0x10000, 0x30008, 0x40000, None, 0x80000, None) == 4
    assert L.ssd_conv_window(ctypes.byref(d), 1, 0x10000, 0x30000, 0x40000, 0x80000, 0x80000, None) == 5
    assert L.ssd_dt_sum(ctypes.byref(d), 1, None, 0x20000, 0x90000, None) == 1
    assert L.ssd_dt_sum(ctypes.byref(dims(headdim=32)), 1, 0x1000, 0x20000, 0x90000, None) == 2
    assert L.ssd_cp_combine(ctypes.byref(d), 4, 5, 0x1000, 0x2000, 0x3000, None, 0x4000, None) == 2  # upto > nseg
    assert L.ssd_cp_combine(ctypes.byref(d), 0, 0, 0x1000, 0x2000, 0x3000, None, 0x4000, None) == 2
    assert L.ssd_cp_combine(ctypes.byref(d), 4, 2, 0x1000, None, 0x3000, None, 0x4000, None) == 1
    assert L.ssd_cp_combine(ctypes.byref(d), 4, 2, 0x1000, 0x2000, 0x3000, 0x4000, 0x4000, None) == 5


def test_gated_rmsnorm_checks_arguments(L):
    f = L.ssd_gated_rmsnorm
    assert f(4, 1024, 3, 1e-5, 1, 0x10000, 0x20000, 0x30000, None) == 2    # groups must divide the channels
    assert f(4, 1020, 2, 1e-5, 1, 0x10000, 0x20000, 0x30000, None) == 2    # group of 510: not a multiple of 8
    assert f(4, 1024, 8, -1.0, 1, 0x10000, 0x20000, 0x30000, None) == 2    # eps < 0
    assert f(4, 1024, 8, 1e-5, 7, 0x10000, 0x20000, 0x30000, None) == 3
    assert f(4, 1024, 8, 1e-5, 1, None, 0x20000, 0x30000, None) == 1
    assert f(4, 1024, 8, 1e-5, 1, 0x10008, 0x20000, 0x30000, None) == 4
    assert f(0, 1024, 8, 1e-5, 1, None, None, None, None) == 0             # no rows: nothing to do


def _call_backward(L, d, dtype=1, params=True, ptrs=None, grads=None, ws=None, ws_bytes=0):
    p = ops.SsdParams(0x1000, 0x2000, 0x3000, 0x4000, 0x5000) if params is True else (params or None)
    ptrs = ptrs or dict(x=0x10000, dt=0x20000, B=0x30000, C=0x40000, z=0x50000, init=None, init_conv=None,
                        dy=0x60000, dfin=None)
    g = ops.SsdGrads(*([0x100000 * (k + 1) for k in range(10)] + [None, None])) if grads is None else grads
    return L.ssd_prefill_backward(ctypes.byref(d), dtype, ctypes.byref(p) if p else None, ptrs["x"], ptrs["dt"],
                                  ptrs["B"], ptrs["C"], ptrs["z"], ptrs["init"], ptrs["init_conv"], ptrs["dy"],
                                  ptrs["dfin"], ctypes.byref(g) if g is not False else None, ws, ws_bytes, None)


def test_backward_rejects_bad_arguments_before_launch(L):
    small = dims(seqlen=16, nheads=4, d_state=32, ngroups=1)
    # post-conv channels and their gradients, dt and its cumsum, two chunk-state arrays and the partials
    conv_dim = 4 * 64 + 2 * 32
    assert L.ssd_prefill_backward_workspace_bytes(ctypes.byref(small)) >= 4 * (
        2 * 16 * conv_dim + 2 * 4 * 16 + 2 * 1 * 4 * 64 * 32)
    d = dims()
    need = L.ssd_prefill_backward_workspace_bytes(ctypes.byref(d))
    assert L.ssd_prefill_backward_workspace_bytes(ctypes.byref(dims(headdim=32))) == 0
    assert L.ssd_prefill_backward(None, 1, None, *([None] * 9), None, None, 0, None) == 1
    assert _call_backward(L, dims(headdim=32)) == 2
    assert _call_backward(L, d, dtype=7) == 3
    assert _call_backward(L, d, params=False) == 1
    assert _call_backward(L, d, grads=False) == 1
    base = dict(x=0x10000, dt=0x20000, B=0x30000, C=0x40000, z=0x50000, init=None, init_conv=None, dy=0x60000,
                dfin=None)
    assert _call_backward(L, d, ptrs={**base, "dy": None}) == 1
    assert _call_backward(L, d, ptrs={**base, "z": 0x50004}) == 4
    missing = ops.SsdGrads(*([0x100000 * (k + 1) for k in range(4)] + [None] + [0x600000] * 5 + [None, None]))
    assert _call_backward(L, d, grads=missing) == 1                      # dz is required
    odd = ops.SsdGrads(*([0x100000 * (k + 1) for k in range(10)] + [0x100008, None]))
    assert _call_backward(L, d, grads=odd) == 4                          # d_init_state misaligned
    assert _call_backward(L, d) == 7                                     # no workspace
    assert _call_backward(L, d, ws=0x900000, ws_bytes=need - 1) == 7
    assert _call_backward(L, dims(seqlen=64 * 65536)) == 2               # beyond the chunk grid
    # zero tokens: the activations and per-token gradients may be NULL, the parameter gradients may not
    none_act = {**base, "x": None, "dt": None, "B": None, "C": None, "z": None, "dy": None}
    no_param = ops.SsdGrads(*([None] * 5 + [0x100000] * 4 + [None] + [None, None]))
    assert _call_backward(L, dims(seqlen=0), ptrs=none_act, grads=no_param) == 1


def _call_mimo(L, d, rank=4, dtype=1, params=True, ptrs=None):
    p = ops.SsdParams(0x1000, 0x2000, 0x3000, None, None) if params is True else params
    q = ptrs or dict(x=0x10000, dt=0x20000, B=0x30000, C=0x40000, z=0x50000, S=0x60000, y=0x70000)
    return L.ssd_mimo_decode_step(ctypes.byref(d), rank, dtype, ctypes.byref(p) if p else None, q["x"], q["dt"],
                                  q["B"], q["C"], q["z"], q["S"], q["y"], None)


def test_mimo_decode_rejects_bad_arguments_before_launch(L):
    d = dims(batch=256, seqlen=1)
    assert _call_mimo(L, d, rank=3) == 2
    assert _call_mimo(L, d, rank=16) == 2
    assert _call_mimo(L, dims(headdim=32), rank=4) == 2
    assert _call_mimo(L, d, dtype=9) == 3
    assert _call_mimo(L, d, params=None) == 1
    assert _call_mimo(L, d, params=ops.SsdParams(0x1000, None, 0x3000, None, None)) == 1
    assert _call_mimo(L, d, params=ops.SsdParams(0x1008, 0x2000, 0x3000, None, None)) == 4
    base = dict(x=0x10000, dt=0x20000, B=0x30000, C=0x40000, z=0x50000, S=0x60000, y=0x70000)
    assert _call_mimo(L, d, ptrs={**base, "S": None}) == 1
    assert _call_mimo(L, d, ptrs={**base, "C": 0x40004}) == 4
    assert _call_mimo(L, d, ptrs={**base, "y": base["z"]}) == 5
    # no sequences: nothing to do, valid
    assert _call_mimo(L, dims(batch=0, seqlen=1)) == 0


def test_backward_rejects_overlapping_gradients(L):
    d = dims(seqlen=64, nheads=4, d_state=32, ngroups=1)
    need = L.ssd_prefill_backward_workspace_bytes(ctypes.byref(d))
    rows, HP = 64, 256
    base = dict(x=0x1000000, dt=0x2000000, B=0x3000000, C=0x4000000, z=0x5000000, init=None, init_conv=None,
                dy=0x6000000, dfin=None)
    ws = 0x40000000
    ok = [0x10000000 + 0x1000000 * k for k in range(10)] + [None, None]
    # every call below overlaps two ranges, so it fails validation before any launch
    g = list(ok)
    g[0] = base["x"] + 64                                   # dx inside x
    assert _call_backward(L, d, ptrs=base, grads=ops.SsdGrads(*g), ws=ws, ws_bytes=need) == 5
    g = list(ok)
    g[6] = g[5]                                             # dD == dA
    assert _call_backward(L, d, ptrs=base, grads=ops.SsdGrads(*g), ws=ws, ws_bytes=need) == 5
    g = list(ok)
    g[10] = ws + 256                                        # d_init_state inside the workspace
    assert _call_backward(L, d, ptrs=base, grads=ops.SsdGrads(*g), ws=ws, ws_bytes=need) == 5
    g = list(ok)
    g[4] = ok[0] + rows * HP * 4 - 16                       # dz starts 16 bytes before the end of dx
    assert _call_backward(L, d, ptrs=base, grads=ops.SsdGrads(*g), ws=ws, ws_bytes=need) == 5


def test_mimo_rejects_an_overlapping_output(L):
    d = dims(batch=2, seqlen=1, nheads=4, d_state=32, ngroups=1)
    base = dict(x=0x1000000, dt=0x2000000, B=0x3000000, C=0x4000000, z=0x5000000, S=0x6000000, y=0x7000000)
    assert _call_mimo(L, d, ptrs={**base, "y": base["S"] + 1024}) == 5
    assert _call_mimo(L, d, ptrs={**base, "y": base["B"]}) == 5


def test_binding_checks_tensors_before_calling_the_library(L):
    import torch
    from selective_state_space_43_b200.synth import Dims, make_backward_grads, make_mimo_decode_inputs, \
        make_prefill_inputs
    d = Dims(1, 32, 4, 64, 16, 2, 64)
    inp = make_prefill_inputs(d, dtype=torch.bfloat16, seed=1)
    gr = make_backward_grads(d, seed=2)
    args = [inp[k] for k in ("x", "dt", "B", "C", "z", "A", "D", "dt_bias", "conv_w", "conv_b")]
    # host tensors are refused: there is no CPU path
    with pytest.raises(ValueError, match="must be on"):
        ops.prefill_backward(*args, gr["dy"])
    data = make_mimo_decode_inputs(d, 2, 1, dtype=torch.bfloat16, seed=3)
    s = data["steps"][0]
    with pytest.raises(ValueError, match="must be on"):
        ops.mimo_decode_step(s["x"], s["dt"], s["B"], s["C"], s["z"], data["params"]["A"], data["params"]["D"],
                             data["params"]["dt_bias"], data["ssm_state"])
    with pytest.raises(ValueError, match="must be on"):
        ops.prefill(*args)
