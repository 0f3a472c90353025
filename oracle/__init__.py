"""fp64 CPU oracle of the Mamba-2 SSD layer core (TEST INFRASTRUCTURE ONLY).

Only the tests, the package smoke check and the benchmark's CPU-baseline /
reference legs may import this package.  The product path (the CUDA library
and its Python binding) never does.

The arithmetic lives in ``ssd_oracle.c`` (plain C, double precision, the
token-by-token recurrence); this file compiles it with gcc on first use and
passes numpy float64 arrays to it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB = os.path.join(_HERE, "libssd_oracle.so")
_lib = None


class _Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_long), ("seqlen", ctypes.c_long), ("nheads", ctypes.c_int),
                ("headdim", ctypes.c_int), ("d_state", ctypes.c_int), ("ngroups", ctypes.c_int)]


def build(force: bool = False) -> str:
    """Compile ssd_oracle.c into libssd_oracle.so next to it (plain gcc -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-shared", "-fPIC", "-pthread", "-o", tmp, _SRC,
                               "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _bind(lib):
    dp = ctypes.POINTER(ctypes.c_double)
    lib.oracle_conv_silu.argtypes = [ctypes.c_long, dp, ctypes.c_long, dp, dp, ctypes.c_double, dp]
    lib.oracle_prefill.argtypes = [ctypes.POINTER(_Dims)] + [dp] * 12 + [ctypes.c_void_p] + [dp] * 3 + [
        ctypes.c_int]
    lib.oracle_decode_step.argtypes = [ctypes.POINTER(_Dims)] + [dp] * 12 + [ctypes.c_void_p, dp]
    if hasattr(lib, "oracle_mimo_decode_step"):
        lib.oracle_mimo_decode_step.argtypes = [ctypes.POINTER(_Dims), ctypes.c_int] + [dp] * 10
    if hasattr(lib, "oracle_prefill_backward"):
        lib.oracle_prefill_backward.argtypes = [ctypes.POINTER(_Dims)] + [dp] * 26 + [ctypes.c_int]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def use_library(path: str | None):
    """Point the wrappers at another compiled copy of ssd_oracle.c (None = the
    default one).  Used by the test that plants mistakes in the oracle to check
    that its pins catch them."""
    global _lib
    _lib = None if path is None else _bind(ctypes.CDLL(path))


def _f64(a):
    """Widen an array (numpy or torch, any float dtype) to a contiguous float64 numpy array (exact)."""
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _dims(batch, seqlen, nheads, headdim, d_state, ngroups):
    return _Dims(int(batch), int(seqlen), int(nheads), int(headdim), int(d_state), int(ngroups))


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def conv_silu(seq, hist, w, b):
    """silu(b + sum_k w[k] * seq[t-3+k]) for one channel; hist = tokens -3..-1 or None."""
    seq = _f64(seq)
    hist = _f64(hist)
    w = _f64(w)
    out = np.empty(seq.shape[0], dtype=np.float64)
    _load().oracle_conv_silu(seq.shape[0], _ptr(seq), 1, _ptr(hist), _ptr(w), float(b), _ptr(out))
    return out


def prefill(inp: dict, unit_mask=None, nthreads: int | None = None):
    """Token-by-token fp64 prefill.  ``inp`` holds x, dt, B, C, z, A, D, dt_bias,
    conv_w, conv_b, init_state (or None), init_conv_state (or None) with the
    layouts x/z [Bt, L, H*P], dt [Bt, L, H], B/C [Bt, L, G, N].

    ``unit_mask`` (bool [Bt, H]) restricts the work to some (b, h) pairs; the
    other entries of y and final_state come back as NaN.
    Returns (y [Bt, L, H*P], final_state [Bt, H, P, N], conv_state [Bt, conv_dim, 3]).
    """
    x = _f64(inp["x"])
    Bt, L, HP = x.shape
    Bm = _f64(inp["B"])
    G, N = Bm.shape[2], Bm.shape[3]
    H = inp["A"].shape[0]
    P = HP // H
    d = _dims(Bt, L, H, P, N, G)
    arrs = [x, _f64(inp["dt"]), Bm, _f64(inp["C"]), _f64(inp["z"]), _f64(inp["A"]), _f64(inp["D"]),
            _f64(inp["dt_bias"]), _f64(inp["conv_w"]), _f64(inp["conv_b"]), _f64(inp.get("init_state")),
            _f64(inp.get("init_conv_state"))]
    mask = None
    if unit_mask is not None:
        mask = np.ascontiguousarray(np.asarray(unit_mask, dtype=np.uint8).reshape(Bt * H))
    y = np.full((Bt, L, HP), np.nan)
    fs = np.full((Bt, H, P, N), np.nan)
    cs = np.empty((Bt, HP + 2 * G * N, 3))
    _load().oracle_prefill(ctypes.byref(d), *[_ptr(a) for a in arrs],
                           None if mask is None else mask.ctypes.data_as(ctypes.c_void_p),
                           _ptr(y), _ptr(fs), _ptr(cs), int(nthreads or default_threads()))
    return y, fs, cs


def prefill_varlen(inp: dict, cu_seqlens, nthreads: int | None = None):
    """Packed variable-length prefill: x/z [T, H*P], dt [T, H], B/C [T, G, N], init_state
    [nseq, H, P, N] or None, init_conv_state [nseq, conv_dim, 3] or None; sequence s is rows
    cu_seqlens[s] .. cu_seqlens[s+1]-1.  Each sequence is an independent prefill from its own
    initial states (the per-sequence chunked prefill of serving stacks, "EP6" survey, vLLM
    section), so this is ``prefill`` run on each slice.
    Returns (y [T, H*P], final_state [nseq, H, P, N], conv_state [nseq, conv_dim, 3]).
    """
    cu = [int(v) for v in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    x = _f64(inp["x"])
    T, HP = x.shape
    G, N = inp["B"].shape[1], inp["B"].shape[2]
    H = inp["A"].shape[0]
    P = HP // H
    nseq = len(cu) - 1
    y = np.empty((T, HP))
    fs = np.empty((nseq, H, P, N))
    cs = np.empty((nseq, HP + 2 * G * N, 3))
    params = {k: inp[k] for k in ("A", "D", "dt_bias", "conv_w", "conv_b")}
    for s in range(nseq):
        r0, r1 = cu[s], cu[s + 1]
        one = dict(params)
        for k in ("x", "dt", "B", "C", "z"):
            one[k] = _f64(inp[k])[r0:r1][None]
        for k in ("init_state", "init_conv_state"):
            one[k] = None if inp.get(k) is None else _f64(inp[k])[s:s + 1]
        ys, fss, css = prefill(one, nthreads=nthreads)
        y[r0:r1] = ys[0]
        fs[s] = fss[0]
        cs[s] = css[0]
    return y, fs, cs


def decode_step(step: dict, params: dict, conv_state, ssm_state, unit_mask=None):
    """One fp64 decode step.  ``conv_state`` and ``ssm_state`` must be float64
    numpy arrays; they are updated in place.  Returns y [Bt, H*P]."""
    assert conv_state.dtype == np.float64 and conv_state.flags.c_contiguous
    assert ssm_state.dtype == np.float64 and ssm_state.flags.c_contiguous
    x = _f64(step["x"])
    Bt, HP = x.shape
    Bm = _f64(step["B"])
    G, N = Bm.shape[1], Bm.shape[2]
    H = params["A"].shape[0]
    P = HP // H
    d = _dims(Bt, 1, H, P, N, G)
    arrs = [x, _f64(step["dt"]), Bm, _f64(step["C"]), _f64(step["z"]), _f64(params["A"]), _f64(params["D"]),
            _f64(params["dt_bias"]), _f64(params["conv_w"]), _f64(params["conv_b"]), conv_state, ssm_state]
    mask = None
    if unit_mask is not None:
        mask = np.ascontiguousarray(np.asarray(unit_mask, dtype=np.uint8).reshape(Bt * H))
    y = np.full((Bt, HP), np.nan)
    _load().oracle_decode_step(ctypes.byref(d), *[_ptr(a) for a in arrs],
                               None if mask is None else mask.ctypes.data_as(ctypes.c_void_p), _ptr(y))
    return y


def prefill_backward(inp: dict, dy, d_final=None, nthreads: int | None = None):
    """Gradients of the fp64 prefill (the adjoint of the token-by-token recurrence, for training:
    "Nemotron-H 스타일 Hybrid Mamba-Transformer 3B 모델 구현 타당성 분석" §3.1/§3.2 checks the new
    Mamba-2 layer's forward and backward).  The loss whose gradients are returned is
    sum(dy * y) + sum(d_final * final_state), y and final_state from ``prefill(inp)``; the conv_state
    output carries none.  ``inp`` as for ``prefill``; dy [Bt, L, H*P]; d_final [Bt, H, P, N] or None.
    Returns a dict of float64 arrays shaped like the inputs they belong to: x, z, dt, B, C (B/C as
    [Bt, L, G, N]), A, D, dt_bias, conv_w, conv_b, init_state, init_conv_state (the last two are the
    gradients for the given initial states, or for zero ones when they are None).
    """
    x = _f64(inp["x"])
    Bt, L, HP = x.shape
    Bm = _f64(inp["B"])
    G, N = Bm.shape[2], Bm.shape[3]
    H = inp["A"].shape[0]
    P = HP // H
    conv_dim = HP + 2 * G * N
    d = _dims(Bt, L, H, P, N, G)
    arrs = [x, _f64(inp["dt"]), Bm, _f64(inp["C"]), _f64(inp["z"]), _f64(inp["A"]), _f64(inp["D"]),
            _f64(inp["dt_bias"]), _f64(inp["conv_w"]), _f64(inp["conv_b"]), _f64(inp.get("init_state")),
            _f64(inp.get("init_conv_state")), _f64(dy), _f64(d_final)]
    out = {"x": np.empty((Bt, L, HP)), "dt": np.empty((Bt, L, H)), "B": np.empty((Bt, L, G, N)),
           "C": np.empty((Bt, L, G, N)), "z": np.empty((Bt, L, HP)), "A": np.empty(H), "D": np.empty(H),
           "dt_bias": np.empty(H), "conv_w": np.empty((conv_dim, 4)), "conv_b": np.empty(conv_dim),
           "init_state": np.empty((Bt, H, P, N)), "init_conv_state": np.empty((Bt, conv_dim, 3))}
    order = ("x", "dt", "B", "C", "z", "A", "D", "dt_bias", "conv_w", "conv_b", "init_state", "init_conv_state")
    _load().oracle_prefill_backward(ctypes.byref(d), *[_ptr(a) for a in arrs], *[_ptr(out[k]) for k in order],
                                    int(nthreads or default_threads()))
    return out


def mimo_decode_step(step: dict, params: dict, ssm_state):
    """One fp64 MIMO decode step (Mamba-3's multi-input multi-output SSM on the Mamba-2 scalar decay, no
    short conv; "Mamba-3: 추론을 우선한 상태 공간 모델", opening section and 아키텍처).  step holds x, z
    [Bt, H, R, P], dt [Bt, H], B, C [Bt, G, R, N]; params A, D, dt_bias [H].  ``ssm_state`` (float64
    [Bt, H, P, N], C-contiguous) is updated in place.  Returns y [Bt, H, R, P]."""
    assert ssm_state.dtype == np.float64 and ssm_state.flags.c_contiguous
    x = _f64(step["x"])
    Bt, H, R, P = x.shape
    Bm = _f64(step["B"])
    G, N = Bm.shape[1], Bm.shape[3]
    d = _dims(Bt, 1, H, P, N, G)
    y = np.empty((Bt, H, R, P))
    arrs = [x, _f64(step["dt"]), Bm, _f64(step["C"]), _f64(step["z"]), _f64(params["A"]), _f64(params["D"]),
            _f64(params["dt_bias"]), ssm_state, y]
    _load().oracle_mimo_decode_step(ctypes.byref(d), int(R), *[_ptr(a) for a in arrs])
    return y


def gated_rmsnorm(y, weight, ngroups: int, eps: float = 1e-5):
    """RMSNorm of the gated output, as the norm that Mamba-2 blocks apply before their output
    projection (the "Mamba-3: 추론을 우선한 상태 공간 모델" page, 정규화 section, keeps it for hybrid
    models and names its variants: before or after the gate, grouped or over all channels).  Reading
    taken: after the SiLU(z) gate, over ``ngroups`` contiguous channel groups (1 = all channels):
    out = v / sqrt(mean over the group of v^2 + eps) * weight, v = the gated y of ``prefill``.
    y [..., H*P], weight [H*P].  Plain fp64 definition."""
    v = _f64(y)
    w = _f64(weight)
    shp = v.shape
    g = v.reshape(shp[:-1] + (ngroups, shp[-1] // ngroups))
    ms = np.mean(g * g, axis=-1, keepdims=True)
    return (g / np.sqrt(ms + eps)).reshape(shp) * w
