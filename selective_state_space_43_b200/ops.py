"""Thin ctypes binding of the C ABI in include/ssd.h.

Argument marshalling only: every step of the layer runs in the CUDA library
(libssd_b200.so).  Tensors are checked for device, dtype, shape and
contiguity, then their data pointers and torch's current CUDA stream are
passed through.  There is no CPU fallback: if the library is missing or the
tensors are not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssd_b200.so")

SSD_F32, SSD_BF16, SSD_BF16_YF32 = 0, 1, 2
STATUS = {0: "SSD_OK", 1: "SSD_ERR_NULL", 2: "SSD_ERR_SHAPE", 3: "SSD_ERR_DTYPE", 4: "SSD_ERR_ALIGN",
          5: "SSD_ERR_UNSUPPORTED", 6: "SSD_ERR_CUDA", 7: "SSD_ERR_WORKSPACE", 8: "SSD_ERR_TIMEOUT",
          9: "SSD_ERR_RANGE"}


class SsdDims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("nheads", ctypes.c_int32),
                ("headdim", ctypes.c_int32), ("d_state", ctypes.c_int32), ("ngroups", ctypes.c_int32),
                ("chunk", ctypes.c_int32), ("d_conv", ctypes.c_int32)]


class SsdParams(ctypes.Structure):
    _fields_ = [("A", ctypes.c_void_p), ("D", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p),
                ("conv_w", ctypes.c_void_p), ("conv_b", ctypes.c_void_p)]


class SsdRowStrides(ctypes.Structure):
    _fields_ = [("x", ctypes.c_int64), ("z", ctypes.c_int64), ("dt", ctypes.c_int64), ("B", ctypes.c_int64),
                ("C", ctypes.c_int64)]


class SsdGrads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("dx", "ddt", "dB", "dC", "dz", "dA", "dD", "ddt_bias", "dconv_w",
                                               "dconv_b", "d_init_state", "d_init_conv_state")]


class SsdError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)} ({lib().ssd_status_string(status).decode()})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -c 'import __graft_entry__ as g; "
                               "g.build()'` (needs nvcc); there is no CPU fallback")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz = ctypes.c_void_p, ctypes.c_size_t
        dimp, parp = ctypes.POINTER(SsdDims), ctypes.POINTER(SsdParams)
        L.ssd_status_string.restype = ctypes.c_char_p
        L.ssd_status_string.argtypes = [ctypes.c_int]
        L.ssd_version.restype = ctypes.c_char_p
        L.ssd_version.argtypes = []
        L.ssd_prefill_workspace_bytes.restype = sz
        L.ssd_prefill_workspace_bytes.argtypes = [dimp, ctypes.c_int]
        L.ssd_prefill_path.restype = ctypes.c_int
        L.ssd_prefill_path.argtypes = [dimp, ctypes.c_int]
        L.ssd_prefill.restype = ctypes.c_int
        L.ssd_prefill.argtypes = [dimp, ctypes.c_int, parp] + [vp] * 11 + [sz, vp]
        L.ssd_decode_step.restype = ctypes.c_int
        L.ssd_decode_step.argtypes = [dimp, ctypes.c_int, parp] + [vp] * 8 + [vp]
        L.ssd_prefill_varlen_workspace_bytes.restype = sz
        L.ssd_prefill_varlen_workspace_bytes.argtypes = [dimp, ctypes.c_int]
        L.ssd_prefill_varlen.restype = ctypes.c_int
        L.ssd_prefill_varlen.argtypes = [dimp, ctypes.c_int, parp] + [vp] * 12 + [sz, vp]
        L.ssd_prefill_strided.restype = ctypes.c_int
        L.ssd_prefill_strided.argtypes = [dimp, ctypes.c_int, parp, ctypes.POINTER(SsdRowStrides)] + [vp] * 11 + [sz, vp]
        L.ssd_conv_window.restype = ctypes.c_int
        L.ssd_conv_window.argtypes = [dimp, ctypes.c_int] + [vp] * 5 + [vp]
        L.ssd_dt_sum.restype = ctypes.c_int
        L.ssd_dt_sum.argtypes = [dimp, ctypes.c_int, vp, vp, vp, vp]
        L.ssd_cp_combine.restype = ctypes.c_int
        L.ssd_cp_combine.argtypes = [dimp, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp, vp, vp]
        L.ssd_gated_rmsnorm.restype = ctypes.c_int
        L.ssd_gated_rmsnorm.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_float, ctypes.c_int,
                                        vp, vp, vp, vp]
        L.ssd_prefill_noalloc.restype = ctypes.c_int
        L.ssd_prefill_noalloc.argtypes = [dimp, ctypes.c_int, parp] + [vp] * 10 + [vp]
        L.ssd_prefill_backward_workspace_bytes.restype = sz
        L.ssd_prefill_backward_workspace_bytes.argtypes = [dimp]
        L.ssd_prefill_backward.restype = ctypes.c_int
        L.ssd_prefill_backward.argtypes = [dimp, ctypes.c_int, parp] + [vp] * 9 + [ctypes.POINTER(SsdGrads)] + [
            vp, sz, vp]
        L.ssd_mimo_decode_step.restype = ctypes.c_int
        L.ssd_mimo_decode_step.argtypes = [dimp, ctypes.c_int32, ctypes.c_int, parp] + [vp] * 7 + [vp]
        L.ssd_device_status.restype = ctypes.c_int
        L.ssd_device_status.argtypes = [vp]
        L.ssd_test_stall_prefill.restype = ctypes.c_int
        L.ssd_test_stall_prefill.argtypes = [ctypes.c_uint64]
        L.ssd_set_timing_events.restype = ctypes.c_int
        L.ssd_set_timing_events.argtypes = [vp, vp]
        _lib = L
    return _lib


def _dtype_code(t: torch.Tensor, y_dtype: torch.dtype) -> int:
    if t.dtype == torch.bfloat16:
        if y_dtype == torch.bfloat16:
            return SSD_BF16
        if y_dtype == torch.float32:
            return SSD_BF16_YF32
    elif t.dtype == torch.float32 and y_dtype == torch.float32:
        return SSD_F32
    raise TypeError(f"unsupported activation / output dtypes {t.dtype} / {y_dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(t, name, shape, dtype, device):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _row_stride(t, name, shape, dtype, device) -> int:
    """Elements between consecutive tokens of a [Bt, L, ...] input.  Contiguous tensors, and views
    whose per-token part is contiguous with batches L rows apart (e.g. slices of a block's in_proj
    output), are accepted; the library reads the views in place."""
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    width = 1
    for n in shape[2:]:
        width *= n
    if t.is_contiguous():
        return width
    expect = 1
    for dim in range(t.dim() - 1, 1, -1):
        if t.shape[dim] > 1 and t.stride(dim) != expect:
            raise ValueError(f"{name}: the elements of one token must be contiguous")
        expect *= t.shape[dim]
    Bt, L = shape[0], shape[1]
    rs = t.stride(1) if L > 1 else (t.stride(0) if Bt > 1 else width)
    if Bt > 1 and L > 1 and t.stride(0) != L * rs:
        raise ValueError(f"{name}: consecutive sequences must be seqlen rows apart")
    return rs


def _stream_ptr(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def make_dims(batch, seqlen, nheads, headdim, d_state, ngroups, chunk=128) -> SsdDims:
    return SsdDims(int(batch), int(seqlen), int(nheads), int(headdim), int(d_state), int(ngroups), int(chunk), 4)


def prefill_workspace_bytes(dims: SsdDims, dtype: torch.dtype) -> int:
    return int(lib().ssd_prefill_workspace_bytes(ctypes.byref(dims), SSD_BF16 if dtype == torch.bfloat16 else
                                                  SSD_F32))


def prefill_path(dims: SsdDims, dtype: torch.dtype) -> int:
    """1 = tcgen05 tensor-core path, 2 = CUDA-core path, <0 = invalid sizes."""
    return int(lib().ssd_prefill_path(ctypes.byref(dims), SSD_BF16 if dtype == torch.bfloat16 else SSD_F32))


def _params(A, D, dt_bias, conv_w, conv_b, H, conv_dim, device):
    for name, t, shp in (("A", A, (H,)), ("D", D, (H,)), ("dt_bias", dt_bias, (H,)),
                         ("conv_w", conv_w, (conv_dim, 4)), ("conv_b", conv_b, (conv_dim,))):
        _check(t, name, shp, torch.float32, device)
    return SsdParams(A.data_ptr(), D.data_ptr(), dt_bias.data_ptr(), conv_w.data_ptr(), conv_b.data_ptr())


def prefill(x, dt, B, C, z, A, D, dt_bias, conv_w, conv_b, init_state=None, init_conv_state=None, chunk=128,
            workspace=None, y=None, final_state=None, conv_state=None, y_dtype=None):
    """Chunked SSD prefill on the GPU.

    x, z [Bt, L, H*P]; dt [Bt, L, H]; B, C [Bt, L, G, N] (bf16 or fp32, one dtype), contiguous or
    views with strided rows (e.g. slices of the in_proj output [Bt, L, z | x | B | C | dt]);
    A, D, dt_bias [H], conv_w [conv_dim, 4], conv_b [conv_dim] fp32;
    init_state [Bt, H, P, N] fp32 or None; init_conv_state [Bt, conv_dim, 3] or None.
    y_dtype: the dtype of y (default: the activation dtype; float32 with bf16
    activations gives the unrounded fp32 y of the same computation).
    Returns (y, final_state, conv_state).
    """
    dev = x.device
    Bt, L, HP = x.shape
    H = A.shape[0]
    P = HP // H
    G, N = B.shape[2], B.shape[3]
    act = x.dtype
    conv_dim = HP + 2 * G * N
    rs = SsdRowStrides(*[_row_stride(t, name, shp, act, dev) for name, t, shp in (
        ("x", x, (Bt, L, HP)), ("z", z, (Bt, L, HP)), ("dt", dt, (Bt, L, H)), ("B", B, (Bt, L, G, N)),
        ("C", C, (Bt, L, G, N)))])
    strided = (rs.x, rs.z, rs.dt, rs.B, rs.C) != (HP, HP, H, G * N, G * N)
    if init_state is not None:
        _check(init_state, "init_state", (Bt, H, P, N), torch.float32, dev)
    if init_conv_state is not None:
        _check(init_conv_state, "init_conv_state", (Bt, conv_dim, 3), act, dev)
    params = _params(A, D, dt_bias, conv_w, conv_b, H, conv_dim, dev)
    dims = make_dims(Bt, L, H, P, N, G, chunk)
    ydt = y_dtype or (y.dtype if y is not None else act)
    code = _dtype_code(x, ydt)
    if y is None:
        y = torch.empty((Bt, L, HP), dtype=ydt, device=dev)
    if final_state is None:
        final_state = torch.empty((Bt, H, P, N), dtype=torch.float32, device=dev)
    if conv_state is None:
        conv_state = torch.empty((Bt, conv_dim, 3), dtype=act, device=dev)
    _check(y, "y", (Bt, L, HP), ydt, dev)
    _check(final_state, "final_state", (Bt, H, P, N), torch.float32, dev)
    _check(conv_state, "conv_state", (Bt, conv_dim, 3), act, dev)
    need = prefill_workspace_bytes(dims, act)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    args = (_ptr(x), _ptr(dt), _ptr(B), _ptr(C), _ptr(z), _ptr(init_state), _ptr(init_conv_state), _ptr(y),
            _ptr(final_state), _ptr(conv_state), _ptr(workspace), ws_bytes, _stream_ptr(dev))
    if strided:
        st = lib().ssd_prefill_strided(ctypes.byref(dims), code, ctypes.byref(params), ctypes.byref(rs), *args)
    else:
        st = lib().ssd_prefill(ctypes.byref(dims), code, ctypes.byref(params), *args)
    if st != 0:
        raise SsdError(st, "ssd_prefill_strided" if strided else "ssd_prefill")
    return y, final_state, conv_state


def prefill_backward_workspace_bytes(dims: SsdDims) -> int:
    return int(lib().ssd_prefill_backward_workspace_bytes(ctypes.byref(dims)))


def prefill_backward(x, dt, B, C, z, A, D, dt_bias, conv_w, conv_b, dy, init_state=None, init_conv_state=None,
                     d_final_state=None, want_init_grads=True, workspace=None, chunk=128):
    """Gradients of ``prefill`` on the GPU (the training backward).

    Inputs as for ``prefill`` (contiguous); dy [Bt, L, H*P] is the gradient of y (the activation dtype,
    or fp32 with bf16 activations when y was fp32); d_final_state [Bt, H, P, N] fp32 or None.
    Returns a dict of fp32 tensors keyed by the input they belong to: x, dt, B, C, z, A, D, dt_bias,
    conv_w, conv_b, and (with ``want_init_grads``) init_state, init_conv_state -- the gradients of
    sum(dy * y) + sum(d_final_state * final_state).
    """
    dev = x.device
    Bt, L, HP = x.shape
    H = A.shape[0]
    P = HP // H
    G, N = B.shape[2], B.shape[3]
    act = x.dtype
    conv_dim = HP + 2 * G * N
    for name, t, shp in (("x", x, (Bt, L, HP)), ("z", z, (Bt, L, HP)), ("dt", dt, (Bt, L, H)),
                         ("B", B, (Bt, L, G, N)), ("C", C, (Bt, L, G, N))):
        _check(t, name, shp, act, dev)
    _check(dy, "dy", (Bt, L, HP), dy.dtype, dev)
    code = _dtype_code(x, dy.dtype)
    if init_state is not None:
        _check(init_state, "init_state", (Bt, H, P, N), torch.float32, dev)
    if init_conv_state is not None:
        _check(init_conv_state, "init_conv_state", (Bt, conv_dim, 3), act, dev)
    if d_final_state is not None:
        _check(d_final_state, "d_final_state", (Bt, H, P, N), torch.float32, dev)
    params = _params(A, D, dt_bias, conv_w, conv_b, H, conv_dim, dev)
    dims = make_dims(Bt, L, H, P, N, G, chunk)
    f32 = dict(dtype=torch.float32, device=dev)
    out = {"x": torch.empty((Bt, L, HP), **f32), "dt": torch.empty((Bt, L, H), **f32),
           "B": torch.empty((Bt, L, G, N), **f32), "C": torch.empty((Bt, L, G, N), **f32),
           "z": torch.empty((Bt, L, HP), **f32), "A": torch.empty(H, **f32), "D": torch.empty(H, **f32),
           "dt_bias": torch.empty(H, **f32), "conv_w": torch.empty((conv_dim, 4), **f32),
           "conv_b": torch.empty(conv_dim, **f32)}
    if want_init_grads:
        out["init_state"] = torch.empty((Bt, H, P, N), **f32)
        out["init_conv_state"] = torch.empty((Bt, conv_dim, 3), **f32)
    grads = SsdGrads(*[None if out.get(k) is None else out[k].data_ptr() for k in (
        "x", "dt", "B", "C", "z", "A", "D", "dt_bias", "conv_w", "conv_b", "init_state", "init_conv_state")])
    need = prefill_backward_workspace_bytes(dims)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().ssd_prefill_backward(ctypes.byref(dims), code, ctypes.byref(params), _ptr(x), _ptr(dt), _ptr(B),
                                    _ptr(C), _ptr(z), _ptr(init_state), _ptr(init_conv_state), _ptr(dy),
                                    _ptr(d_final_state), ctypes.byref(grads), _ptr(workspace), ws_bytes,
                                    _stream_ptr(dev))
    if st != 0:
        raise SsdError(st, "ssd_prefill_backward")
    return out


def prefill_varlen_workspace_bytes(dims: SsdDims, dtype: torch.dtype) -> int:
    code = SSD_F32 if dtype == torch.float32 else SSD_BF16
    return int(lib().ssd_prefill_varlen_workspace_bytes(ctypes.byref(dims), code))


def prefill_varlen(x, dt, B, C, z, A, D, dt_bias, conv_w, conv_b, cu_seqlens, init_state=None,
                   init_conv_state=None, chunk=128, workspace=None, y=None, final_state=None, conv_state=None,
                   y_dtype=None):
    """Packed variable-length prefill: sequence s is rows cu_seqlens[s] .. cu_seqlens[s+1]-1.

    x, z [T, H*P]; dt [T, H]; B, C [T, G, N]; cu_seqlens: nseq+1 non-decreasing offsets from 0 to T,
    an int64 tensor on the device (a list or CPU tensor is copied there first); init_state
    [nseq, H, P, N] fp32 or None; init_conv_state [nseq, conv_dim, 3] or None.
    Returns (y [T, H*P], final_state [nseq, H, P, N], conv_state [nseq, conv_dim, 3]).
    Offsets that are out of order or out of range are reported by device_status().
    """
    dev = x.device
    T, HP = x.shape
    H = A.shape[0]
    P = HP // H
    G, N = B.shape[1], B.shape[2]
    act = x.dtype
    conv_dim = HP + 2 * G * N
    if not torch.is_tensor(cu_seqlens) or cu_seqlens.device != dev:
        cu_seqlens = torch.as_tensor(cu_seqlens, dtype=torch.int64).to(dev)
    if cu_seqlens.dtype != torch.int64 or cu_seqlens.dim() != 1 or not cu_seqlens.is_contiguous():
        raise ValueError("cu_seqlens must be a contiguous 1-D int64 tensor")
    nseq = cu_seqlens.numel() - 1
    if nseq < 0:
        raise ValueError("cu_seqlens needs at least one entry")
    for name, t, shp in (("x", x, (T, HP)), ("z", z, (T, HP)), ("dt", dt, (T, H)), ("B", B, (T, G, N)),
                         ("C", C, (T, G, N))):
        _check(t, name, shp, act, dev)
    if init_state is not None:
        _check(init_state, "init_state", (nseq, H, P, N), torch.float32, dev)
    if init_conv_state is not None:
        _check(init_conv_state, "init_conv_state", (nseq, conv_dim, 3), act, dev)
    params = _params(A, D, dt_bias, conv_w, conv_b, H, conv_dim, dev)
    dims = make_dims(nseq, T, H, P, N, G, chunk)
    ydt = y_dtype or (y.dtype if y is not None else act)
    code = _dtype_code(x, ydt)
    if y is None:
        y = torch.empty((T, HP), dtype=ydt, device=dev)
    if final_state is None:
        final_state = torch.empty((nseq, H, P, N), dtype=torch.float32, device=dev)
    if conv_state is None:
        conv_state = torch.empty((nseq, conv_dim, 3), dtype=act, device=dev)
    _check(y, "y", (T, HP), ydt, dev)
    _check(final_state, "final_state", (nseq, H, P, N), torch.float32, dev)
    _check(conv_state, "conv_state", (nseq, conv_dim, 3), act, dev)
    need = prefill_varlen_workspace_bytes(dims, act)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().ssd_prefill_varlen(ctypes.byref(dims), code, ctypes.byref(params), _ptr(cu_seqlens), _ptr(x), _ptr(dt),
                                  _ptr(B), _ptr(C), _ptr(z), _ptr(init_state), _ptr(init_conv_state), _ptr(y),
                                  _ptr(final_state), _ptr(conv_state), _ptr(workspace), ws_bytes, _stream_ptr(dev))
    if st != 0:
        raise SsdError(st, "ssd_prefill_varlen")
    return y, final_state, conv_state


def conv_window(x, B, C, init_conv_state=None, out=None):
    """Pre-conv x|B|C of the last 3 tokens of each sequence, [Bt, conv_dim, 3] (history before token 0):
    the conv_state that ssd_prefill would return, without the scan."""
    dev = x.device
    Bt, L, HP = x.shape
    G, N = B.shape[2], B.shape[3]
    conv_dim = HP + 2 * G * N
    for name, t, shp in (("x", x, (Bt, L, HP)), ("B", B, (Bt, L, G, N)), ("C", C, (Bt, L, G, N))):
        _check(t, name, shp, x.dtype, dev)
    if init_conv_state is not None:
        _check(init_conv_state, "init_conv_state", (Bt, conv_dim, 3), x.dtype, dev)
    if out is None:
        out = torch.empty((Bt, conv_dim, 3), dtype=x.dtype, device=dev)
    dims = make_dims(Bt, L, HP // 64, 64, N, G)
    st = lib().ssd_conv_window(ctypes.byref(dims), SSD_F32 if x.dtype == torch.float32 else SSD_BF16, _ptr(x),
                               _ptr(B), _ptr(C), _ptr(init_conv_state), _ptr(out), _stream_ptr(dev))
    if st != 0:
        raise SsdError(st, "ssd_conv_window")
    return out


def dt_sum(dt, dt_bias, ngroups=1, d_state=128):
    """sum_t softplus(dt_raw + dt_bias[h]) per sequence and head, [Bt, H] fp32."""
    dev = dt.device
    Bt, L, H = dt.shape
    _check(dt, "dt", (Bt, L, H), dt.dtype, dev)
    _check(dt_bias, "dt_bias", (H,), torch.float32, dev)
    out = torch.empty((Bt, H), dtype=torch.float32, device=dev)
    dims = make_dims(Bt, L, H, 64, d_state, ngroups)
    st = lib().ssd_dt_sum(ctypes.byref(dims), SSD_F32 if dt.dtype == torch.float32 else SSD_BF16, _ptr(dt_bias),
                          _ptr(dt), _ptr(out), _stream_ptr(dev))
    if st != 0:
        raise SsdError(st, "ssd_dt_sum")
    return out


def cp_combine(seg_states, dt_sums, A, upto, init_state=None):
    """Initial state of segment ``upto``: init_state (or zero) folded with segments 0 .. upto-1,
    S <- exp(A_h dt_sums[q]) S + seg_states[q].  seg_states [W, Bt, H, P, N], dt_sums [W, Bt, H]."""
    dev = seg_states.device
    W, Bt, H, P, N = seg_states.shape
    _check(seg_states, "seg_states", (W, Bt, H, P, N), torch.float32, dev)
    _check(dt_sums, "dt_sums", (W, Bt, H), torch.float32, dev)
    _check(A, "A", (H,), torch.float32, dev)
    if init_state is not None:
        _check(init_state, "init_state", (Bt, H, P, N), torch.float32, dev)
    out = torch.empty((Bt, H, P, N), dtype=torch.float32, device=dev)
    dims = make_dims(Bt, 0, H, P, N, 1)
    st = lib().ssd_cp_combine(ctypes.byref(dims), W, int(upto), _ptr(A), _ptr(dt_sums), _ptr(seg_states),
                              _ptr(init_state), _ptr(out), _stream_ptr(dev))
    if st != 0:
        raise SsdError(st, "ssd_cp_combine")
    return out


def gated_rmsnorm(y, weight, norm_groups, eps=1e-5, out=None):
    """RMSNorm over ``norm_groups`` contiguous channel groups of the gated output y [..., channels]
    (bf16 or fp32), times the per-channel fp32 ``weight``; ``out`` may be ``y`` (in place)."""
    dev = y.device
    channels = y.shape[-1]
    if not y.is_contiguous():
        raise ValueError("y must be contiguous")
    _check(weight, "weight", (channels,), torch.float32, dev)
    if out is None:
        out = torch.empty_like(y)
    _check(out, "out", tuple(y.shape), y.dtype, dev)
    code = SSD_F32 if y.dtype == torch.float32 else SSD_BF16
    st = lib().ssd_gated_rmsnorm(y.numel() // channels, channels, int(norm_groups), float(eps), code, _ptr(y),
                                 _ptr(weight), _ptr(out), _stream_ptr(dev))
    if st != 0:
        raise SsdError(st, "ssd_gated_rmsnorm")
    return out


def decode_step(x, dt, B, C, z, A, D, dt_bias, conv_w, conv_b, conv_state, ssm_state, y=None, y_dtype=None):
    """One decode token for Bt sequences; conv_state and ssm_state update in place.

    x, z [Bt, H*P]; dt [Bt, H]; B, C [Bt, G, N]; conv_state [Bt, conv_dim, 3];
    ssm_state [Bt, H, P, N] fp32.  Returns y [Bt, H*P].
    """
    dev = x.device
    Bt, HP = x.shape
    H = A.shape[0]
    P = HP // H
    G, N = B.shape[1], B.shape[2]
    act = x.dtype
    conv_dim = HP + 2 * G * N
    for name, t, shp in (("x", x, (Bt, HP)), ("z", z, (Bt, HP)), ("dt", dt, (Bt, H)), ("B", B, (Bt, G, N)),
                         ("C", C, (Bt, G, N)), ("conv_state", conv_state, (Bt, conv_dim, 3))):
        _check(t, name, shp, act, dev)
    _check(ssm_state, "ssm_state", (Bt, H, P, N), torch.float32, dev)
    params = _params(A, D, dt_bias, conv_w, conv_b, H, conv_dim, dev)
    ydt = y_dtype or (y.dtype if y is not None else act)
    code = _dtype_code(x, ydt)
    if y is None:
        y = torch.empty((Bt, HP), dtype=ydt, device=dev)
    _check(y, "y", (Bt, HP), ydt, dev)
    dims = make_dims(Bt, 1, H, P, N, G)
    st = lib().ssd_decode_step(ctypes.byref(dims), code, ctypes.byref(params), _ptr(x), _ptr(dt), _ptr(B),
                               _ptr(C), _ptr(z), _ptr(conv_state), _ptr(ssm_state), _ptr(y), _stream_ptr(dev))
    if st != 0:
        raise SsdError(st, "ssd_decode_step")
    return y


NOALLOC_SCRATCH_BYTES = 16 << 20


def prefill_noalloc(x, dt, B, C, z, A, D, dt_bias, conv_w, conv_b, init_state=None, init_conv_state=None,
                    chunk=128, y=None, final_state=None, conv_state=None, y_dtype=None):
    """ssd_prefill_noalloc: the same prefill with the library's built-in scratch
    (for callers that cannot allocate a workspace).  Outputs must be passed in
    if the caller cannot allocate them either.  Raises SsdError
    (SSD_ERR_WORKSPACE) when the sizes need more than 16 MiB of scratch."""
    dev = x.device
    Bt, L, HP = x.shape
    H = A.shape[0]
    P = HP // H
    G, N = B.shape[2], B.shape[3]
    act = x.dtype
    conv_dim = HP + 2 * G * N
    for name, t, shp in (("x", x, (Bt, L, HP)), ("z", z, (Bt, L, HP)), ("dt", dt, (Bt, L, H)),
                         ("B", B, (Bt, L, G, N)), ("C", C, (Bt, L, G, N))):
        _check(t, name, shp, act, dev)
    if init_state is not None:
        _check(init_state, "init_state", (Bt, H, P, N), torch.float32, dev)
    if init_conv_state is not None:
        _check(init_conv_state, "init_conv_state", (Bt, conv_dim, 3), act, dev)
    params = _params(A, D, dt_bias, conv_w, conv_b, H, conv_dim, dev)
    ydt = y_dtype or (y.dtype if y is not None else act)
    code = _dtype_code(x, ydt)
    if y is None:
        y = torch.empty((Bt, L, HP), dtype=ydt, device=dev)
    if final_state is None:
        final_state = torch.empty((Bt, H, P, N), dtype=torch.float32, device=dev)
    if conv_state is None:
        conv_state = torch.empty((Bt, conv_dim, 3), dtype=act, device=dev)
    _check(y, "y", (Bt, L, HP), ydt, dev)
    _check(final_state, "final_state", (Bt, H, P, N), torch.float32, dev)
    _check(conv_state, "conv_state", (Bt, conv_dim, 3), act, dev)
    dims = make_dims(Bt, L, H, P, N, G, chunk)
    st = lib().ssd_prefill_noalloc(ctypes.byref(dims), code, ctypes.byref(params), _ptr(x), _ptr(dt), _ptr(B),
                                   _ptr(C), _ptr(z), _ptr(init_state), _ptr(init_conv_state), _ptr(y),
                                   _ptr(final_state), _ptr(conv_state), _stream_ptr(dev))
    if st != 0:
        raise SsdError(st, "ssd_prefill_noalloc")
    return y, final_state, conv_state


def mimo_decode_step(x, dt, B, C, z, A, D, dt_bias, ssm_state, y=None, y_dtype=None):
    """One MIMO decode step on the GPU (rank R = x.shape[2]; see include/ssd.h).  x, z [Bt, H, R, P];
    dt [Bt, H]; B, C [Bt, G, R, N] (bf16 or fp32, one dtype); A, D, dt_bias [H] fp32; ssm_state
    [Bt, H, P, N] fp32, updated in place.  Returns y [Bt, H, R, P] (the activation dtype, or y_dtype)."""
    dev = x.device
    Bt, H, R, P = x.shape
    G, N = B.shape[1], B.shape[3]
    act = x.dtype
    for name, t, shp in (("x", x, (Bt, H, R, P)), ("z", z, (Bt, H, R, P)), ("dt", dt, (Bt, H)),
                         ("B", B, (Bt, G, R, N)), ("C", C, (Bt, G, R, N))):
        _check(t, name, shp, act, dev)
    for name, t in (("A", A), ("D", D), ("dt_bias", dt_bias)):
        _check(t, name, (H,), torch.float32, dev)
    _check(ssm_state, "ssm_state", (Bt, H, P, N), torch.float32, dev)
    ydt = y_dtype or (y.dtype if y is not None else act)
    code = _dtype_code(x, ydt)
    if y is None:
        y = torch.empty((Bt, H, R, P), dtype=ydt, device=dev)
    _check(y, "y", (Bt, H, R, P), ydt, dev)
    params = SsdParams(A.data_ptr(), D.data_ptr(), dt_bias.data_ptr(), None, None)
    dims = make_dims(Bt, 1, H, P, N, G)
    st = lib().ssd_mimo_decode_step(ctypes.byref(dims), int(R), code, ctypes.byref(params), _ptr(x), _ptr(dt),
                                    _ptr(B), _ptr(C), _ptr(z), _ptr(ssm_state), _ptr(y), _stream_ptr(dev))
    if st != 0:
        raise SsdError(st, "ssd_mimo_decode_step")
    return y


def device_status(device="cuda"):
    """Synchronise the current stream; raise if a kernel gave up on a bounded device-side wait
    (SSD_ERR_TIMEOUT), met invalid packed-sequence offsets (SSD_ERR_SHAPE) or, in the tensor-core backward,
    an operand beyond fp16 range (SSD_ERR_RANGE)."""
    st = lib().ssd_device_status(_stream_ptr(torch.device(device)))
    if st != 0:
        raise SsdError(st, "ssd_device_status")


def set_timing_events(before, after):
    """Record two torch.cuda.Event objects around the dominant kernel of the next calls (None, None = off)."""
    if before is None:
        st = lib().ssd_set_timing_events(None, None)
    else:
        for ev in (before, after):
            if not ev.cuda_event:   # torch creates the CUDA event lazily, on its first record
                ev.record()
        st = lib().ssd_set_timing_events(ctypes.c_void_p(before.cuda_event), ctypes.c_void_p(after.cuda_event))
    if st != 0:
        raise SsdError(st, "ssd_set_timing_events")


_side_streams = {}


def _host_streams(dev):
    """Two side streams per device (host->device copies, device->host copies), created once."""
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    if key not in _side_streams:
        _side_streams[key] = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
    return _side_streams[key]


def host_pieces(L: int, chunk: int, segments=None) -> list:
    """Row ranges [r0, r1) of the pieces prefill_host cuts a sequence of L tokens into: ``segments`` pieces
    (default: as many as fit at two chunks each, at most 8) of equal length rounded up to whole chunks,
    the last one shorter; one piece when L fits in one."""
    if segments is None:
        segments = max(1, min(8, L // (2 * chunk)))
    seg = -(-L // max(1, int(segments)))
    seg = max(chunk, -(-seg // chunk) * chunk)
    return [(r0, min(L, r0 + seg)) for r0 in range(0, L, seg)] if L > 0 else [(0, 0)]


def _host_outputs(inputs: dict, out):
    """The pinned host tensors prefill_host writes y, final_state and conv_state into: the caller's ``out``
    (checked) or new ones."""
    x = inputs["x"]
    Bt, L, HP = x.shape
    H = inputs["A"].shape[0]
    G, N = inputs["B"].shape[2], inputs["B"].shape[3]
    shapes = ((Bt, L, HP), (Bt, H, HP // H, N), (Bt, HP + 2 * G * N, 3))
    dtypes = (x.dtype, torch.float32, x.dtype)
    if out is None:
        return [torch.empty(sh, dtype=dt, pin_memory=True) for sh, dt in zip(shapes, dtypes)]
    out = list(out)
    for name, t, sh, dt in zip(("y", "final_state", "conv_state"), out, shapes, dtypes):
        if t.is_cuda or tuple(t.shape) != sh or t.dtype != dt or not t.is_contiguous():
            raise ValueError(f"out {name} must be a contiguous host tensor {sh} of {dt}")
    return out


def prefill_host(inputs: dict, chunk=128, device="cuda", segments=None, out=None):
    """End-to-end prefill from HOST tensors (pinned for asynchronous copies): the inputs go to the device,
    ssd_prefill runs, and y, final_state and conv_state come back into pinned host tensors -- the caller's
    ``out`` = (y, final_state, conv_state) when given (reused across calls, no host allocation), else new
    ones (a pinned allocation of y's size per call).

    The work is cut into pieces of one sequence (batch row) and a chunk-aligned token range: ``segments``
    ranges per sequence (default: about eight pieces in all, each at least two chunks long), so every
    tensor of a piece is one contiguous host range and moves in one copy.  Piece k is copied in on one
    side stream while piece k-1 is scanned on the current stream and piece k-2's y is copied out on
    another, so the two copy directions and the scan overlap.  A piece starts from the states the previous
    piece of its sequence left (final_state and conv_state as init_state and init_conv_state), which on
    chunk boundaries gives the same values as one call over the whole sequence.  The current stream waits
    for every copy before the call returns, so events recorded on it around the call time the whole
    transfer.  Returns ([y, final_state, conv_state] on the host, bytes in, bytes out).
    """
    dev = torch.device(device)
    x = inputs["x"]
    Bt, L = x.shape[0], x.shape[1]
    h2d = sum(t.numel() * t.element_size() for t in inputs.values() if t is not None)
    if segments is None:
        segments = max(1, min(L // (2 * chunk), -(-8 // max(Bt, 1))))
    ranges = host_pieces(L, chunk, segments)
    y_host, fs_host, cs_host = _host_outputs(inputs, out)
    if Bt * len(ranges) <= 1:
        return _prefill_host_whole(inputs, chunk, dev, h2d, (y_host, fs_host, cs_host))

    cur = torch.cuda.current_stream(dev)
    s_in, s_out = _host_streams(dev)
    s_in.wait_stream(cur)
    s_out.wait_stream(cur)
    names = ("A", "D", "dt_bias", "conv_w", "conv_b", "init_state", "init_conv_state")
    with torch.cuda.stream(s_in):
        p = {k: (None if inputs.get(k) is None else inputs[k].to(dev, non_blocking=True)) for k in names}
    for t in p.values():
        if t is not None:
            t.record_stream(cur)
    for b in range(Bt):
        fs_prev = None if p["init_state"] is None else p["init_state"][b:b + 1]
        cs_prev = None if p["init_conv_state"] is None else p["init_conv_state"][b:b + 1]
        for r0, r1 in ranges:
            with torch.cuda.stream(s_in):
                d = {k: inputs[k][b:b + 1, r0:r1].to(dev, non_blocking=True) for k in ("x", "dt", "B", "C", "z")}
                ready = torch.cuda.Event()
                ready.record(s_in)
            cur.wait_event(ready)
            for t in d.values():
                t.record_stream(cur)
            y, fs, cs = prefill(d["x"], d["dt"], d["B"], d["C"], d["z"], p["A"], p["D"], p["dt_bias"], p["conv_w"],
                                p["conv_b"], fs_prev, cs_prev, chunk=chunk)
            done = torch.cuda.Event()
            done.record(cur)
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                y_host[b, r0:r1].copy_(y[0], non_blocking=True)
                if r1 == L:
                    fs_host[b].copy_(fs[0], non_blocking=True)
                    cs_host[b].copy_(cs[0], non_blocking=True)
            for t in (y, fs, cs):
                t.record_stream(s_out)
            fs_prev, cs_prev = fs, cs
    out_done = torch.cuda.Event()
    out_done.record(s_out)
    cur.wait_event(out_done)
    outs = [y_host, fs_host, cs_host]
    return outs, h2d, sum(t.numel() * t.element_size() for t in outs)


def _prefill_host_whole(inputs: dict, chunk, dev, h2d, outs):
    """prefill_host in one piece on the current stream: copy in, scan, copy out."""
    names = ("x", "dt", "B", "C", "z", "A", "D", "dt_bias", "conv_w", "conv_b", "init_state", "init_conv_state")
    d = {k: (None if inputs.get(k) is None else inputs[k].to(dev, non_blocking=True)) for k in names}
    y, fs, cs = prefill(d["x"], d["dt"], d["B"], d["C"], d["z"], d["A"], d["D"], d["dt_bias"], d["conv_w"],
                        d["conv_b"], d["init_state"], d["init_conv_state"], chunk=chunk)
    outs = list(outs)
    for o, t in zip(outs, (y, fs, cs)):
        o.copy_(t, non_blocking=True)
    return outs, h2d, sum(t.numel() * t.element_size() for t in outs)
