"""Runs kernels' own CUDA source on the CPU through the host emulation of the CUDA execution model
(tests/emu), built with AddressSanitizer and UBSan: a bounds and logic check of the CUDA code that
needs no GPU.  Harnesses: run_backward (ssd_backward.cu) and run_mimo (ssd_mimo.cu).  Test helper,
imported by the CPU tests only."""
from __future__ import annotations

import os
import subprocess
import tempfile

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
EMU = os.path.join(HERE, "emu")
CSRC = os.path.join(ROOT, "selective_state_space_43_b200", "csrc")

_exes = {}


def build(out_dir: str, target: str = "run_backward") -> str:
    """Compiles tests/emu/<target>.cpp (which includes the kernel's .cu file) with g++ and ASan/UBSan."""
    if target in _exes and os.path.exists(_exes[target]):
        return _exes[target]
    exe = os.path.join(out_dir, target)
    cmd = ["g++", "-std=c++20", "-O1", "-g", "-fsanitize=address,undefined", "-fno-sanitize-recover=undefined",
           "-fno-omit-frame-pointer", "-Wall", "-Wno-unknown-pragmas", "-I", EMU, "-I", CSRC,
           "-o", exe, os.path.join(EMU, target + ".cpp"), "-pthread"]
    subprocess.check_call(cmd)
    _exes[target] = exe
    return exe


def _exec(exe: str, payload: bytes, timeout: float) -> np.ndarray:
    with tempfile.TemporaryDirectory() as tmp:
        fin, fout = os.path.join(tmp, "in.bin"), os.path.join(tmp, "out.bin")
        with open(fin, "wb") as f:
            f.write(payload)
        env = dict(os.environ, ASAN_OPTIONS="detect_leaks=0:abort_on_error=0", UBSAN_OPTIONS="print_stacktrace=1")
        r = subprocess.run([exe, fin, fout], capture_output=True, text=True, timeout=timeout, env=env)
        if r.returncode != 0:
            raise RuntimeError(f"emulated kernel run failed ({r.returncode}):\n{r.stderr[-4000:]}")
        return np.fromfile(fout, dtype=np.uint8)


def _raw(t, bf16: bool) -> bytes:
    t = t.detach().cpu().contiguous()
    if bf16:
        return t.to(torch.bfloat16).view(torch.int16).numpy().tobytes()
    return t.to(torch.float32).numpy().tobytes()


def run_backward(exe: str, inp: dict, dy, d_final=None, dy_bf16=None, timeout: float = 600.0) -> dict:
    """Backward through the emulated kernels.  ``inp`` as make_prefill_inputs (torch, CPU)."""
    x = inp["x"]
    act_bf16 = x.dtype == torch.bfloat16
    dy_bf16 = act_bf16 if dy_bf16 is None else dy_bf16
    Bt, L, HP = x.shape
    G, N = inp["B"].shape[2], inp["B"].shape[3]
    H = inp["A"].shape[0]
    P = HP // H
    conv_dim = HP + 2 * G * N
    ist, ics = inp.get("init_state"), inp.get("init_conv_state")
    hdr = np.array([Bt, L, H, P, N, G, int(act_bf16), int(dy_bf16), int(ist is not None), int(ics is not None),
                    int(d_final is not None)], dtype=np.int64)
    parts = [hdr.tobytes()]
    for k in ("A", "D", "dt_bias", "conv_w", "conv_b"):
        parts.append(_raw(inp[k], False))
    for k in ("x", "dt", "B", "C", "z"):
        parts.append(_raw(inp[k], act_bf16))
    parts.append(_raw(dy, dy_bf16))
    if ist is not None:
        parts.append(_raw(ist, False))
    if ics is not None:
        parts.append(_raw(ics, act_bf16))
    if d_final is not None:
        parts.append(_raw(d_final, False))
    shapes = [("x", (Bt, L, HP)), ("dt", (Bt, L, H)), ("B", (Bt, L, G, N)), ("C", (Bt, L, G, N)),
              ("z", (Bt, L, HP)), ("A", (H,)), ("D", (H,)), ("dt_bias", (H,)), ("conv_w", (conv_dim, 4)),
              ("conv_b", (conv_dim,)), ("init_state", (Bt, H, P, N)), ("init_conv_state", (Bt, conv_dim, 3))]
    flat = _exec(exe, b"".join(parts), timeout).view(np.float32)
    out, off = {}, 0
    for k, shp in shapes:
        n = int(np.prod(shp))
        out[k] = flat[off:off + n].reshape(shp)
        off += n
    assert off == flat.size
    return out


def run_mimo(exe: str, data: dict, rank: int, y_bf16=None, timeout: float = 600.0):
    """MIMO decode steps through the emulated kernel.  ``data`` as make_mimo_decode_inputs (torch, CPU).
    Returns (list of y [Bt, H, R, P] as float32, final state [Bt, H, P, N])."""
    st0 = data["steps"][0]
    act_bf16 = st0["x"].dtype == torch.bfloat16
    y_bf16 = act_bf16 if y_bf16 is None else y_bf16
    Bt, H, R, P = st0["x"].shape
    G, N = st0["B"].shape[1], st0["B"].shape[3]
    assert R == rank
    hdr = np.array([Bt, H, P, N, G, R, int(act_bf16), int(y_bf16), len(data["steps"])], dtype=np.int64)
    parts = [hdr.tobytes()] + [_raw(data["params"][k], False) for k in ("A", "D", "dt_bias")]
    parts.append(_raw(data["ssm_state"], False))
    for s in data["steps"]:
        for k in ("x", "dt", "B", "C", "z"):
            parts.append(_raw(s[k], act_bf16))
    raw = _exec(exe, b"".join(parts), timeout)
    ny = Bt * H * R * P * (2 if y_bf16 else 4)
    ys = []
    for i in range(len(data["steps"])):
        chunk = raw[i * ny:(i + 1) * ny]
        if y_bf16:
            y = torch.from_numpy(chunk.view(np.int16).copy()).view(torch.bfloat16).float().numpy()
        else:
            y = chunk.view(np.float32).copy()
        ys.append(y.reshape(Bt, H, R, P))
    state = raw[len(data["steps"]) * ny:].view(np.float32).reshape(Bt, H, P, N)
    return ys, state
