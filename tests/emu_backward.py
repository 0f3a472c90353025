"""Runs the backward kernels' own source on the CPU through the host emulation of the CUDA
execution model (tests/emu), built with AddressSanitizer: a bounds and logic check of the
CUDA code that needs no GPU.  Test helper, imported by the CPU tests only."""
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

_exe = None


def build(out_dir: str) -> str:
    """Compiles run_backward.cpp (which includes ssd_backward.cu) with g++ and ASan/UBSan."""
    global _exe
    if _exe and os.path.exists(_exe):
        return _exe
    exe = os.path.join(out_dir, "run_backward")
    cmd = ["g++", "-std=c++20", "-O1", "-g", "-fsanitize=address,undefined", "-fno-sanitize-recover=undefined",
           "-fno-omit-frame-pointer", "-Wall", "-Wno-unknown-pragmas", "-I", EMU, "-I", CSRC,
           "-o", exe, os.path.join(EMU, "run_backward.cpp"), "-pthread"]
    subprocess.check_call(cmd)
    _exe = exe
    return exe


def _raw(t, bf16: bool) -> bytes:
    t = t.detach().cpu().contiguous()
    if bf16:
        return t.to(torch.bfloat16).view(torch.int16).numpy().tobytes()
    return t.to(torch.float32).numpy().tobytes()


def run(exe: str, inp: dict, dy, d_final=None, dy_bf16=None, timeout: float = 600.0) -> dict:
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
    with tempfile.TemporaryDirectory() as tmp:
        fin, fout = os.path.join(tmp, "in.bin"), os.path.join(tmp, "out.bin")
        with open(fin, "wb") as f:
            f.write(b"".join(parts))
        env = dict(os.environ, ASAN_OPTIONS="detect_leaks=0:abort_on_error=0", UBSAN_OPTIONS="print_stacktrace=1")
        r = subprocess.run([exe, fin, fout], capture_output=True, text=True, timeout=timeout, env=env)
        if r.returncode != 0:
            raise RuntimeError(f"emulated backward failed ({r.returncode}):\n{r.stderr[-4000:]}")
        flat = np.fromfile(fout, dtype=np.float32)
    out, off = {}, 0
    for k, shp in shapes:
        n = int(np.prod(shp))
        out[k] = flat[off:off + n].reshape(shp)
        off += n
    assert off == flat.size
    return out
