"""The host emulation of the kernels is a strong enough check: faults planted in temporary copies of
the backward and MIMO kernels' source (an access outside a buffer, a misaligned 16-byte shared load, a read of
shared memory that was never written, a dropped term) each make the emulated run fail, through
AddressSanitizer, the emulator's alignment check, the NaN-filled outputs and shared memory, or the
comparison with the oracle.  CPU only; the
faults are planted in copies, never in the library's source."""
import concurrent.futures as cf
import os
import subprocess

import numpy as np
import pytest
import torch

import emu_harness
import oracle
from selective_state_space_43_b200.synth import Dims, make_backward_grads, make_prefill_inputs

SRC = os.path.join(emu_harness.CSRC, "ssd_backward.cu")

MUTANTS = {
    # reads x one token past the tile: beyond the array for the last tile of the last sequence
    "post-conv reads past its tile": ("r[i] = act_pair(src + (i - 3) * rs);", "r[i] = act_pair(src + (i - 2) * rs);"),
    # writes each pre-conv gradient one token late: beyond dx / dB / dC for the last token
    "conv backward writes one row late": ("if (j < n) *reinterpret_cast<float2*>(out + j * rs) = o;",
                                          "if (j < n) *reinterpret_cast<float2*>(out + (j + 1) * rs) = o;"),
    # leaves the rows of a ragged chunk past its end as they were (NaN bytes for the first head)
    "ragged rows not cleared": ("            xs[j * kS + p] = xv;", "            if (j < Qv) xs[j * kS + p] = xv;"),
    # shared rows no longer 16-byte aligned: the emulation's alignment check must stop the vector loads
    "unaligned shared rows": ("constexpr int kS = kQ + 4;", "constexpr int kS = kQ + 1;"),
    # drops the D skip term of dx
    "dx without the D skip": ("dts[j] * el[j] * lmb[r][q] + Dh * gs[j * kS + p];", "dts[j] * el[j] * lmb[r][q];"),
}


def _build(name, old, new, tmp):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for '{name}' not unique"
    d = os.path.join(tmp, name.replace(" ", "_"))
    os.makedirs(d)
    with open(os.path.join(d, "ssd_backward.cu"), "w") as f:
        f.write(src.replace(old, new))
    exe = os.path.join(d, "run_backward")
    cmd = ["g++", "-std=c++20", "-O1", "-g", "-fsanitize=address,undefined", "-fno-sanitize-recover=undefined",
           "-fno-omit-frame-pointer", "-w", "-I", d, "-I", emu_harness.EMU, "-I", emu_harness.CSRC, "-o", exe,
           os.path.join(emu_harness.EMU, "run_backward.cpp"), "-pthread"]
    subprocess.check_call(cmd)
    return exe


@pytest.fixture(scope="module")
def mutant_exes(tmp_path_factory):
    tmp = str(tmp_path_factory.mktemp("emu_mutants"))
    with cf.ThreadPoolExecutor(max_workers=len(MUTANTS)) as ex:
        futs = {name: ex.submit(_build, name, old, new, tmp) for name, (old, new) in MUTANTS.items()}
        return {name: f.result() for name, f in futs.items()}


def _case():
    d = Dims(2, 150, 4, 64, 32, 2, 64)
    inp = make_prefill_inputs(d, dtype=torch.float32, seed=8, init_state=True, init_conv_state=True, random_D=True)
    gr = make_backward_grads(d, dtype=torch.float32, seed=9)
    return inp, gr


def _caught(exe, inp, gr, want):
    try:
        got = emu_harness.run_backward(exe, inp, gr["dy"], gr["d_final"], dy_bf16=False)
    except RuntimeError:
        return True                                   # sanitizer report or a failed run
    for k, ref in want.items():
        g = got[k].astype(np.float64)
        if np.isnan(g).any():
            return True
        if np.linalg.norm(g - ref) > 2e-5 * max(np.linalg.norm(ref), 1e-30):
            return True
    return False


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_kernel_fault_is_caught(mutant_exes, name):
    inp, gr = _case()
    want = oracle.prefill_backward(inp, gr["dy"], gr["d_final"])
    assert _caught(mutant_exes[name], inp, gr, want), f"the emulation missed the planted fault '{name}'"


MIMO_SRC = os.path.join(emu_harness.CSRC, "ssd_mimo.cu")

MIMO_MUTANTS = {
    # the reduce-scatter keeps the other half: each lane writes another output's sum
    "read-out keeps the wrong half": ("if (upper) first += HALF;", "if (!upper) first += HALF;"),
    # only the first lane of each row writes: the other outputs stay unwritten (NaN)
    "read-outs written by too few lanes": ("if ((lane % (LPR / SCAT)) == 0) {", "if ((lane % LPR) == 0) {"),
    # the head's state loaded one vector late: past the state array for the last head
    "state read one vector late": ("bulk_load(s_st, gstate, kStateBytes, bar);",
                                   "bulk_load(s_st, gstate + 4, kStateBytes, bar);"),
    # each lane updates the next lane's columns: the last lane of a row reads and writes past the row
    "state columns one vector late": ("float* srow = s_st + p * N + n0;", "float* srow = s_st + p * N + n0 + 4;"),
    # the updated state is never written back
    "state store dropped": ("bulk_store(gstate, s_st, kStateBytes);", "(void)gstate;"),
}


def _build_mimo(name, old, new, tmp):
    src = open(MIMO_SRC).read()
    assert src.count(old) == 1, f"mutation site for '{name}' not unique"
    d = os.path.join(tmp, name.replace(" ", "_"))
    os.makedirs(d)
    with open(os.path.join(d, "ssd_mimo.cu"), "w") as f:
        f.write(src.replace(old, new))
    exe = os.path.join(d, "run_mimo")
    cmd = ["g++", "-std=c++20", "-O1", "-g", "-fsanitize=address,undefined", "-fno-sanitize-recover=undefined",
           "-fno-omit-frame-pointer", "-w", "-I", d, "-I", emu_harness.EMU, "-I", emu_harness.CSRC, "-o", exe,
           os.path.join(emu_harness.EMU, "run_mimo.cpp"), "-pthread"]
    subprocess.check_call(cmd)
    return exe


@pytest.fixture(scope="module")
def mimo_mutant_exes(tmp_path_factory):
    tmp = str(tmp_path_factory.mktemp("emu_mimo_mutants"))
    with cf.ThreadPoolExecutor(max_workers=len(MIMO_MUTANTS)) as ex:
        futs = {name: ex.submit(_build_mimo, name, old, new, tmp) for name, (old, new) in MIMO_MUTANTS.items()}
        return {name: f.result() for name, f in futs.items()}


@pytest.mark.parametrize("name", sorted(MIMO_MUTANTS))
def test_planted_mimo_kernel_fault_is_caught(mimo_mutant_exes, name):
    from pins import f64
    from selective_state_space_43_b200.synth import make_mimo_decode_inputs
    d = Dims(2, 1, 4, 64, 64, 2, 64)
    data = make_mimo_decode_inputs(d, 4, 2, dtype=torch.float32, seed=3, random_D=True)
    prm = {k: f64(v) for k, v in data["params"].items()}
    S = f64(data["ssm_state"]).copy()
    want = [oracle.mimo_decode_step(s, prm, S) for s in data["steps"]]
    try:
        ys, _ = emu_harness.run_mimo(mimo_mutant_exes[name], data, 4, y_bf16=False)
    except RuntimeError:
        return                                         # sanitizer report or a failed run
    caught = any(np.isnan(y).any() or np.max(np.abs(y - w)) > 2e-5 * max(1.0, np.max(np.abs(w)))
                 for y, w in zip(ys, want))
    assert caught, f"the emulation missed the planted fault '{name}'"
