"""The backward kernels' CUDA source, run on the CPU through the host emulation of the CUDA
execution model (tests/emu/emu_cuda.h: one thread per CUDA thread, a real barrier for
__syncthreads, shared memory pre-filled with NaN bytes) and built with AddressSanitizer and
UBSan, against the fp64 oracle's backward.

This checks, with no GPU, that every access of every kernel stays inside its buffer for these
sizes (ragged chunks, one to several chunks, every supported d_state, empty and short
sequences), that every output element is written (outputs start as NaN), and that the
arithmetic is the backward the oracle defines.  The same source is compiled by nvcc into the
library; the GPU parity tests call that build through the C ABI.
"""
import numpy as np
import pytest
import torch

import emu_harness
import oracle
from selective_state_space_43_b200.synth import Dims, make_backward_grads, make_prefill_inputs


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    return emu_harness.build(str(tmp_path_factory.mktemp("emu")))


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def check(got, want, tol=2e-5):
    for k in want:
        if want[k].size == 0:
            assert got[k].size == 0, k
            continue
        g = got[k].astype(np.float64)
        assert not np.isnan(g).any(), f"{k}: unwritten (NaN) elements"
        assert rel_l2(g, want[k]) <= tol, (k, rel_l2(g, want[k]))
        assert np.max(np.abs(g - want[k])) <= tol * max(1.0, np.max(np.abs(want[k]))), k


CASES = [
    # batch, L, H, G, N, dtype, init states, d_final, dy fp32 with bf16 activations
    (2, 150, 4, 2, 32, torch.bfloat16, True, True, False),   # ragged third chunk, groups of 2
    (1, 64, 2, 1, 16, torch.float32, False, False, False),   # exactly one chunk, zero states
    (1, 70, 2, 1, 128, torch.bfloat16, True, True, True),    # d_state 128 (largest shared tile)
    (1, 129, 3, 3, 64, torch.float32, True, False, False),   # one head per group, 1-token last chunk
    (1, 100, 6, 2, 32, torch.bfloat16, True, True, False),   # three heads per group: halves of 1 and 2 heads
    (1, 200, 8, 2, 128, torch.bfloat16, True, True, False),  # d_state 128, 4 heads per group, 4 chunks (8-token tail)
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}L{c[1]}H{c[2]}G{c[3]}N{c[4]}")
def test_emulated_backward_matches_oracle(exe, case):
    Bt, L, H, G, N, dtype, init, dfin, dy32 = case
    d = Dims(Bt, L, H, 64, N, G, 64)
    inp = make_prefill_inputs(d, dtype=dtype, seed=L + N, init_state=init, init_conv_state=init, random_D=True)
    gr = make_backward_grads(d, dtype=torch.float32 if dy32 else dtype, seed=L + N + 1, d_final=dfin)
    got = emu_harness.run_backward(exe, inp, gr["dy"], gr["d_final"], dy_bf16=(dtype == torch.bfloat16 and not dy32))
    want = oracle.prefill_backward(inp, gr["dy"], gr["d_final"])
    check(got, want)


@pytest.mark.parametrize("L", [0, 1, 3])
def test_emulated_backward_short_sequences(exe, L):
    d = Dims(2, L, 2, 64, 16, 1, 64)
    inp = make_prefill_inputs(d, dtype=torch.float32, seed=9, init_state=True, init_conv_state=True)
    gr = make_backward_grads(d, dtype=torch.float32, seed=10, d_final=True)
    got = emu_harness.run_backward(exe, inp, gr["dy"], gr["d_final"], dy_bf16=False)
    want = oracle.prefill_backward(inp, gr["dy"], gr["d_final"])
    check(got, want)
    if L == 0:
        # no tokens: the state gradient passes straight through, the rest is zero
        assert np.array_equal(got["init_state"], gr["d_final"].numpy())
        assert not got["conv_w"].any() and not got["init_conv_state"].any()
