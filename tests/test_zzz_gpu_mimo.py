"""GPU parity of ssd_mimo_decode_step (Mamba-3's MIMO SSM decode on the Mamba-2 scalar decay)
against the fp64 oracle over consecutive steps (needs a B200).  Tolerance as for the decode step:
rel-L2 <= 5e-3 and max-abs <= 2e-2 on the fp32 y and on the state; the bf16 y equals the
round-to-nearest-even of the fp32 y bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_bf16_is_rounded, assert_close, np64
from pins import f64
from selective_state_space_43_b200 import ops
from selective_state_space_43_b200.synth import WORKLOADS, Dims, make_mimo_decode_inputs

pytestmark = pytest.mark.gpu


def run(d, R, dtype, steps, seed, y_dtype=None):
    data = make_mimo_decode_inputs(d, R, steps, dtype=dtype, seed=seed, random_D=True)
    p = {k: v.cuda() for k, v in data["params"].items()}
    S = data["ssm_state"].cuda()
    ys = []
    for s in data["steps"]:
        g = {k: v.cuda() for k, v in s.items()}
        ys.append(ops.mimo_decode_step(g["x"], g["dt"], g["B"], g["C"], g["z"], p["A"], p["D"], p["dt_bias"], S,
                                       y_dtype=y_dtype))
    torch.cuda.synchronize()
    prm = {k: f64(v) for k, v in data["params"].items()}
    So = f64(data["ssm_state"]).copy()
    yo = [oracle.mimo_decode_step(s, prm, So) for s in data["steps"]]
    return ys, S, yo, So


@pytest.mark.parametrize("R,N,G,dtype", [(1, 128, 2, torch.float32), (2, 64, 1, torch.bfloat16),
                                         (4, 128, 4, torch.bfloat16), (8, 32, 2, torch.float32),
                                         (4, 16, 1, torch.float32)])
def test_mimo_decode_matches_oracle(R, N, G, dtype):
    d = Dims(3, 1, 8, 64, N, G, 64)
    ys, S, yo, So = run(d, R, dtype, steps=4, seed=R * 100 + N, y_dtype=torch.float32)
    for t, (a, b) in enumerate(zip(ys, yo)):
        assert_close(np64(a), b, f"R{R} N{N} step {t} y")
    assert_close(np64(S), So, f"R{R} N{N} state")


def test_mimo_decode_bf16_output_is_rounded():
    d = Dims(2, 1, 8, 64, 128, 2, 64)
    y16, S16, _, _ = run(d, 4, torch.bfloat16, steps=2, seed=9)
    y32, S32, _, _ = run(d, 4, torch.bfloat16, steps=2, seed=9, y_dtype=torch.float32)
    assert torch.equal(S16, S32)
    for a, b in zip(y16, y32):
        assert_bf16_is_rounded(a, b, "MIMO y")


def test_mimo_decode_full_decode_workload():
    # the benchmark's layer and batch: 256 sequences, H128 P64 N128 G8, rank 4, two steps
    d = WORKLOADS["decode_nemotron_h_8b"]["dims"]
    ys, S, yo, So = run(d, 4, torch.bfloat16, steps=2, seed=77, y_dtype=torch.float32)
    for t, (a, b) in enumerate(zip(ys, yo)):
        assert_close(np64(a), b, f"full workload step {t} y")
    assert_close(np64(S), So, "full workload state")
