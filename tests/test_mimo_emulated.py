"""The MIMO decode kernel's CUDA source, run on the CPU through the host emulation of the CUDA
execution model (tests/emu/emu_cuda.h: one thread per CUDA thread, real barriers for
__syncthreads and for the warp shuffles) built with AddressSanitizer and UBSan, against the fp64
oracle's MIMO step over several consecutive steps.  Shows with no GPU that every access stays in
its buffer, every y element is written, and the arithmetic is the oracle's; the GPU parity tests
call the nvcc build of the same source through the C ABI."""
import numpy as np
import pytest
import torch

import emu_harness
import oracle
from pins import f64
from selective_state_space_43_b200.synth import Dims, make_mimo_decode_inputs


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    return emu_harness.build(str(tmp_path_factory.mktemp("emu")), "run_mimo")


def oracle_steps(data):
    params = {k: f64(v) for k, v in data["params"].items()}
    S = f64(data["ssm_state"]).copy()
    ys = [oracle.mimo_decode_step(s, params, S) for s in data["steps"]]
    return ys, S


@pytest.mark.parametrize("R,N,G,Bt", [(1, 128, 2, 2), (2, 64, 1, 3), (4, 128, 2, 2), (8, 32, 4, 1), (4, 16, 1, 2)])
def test_emulated_mimo_matches_oracle(exe, R, N, G, Bt):
    d = Dims(Bt, 1, 4, 64, N, G, 64)
    data = make_mimo_decode_inputs(d, R, steps=3, dtype=torch.float32, seed=R * N + G, random_D=True)
    ys, S = emu_harness.run_mimo(exe, data, R, y_bf16=False)
    yo, So = oracle_steps(data)
    for t, (a, b) in enumerate(zip(ys, yo)):
        assert not np.isnan(a).any(), f"step {t}: unwritten y"
        assert np.max(np.abs(a - b)) <= 2e-5 * max(1.0, np.max(np.abs(b))), t
    assert np.max(np.abs(S - So)) <= 2e-5


def test_emulated_mimo_bf16_output_is_rounded_fp32(exe):
    d = Dims(2, 1, 4, 64, 64, 2, 64)
    data = make_mimo_decode_inputs(d, 4, steps=2, dtype=torch.bfloat16, seed=5)
    y16, S16 = emu_harness.run_mimo(exe, data, 4, y_bf16=True)
    y32, S32 = emu_harness.run_mimo(exe, data, 4, y_bf16=False)
    assert np.array_equal(S16, S32)
    for a, b in zip(y16, y32):
        assert np.array_equal(a, torch.from_numpy(b).to(torch.bfloat16).float().numpy())
    yo, So = oracle_steps(data)
    for a, b in zip(y32, yo):
        assert np.max(np.abs(a - b)) <= 2e-5 * max(1.0, np.max(np.abs(b)))
