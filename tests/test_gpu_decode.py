"""GPU parity of ssd_decode_step against the fp64 oracle (needs a B200)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_bf16_is_rounded, assert_close, dev_inputs, gpu_decode, gpu_prefill, np64
from selective_state_space_43_b200.synth import Dims, make_decode_inputs, make_prefill_inputs

pytestmark = pytest.mark.gpu


def _run(d, steps, dtype, seed, sub=None, random_D=True):
    """Run `steps` decode steps on the GPU; the oracle follows the sequences in `sub` (all if None).

    With bf16 activations two copies of the states advance side by side, one
    writing bf16 y and one fp32 y: they must stay bit-identical, the bf16 y
    must be the rounded fp32 y, and the fp32 y is held to the tolerance."""
    data = make_decode_inputs(d, steps, dtype=dtype, seed=seed, random_D=random_D)
    params = dev_inputs(data["params"])
    conv = data["conv_state"].to("cuda")
    ssm = data["ssm_state"].to("cuda")
    twin = dtype == torch.bfloat16
    if twin:
        conv32, ssm32 = conv.clone(), ssm.clone()
    sel = list(range(d.batch)) if sub is None else list(sub)
    conv_o = data["conv_state"][sel].double().numpy().copy()
    ssm_o = data["ssm_state"][sel].double().numpy().copy()
    worst = (0.0, 0.0)
    for t in range(steps):
        step = data["steps"][t]
        sd = dev_inputs(step)
        y = gpu_decode(sd, params, conv, ssm)
        if twin:
            y32 = gpu_decode(sd, params, conv32, ssm32, y_dtype=torch.float32)
            assert_bf16_is_rounded(y, y32, f"decode step {t} y")
            y = y32
        yo = oracle.decode_step({k: v[sel] for k, v in step.items()}, data["params"], conv_o, ssm_o)
        r = assert_close(np64(y)[sel], yo, f"decode step {t} y")
        worst = (max(worst[0], r[0]), max(worst[1], r[1]))
    if twin:
        assert torch.equal(ssm, ssm32) and torch.equal(conv, conv32)
    torch.cuda.synchronize()
    assert_close(np64(ssm)[sel], ssm_o, "decode ssm_state after all steps")
    assert np.array_equal(np64(conv)[sel], conv_o), "decode conv_state"
    assert torch.isfinite(ssm).all()
    return worst


@pytest.mark.parametrize("N", [16, 32, 64, 128])
def test_decode_small_matches_oracle(N):
    d = Dims(6, 1, 16, 64, N, 4, 128)
    _run(d, 8, torch.bfloat16, seed=31 + N)


def test_decode_fp32_matches_oracle():
    d = Dims(4, 1, 8, 64, 32, 2, 128)
    _run(d, 6, torch.float32, seed=33)


def test_decode_nemotron_h_shape_64_steps_all_heads():
    # the decode workload's layer shape with a batch the oracle follows fully
    d = Dims(8, 1, 128, 64, 128, 8, 128)
    _run(d, 64, torch.bfloat16, seed=34, random_D=False)


def test_decode_full_size_64_steps_sampled():
    # 256 sequences x 128 heads x 64 x 128 fp32 state (1.07 GB), 64 consecutive steps;
    # the oracle follows sequences 0, 131 and 255 (all their heads) through every step
    d = Dims(256, 1, 128, 64, 128, 8, 128)
    _run(d, 64, torch.bfloat16, seed=47, sub=[0, 131, 255], random_D=False)


def test_prefill_then_decode_continues_the_sequence():
    d = Dims(2, 200, 16, 64, 128, 4, 128)
    inp = make_prefill_inputs(d, dtype=torch.bfloat16, seed=35, init_state=True, init_conv_state=True)
    dev = dev_inputs(inp)
    L1 = 190
    first = {k: (v[:, :L1].contiguous() if k in ("x", "z", "dt", "B", "C") else v) for k, v in dev.items()}
    _, fs, cs = gpu_prefill(first, 128)
    params = {k: dev[k] for k in ("A", "D", "dt_bias", "conv_w", "conv_b")}
    ys = []
    for t in range(L1, d.seqlen):
        step = {k: dev[k][:, t].contiguous() for k in ("x", "z", "dt", "B", "C")}
        ys.append(gpu_decode(step, params, cs, fs, y_dtype=torch.float32))
    yo, fo, co = oracle.prefill(inp)
    assert_close(np64(torch.stack(ys, dim=1)), yo[:, L1:], "decode after prefill y")
    assert_close(np64(fs), fo, "decode after prefill state")
    assert np.array_equal(np64(cs), co)
