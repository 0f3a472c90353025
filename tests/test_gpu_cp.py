"""Context-parallel prefill on one GPU: W ranks emulated in one process (the
three phases of selective_state_space_43_b200.cp run rank by rank, the gathers
are Python lists), against the whole-sequence ssd_prefill and the oracle."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close, dev_inputs, np64
from selective_state_space_43_b200 import cp, ops
from selective_state_space_43_b200.synth import Dims, make_prefill_inputs

pytestmark = pytest.mark.gpu


class Fp32YKernels(cp.CudaKernels):
    """The library's kernels with y in fp32 (the tolerance is stated on the unrounded y)."""

    @staticmethod
    def prefill(inp, init_state, init_conv_state, chunk):
        return ops.prefill(inp["x"], inp["dt"], inp["B"], inp["C"], inp["z"], inp["A"], inp["D"], inp["dt_bias"],
                           inp["conv_w"], inp["conv_b"], init_state, init_conv_state, chunk=chunk,
                           y_dtype=torch.float32)


def emulate(inp, segments, chunk, init=False, kernels=cp.CudaKernels):
    scans, t0 = [], 0
    for r, n in enumerate(segments):
        seg = {k: (v[:, t0:t0 + n].contiguous() if k in ("x", "z", "dt", "B", "C") else v) for k, v in inp.items()}
        scans.append(cp.SegmentScan(seg, r, len(segments), inp["init_state"] if init else None,
                                    inp["init_conv_state"] if init else None, chunk, kernels))
        t0 += n
    windows = [s.window() for s in scans]
    parts = [s.local_pass(windows) for s in scans]
    states = torch.stack([p[0] for p in parts])
    sums = torch.stack([p[1] for p in parts])
    return [s.final_pass(states, sums) for s in scans]


def test_two_segments_on_chunk_boundaries_are_bit_exact():
    d = Dims(2, 640, 16, 64, 128, 2, 128)
    inp = dev_inputs(make_prefill_inputs(d, dtype=torch.bfloat16, seed=501))
    outs = emulate(inp, [256, 384], d.chunk)
    y, fs, cs = ops.prefill(inp["x"], inp["dt"], inp["B"], inp["C"], inp["z"], inp["A"], inp["D"], inp["dt_bias"],
                            inp["conv_w"], inp["conv_b"], chunk=d.chunk)
    ops.device_status()
    assert torch.equal(torch.cat([o[0] for o in outs], dim=1), y)
    assert torch.equal(outs[1][1], fs) and torch.equal(outs[1][2], cs)


@pytest.mark.parametrize("d,dtype", [(Dims(1, 701, 32, 64, 128, 4, 128), torch.bfloat16),
                                     (Dims(2, 701, 4, 64, 32, 1, 64), torch.float32)])
def test_four_ragged_segments_match_the_oracle(d, dtype):
    segments = [200, 137, 300, 64]
    host = make_prefill_inputs(d, dtype=dtype, seed=502, init_state=True, init_conv_state=True)
    inp = dev_inputs(host)
    outs = emulate(inp, segments, d.chunk, init=True, kernels=Fp32YKernels)
    ops.device_status()
    yo, fo, co = oracle.prefill(host)
    assert_close(np64(torch.cat([o[0] for o in outs], dim=1)), yo, "context-parallel y")
    assert_close(np64(outs[-1][1]), fo, "context-parallel final state")
    assert np.array_equal(np64(outs[-1][2]), co)


def test_helpers_match_their_definitions():
    d = Dims(3, 300, 8, 64, 64, 2, 128)
    host = make_prefill_inputs(d, dtype=torch.bfloat16, seed=503, init_state=True, init_conv_state=True)
    inp = dev_inputs(host)
    # the window is the conv_state ssd_prefill returns
    _, _, cs = ops.prefill(inp["x"], inp["dt"], inp["B"], inp["C"], inp["z"], inp["A"], inp["D"], inp["dt_bias"],
                           inp["conv_w"], inp["conv_b"], None, inp["init_conv_state"], chunk=d.chunk)
    assert torch.equal(ops.conv_window(inp["x"], inp["B"], inp["C"], inp["init_conv_state"]), cs)
    short = {k: inp[k][:, :2].contiguous() for k in ("x", "B", "C")}
    _, _, cs2 = oracle.prefill({**host, **{k: host[k][:, :2] for k in ("x", "z", "dt", "B", "C")}})
    assert np.array_equal(np64(ops.conv_window(short["x"], short["B"], short["C"], inp["init_conv_state"])), cs2)
    # sum of softplus(dt + bias), against fp64
    got = np64(ops.dt_sum(inp["dt"], inp["dt_bias"]))
    want = np.log1p(np.exp(host["dt"].double().numpy() + host["dt_bias"].double().numpy())).sum(axis=1)
    np.testing.assert_allclose(got, want, rtol=2e-5)
    # the fold of two segments over an initial state
    seg = torch.randn((2, 3, 8, 64, 64), device="cuda")
    sums = torch.rand((2, 3, 8), device="cuda") * 3
    s_in = ops.cp_combine(seg, sums, inp["A"], 2, inp["init_state"])
    e = lambda q: torch.exp(inp["A"].double()[None, :, None, None] * sums[q].double()[:, :, None, None])
    want = e(1) * (e(0) * inp["init_state"].double() + seg[0].double()) + seg[1].double()
    np.testing.assert_allclose(np64(s_in), want.cpu().numpy(), rtol=1e-5, atol=1e-6)
    assert torch.equal(ops.cp_combine(seg, sums, inp["A"], 0, None), torch.zeros_like(s_in))
