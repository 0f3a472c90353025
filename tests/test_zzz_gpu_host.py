"""The end-to-end host API (ops.prefill_host: pinned host tensors in and out) on the GPU: the
segmented pipeline (copies in, scans and copies out overlapped on three streams, states chained
from piece to piece on chunk boundaries) returns exactly what one device-side ssd_prefill call
returns on the tensor-core path, and agrees with the oracle on the CUDA-core path (needs a B200)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close, dev_inputs, gpu_prefill, np64
from selective_state_space_43_b200 import ops
from selective_state_space_43_b200.synth import Dims, make_prefill_inputs

pytestmark = pytest.mark.gpu


def pinned(inp):
    return {k: (None if v is None else v.pin_memory()) for k, v in inp.items()}


@pytest.mark.parametrize("Bt,L,segments", [(1, 1024, 4), (2, 1000, 3), (1, 4096, None), (2, 300, 8)])
def test_pipelined_host_prefill_is_bit_exact(Bt, L, segments):
    d = Dims(Bt, L, 16, 64, 128, 2, 128)
    inp = make_prefill_inputs(d, dtype=torch.bfloat16, seed=L + Bt, init_state=True, init_conv_state=True)
    (yh, fh, ch), h2d, d2h = ops.prefill_host(pinned(inp), chunk=d.chunk, segments=segments)
    torch.cuda.synchronize()
    y, fs, cs = gpu_prefill(dev_inputs(inp), d.chunk)
    torch.cuda.synchronize()
    assert torch.equal(yh, y.cpu()) and torch.equal(fh, fs.cpu()) and torch.equal(ch, cs.cpu())
    assert h2d == sum(t.numel() * t.element_size() for t in inp.values() if t is not None)
    assert d2h == yh.numel() * 2 + fh.numel() * 4 + ch.numel() * 2
    (yw, fw, cw), _, _ = ops.prefill_host(pinned(inp), chunk=d.chunk, segments=1)
    torch.cuda.synchronize()
    assert torch.equal(yw, yh) and torch.equal(fw, fh) and torch.equal(cw, ch)


def test_pipelined_host_prefill_cuda_core_path():
    d = Dims(2, 200, 4, 64, 32, 1, 64)
    inp = make_prefill_inputs(d, dtype=torch.float32, seed=7, init_state=True, init_conv_state=True)
    (yh, fh, ch), _, _ = ops.prefill_host(pinned(inp), chunk=d.chunk, segments=3)
    torch.cuda.synchronize()
    yo, fo, co = oracle.prefill(inp)
    assert_close(np64(yh), yo, "host pipeline y (CUDA-core path)")
    assert_close(np64(fh), fo, "host pipeline final_state (CUDA-core path)")
    assert np.array_equal(np64(ch), co)


def test_repeated_calls_reuse_memory_safely():
    # back-to-back calls without a synchronisation between them: buffers freed by one call and
    # reused by the next must not be overwritten while a side stream still reads them
    d = Dims(1, 2048, 16, 64, 128, 2, 128)
    inps = [make_prefill_inputs(d, dtype=torch.bfloat16, seed=s, init_state=True) for s in (1, 2, 3)]
    outs = [ops.prefill_host(pinned(i), chunk=d.chunk)[0] for i in inps]
    torch.cuda.synchronize()
    for i, o in zip(inps, outs):
        y, fs, _ = gpu_prefill(dev_inputs(i), d.chunk)
        torch.cuda.synchronize()
        assert torch.equal(o[0], y.cpu()) and torch.equal(o[1], fs.cpu())


@pytest.mark.parametrize("segments", [1, 4])
def test_host_prefill_into_callers_pinned_outputs(segments):
    # the caller's pinned output buffers are written in place and returned, on both the one-piece and the
    # pipelined path; reusing them on the next call gives that call's results
    d = Dims(2, 700, 16, 64, 128, 2, 128)
    first = make_prefill_inputs(d, dtype=torch.bfloat16, seed=31, init_state=True, init_conv_state=True)
    second = make_prefill_inputs(d, dtype=torch.bfloat16, seed=32, init_state=True, init_conv_state=True)
    want = [ops.prefill_host(pinned(i), chunk=d.chunk, segments=segments)[0] for i in (first, second)]
    torch.cuda.synchronize()
    out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in want[0]]
    for inp, w in zip((first, second), want):
        got, _, _ = ops.prefill_host(pinned(inp), chunk=d.chunk, segments=segments, out=out)
        torch.cuda.synchronize()
        assert all(g is o for g, o in zip(got, out))
        assert all(torch.equal(g, x) for g, x in zip(got, w))
    with pytest.raises(ValueError):
        ops.prefill_host(pinned(first), chunk=d.chunk, out=[out[0], out[1], out[1]])
