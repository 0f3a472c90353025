"""ssd_prefill_noalloc: the prefill entry point for callers that cannot
allocate device memory (no allocator they may use, or an allocation would
break their memory plan), which keeps its scratch in a fixed array inside the
library.  The same kernels run on the same inputs as ssd_prefill, so its
results must equal ssd_prefill's bit for bit, on two calls in a row (the second
call finds the first call's leftovers in the shared array), and after a longer
call has filled more of the array than a shorter one with a ragged last chunk
rewrites (the shorter call must read none of the longer call's rows).

Collected last on purpose (file name), so that a run stopping at the first
failure has already run every other test."""
import ctypes

import pytest
import torch

from gpu_util import dev_inputs
from selective_state_space_43_b200 import ops
from selective_state_space_43_b200.synth import Dims, make_prefill_inputs

pytestmark = pytest.mark.gpu


def _run(fn, d, seed, y_dtype):
    inp = dev_inputs(make_prefill_inputs(d, dtype=torch.bfloat16, seed=seed, init_state=True, init_conv_state=True))
    return fn(inp["x"], inp["dt"], inp["B"], inp["C"], inp["z"], inp["A"], inp["D"], inp["dt_bias"],
              inp["conv_w"], inp["conv_b"], inp["init_state"], inp["init_conv_state"], chunk=d.chunk,
              y_dtype=y_dtype)


def _scratch_bytes(d):
    dims = ops.make_dims(d.batch, d.seqlen, d.nheads, d.headdim, d.d_state, d.ngroups, d.chunk)
    return ops.prefill_workspace_bytes(dims, torch.bfloat16)


def _assert_equal(got, want, what):
    torch.cuda.synchronize()
    ops.device_status()
    for name, g, w in zip(("y", "final_state", "conv_state"), got, want):
        assert torch.equal(g, w), f"{what}: {name} differs from ssd_prefill's"


@pytest.mark.parametrize("y_dtype", [torch.float32, torch.bfloat16])
def test_noalloc_matches_prefill_on_two_calls_in_a_row(y_dtype):
    # Nemotron-H 8B layer shape (16 heads per group), 2 x 1000 tokens with a ragged last chunk:
    # 2 * 1000 * 2 * 2 * 128 * 2 bytes of post-conv B/C scratch, inside the 16 MiB built-in array
    d = Dims(2, 1000, 32, 64, 128, 2, 128)
    assert _scratch_bytes(d) == 2 * 1000 * 2 * 2 * 128 * 2 <= ops.NOALLOC_SCRATCH_BYTES
    for seed in (201, 202):
        want = _run(ops.prefill, d, seed, y_dtype)
        got = _run(ops.prefill_noalloc, d, seed, y_dtype)
        _assert_equal(got, want, f"seed {seed}")


def test_noalloc_shorter_call_after_a_longer_one():
    # a call over 2 x 2000 tokens fills 4 MB of the array; the next call (2 x 1000 tokens, last chunk
    # of 104 rows) reuses its first 2 MB, and must match ssd_prefill with a fresh workspace
    long_d, short_d = Dims(2, 2000, 32, 64, 128, 2, 128), Dims(2, 1000, 32, 64, 128, 2, 128)
    assert _scratch_bytes(short_d) < _scratch_bytes(long_d) <= ops.NOALLOC_SCRATCH_BYTES
    _run(ops.prefill_noalloc, long_d, 211, torch.bfloat16)
    want = _run(ops.prefill, short_d, 212, torch.bfloat16)
    got = _run(ops.prefill_noalloc, short_d, 212, torch.bfloat16)
    _assert_equal(got, want, "after a longer call")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # 4 x 8192 tokens of the Nemotron 3 Nano layer need 128 MiB of scratch: rejected before any launch
    d = Dims(4, 8192, 64, 64, 128, 8, 128)
    dims = ops.make_dims(d.batch, d.seqlen, d.nheads, d.headdim, d.d_state, d.ngroups, d.chunk)
    assert ops.prefill_workspace_bytes(dims, torch.bfloat16) > ops.NOALLOC_SCRATCH_BYTES
    prm = ops.SsdParams(0x1000, 0x2000, 0x3000, 0x4000, 0x5000)
    code = ops.lib().ssd_prefill_noalloc(ctypes.byref(dims), ops.SSD_BF16, ctypes.byref(prm), 0x10000, 0x20000,
                                         0x30000, 0x40000, 0x50000, None, None, 0x60000, 0x70000, 0x80000, None)
    assert code == 7
