"""GPU parity of ssd_prefill_varlen (packed variable-length batch) against the
fp64 oracle run on each sequence (needs a B200)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_bf16_is_rounded, assert_close, dev_inputs, np64
from selective_state_space_43_b200 import ops
from selective_state_space_43_b200.synth import Dims, make_varlen_inputs, varlen_lengths

pytestmark = pytest.mark.gpu


def gpu_varlen(dev, cu, chunk, y_dtype=None):
    return ops.prefill_varlen(dev["x"], dev["dt"], dev["B"], dev["C"], dev["z"], dev["A"], dev["D"],
                              dev["dt_bias"], dev["conv_w"], dev["conv_b"], cu, dev.get("init_state"),
                              dev.get("init_conv_state"), chunk=chunk, y_dtype=y_dtype)


def check_varlen(d, dtype, lengths, init, seed, tag):
    inp, cu = make_varlen_inputs(d, lengths, dtype=dtype, seed=seed, init_state=init, init_conv_state=init)
    dev = dev_inputs(inp)
    cu_dev = torch.tensor(cu, dtype=torch.int64, device="cuda")
    y, fs, cs = gpu_varlen(dev, cu_dev, d.chunk)
    if y.dtype == torch.bfloat16:
        y32, fs32, cs32 = gpu_varlen(dev, cu_dev, d.chunk, y_dtype=torch.float32)
        assert_bf16_is_rounded(y, y32, f"{tag} y")
        assert torch.equal(fs, fs32) and torch.equal(cs, cs32)
    else:
        y32 = y
    ops.device_status()
    yo, fo, co = oracle.prefill_varlen(inp, cu)
    yg, fg = np64(y32), np64(fs)
    for s in range(len(lengths)):
        r0, r1 = cu[s], cu[s + 1]
        if r1 > r0:
            assert_close(yg[r0:r1], yo[r0:r1], f"{tag} y of sequence {s} (length {r1 - r0})")
        assert_close(fg[s], fo[s], f"{tag} final_state of sequence {s} (length {r1 - r0})")
    assert np.array_equal(np64(cs), co), f"{tag} conv_state"
    return inp, cu, y, fs, cs


# empty, shorter than the conv window, ragged, exactly one chunk, several chunks
EDGE = [0, 1, 2, 3, 5, 127, 128, 129, 300, 0, 700]


@pytest.mark.parametrize("init", [False, True])
def test_varlen_tensor_core_path_matches_oracle(init):
    d = Dims(1, 1, 16, 64, 128, 2, 128)
    assert ops.prefill_path(ops.make_dims(len(EDGE), sum(EDGE), 16, 64, 128, 2, 128), torch.bfloat16) == 1
    check_varlen(d, torch.bfloat16, EDGE, init, seed=301, tag=f"varlen tc init={init}")


def test_varlen_tensor_core_path_d_state_64():
    d = Dims(1, 1, 8, 64, 64, 2, 64)
    assert ops.prefill_path(ops.make_dims(len(EDGE), sum(EDGE), 8, 64, 64, 2, 64), torch.bfloat16) == 1
    check_varlen(d, torch.bfloat16, EDGE, True, seed=306, tag="varlen tc n64")


@pytest.mark.parametrize("name,d,dtype", [
    ("fp32_q64", Dims(1, 1, 4, 64, 32, 1, 64), torch.float32),
    ("bf16_n32", Dims(1, 1, 8, 64, 32, 2, 128), torch.bfloat16),
])
def test_varlen_cuda_core_path_matches_oracle(name, d, dtype):
    assert ops.prefill_path(ops.make_dims(len(EDGE), sum(EDGE), d.nheads, 64, d.d_state, d.ngroups, d.chunk),
                            dtype) == 2
    check_varlen(d, dtype, EDGE, True, seed=302, tag=f"varlen simt {name}")


def test_varlen_layer_shape_mixed_lengths():
    # Nemotron-H 8B head / group shape, a continuous-batching mix of lengths; a sample of heads is
    # checked by the oracle sequence by sequence
    d = Dims(1, 1, 32, 64, 128, 4, 128)
    lengths = varlen_lengths(6, 40, 1500, seed=303)
    check_varlen(d, torch.bfloat16, lengths, True, seed=304, tag="varlen layer shape")


def test_equal_lengths_match_the_batched_entry_point_bit_for_bit():
    d = Dims(3, 300, 16, 64, 128, 2, 128)
    inp, cu = make_varlen_inputs(d, [300, 300, 300], dtype=torch.bfloat16, seed=305, init_state=True,
                                 init_conv_state=True)
    dev = dev_inputs(inp)
    y, fs, cs = gpu_varlen(dev, torch.tensor(cu, dtype=torch.int64, device="cuda"), d.chunk)
    yb, fsb, csb = ops.prefill(dev["x"].view(3, 300, -1), dev["dt"].view(3, 300, -1),
                               dev["B"].view(3, 300, d.ngroups, d.d_state),
                               dev["C"].view(3, 300, d.ngroups, d.d_state), dev["z"].view(3, 300, -1),
                               dev["A"], dev["D"], dev["dt_bias"], dev["conv_w"], dev["conv_b"],
                               dev["init_state"], dev["init_conv_state"], chunk=d.chunk)
    ops.device_status()
    assert torch.equal(y.view(3, 300, -1), yb) and torch.equal(fs, fsb) and torch.equal(cs, csb)


def test_invalid_offsets_are_reported_and_treated_as_empty():
    d = Dims(1, 1, 16, 64, 128, 2, 128)
    lengths = [5, 200, 40]
    inp, cu = make_varlen_inputs(d, lengths, dtype=torch.bfloat16, seed=306, init_state=True)
    dev = dev_inputs(inp)
    bad = [0, 5, 3, cu[-1]]  # sequence 1 runs backwards: it is skipped, sequences 0 and 2 are scanned
    y, fs, cs = gpu_varlen(dev, torch.tensor(bad, dtype=torch.int64, device="cuda"), d.chunk)
    with pytest.raises(ops.SsdError) as e:
        ops.device_status()
    assert e.value.status == 2
    ops.device_status()  # the report clears the flag
    assert torch.equal(fs[1], dev["init_state"][1])  # an empty sequence passes its state through
    yo, fo, co = oracle.prefill_varlen(inp, [0, 5, 5, cu[-1]])
    assert_close(np64(fs[0]), fo[0], "valid sequence 0 next to an invalid one")
