"""Head-group sharding on one GPU: W ranks emulated in one process, each running
the library's prefill on its groups (strided views of the full layer's x, z, B,
C); the gathered shards must be bit-equal to one ssd_prefill of the whole layer
(each head's CTA does the same arithmetic either way) and, with y in fp32,
within the tolerance of the oracle."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close, dev_inputs, np64
from selective_state_space_43_b200 import ops, shard
from selective_state_space_43_b200.synth import Dims, make_prefill_inputs

pytestmark = pytest.mark.gpu


def _whole(inp, chunk, y_dtype=None):
    return ops.prefill(inp["x"], inp["dt"], inp["B"], inp["C"], inp["z"], inp["A"], inp["D"], inp["dt_bias"],
                       inp["conv_w"], inp["conv_b"], inp["init_state"], inp["init_conv_state"], chunk=chunk,
                       y_dtype=y_dtype)


@pytest.mark.parametrize("world", [2, 4, 8])
def test_group_shards_equal_the_whole_layer(world):
    # the Nemotron-H 8B layer (128 heads, 8 groups) over 1000 tokens: 16 * 8 / world heads per rank, all on
    # the tensor-core path
    d = Dims(1, 1000, 128, 64, 128, 8, 128)
    inp = dev_inputs(make_prefill_inputs(d, dtype=torch.bfloat16, seed=621, init_state=True, init_conv_state=True))
    parts = [shard.prefill_group_sharded(inp, world, r, chunk=d.chunk) for r in range(world)]
    want = _whole(inp, d.chunk)
    got = shard.gather_shards(parts, d.nheads, d.headdim, d.ngroups, d.d_state)
    ops.device_status()
    for name, g, w in zip(("y", "final_state", "conv_state"), got, want):
        assert torch.equal(g, w), f"{name} of {world} group shards differs from the whole layer"


def test_group_shards_match_the_oracle():
    d = Dims(2, 300, 16, 64, 128, 4, 128)
    host = make_prefill_inputs(d, dtype=torch.bfloat16, seed=622, init_state=True, init_conv_state=True)
    inp = dev_inputs(host)
    parts = [shard.prefill_group_sharded(inp, 2, r, chunk=d.chunk, y_dtype=torch.float32) for r in range(2)]
    y, fs, cs = shard.gather_shards(parts, d.nheads, d.headdim, d.ngroups, d.d_state)
    ops.device_status()
    yo, fo, co = oracle.prefill(host)
    assert_close(np64(y), yo, "group-sharded y")
    assert_close(np64(fs), fo, "group-sharded final_state")
    assert np.array_equal(np64(cs), co)
