"""Head-group sharding of one layer's prefill, host logic: W gloo ranks on CPU,
each taking G/W whole groups through selective_state_space_43_b200.shard with
the fp64 oracle standing in for the CUDA prefill; the gathered shards must
equal the oracle's whole-layer prefill exactly (the groups are independent, so
each head's arithmetic is the same with or without the others)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from selective_state_space_43_b200 import shard
from selective_state_space_43_b200.synth import Dims, make_prefill_inputs

D_SHARD = Dims(2, 77, 8, 64, 16, 4, 32)   # 2 heads per group, ragged chunks


class Fp64Kernels:
    @staticmethod
    def prefill(inp, chunk, y_dtype=None):
        full = {k: (None if v is None else v.contiguous()) for k, v in inp.items()}
        y, fs, cs = oracle.prefill(full)
        return torch.from_numpy(y), torch.from_numpy(fs), torch.from_numpy(cs)


def _inputs():
    return make_prefill_inputs(D_SHARD, dtype=torch.float32, seed=611, init_state=True, init_conv_state=True,
                               random_D=True)


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    y, fs, cs = shard.prefill_group_sharded_dist(_inputs(), chunk=D_SHARD.chunk, kernels=Fp64Kernels)
    # the gather is the test's, not the path's: every rank's shard on every rank
    parts = []
    for t in (y, fs, cs):
        g = [torch.empty_like(t) for _ in range(world)]
        dist.all_gather(g, t.contiguous())
        parts.append(g)
    if rank == 0:
        out["parts"] = [tuple(parts[k][r].numpy() for k in range(3)) for r in range(world)]
    dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_ranks_reproduce_the_whole_layer(world):
    if not torch.distributed.is_gloo_available():
        pytest.skip("gloo backend not available")
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    parts = [tuple(torch.from_numpy(a) for a in p) for p in out["parts"]]
    d = D_SHARD
    y, fs, cs = shard.gather_shards(parts, d.nheads, d.headdim, d.ngroups, d.d_state)
    yo, fo, co = oracle.prefill(_inputs())
    assert np.array_equal(y.numpy(), yo)
    assert np.array_equal(fs.numpy(), fo)
    assert np.array_equal(cs.numpy(), co)


def test_group_ranges_and_channels():
    assert [shard.group_range(8, 4, r) for r in range(4)] == [(0, 2), (2, 4), (4, 6), (6, 8)]
    with pytest.raises(ValueError):
        shard.group_range(8, 3, 0)
    with pytest.raises(ValueError):
        shard.group_range(8, 2, 2)
    # Nemotron-H 8B layer, rank 1 of 4: heads 32..63, groups 2..3
    rx, rb, rc = shard.shard_channels(128, 64, 8, 128, 2, 4)
    assert rx == (32 * 64, 64 * 64) and rb == (8192 + 256, 8192 + 512) and rc == (8192 + 1024 + 256, 8192 + 1024 + 512)


def test_shard_inputs_pick_the_groups_channels():
    inp = _inputs()
    d = D_SHARD
    s = shard.shard_inputs(inp, 2, 1)   # groups 2, 3 -> heads 4..7
    assert torch.equal(s["x"], inp["x"][:, :, 4 * 64:8 * 64]) and not s["x"].is_contiguous()
    assert torch.equal(s["B"], inp["B"][:, :, 2:4]) and torch.equal(s["dt"], inp["dt"][:, :, 4:8])
    assert torch.equal(s["A"], inp["A"][4:8]) and torch.equal(s["init_state"], inp["init_state"][:, 4:8])
    HP, GN = d.nheads * d.headdim, d.ngroups * d.d_state
    want = torch.cat([inp["conv_w"][256:512], inp["conv_w"][HP + 32:HP + 64], inp["conv_w"][HP + GN + 32:HP + GN + 64]])
    assert torch.equal(s["conv_w"], want)
    assert torch.equal(s["init_conv_state"][:, 256:256 + 32], inp["init_conv_state"][:, HP + 32:HP + 64])
