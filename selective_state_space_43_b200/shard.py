"""Head-group sharding of one Mamba-2 layer's prefill across ranks (one process per GPU).

A Mamba-2 layer's H heads fall into G groups, and the heads of a group share one
B and one C ("Nemotron-H 스타일 Hybrid Mamba-Transformer 3B 모델 구현 타당성 분석",
table 1.4: n_groups = 8).  The groups are independent of one another: a head's
conv channels, state and output depend only on its own x, z and dt channels and
on its group's B and C.  Giving each of W ranks G/W whole groups therefore needs
no exchange at all, and no rank holds another rank's B or C.  Rank r takes groups
[r*G/W, (r+1)*G/W) and their heads, reads its slices of the layer's x, z, B and C
in place (strided views of the full arrays), and returns its shard of every
output:

  y            [Bt, L, H_r*P]       the rank's heads (what a row-parallel
                                     out_proj consumes without a gather)
  final_state  [Bt, H_r, P, N]
  conv_state   [Bt, conv_dim_r, 3]  channels [x of its heads | its B | its C]

``gather_shards`` puts the W shards back into the whole layer's layout (tests,
or a caller that wants the full outputs).  The CUDA path is the library's
prefill on the shard; ``kernels`` lets the host logic run with other kernels
(the tests' fp64 stand-ins on CPU ranks).
"""
from __future__ import annotations

import torch

from . import ops


def group_range(G: int, world: int, rank: int) -> tuple[int, int]:
    """Groups [g0, g1) of ``rank``: G/W consecutive groups each (G must be a multiple of W)."""
    if world <= 0 or G % world != 0:
        raise ValueError(f"{G} groups cannot be split evenly over {world} ranks")
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside [0, {world})")
    per = G // world
    return rank * per, (rank + 1) * per


def shard_channels(H: int, P: int, G: int, N: int, g0: int, g1: int):
    """The conv channels of groups [g0, g1) in the layer's [x | B | C] order, as three index ranges."""
    hpg = H // G
    h0, h1 = g0 * hpg, g1 * hpg
    HP, GN = H * P, G * N
    return (h0 * P, h1 * P), (HP + g0 * N, HP + g1 * N), (HP + GN + g0 * N, HP + GN + g1 * N)


def shard_inputs(inp: dict, world: int, rank: int) -> dict:
    """The inputs of ``rank``'s shard of a prefill (``inp`` as make_prefill_inputs: x, z [Bt, L, H*P], dt
    [Bt, L, H], B, C [Bt, L, G, N], the parameters and the optional initial states).  x, z, B and C are
    views of the full arrays (read in place); dt (H_r values per token, rarely 16-byte aligned as a view),
    the per-head parameters, the conv taps of the shard's channels and the initial states are copied."""
    Bt, L, HP = inp["x"].shape
    G, N = inp["B"].shape[2], inp["B"].shape[3]
    H = inp["A"].shape[0]
    P = HP // H
    if H % G != 0:
        raise ValueError("nheads must be a multiple of ngroups")
    g0, g1 = group_range(G, world, rank)
    hpg = H // G
    h0, h1 = g0 * hpg, g1 * hpg
    rx, rb, rc = shard_channels(H, P, G, N, g0, g1)
    chans = torch.cat([torch.arange(*rx), torch.arange(*rb), torch.arange(*rc)]).to(inp["conv_w"].device)
    out = {
        "x": inp["x"][:, :, rx[0]:rx[1]], "z": inp["z"][:, :, rx[0]:rx[1]],
        "dt": inp["dt"][:, :, h0:h1].contiguous(),
        "B": inp["B"][:, :, g0:g1], "C": inp["C"][:, :, g0:g1],
        "A": inp["A"][h0:h1].contiguous(), "D": inp["D"][h0:h1].contiguous(),
        "dt_bias": inp["dt_bias"][h0:h1].contiguous(),
        "conv_w": inp["conv_w"].index_select(0, chans).contiguous(),
        "conv_b": inp["conv_b"].index_select(0, chans).contiguous(),
        "init_state": None, "init_conv_state": None,
    }
    if inp.get("init_state") is not None:
        out["init_state"] = inp["init_state"][:, h0:h1].contiguous()
    if inp.get("init_conv_state") is not None:
        out["init_conv_state"] = inp["init_conv_state"].index_select(
            1, chans.to(inp["init_conv_state"].device)).contiguous()
    return out


class CudaKernels:
    """The library's prefill (strided entry point for the views)."""

    @staticmethod
    def prefill(inp, chunk, y_dtype=None):
        return ops.prefill(inp["x"], inp["dt"], inp["B"], inp["C"], inp["z"], inp["A"], inp["D"], inp["dt_bias"],
                           inp["conv_w"], inp["conv_b"], inp["init_state"], inp["init_conv_state"], chunk=chunk,
                           y_dtype=y_dtype)


def prefill_group_sharded(inp: dict, world: int, rank: int, chunk: int = 128, kernels=CudaKernels, y_dtype=None):
    """``rank``'s shard of the layer's prefill: (y, final_state, conv_state) of its groups (layouts above).
    No collective: every rank reads only its own groups' inputs."""
    return kernels.prefill(shard_inputs(inp, world, rank), chunk, y_dtype)


def gather_shards(parts, H: int, P: int, G: int, N: int):
    """The W ranks' (y, final_state, conv_state) shards, rank order, back in the whole layer's layout."""
    world = len(parts)
    y = torch.cat([p[0] for p in parts], dim=2)
    fs = torch.cat([p[1] for p in parts], dim=1)
    per = [shard_channels(H, P, G, N, *group_range(G, world, r)) for r in range(world)]
    cs_parts = [p[2] for p in parts]
    xs, bs, cs = [], [], []
    for (rx, rb, rc), c in zip(per, cs_parts):
        nx, nb = rx[1] - rx[0], rb[1] - rb[0]
        xs.append(c[:, :nx])
        bs.append(c[:, nx:nx + nb])
        cs.append(c[:, nx + nb:])
    conv = torch.cat(xs + bs + cs, dim=1)
    return y, fs, conv


def prefill_group_sharded_dist(inp: dict, chunk: int = 128, group=None, kernels=CudaKernels, y_dtype=None):
    """prefill_group_sharded for this process's rank of ``group`` (torch.distributed)."""
    import torch.distributed as dist
    return prefill_group_sharded(inp, dist.get_world_size(group), dist.get_rank(group), chunk, kernels, y_dtype)
