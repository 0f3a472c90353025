"""Context-parallel prefill: every sequence of a batch split into consecutive
segments, one per rank (one process per GPU, torch.distributed for the exchange).

The state after a segment is affine in the state before it,
S_out = exp(A * sum dt) * S_in + S_loc, so the ranks need one exchange (the
chunked SSD state passing of "EP6. 트랜스포머 대체 신경망 연구" §7-§8, carried
across devices): each rank scans its segment from zero, the (S_loc, sum dt) of
all ranks are gathered, each rank folds the segments before its own into its
initial state and scans its segment again from it.  The causal conv needs the
3 pre-conv tokens before a segment, which the previous rank provides.

``SegmentScan`` runs one rank's part in three phases, so that W ranks can also
be emulated in one process (tests); ``prefill_context_parallel`` drives the
phases with ``torch.distributed.all_gather`` (NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations

import torch

from . import ops


class CudaKernels:
    """The library's kernels (ssd_prefill, ssd_conv_window, ssd_dt_sum, ssd_cp_combine)."""

    @staticmethod
    def prefill(inp, init_state, init_conv_state, chunk):
        return ops.prefill(inp["x"], inp["dt"], inp["B"], inp["C"], inp["z"], inp["A"], inp["D"], inp["dt_bias"],
                           inp["conv_w"], inp["conv_b"], init_state, init_conv_state, chunk=chunk)

    @staticmethod
    def conv_window(inp):
        return ops.conv_window(inp["x"], inp["B"], inp["C"])

    @staticmethod
    def dt_sum(inp):
        return ops.dt_sum(inp["dt"], inp["dt_bias"])

    @staticmethod
    def combine(seg_states, dt_sums, A, upto, init_state):
        return ops.cp_combine(seg_states, dt_sums, A, upto, init_state)


class SegmentScan:
    """Rank ``rank`` of ``world``: ``inp`` holds this rank's segment of every sequence (x, z [Bt, Ls, H*P],
    dt [Bt, Ls, H], B, C [Bt, Ls, G, N]) and the layer parameters; ``init_state`` / ``init_conv_state`` are the
    sequences' initial states (used by rank 0; None = zeros).  Segments must hold at least 3 tokens."""

    def __init__(self, inp, rank, world, init_state=None, init_conv_state=None, chunk=128, kernels=CudaKernels):
        if inp["x"].shape[1] < 3 and world > 1:
            raise ValueError("context-parallel segments need at least 3 tokens")
        self.inp, self.rank, self.world, self.chunk, self.k = inp, rank, world, chunk, kernels
        self.init_state, self.init_conv_state = init_state, init_conv_state
        self.halo = None

    def window(self):
        """Phase 0: the pre-conv window this segment hands to the next rank, [Bt, conv_dim, 3]."""
        return self.k.conv_window(self.inp)

    def local_pass(self, windows):
        """Phase 1 (``windows`` = every rank's phase-0 result): scan the segment from zero.
        Returns (S_loc [Bt, H, P, N] fp32, sum dt [Bt, H] fp32) for the gather."""
        self.halo = self.init_conv_state if self.rank == 0 else windows[self.rank - 1]
        _, s_loc, _ = self.k.prefill(self.inp, None, self.halo, self.chunk)
        return s_loc, self.k.dt_sum(self.inp)

    def final_pass(self, seg_states, dt_sums):
        """Phase 2 (``seg_states`` [W, Bt, H, P, N], ``dt_sums`` [W, Bt, H] from every rank): scan the segment
        from its true initial state.  Returns (y, the state after this segment, its conv window)."""
        s_in = self.k.combine(seg_states, dt_sums, self.inp["A"], self.rank, self.init_state)
        return self.k.prefill(self.inp, s_in, self.halo, self.chunk)


def prefill_context_parallel(inp, init_state=None, init_conv_state=None, chunk=128, group=None,
                             kernels=CudaKernels):
    """This rank's segment of a context-parallel prefill over ``group``.  Returns (y of the segment, the
    state after it, its conv window); on the last rank these are the sequences' final states."""
    import torch.distributed as dist
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    scan = SegmentScan(inp, rank, world, init_state, init_conv_state, chunk, kernels)

    def gather(t):
        parts = [torch.empty_like(t) for _ in range(world)]
        dist.all_gather(parts, t.contiguous(), group=group)
        return parts

    windows = gather(scan.window())
    s_loc, dsum = scan.local_pass(windows)
    return scan.final_pass(torch.stack(gather(s_loc)), torch.stack(gather(dsum)))
