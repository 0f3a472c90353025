"""Context-parallel prefill, host logic: W gloo ranks on CPU, each holding a
segment of the sequences, run selective_state_space_43_b200.cp with fp64
kernels (the oracle's prefill plus the plain definitions of the three helper
steps); the stitched result must equal the oracle's whole-sequence prefill."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from selective_state_space_43_b200 import cp
from selective_state_space_43_b200.synth import Dims, make_prefill_inputs

SEGMENTS = [37, 64, 3, 40]  # unequal, one of the minimum length 3


class Fp64Kernels:
    @staticmethod
    def prefill(inp, init_state, init_conv_state, chunk):
        y, fs, cs = oracle.prefill({**inp, "init_state": init_state, "init_conv_state": init_conv_state})
        return torch.from_numpy(y), torch.from_numpy(fs), torch.from_numpy(cs)

    @staticmethod
    def conv_window(inp):
        Bt, L = inp["x"].shape[:2]
        xbc = torch.cat([inp["x"], inp["B"].reshape(Bt, L, -1), inp["C"].reshape(Bt, L, -1)], dim=2)
        return xbc[:, L - 3:].transpose(1, 2).to(torch.float64).contiguous()

    @staticmethod
    def dt_sum(inp):
        return torch.nn.functional.softplus(inp["dt"].double() + inp["dt_bias"].double()).sum(dim=1)

    @staticmethod
    def combine(seg_states, dt_sums, A, upto, init_state):
        s = torch.zeros_like(seg_states[0]) if init_state is None else init_state.double().clone()
        for q in range(upto):
            s = torch.exp(A.double()[None, :, None, None] * dt_sums[q][:, :, None, None]) * s + seg_states[q]
        return s


def _inputs():
    d = Dims(2, sum(SEGMENTS), 4, 64, 16, 2, 16)
    return d, make_prefill_inputs(d, dtype=torch.float32, seed=404, init_state=True, init_conv_state=True)


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    d, inp = _inputs()
    t0 = sum(SEGMENTS[:rank])
    seg = {k: (v[:, t0:t0 + SEGMENTS[rank]] if k in ("x", "z", "dt", "B", "C") else v) for k, v in inp.items()}
    y, fs, cs = cp.prefill_context_parallel(seg, inp["init_state"].double(), inp["init_conv_state"].double(),
                                            chunk=d.chunk, kernels=Fp64Kernels)
    out[rank] = (y.numpy(), fs.numpy(), cs.numpy())
    dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_four_gloo_ranks_reproduce_the_whole_sequence():
    if not torch.distributed.is_gloo_available():
        pytest.skip("gloo backend not available")
    world = len(SEGMENTS)
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    d, inp = _inputs()
    yo, fo, co = oracle.prefill(inp)
    y = np.concatenate([out[r][0] for r in range(world)], axis=1)
    np.testing.assert_allclose(y, yo, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(out[world - 1][1], fo, rtol=1e-9, atol=1e-12)
    assert np.array_equal(out[world - 1][2], co)
    # every rank ends with the state after its own segment
    t1 = SEGMENTS[0]
    _, f0, _ = oracle.prefill({**inp, **{k: inp[k][:, :t1] for k in ("x", "z", "dt", "B", "C")}})
    np.testing.assert_allclose(out[0][1], f0, rtol=1e-9, atol=1e-12)
