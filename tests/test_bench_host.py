"""Host-side logic of the multi-GPU bench (one process per GPU, independent
sequences per rank, max-over-ranks timing), exercised with 2 gloo ranks on CPU."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    w, r, local = bench.dist_setup()
    assert (w, r, local) == (world, rank, rank)
    bench.barrier(w)
    # rank 1 is the slower one: the job's step time is the max, tokens add up over ranks
    value, ms = bench.weak_scaling_value(4096, 1.0 + rank, w, torch.device("cpu"))
    out[rank] = (value, ms)
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_rank_weak_scaling_aggregation():
    if not torch.distributed.is_gloo_available():
        pytest.skip("gloo backend not available")
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        value, ms = out[r]
        assert ms == pytest.approx(2.0)
        assert value == pytest.approx(2 * 4096 / 2.0e-3)


def test_single_rank_needs_no_process_group():
    os.environ.pop("WORLD_SIZE", None)
    w, r, local = bench.dist_setup()
    assert (w, r) == (1, 0)
    value, ms = bench.weak_scaling_value(4096, 0.5, 1, torch.device("cpu"))
    assert ms == 0.5 and value == pytest.approx(4096 / 0.5e-3)


def test_algorithmic_byte_and_flop_counts_match_the_survey_figures():
    from selective_state_space_43_b200.synth import WORKLOADS
    d = WORKLOADS["nemotron_h_8b"]["dims"]
    # 53,504 B per token of activations plus the 4.19 MB final state and the conv tail
    assert bench.prefill_bytes(d, 2, False) == 4096 * 53504 + 128 * 64 * 128 * 4 + 10240 * 3 * 2
    assert bench.prefill_flops(d) == 4096 * 6553600
    dd = WORKLOADS["decode_nemotron_h_8b"]["dims"]
    total, _ = bench.decode_bytes(dd, 2)
    assert abs(total / 1e6 - 2192.6) < 0.1


def test_backward_work_counts():
    from selective_state_space_43_b200.synth import WORKLOADS
    d = WORKLOADS["nemotron_h_8b"]["dims"]
    # per token: x, z, dt, B, C and dy read as bf16, their fp32 gradients written; two fp32 states
    per_token = (2 * 8192 + 128 + 2 * 1024) * 2 + 8192 * 2 + (2 * 8192 + 128 + 2 * 1024) * 4
    assert bench.backward_bytes(d, 2) == 4096 * per_token + 2 * 128 * 64 * 128 * 4
    # 64 chunks of 64 tokens; per head 8QPN + 4Q^2P + 2Q^2N, per group 2Q^2N
    per_head = 8 * 64 * 64 * 128 + 4 * 64 * 64 * 64 + 2 * 64 * 64 * 128
    assert bench.backward_chunk_flops(d) == 64 * (128 * per_head + 8 * 2 * 64 * 64 * 128)
    assert abs(bench.FP32_ALU_TFLOPS - 74.45) < 0.01


def test_mimo_decode_byte_count():
    from selective_state_space_43_b200.synth import WORKLOADS
    d = WORKLOADS["decode_nemotron_h_8b"]["dims"]
    # the fp32 state read and written dominates: 2 x 1.07 GB, plus x, z, y (rank 4) and B, C (rank 4)
    state = 2 * 256 * 128 * 64 * 128 * 4
    assert bench.mimo_decode_bytes(d, 4, 2) == state + 3 * 256 * 128 * 4 * 64 * 2 + 2 * 256 * 8 * 4 * 128 * 2 + \
        256 * 128 * 2
    assert bench.mimo_decode_bytes(d, 1, 2) < bench.mimo_decode_bytes(d, 4, 2) < 1.03 * state
