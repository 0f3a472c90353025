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


def test_algorithmic_byte_and_flop_counts_per_token():
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
    # the tensor-core chunk backward: fp32 post-conv x|B|C, dt, cs; bf16 dy, z, dt; fp16 states and adjoints
    # with an fp32 scale per state row; dz, dx, two halves of dB|dC, ddt written (fp32), the per-chunk partials
    reads = 4096 * (8192 + 2048) * 4 + 4096 * 2 * 128 * 4 + 4096 * (2 * 8192 + 128) * 2 + \
        2 * 64 * 128 * 64 * (128 * 2 + 4) + 64 * 128 * 16
    writes = 4096 * 2 * 8192 * 4 + 2 * 4096 * 2048 * 4 + 4096 * 128 * 4 + 64 * 128 * 12
    assert bench.backward_chunk_bytes(d, 2) == reads + writes


def test_mimo_decode_byte_count():
    from selective_state_space_43_b200.synth import WORKLOADS
    d = WORKLOADS["decode_nemotron_h_8b"]["dims"]
    # the fp32 state read and written dominates: 2 x 1.07 GB, plus x, z, y (rank 4) and B, C (rank 4)
    state = 2 * 256 * 128 * 64 * 128 * 4
    assert bench.mimo_decode_bytes(d, 4, 2) == state + 3 * 256 * 128 * 4 * 64 * 2 + 2 * 256 * 8 * 4 * 128 * 2 + \
        256 * 128 * 2
    assert bench.mimo_decode_bytes(d, 1, 2) < bench.mimo_decode_bytes(d, 4, 2) < 1.03 * state


class _FakeEvent:
    def __init__(self, enable_timing=False):
        pass

    def record(self, *a):
        pass

    def elapsed_time(self, other):
        return 2.0  # ms


class _FakeSampler:
    def load(self, on):
        pass


class _FakeOps:
    """Stands in for the binding: checks the call shapes the bench legs make, computes nothing."""

    def __init__(self):
        from selective_state_space_43_b200 import ops
        self.make_dims = ops.make_dims
        self.calls = {"backward": 0, "mimo": 0, "events": []}

    def prefill_backward_workspace_bytes(self, dims):
        return 1024

    def prefill_backward(self, x, dt, B, C, z, A, D, dt_bias, conv_w, conv_b, dy, init_state, init_conv_state,
                         d_final_state, workspace=None):
        assert dy.shape == x.shape and d_final_state.shape[0] == x.shape[0] and workspace.numel() >= 1024
        self.calls["backward"] += 1
        return {}

    def mimo_decode_step(self, x, dt, B, C, z, A, D, dt_bias, ssm_state, y=None):
        assert x.shape[2] == bench.MIMO_RANK and y.shape == x.shape and ssm_state.dtype == torch.float32
        self.calls["mimo"] += 1
        return y

    def set_timing_events(self, before, after):
        self.calls["events"].append(before is None)


def test_backward_and_mimo_bench_legs_on_a_fake_device(monkeypatch):
    from selective_state_space_43_b200.synth import Dims
    monkeypatch.setattr(torch.cuda, "Event", _FakeEvent)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    fake = _FakeOps()
    d = Dims(1, 256, 4, 64, 32, 2, 128)
    flush = torch.empty(16)
    peaks = {"hbm_gbs": 6554.6}
    b = bench.bench_backward(fake, d, torch.bfloat16, torch.device("cpu"), flush, 5, 3, 1, _FakeSampler(), peaks)
    assert fake.calls["backward"] == 3 + 5 and fake.calls["events"][-1] is True   # hook cleared afterwards
    assert b["ms_per_step"] == 2.0 and b["value"] == 256 / 2e-3
    rf = b["dominant_kernel"]["roofline"]
    assert rf["bound"] == "hbm" and rf["unit"] == "GB/s" and rf["peak"] == 6554.6
    assert abs(rf["achieved"] - bench.backward_chunk_bytes(d, 2) / 2e-3 / 1e9) < 1e-6
    m = bench.bench_mimo(fake, d, torch.bfloat16, torch.device("cpu"), 1, _FakeSampler(), peaks, 4)
    assert fake.calls["mimo"] == 3 + 4
    # the 4 timed steps run back to back between one pair of events (2 ms on the fake clock)
    assert m["ms_per_step"] == 2.0 / 4
    assert abs(m["value"] - bench.mimo_decode_bytes(d, bench.MIMO_RANK, 2) / 0.5e-3 / 1e9) < 1e-6
    assert m["roofline"]["frac"] == m["roofline"]["achieved"] / 6554.6


def test_oracle_baselines_of_the_backward_and_mimo_lines():
    from selective_state_space_43_b200.synth import Dims
    d = Dims(1, 96, 4, 64, 16, 2, 64)
    b = bench.cpu_backward_baseline(d, torch.bfloat16)
    assert b["kind"] == "oracle" and b["unit"] == "tokens/s" and b["value"] > 0 and "2 of 4 heads" in b["sample"]
    m = bench.cpu_mimo_baseline(Dims(4, 1, 4, 64, 16, 2, 64), torch.bfloat16, nseq=2)
    assert m["kind"] == "oracle" and m["unit"] == "GB/s" and m["value"] > 0


def test_host_prefill_pieces():
    from selective_state_space_43_b200.ops import host_pieces
    assert host_pieces(4096, 128) == [(r, r + 512) for r in range(0, 4096, 512)]   # 8 pieces of 4 chunks
    assert host_pieces(1000, 128, 3) == [(0, 384), (384, 768), (768, 1000)]       # rounded up to chunks
    assert host_pieces(300, 128) == [(0, 300)]                                       # one piece
    assert host_pieces(300, 128, 8) == [(0, 128), (128, 256), (256, 300)]
    assert host_pieces(0, 128) == [(0, 0)]
    for L in (1, 127, 129, 777, 5000):
        for segs in (None, 1, 2, 5, 9):
            p = host_pieces(L, 64, segs)
            assert p[0][0] == 0 and p[-1][1] == L
            assert all(a[1] == b[0] for a, b in zip(p, p[1:]))
            assert all(r0 % 64 == 0 for r0, _ in p)                                 # chunk-aligned starts


def test_oracle_baselines_of_the_prefill_and_decode_lines():
    from selective_state_space_43_b200.synth import Dims, make_decode_inputs, make_prefill_inputs
    d = Dims(2, 96, 4, 64, 16, 2, 64)
    inp = make_prefill_inputs(d, dtype=torch.bfloat16, seed=5, init_state=True)
    p = bench.cpu_baseline(inp, d, 0.0, "tiny")
    assert p["kind"] == "oracle" and p["unit"] == "tokens/s" and p["value"] > 0 and "of the tiny workload" in p["sample"]
    dd = Dims(4, 1, 4, 64, 16, 2, 64)
    data = make_decode_inputs(dd, steps=3, seed=6)
    sample = {"params": data["params"], "ssm_state": data["ssm_state"][:2].clone(),
              "conv_state": data["conv_state"][:2].clone(),
              "steps": [{k: v[:2].clone() for k, v in s.items()} for s in data["steps"]]}
    r = bench.cpu_decode_baseline(sample, dd, 3, 2)
    assert r["kind"] == "oracle" and r["unit"] == "GB/s" and r["value"] > 0 and "2 of the 4 sequences" in r["sample"]
    # the baseline leaves the sample's states untouched (it steps copies)
    assert torch.equal(sample["ssm_state"], data["ssm_state"][:2])


def test_headline_is_the_largest_single_gpu_prefill_workload():
    from selective_state_space_43_b200.synth import WORKLOADS
    prefill = [n for n in WORKLOADS if not n.startswith("decode")]
    tokens = {n: WORKLOADS[n]["dims"].batch * WORKLOADS[n]["dims"].seqlen for n in prefill}
    nbytes = {n: bench.prefill_bytes(WORKLOADS[n]["dims"], 2, WORKLOADS[n]["init_state"]) for n in prefill}
    assert bench.HEADLINE_WORKLOAD == max(prefill, key=lambda n: (nbytes[n], tokens[n]))
    assert set(bench.OTHER_PREFILL_WORKLOADS) == set(prefill) - {bench.HEADLINE_WORKLOAD}


def test_bidirectional_link_floor():
    # no slowdown when both directions run: the floor is the longer direction alone
    same = {"h2d_gbs": 50.0, "d2h_gbs": 40.0, "h2d_both_gbs": 50.0, "d2h_both_gbs": 40.0}
    assert abs(bench.link_floor_bidir_ms(500e6, 200e6, same) - 10.0) < 1e-9
    # both directions at half rate while together: 100 MB out overlaps 4 ms of the way in
    slow = {"h2d_gbs": 50.0, "d2h_gbs": 50.0, "h2d_both_gbs": 25.0, "d2h_both_gbs": 25.0}
    # together 4 ms (100 MB in, 100 MB out), then 400 MB in alone at 50 GB/s = 8 ms
    assert abs(bench.link_floor_bidir_ms(500e6, 100e6, slow) - 12.0) < 1e-9
