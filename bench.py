#!/usr/bin/env python
"""Benchmark of the Mamba-2 SSD layer core on B200.

Headline (`value`): SSD prefill throughput in tokens/s for one Mamba-2 layer of
the Nemotron 3 Nano shape (batch 4, seqlen 8192, 64 heads x 64, d_state 128,
8 groups, chunk 128, bf16 activations, fp32 initial state ~ N(0, 0.1^2)), the
largest of the layer workloads that fit one GPU, inputs resident in HBM, L2
flushed between timed steps.  Also reported on the same line:
  roofline    the dominant prefill kernel's algorithmic bytes per launch over
              its own CUDA-event duration, against measured HBM bandwidth;
  tensor      algorithmic TFLOP/s of the step and its fraction of bf16 peak;
  e2e         the same prefill through the public API from pinned HOST
              tensors, host<->device copies inside the timed region;
  cpu_baseline the fp64 oracle timed on this host's cores on a sample of the
              same workload;
  configs     the same measurements (and an oracle sample each) for the other
              prefill workloads: the tiny fp32 case, the Nemotron-H 8B layer
              (B1 L4096) and the proposed 3B hybrid layer (B8 L4096);
  decode      GB/s of 64 consecutive decode steps for 256 sequences of the
              Nemotron-H 8B layer, fraction of measured HBM, oracle sample;
  varlen, gated_rmsnorm, backward, mimo_decode   the widened rows;
  clocks      SM clocks and throttle reasons sampled while timing.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Multi-GPU (weak scaling, no data-path collective: every rank runs its own
sequences): python -m torch.distributed.run --nproc-per-node N bench.py --gpus N
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from selective_state_space_43_b200.synth import (Dims, WORKLOADS, make_backward_grads,  # noqa: E402
                                                 make_decode_inputs, make_mimo_decode_inputs, make_prefill_inputs,
                                                 make_varlen_inputs, seed_of, varlen_lengths)

METRIC = "SSD prefill tokens/s per layer (% bf16 TC peak); decode GB/s (% of HBM peak)"
# the headline: the largest single-GPU prefill workload (B4 L8192 of the Nemotron 3 Nano layer, initial state);
# the other prefill workloads get lines of their own under "configs"
HEADLINE_WORKLOAD = "nemotron3_nano"
OTHER_PREFILL_WORKLOADS = ("tiny_fp32", "nemotron_h_8b", "hybrid_3b")
DECODE_WORKLOAD = "decode_nemotron_h_8b"
# the widened rows' lines run on the Nemotron-H 8B layer (B1 L4096)
BACKWARD_WORKLOAD = VARLEN_WORKLOAD = NORM_WORKLOAD = "nemotron_h_8b"
# the decode line's oracle sample: the first sequences of the batch for the first steps
DECODE_ORACLE_SEQS, DECODE_ORACLE_STEPS = 8, 4
L2_FLUSH_BYTES = 256 << 20
# continuous-batching mix for the packed variable-length prefill: this many sequences of the prefill
# workload's layer, lengths log-uniform in [VARLEN_MIN, VARLEN_MAX], each with its own initial state
VARLEN_NSEQ, VARLEN_MIN, VARLEN_MAX = 32, 64, 4096
# fp32 FMA peak of the CUDA cores, for the backward's SIMT chunk kernel: 148 SMs x 128 fp32 lanes x 2 flops
# per FMA x the 1965 MHz maximum SM clock
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
BWD_Q = 64  # the backward's chunk length
MIMO_RANK = 4     # rank of the MIMO decode line (the pages give no rank; 4 = a few SSMs per head)
MIMO_INPUTS = 4   # distinct step inputs the MIMO decode line cycles through
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------------------------------------
# algorithmic work (what the layer must read, write and compute, independent of the implementation)

def prefill_bytes(d: Dims, act_bytes: int, init_state: bool) -> int:
    tok = d.batch * d.seqlen
    inputs = tok * (2 * d.d_inner + d.nheads + 2 * d.ngroups * d.d_state) * act_bytes   # x, z, dt, B, C
    out = tok * d.d_inner * act_bytes                                                 # y
    state = d.batch * d.nheads * d.headdim * d.d_state * 4 * (2 if init_state else 1)
    conv = d.batch * d.conv_dim * 3 * act_bytes
    return inputs + out + state + conv


def varlen_bytes(d: Dims, T: int, nseq: int, act_bytes: int) -> int:
    """Algorithmic bytes of one packed prefill: T rows of inputs and y, per-sequence states in and out."""
    inputs = T * (2 * d.d_inner + d.nheads + 2 * d.ngroups * d.d_state) * act_bytes
    out = T * d.d_inner * act_bytes
    state = nseq * d.nheads * d.headdim * d.d_state * 4 * 2
    conv = nseq * d.conv_dim * 3 * act_bytes
    return inputs + out + state + conv


def prefill_flops(d: Dims) -> int:
    # per token: C.B^T once per group (2QN per group), then per head the masked
    # Q x Q times X (2QP), the chunk state B^T X (2NP) and C times the state (2NP)
    per_tok = 2 * d.chunk * d.d_state * d.ngroups + d.nheads * (2 * d.chunk * d.headdim + 4 * d.d_state * d.headdim)
    return d.batch * d.seqlen * per_tok


def backward_bytes(d: Dims, act_bytes: int) -> int:
    """Bytes the backward must move: the forward inputs and dy read (activation dtype), d_final read,
    the fp32 gradients of the activations and of the initial state written."""
    rows = d.batch * d.seqlen
    act_in = rows * (2 * d.d_inner + d.nheads + 2 * d.ngroups * d.d_state) * act_bytes
    dy = rows * d.d_inner * act_bytes
    grads = rows * (2 * d.d_inner + d.nheads + 2 * d.ngroups * d.d_state) * 4
    states = 2 * d.batch * d.nheads * d.headdim * d.d_state * 4
    return act_in + dy + grads + states


def backward_chunk_flops(d: Dims) -> int:
    """Algorithmic flops of the per-chunk backward (chunk_bwd_kernel) for Q = 64 chunks: per (chunk, head)
    the four Q x P x N contractions (Sp C, g Sp, Lm B, x Lm), the full Q x Q x P product g.x and the two
    causal-triangle Q x Q x P (y, dx) and Q x Q x N (dB, dC) sums; per (chunk, group) C.B."""
    Q, P, N = BWD_Q, d.headdim, d.d_state
    nc = -(-d.seqlen // Q)
    per_head = 8 * Q * P * N + 2 * Q * Q * P + 2 * Q * Q * P + 2 * Q * Q * N
    per_group = 2 * Q * Q * N
    return d.batch * nc * (d.nheads * per_head + d.ngroups * per_group)


def backward_chunk_bytes(d: Dims, act_bytes: int) -> int:
    """Algorithmic bytes of one launch of the tensor-core per-chunk backward (chunk_bwd_tc_kernel), Q = 64:
    reads the fp32 post-conv x, B, C, dt and in-chunk cumsum (workspace), dy and z and the raw dt (activation
    dtype), the entering states and leaving adjoints (the state pass's fp16 [nc][H][P][N] tiles, with an fp32
    scale per row p) and the per-chunk F partials; writes dz, the post-conv gradients of x (fp32), of B and C
    (fp32, one copy per half of each group's heads), ddt and the per-chunk partials.  Each byte counted once."""
    Q, P, N = BWD_Q, d.headdim, d.d_state
    rows, nc = d.batch * d.seqlen, d.batch * -(-d.seqlen // Q)
    HP, GN = d.nheads * P, d.ngroups * N
    halves = 2 if d.nheads // d.ngroups >= 2 else 1
    reads = rows * (HP + 2 * GN) * 4 + rows * 2 * d.nheads * 4 + rows * (2 * HP + d.nheads) * act_bytes + \
        2 * nc * d.nheads * P * (N * 2 + 4) + nc * d.nheads * 4 * 4
    writes = rows * 2 * HP * 4 + halves * rows * 2 * GN * 4 + rows * d.nheads * 4 + nc * d.nheads * 3 * 4
    return reads + writes


def bench_backward(ops, d: Dims, act, dev, flush, K: int, warmup: int, world: int, sampler, peaks):
    """Times ssd_prefill_backward on the prefill workload (bf16 activations and dy, d_final given)."""
    inp = make_prefill_inputs(d, dtype=act, seed=seed_of(BACKWARD_WORKLOAD) + 7)
    gr = make_backward_grads(d, dtype=act, seed=seed_of(BACKWARD_WORKLOAD) + 8)
    g = {k: (None if v is None else v.to(dev)) for k, v in inp.items()}
    dy, dfin = gr["dy"].to(dev), gr["d_final"].to(dev)
    dims = ops.make_dims(d.batch, d.seqlen, d.nheads, d.headdim, d.d_state, d.ngroups, d.chunk)
    ws = torch.empty(max(ops.prefill_backward_workspace_bytes(dims), 16), dtype=torch.uint8, device=dev)

    def once():
        return ops.prefill_backward(g["x"], g["dt"], g["B"], g["C"], g["z"], g["A"], g["D"], g["dt_bias"],
                                    g["conv_w"], g["conv_b"], dy, None, None, dfin, workspace=ws)
    for _ in range(warmup):
        flush.zero_()
        once()
    torch.cuda.synchronize(dev)
    KB = max(3, min(K, 10))
    st = [torch.cuda.Event(enable_timing=True) for _ in range(KB)]
    en = [torch.cuda.Event(enable_timing=True) for _ in range(KB)]
    ks = [torch.cuda.Event(enable_timing=True) for _ in range(KB)]
    ke = [torch.cuda.Event(enable_timing=True) for _ in range(KB)]
    barrier(world)
    sampler.load(True)
    for k in range(KB):
        flush.zero_()
        ops.set_timing_events(ks[k], ke[k])
        st[k].record()
        once()
        en[k].record()
    torch.cuda.synchronize(dev)
    ops.set_timing_events(None, None)
    sampler.load(False)
    barrier(world)
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(st, en)) / KB, world, dev)
    kms = sum(a.elapsed_time(b) for a, b in zip(ks, ke)) / KB
    tokens = d.batch * d.seqlen
    abytes = 2 if act == torch.bfloat16 else 4
    nbytes = backward_bytes(d, abytes)
    kbytes = backward_chunk_bytes(d, abytes)
    kgbs = kbytes / (kms * 1e-3) / 1e9
    return {"value": tokens * world / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "steps": KB,
            "workload": f"gradients of the {BACKWARD_WORKLOAD} layer prefill (bf16 inputs and dy, fp32 d_final; "
                        "every input, parameter and initial-state gradient, fp32)",
            "launch": "eager (7 kernels: post-conv, dt, chunk states (tcgen05), state scans, chunk backward "
                      "(tcgen05), conv backward, reductions; the tcgen05 kernels for bf16, d_state 64/128)",
            "algorithmic_bytes_per_step": nbytes, "achieved_gbs": nbytes / (ms * 1e-3) / 1e9,
            "dominant_kernel": {"kernel": "chunk_bwd_tc_kernel", "ms": kms, "share": kms / ms,
                                "algorithmic_flops_per_launch": backward_chunk_flops(d),
                                "roofline": {"bound": "hbm", "achieved": kgbs, "peak": peaks["hbm_gbs"],
                                             "unit": "GB/s", "frac": kgbs / peaks["hbm_gbs"],
                                             "traffic": kernel_traffic(f"chunk_bwd_tc_kernel@{BACKWARD_WORKLOAD}"),
                                             "algorithmic_bytes_per_launch": kbytes}},
            "l2": "flushed between timed steps (256 MB write outside the step events)"}


def decode_bytes(d: Dims, act_bytes: int) -> tuple[int, int]:
    """(bytes of the whole step, bytes of the state-stream kernel alone)."""
    B = d.batch
    state = 2 * B * d.nheads * d.headdim * d.d_state * 4
    conv = 2 * B * d.conv_dim * 3 * act_bytes
    inputs = B * (2 * d.d_inner + d.nheads + 2 * d.ngroups * d.d_state) * act_bytes
    y = B * d.d_inner * act_bytes
    roll = B * 2 * d.ngroups * d.d_state * (3 + 3) * act_bytes     # B/C conv window rewritten by the roll kernel
    total = state + conv + inputs + y
    return total, total - roll


def mimo_decode_bytes(d: Dims, rank: int, act_bytes: int) -> int:
    """Bytes of one MIMO decode step: the fp32 state read and written, x, z, B, C, dt read, y written."""
    B = d.batch
    state = 2 * B * d.nheads * d.headdim * d.d_state * 4
    xzy = 3 * B * d.nheads * rank * d.headdim * act_bytes
    bc = 2 * B * d.ngroups * rank * d.d_state * act_bytes
    return state + xzy + bc + B * d.nheads * act_bytes


def bench_mimo(ops, d: Dims, act, dev, world: int, sampler, peaks, nsteps: int):
    """Times ssd_mimo_decode_step (rank MIMO_RANK) on the decode workload's layer and batch."""
    data = make_mimo_decode_inputs(d, MIMO_RANK, MIMO_INPUTS, dtype=act, seed=seed_of(DECODE_WORKLOAD) + 5)
    p = {k: v.to(dev) for k, v in data["params"].items()}
    ssm = data["ssm_state"].to(dev)
    steps = [{k: v.to(dev) for k, v in s.items()} for s in data["steps"]]
    ys = [torch.empty_like(s["x"]) for s in steps]
    del data

    def mstep(i):
        s = steps[i % len(steps)]
        ops.mimo_decode_step(s["x"], s["dt"], s["B"], s["C"], s["z"], p["A"], p["D"], p["dt_bias"], ssm,
                             y=ys[i % len(steps)])
    for i in range(3):
        mstep(i)
    torch.cuda.synchronize(dev)
    # the steps back to back between one pair of events, as a decode loop runs them
    ms_, me = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    sampler.load(True)
    ms_.record()
    for k in range(nsteps):
        mstep(k)
    me.record()
    torch.cuda.synchronize(dev)
    sampler.load(False)
    barrier(world)
    ms = max_over_ranks(ms_.elapsed_time(me) / nsteps, world, dev)
    nbytes = mimo_decode_bytes(d, MIMO_RANK, 2 if act == torch.bfloat16 else 4)
    gbs = nbytes / (ms * 1e-3) / 1e9
    flops = 4 * MIMO_RANK * d.batch * d.nheads * d.headdim * d.d_state
    return {"value": gbs * world, "unit": "GB/s", "ms_per_step": ms, "steps": nsteps, "rank": MIMO_RANK,
            "workload": f"MIMO decode step, rank {MIMO_RANK}, on the {DECODE_WORKLOAD} layer and batch "
                        f"({d.batch} sequences, H{d.nheads} P{d.headdim} N{d.d_state} G{d.ngroups}), bf16 "
                        "activations, fp32 state, no conv",
            "algorithmic_bytes_per_step": nbytes, "algorithmic_flops_per_step": flops,
            "roofline": {"bound": "hbm", "kernel": "mimo_decode_kernel", "achieved": gbs, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "traffic": kernel_traffic("mimo_decode_kernel")},
            "l2": "state (1.07 GB) larger than L2; no flush"}


# ---------------------------------------------------------------------------------------------------------

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None if
    the summary is missing or the kernel's source changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        t = json.load(f).get(kernel)
    if not t:
        return None
    src = os.path.join(ROOT, t["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != t["source_sha256_16"]:
        return None
    return t["dram_bytes_per_launch"]


class ClockSampler:
    """Samples SM clock and clock-event (throttle) reasons through NVML while running."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting", 0x10: "sync_boost"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples = []
        self.period = period_s
        self.ok = False
        self._stop = threading.Event()
        self._load = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
            self.ok = True
        except Exception as e:  # no NVML: report that, never guess
            self.err = str(e)

    def _run(self):
        while not self._stop.is_set():
            if self._load.is_set():
                try:
                    mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                    rs = self._reasons(self.h)
                    self.samples.append((mhz, rs))
                except Exception:
                    pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def load(self, on: bool):
        (self._load.set if on else self._load.clear)()

    def stop(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "error": self.err}
        self._stop.set()
        self.t.join()
        mhz = [m for m, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= r
        reasons = sorted(name for b, name in self.REASONS.items() if bits & b)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(mhz), "source": "NVML, sampled every 5 ms during the timed regions"}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def weak_scaling_value(tokens_per_rank: int, ms_per_rank: float, world: int, device) -> tuple[float, float]:
    """Whole-job tokens/s for independent per-rank work: all ranks' tokens over the
    slowest rank's step time.  Returns (tokens/s, max ms)."""
    ms = max_over_ranks(ms_per_rank, world, device)
    return tokens_per_rank * world / (ms * 1e-3), ms


def max_over_ranks(value: float, world: int, device) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------------------------------------
# CPU oracle baseline

def oracle_inputs_f64(inp):
    return {k: (None if v is None else np.ascontiguousarray(v.double().numpy())) for k, v in inp.items()}


def oracle_sample(inp64, d: Dims, first_unit: int, n_units: int, threads: int):
    """Run the oracle on n_units (b, h) pairs starting at first_unit; returns seconds."""
    import oracle
    mask = np.zeros(d.batch * d.nheads, dtype=bool)
    idx = [(first_unit + i) % (d.batch * d.nheads) for i in range(n_units)]
    mask[idx] = True
    t0 = time.perf_counter()
    oracle.prefill(inp64, unit_mask=mask.reshape(d.batch, d.nheads), nthreads=threads)
    return time.perf_counter() - t0


def cpu_baseline(inp, d: Dims, budget_s: float, workload: str):
    """The fp64 oracle on this host's cores, on (sequence, head) pairs of ``workload`` until about
    ``budget_s`` seconds have passed (at least one round of ``threads`` pairs)."""
    import oracle
    threads = oracle.default_threads()
    inp64 = oracle_inputs_f64(inp)
    done, elapsed, u = 0, 0.0, 0
    while (elapsed < budget_s or done == 0) and done < d.batch * d.nheads:
        n = min(threads, d.batch * d.nheads - done)
        elapsed += oracle_sample(inp64, d, u, n, threads)
        done += n
        u += n
    tokens_equiv = done * d.seqlen / d.nheads      # each (b, h) pair is one head's share of L tokens
    return {"value": tokens_equiv / elapsed, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{done} of the {d.batch * d.nheads} (sequence, head) pairs of the {workload} "
                      f"workload ({d.seqlen} tokens each), fp64 token-by-token recurrence, {elapsed:.1f} s; "
                      f"tokens/s = pairs x L / H / seconds"}


def cpu_decode_baseline(sample: dict, d: Dims, steps: int, act_bytes: int):
    """The oracle's decode step timed on the first few sequences of the decode workload for ``steps``
    consecutive steps; GB/s of the algorithmic bytes those sequences' steps move."""
    import oracle
    nseq = sample["ssm_state"].shape[0]
    conv = sample["conv_state"].double().numpy().copy()
    ssm = sample["ssm_state"].double().numpy().copy()
    t0 = time.perf_counter()
    for s in sample["steps"][:steps]:
        oracle.decode_step(s, sample["params"], conv, ssm)
    el = time.perf_counter() - t0
    sub = Dims(nseq, 1, d.nheads, d.headdim, d.d_state, d.ngroups, d.chunk)
    nbytes = decode_bytes(sub, act_bytes)[0] * steps
    return {"value": nbytes / el / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{nseq} of the {d.batch} sequences, {steps} consecutive steps, fp64, {el:.2f} s; "
                      f"GB/s = those sequences' algorithmic bytes per step x steps / seconds"}


def cpu_backward_baseline(d: Dims, act):
    """The oracle's backward timed on one group of the prefill workload's layer (H/G heads, all L tokens,
    the same per-head shapes), reported as tokens/s of the whole layer: one group is 1/G of the work."""
    import oracle
    sub = Dims(d.batch, d.seqlen, d.nheads // d.ngroups, d.headdim, d.d_state, 1, d.chunk)
    inp = make_prefill_inputs(sub, dtype=act, seed=seed_of(BACKWARD_WORKLOAD) + 7)
    gr = make_backward_grads(sub, dtype=act, seed=seed_of(BACKWARD_WORKLOAD) + 8)
    t0 = time.perf_counter()
    oracle.prefill_backward(inp, gr["dy"], gr["d_final"])
    el = time.perf_counter() - t0
    tokens = d.batch * d.seqlen / d.ngroups
    return {"value": tokens / el, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"one group ({sub.nheads} of {d.nheads} heads, {d.seqlen} tokens) of the {BACKWARD_WORKLOAD} "
                      f"layer, fp64 adjoint of the token recurrence, {el:.1f} s; tokens/s = L / G / seconds"}


def cpu_mimo_baseline(d: Dims, act, nseq: int = 16):
    """The oracle's MIMO step timed on ``nseq`` of the decode workload's sequences, as GB/s of the
    step's algorithmic bytes for those sequences."""
    import oracle
    sub = Dims(nseq, 1, d.nheads, d.headdim, d.d_state, d.ngroups, d.chunk)
    data = make_mimo_decode_inputs(sub, MIMO_RANK, 1, dtype=act, seed=seed_of(DECODE_WORKLOAD) + 5)
    state = data["ssm_state"].double().numpy().copy()
    t0 = time.perf_counter()
    oracle.mimo_decode_step(data["steps"][0], data["params"], state)
    el = time.perf_counter() - t0
    nbytes = mimo_decode_bytes(sub, MIMO_RANK, 2 if act == torch.bfloat16 else 4)
    return {"value": nbytes / el / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{nseq} of the {d.batch} sequences of one step, rank {MIMO_RANK}, fp64, {el:.2f} s"}


# ---------------------------------------------------------------------------------------------------------

def run_reference(args):
    """The reference arm: the fp64 CPU oracle as it stands, on the host cores, on the headline workload."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    w = WORKLOADS[HEADLINE_WORKLOAD]
    d = w["dims"]
    inp = make_prefill_inputs(d, dtype=w["dtype"], seed=seed_of(HEADLINE_WORKLOAD), init_state=w["init_state"])
    inp64 = oracle_inputs_f64(inp)
    threads = oracle.default_threads()
    n = threads
    for i in range(args.warmup):
        oracle_sample(inp64, d, i * n, n, threads)
    times = [oracle_sample(inp64, d, (args.warmup + k) * n, n, threads) for k in range(args.steps)]
    sec = sum(times) / len(times)
    value = n * d.seqlen / d.nheads / sec
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w["desc"], "sample_per_step": f"{n} (sequence, head) pairs of {d.seqlen} tokens"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": f"{n} (sequence, head) pairs per step, {args.steps} steps"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


class PrefillRun:
    """One prefill workload resident on the device, with its outputs and workspace."""

    def __init__(self, ops, name: str, dev, rank: int):
        w = WORKLOADS[name]
        self.name, self.w, self.d, self.act = name, w, w["dims"], w["dtype"]
        d = self.d
        self.inp = make_prefill_inputs(d, dtype=self.act, seed=seed_of(name) + 1000 * rank,
                                       init_state=w["init_state"])
        self.g = {k: (None if v is None else v.to(dev)) for k, v in self.inp.items()}
        self.dims = ops.make_dims(d.batch, d.seqlen, d.nheads, d.headdim, d.d_state, d.ngroups, d.chunk)
        self.path = ops.prefill_path(self.dims, self.act)
        self.ws = torch.empty(max(ops.prefill_workspace_bytes(self.dims, self.act), 16), dtype=torch.uint8,
                              device=dev)
        self.y = torch.empty_like(self.g["x"])
        self.fs = torch.empty((d.batch, d.nheads, d.headdim, d.d_state), dtype=torch.float32, device=dev)
        self.cs = torch.empty((d.batch, d.conv_dim, 3), dtype=self.act, device=dev)
        self.ops = ops

    def once(self):
        g = self.g
        self.ops.prefill(g["x"], g["dt"], g["B"], g["C"], g["z"], g["A"], g["D"], g["dt_bias"], g["conv_w"],
                         g["conv_b"], g["init_state"], None, chunk=self.d.chunk, workspace=self.ws, y=self.y,
                         final_state=self.fs, conv_state=self.cs)

    def free_device(self):
        self.g = self.ws = self.y = self.fs = self.cs = None


def bench_prefill(run: PrefillRun, dev, flush, K: int, warmup: int, world: int, sampler, peaks, peak_src,
                  use_graph: bool):
    """Times one prefill step (B/C prologue + chunk scan) of ``run``: ``K`` steps bracketed by CUDA events,
    L2 flushed between them outside the events, then the dominant kernel alone through the library's timing
    hook.  Returns the result dict (tokens/s, roofline of the dominant kernel, tensor-core fraction)."""
    ops, d, act = run.ops, run.d, run.act
    for _ in range(warmup):
        flush.zero_()
        run.once()
    torch.cuda.synchronize(dev)
    # the step captured once into a CUDA graph and replayed, so that the timed region holds the device
    # work and not the host-side argument marshalling between launches
    step, launch = run.once, "eager"
    graph = None
    if use_graph:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                run.once()
            graph.replay()
            torch.cuda.synchronize(dev)
            step, launch = graph.replay, "CUDA graph replay of the two-kernel step"
        except RuntimeError as exc:  # capture refused: time the eager launches instead
            print(f"bench: CUDA graph capture failed ({exc}); timing eager launches", file=sys.stderr)
            torch.cuda.synchronize(dev)
            graph = None
    for _ in range(warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    st = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    en = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize(dev)
    sampler.load(True)
    for k in range(K):
        flush.zero_()                      # L2 flush, outside the step's events
        st[k].record()
        step()
        en[k].record()
    torch.cuda.synchronize(dev)
    sampler.load(False)
    barrier(world)
    step_ms = sum(s.elapsed_time(e) for s, e in zip(st, en)) / K
    # the dominant kernel alone, in a second pass: events recorded between the two launches of a
    # step would also serialise them, so they are kept out of the pass that gives `value`
    ks = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ke = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    for k in range(K):
        flush.zero_()
        ops.set_timing_events(ks[k], ke[k])
        run.once()
    torch.cuda.synchronize(dev)
    ops.set_timing_events(None, None)
    ops.device_status(dev)   # raises if a bounded device-side wait gave up
    kern_ms = sum(s.elapsed_time(e) for s, e in zip(ks, ke)) / K
    tokens_per_rank = d.batch * d.seqlen
    value, step_ms_max = weak_scaling_value(tokens_per_rank, step_ms, world, dev)
    act_bytes = 2 if act == torch.bfloat16 else 4
    pbytes = prefill_bytes(d, act_bytes, run.w["init_state"])
    pflops = prefill_flops(d)
    kernel_name = "ssd_chunk_scan_tc" if run.path == 1 else "prefill_simt_kernel"
    achieved_gbs = pbytes / (kern_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "kernel": kernel_name, "achieved": achieved_gbs, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": achieved_gbs / peaks["hbm_gbs"],
                "traffic": kernel_traffic(f"{kernel_name}@{run.name}"),
                "algorithmic_bytes_per_launch": pbytes, "kernel_ms": kern_ms,
                "peak_source": f"{peak_src} (copy bandwidth)"}
    tflops = pflops / (step_ms * 1e-3) / 1e12
    tc = {"algorithmic_tflops": tflops, "frac_bf16_peak": tflops / peaks["bf16_tflops"],
          "frac_bf16_sustained": tflops / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]),
          "algorithmic_flops_per_step": pflops, "peak_source": peak_src}
    step_gbs = pbytes / (step_ms_max * 1e-3) / 1e9
    del graph
    return {"value": value, "unit": "tokens/s", "ms_per_step": step_ms_max, "steps": K,
            "workload": run.w["desc"], "dtype": "bf16" if act == torch.bfloat16 else "f32",
            "kernel_path": "tcgen05 tensor-core" if run.path == 1 else "CUDA-core", "launch": launch,
            "ctas": d.batch * d.nheads if run.path == 1 else None,
            "step_frac_hbm": step_gbs / peaks["hbm_gbs"], "tensor": tc, "roofline": roofline,
            "gpu_launches_per_step": 2 if run.path == 1 else 1,
            "l2": "flushed between timed steps (256 MB write outside the step events)"}


def link_bandwidth(dev, nbytes: int = 256 << 20):
    """Pinned host -> device and device -> host copies of ``nbytes``, timed with CUDA events: each direction
    alone, then both at once on two streams (the PCIe link is full duplex, but each direction slows while
    the other runs)."""
    h = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    h2 = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    dbuf = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    dbuf2 = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    out = {}
    for name, fn in (("h2d_gbs", lambda: dbuf.copy_(h, non_blocking=True)),
                     ("d2h_gbs", lambda: h.copy_(dbuf, non_blocking=True))):
        fn()
        torch.cuda.synchronize(dev)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(3):
            fn()
        e.record()
        torch.cuda.synchronize(dev)
        out[name] = 3 * nbytes / (s.elapsed_time(e) * 1e-3) / 1e9
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    cur = torch.cuda.current_stream(dev)
    s = torch.cuda.Event(enable_timing=True)
    e_in, e_out = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    s_in.wait_stream(cur)
    s_out.wait_stream(cur)
    with torch.cuda.stream(s_in):
        dbuf.copy_(h, non_blocking=True)
        e_in.record()
    with torch.cuda.stream(s_out):
        h2.copy_(dbuf2, non_blocking=True)
        e_out.record()
    torch.cuda.synchronize(dev)
    # both streams run the whole time only until the first of them finishes: rate = bytes / own time
    out["h2d_both_gbs"] = nbytes / (s.elapsed_time(e_in) * 1e-3) / 1e9
    out["d2h_both_gbs"] = nbytes / (s.elapsed_time(e_out) * 1e-3) / 1e9
    return out


def link_floor_bidir_ms(h2d: int, d2h: int, link: dict) -> float:
    """The shortest time to move h2d bytes in and d2h bytes out over the link: both directions at once for as
    long as both have bytes left, then the remainder alone (each direction's rates from link_bandwidth)."""
    t_both = min(h2d / (link["h2d_both_gbs"] * 1e9), d2h / (link["d2h_both_gbs"] * 1e9))
    rest_in = h2d - link["h2d_both_gbs"] * 1e9 * t_both
    rest_out = d2h - link["d2h_both_gbs"] * 1e9 * t_both
    return (t_both + rest_in / (link["h2d_gbs"] * 1e9) + rest_out / (link["d2h_gbs"] * 1e9)) * 1e3


def bench_e2e(ops, run: PrefillRun, dev, K: int, world: int, sampler):
    """The prefill of ``run`` through the public API from pinned host tensors, copies inside the events."""
    d = run.d
    host = {k: (None if v is None else v.pin_memory()) for k, v in run.inp.items()}
    # the outputs' pinned host buffers are allocated once and reused, as a serving loop would
    outs = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (run.y, run.fs, run.cs)]
    segments = None   # the API's default: about 8 pieces overlapped on three streams
    try:
        for _ in range(3):
            ops.prefill_host(host, chunk=d.chunk, device=dev, segments=segments, out=outs)
        torch.cuda.synchronize(dev)
    except RuntimeError as exc:   # keep an end-to-end number: one piece on one stream
        print(f"bench: segmented host prefill failed ({exc}); timing the one-piece call", file=sys.stderr)
        torch.cuda.synchronize(dev)
        segments = 1
    KE = max(3, min(K, 10))
    es = [torch.cuda.Event(enable_timing=True) for _ in range(KE)]
    ee = [torch.cuda.Event(enable_timing=True) for _ in range(KE)]
    barrier(world)
    sampler.load(True)
    h2d = d2h = 0
    for k in range(KE):
        es[k].record()
        _, h2d, d2h = ops.prefill_host(host, chunk=d.chunk, device=dev, segments=segments, out=outs)
        ee[k].record()
    torch.cuda.synchronize(dev)
    sampler.load(False)
    barrier(world)
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(es, ee)) / KE, world, dev)
    link = link_bandwidth(dev)
    del host
    return {"value": d.batch * d.seqlen * world / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": KE, "workload": run.w["desc"],
            "link": link,
            "link_floor_ms": max(h2d / link["h2d_gbs"], d2h / link["d2h_gbs"]) / 1e6,
            "link_floor_bidir_ms": link_floor_bidir_ms(h2d, d2h, link),
            "how": "ops.prefill_host: pinned host inputs -> device, ssd_prefill, outputs -> pinned host buffers "
                   "reused across steps; "
                   + ("one piece on one stream" if segments == 1 else
                      "about 8 pieces of one sequence and a chunk-aligned token range (one contiguous copy per "
                      "tensor), copies in, scans and copies out overlapped on three streams, states chained "
                      "along each sequence")
                   + "; CUDA events on the calling stream around the whole call"}


def bench_norm(ops, run: PrefillRun, dev, flush, K: int, warmup: int, peaks, use_graph: bool):
    """Gated RMSNorm (ngroups groups) of ``run``'s prefill output, HBM-bound."""
    d = run.d
    wn = torch.rand(d.d_inner, generator=torch.Generator().manual_seed(11)).add_(0.5).to(dev)
    yn = torch.empty_like(run.y)

    def norm_once():
        ops.gated_rmsnorm(run.y, wn, d.ngroups, out=yn)
    for _ in range(warmup):
        norm_once()
    torch.cuda.synchronize(dev)
    nstep = norm_once
    if use_graph:
        ngraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(ngraph):
            norm_once()
        nstep = ngraph.replay
    ns = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ne = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    for k in range(K):
        flush.zero_()
        ns[k].record()
        nstep()
        ne[k].record()
    torch.cuda.synchronize(dev)
    nms = sum(a.elapsed_time(b) for a, b in zip(ns, ne)) / K
    nbytes = 2 * run.y.numel() * run.y.element_size() + d.d_inner * 4
    ngbs = nbytes / (nms * 1e-3) / 1e9
    return {"kernel": "group_rmsnorm_kernel", "us_per_call": nms * 1e3, "groups": d.ngroups,
            "workload": f"output of the {run.name} prefill, {d.ngroups} groups of {d.d_inner // d.ngroups} channels",
            "algorithmic_bytes": nbytes,
            "roofline": {"bound": "hbm", "achieved": ngbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": ngbs / peaks["hbm_gbs"],
                         "traffic": kernel_traffic(f"group_rmsnorm_kernel@{run.name}")}}


def bench_decode(ops, dev, world: int, sampler, peaks, nsteps: int):
    """``nsteps`` consecutive decode steps of the decode workload.  Returns (result, CPU sample of the first
    sequences for the oracle baseline)."""
    wd = WORKLOADS[DECODE_WORKLOAD]
    dd = wd["dims"]
    data = make_decode_inputs(dd, steps=nsteps, dtype=wd["dtype"], seed=seed_of(DECODE_WORKLOAD))
    ns = DECODE_ORACLE_SEQS
    sample = {"params": data["params"], "ssm_state": data["ssm_state"][:ns].clone(),
              "conv_state": data["conv_state"][:ns].clone(),
              "steps": [{k: v[:ns].clone() for k, v in s.items()} for s in data["steps"][:DECODE_ORACLE_STEPS]]}
    p = {k: v.to(dev) for k, v in data["params"].items()}
    conv = data["conv_state"].to(dev)
    ssm = data["ssm_state"].to(dev)
    steps = [{k: v.to(dev) for k, v in s.items()} for s in data["steps"]]
    del data

    def dstep(s):
        ops.decode_step(s["x"], s["dt"], s["B"], s["C"], s["z"], p["A"], p["D"], p["dt_bias"], p["conv_w"],
                        p["conv_b"], conv, ssm)
    for i in range(3):
        dstep(steps[i % len(steps)])
    torch.cuda.synchronize(dev)
    KD = len(steps)
    # the steps back to back between one pair of events (an event between two steps would keep the next
    # step's state kernel from starting under the previous step's roll, as it does in a decode loop)
    ds, de = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    sampler.load(True)
    ds.record()
    for k in range(KD):
        dstep(steps[k])
    de.record()
    torch.cuda.synchronize(dev)
    sampler.load(False)
    barrier(world)
    dms = max_over_ranks(ds.elapsed_time(de) / KD, world, dev)
    # the state kernel alone: a second pass with events around each of its launches
    dks = [torch.cuda.Event(enable_timing=True) for _ in range(KD)]
    dke = [torch.cuda.Event(enable_timing=True) for _ in range(KD)]
    for k in range(KD):
        ops.set_timing_events(dks[k], dke[k])
        dstep(steps[k])
    torch.cuda.synchronize(dev)
    ops.set_timing_events(None, None)
    dkms = sum(a.elapsed_time(b) for a, b in zip(dks, dke)) / KD
    tot_b, kern_b = decode_bytes(dd, 2 if wd["dtype"] == torch.bfloat16 else 4)
    gbs = tot_b * world / (dms * 1e-3) / 1e9
    kgbs = kern_b / (dkms * 1e-3) / 1e9
    res = {"value": gbs, "unit": "GB/s", "ms_per_step": dms, "steps": KD, "workload": wd["desc"],
           "frac_hbm_peak": gbs / world / peaks["hbm_gbs"], "frac_8tbs_spec": gbs / world / 8000.0,
           "algorithmic_bytes_per_step": tot_b,
           "roofline": {"bound": "hbm", "kernel": "decode_state_kernel", "achieved": kgbs,
                        "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": kgbs / peaks["hbm_gbs"],
                        "traffic": kernel_traffic("decode_state_kernel"),
                        "algorithmic_bytes_per_launch": kern_b, "kernel_ms": dkms},
           "l2": "state (1.07 GB) larger than L2; no flush"}
    return res, sample


def bench_varlen(ops, dev, flush, K: int, warmup: int, world: int, sampler, peaks, use_graph: bool):
    """Packed variable-length prefill: a continuous-batching mix of lengths on the Nemotron-H 8B layer."""
    wv = WORKLOADS[VARLEN_WORKLOAD]
    dv = wv["dims"]
    lengths = varlen_lengths(VARLEN_NSEQ, VARLEN_MIN, VARLEN_MAX, seed=seed_of(VARLEN_WORKLOAD) + 100)
    vin, cu = make_varlen_inputs(dv, lengths, dtype=wv["dtype"], seed=seed_of(VARLEN_WORKLOAD) + 101,
                                 init_state=True, init_conv_state=True)
    gv = {k: (None if t is None else t.to(dev)) for k, t in vin.items()}
    cu_dev = torch.tensor(cu, dtype=torch.int64, device=dev)
    T = cu[-1]
    vdims = ops.make_dims(len(lengths), T, dv.nheads, dv.headdim, dv.d_state, dv.ngroups, dv.chunk)
    vws = torch.empty(max(ops.prefill_varlen_workspace_bytes(vdims, wv["dtype"]), 16), dtype=torch.uint8,
                      device=dev)
    vy = torch.empty_like(gv["x"])
    vfs = torch.empty((len(lengths), dv.nheads, dv.headdim, dv.d_state), dtype=torch.float32, device=dev)
    vcs = torch.empty((len(lengths), dv.conv_dim, 3), dtype=wv["dtype"], device=dev)

    def vstep_eager():
        ops.prefill_varlen(gv["x"], gv["dt"], gv["B"], gv["C"], gv["z"], gv["A"], gv["D"], gv["dt_bias"],
                           gv["conv_w"], gv["conv_b"], cu_dev, gv["init_state"], gv["init_conv_state"],
                           chunk=dv.chunk, workspace=vws, y=vy, final_state=vfs, conv_state=vcs)
    for _ in range(warmup):
        flush.zero_()
        vstep_eager()
    torch.cuda.synchronize(dev)
    vstep, launch = vstep_eager, "eager"
    if use_graph:
        vgraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(vgraph):
            vstep_eager()
        vstep, launch = vgraph.replay, "CUDA graph replay of the two-kernel step"
    KV = max(3, min(K, 20))
    vs = [torch.cuda.Event(enable_timing=True) for _ in range(KV)]
    ve = [torch.cuda.Event(enable_timing=True) for _ in range(KV)]
    barrier(world)
    sampler.load(True)
    for k in range(KV):
        flush.zero_()
        vs[k].record()
        vstep()
        ve[k].record()
    torch.cuda.synchronize(dev)
    sampler.load(False)
    barrier(world)
    ops.device_status(dev)
    vms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(vs, ve)) / KV, world, dev)
    vbytes = varlen_bytes(dv, T, len(lengths), 2 if wv["dtype"] == torch.bfloat16 else 4)
    vgbs = vbytes / (vms * 1e-3) / 1e9
    return {"value": T * world / (vms * 1e-3), "unit": "tokens/s", "ms_per_step": vms, "steps": KV,
            "workload": f"{len(lengths)} packed sequences of the {VARLEN_WORKLOAD} layer, lengths "
                        f"log-uniform in [{VARLEN_MIN}, {VARLEN_MAX}] ({T} tokens; min {min(lengths)}, "
                        f"max {max(lengths)}), per-sequence initial states",
            "algorithmic_bytes_per_step": vbytes, "achieved_gbs": vgbs,
            "frac_hbm_peak": vgbs / peaks["hbm_gbs"], "launch": launch,
            "l2": "flushed between timed steps (256 MB write outside the step events)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--decode-steps", type=int, default=64)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--configs", default=",".join(OTHER_PREFILL_WORKLOADS),
                    help="comma-separated prefill workloads timed beside the headline ('' for none)")
    ap.add_argument("--only", choices=["prefill", "decode", "varlen", "backward", "mimo"],
                    help="run one leg alone, without the CPU baselines (for profiling); 'prefill' times the "
                         "headline and the --configs workloads without e2e or the norm")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time eager launches instead of a CUDA graph replay")
    ap.add_argument("--no-varlen", action="store_true", help="skip the packed variable-length prefill line")
    ap.add_argument("--no-norm", action="store_true", help="skip the gated RMSNorm line")
    ap.add_argument("--no-backward", action="store_true", help="skip the training-backward line")
    ap.add_argument("--no-mimo", action="store_true", help="skip the MIMO decode line")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.only:
        args.no_cpu = args.no_e2e = args.no_norm = True
        args.no_decode, args.no_varlen = args.only != "decode", args.only != "varlen"
        args.no_backward, args.no_mimo = args.only != "backward", args.only != "mimo"
    run_prefill = args.only in (None, "prefill")
    others = [c for c in args.configs.split(",") if c] if run_prefill else []
    for c in others:
        if c not in WORKLOADS or c == HEADLINE_WORKLOAD or c == DECODE_WORKLOAD:
            ap.error(f"--configs: unknown or repeated prefill workload {c!r}")

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from selective_state_space_43_b200 import ops
    ops.lib()   # fail loudly here if the CUDA library is missing

    peaks, peak_src = load_peaks()
    use_graph = not args.no_graph
    K = args.steps
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    sampler = ClockSampler(local)
    sampler.start()

    # ---- headline: prefill of the largest single-GPU layer workload, device-resident inputs ---------------
    head = headline = e2e = None
    if run_prefill:
        head = PrefillRun(ops, HEADLINE_WORKLOAD, dev, rank)
        headline = bench_prefill(head, dev, flush, K, args.warmup, world, sampler, peaks, peak_src, use_graph)
        if not args.no_e2e:
            e2e = bench_e2e(ops, head, dev, K, world, sampler)
        head.free_device()

    # ---- the other prefill workloads (the pages' other layer shapes and the tiny fp32 case) ---------------
    per_config = {}
    runs = {}
    norm = None
    for name in others:
        run = PrefillRun(ops, name, dev, rank)
        per_config[name] = bench_prefill(run, dev, flush, max(3, min(K, 20)), args.warmup, world, sampler, peaks,
                                         peak_src, use_graph)
        if name == NORM_WORKLOAD and not args.no_norm and run.path == 1:
            norm = bench_norm(ops, run, dev, flush, K, args.warmup, peaks, use_graph)
        run.free_device()
        runs[name] = run
    torch.cuda.empty_cache()

    # ---- decode -------------------------------------------------------------------------------------------
    decode = decode_sample = None
    if not args.no_decode:
        decode, decode_sample = bench_decode(ops, dev, world, sampler, peaks, args.decode_steps)
        torch.cuda.empty_cache()

    # ---- packed variable-length prefill (a continuous-batching mix of lengths) -----------------------
    varlen = None
    if not args.no_varlen:
        varlen = bench_varlen(ops, dev, flush, K, args.warmup, world, sampler, peaks, use_graph)
        torch.cuda.empty_cache()

    # ---- training backward of the Nemotron-H 8B layer -------------------------------------------------------
    backward = None
    if not args.no_backward:
        try:
            wb = WORKLOADS[BACKWARD_WORKLOAD]
            backward = bench_backward(ops, wb["dims"], wb["dtype"], dev, flush, K, args.warmup, world, sampler, peaks)
        except (RuntimeError, ValueError) as exc:  # report it and keep the forward numbers
            backward = {"error": f"{type(exc).__name__}: {exc}"[:300]}
        torch.cuda.empty_cache()

    # ---- MIMO decode step on the decode workload ------------------------------------------------------------
    mimo = None
    if not args.no_mimo:
        try:
            wd = WORKLOADS[DECODE_WORKLOAD]
            mimo = bench_mimo(ops, wd["dims"], wd["dtype"], dev, world, sampler, peaks, max(3, min(K, 16)))
        except (RuntimeError, ValueError) as exc:  # report it and keep the other numbers
            mimo = {"error": f"{type(exc).__name__}: {exc}"[:300]}

    clocks = sampler.stop()

    # ---- CPU oracle baselines (rank 0, N = 1 only) --------------------------------------------------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(head.inp, head.d, args.cpu_seconds, HEADLINE_WORKLOAD)
        for name, run in runs.items():
            per_config[name]["cpu_baseline"] = cpu_baseline(run.inp, run.d, args.cpu_seconds / 4, name)
        if decode is not None:
            wd = WORKLOADS[DECODE_WORKLOAD]
            decode["cpu_baseline"] = cpu_decode_baseline(decode_sample, wd["dims"], DECODE_ORACLE_STEPS,
                                                         2 if wd["dtype"] == torch.bfloat16 else 4)
        if backward is not None and "error" not in backward:
            wb = WORKLOADS[BACKWARD_WORKLOAD]
            backward["cpu_baseline"] = cpu_backward_baseline(wb["dims"], wb["dtype"])
        if mimo is not None and "error" not in mimo:
            wd = WORKLOADS[DECODE_WORKLOAD]
            mimo["cpu_baseline"] = cpu_mimo_baseline(wd["dims"], wd["dtype"])

    if rank == 0 and headline is None:   # one leg alone (--only): its own result, not a bench line
        print(json.dumps({"only": args.only, "decode": decode, "varlen": varlen, "backward": backward,
                          "mimo_decode": mimo, "clocks": clocks}), flush=True)
    elif rank == 0:
        d = head.d
        line = {
            "metric": METRIC, "value": headline["value"], "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": headline["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": headline["dtype"],
            "data": "synthetic (seeded recipe: x,z,dt~N(0,1), B,C~N(0,1)/sqrt(N), A=-exp(U[0,ln16]), "
                    "init state~N(0,0.1^2))",
            "config": {"workload": head.w["desc"], "batch_per_gpu": d.batch, "seqlen": d.seqlen,
                       "nheads": d.nheads, "headdim": d.headdim, "d_state": d.d_state, "ngroups": d.ngroups,
                       "chunk": d.chunk, "init_state": head.w["init_state"],
                       "parallelism": f"dp{world} (independent sequences per GPU, no collective)",
                       "l2": headline["l2"], "kernel_path": headline["kernel_path"], "launch": headline["launch"]},
            "tensor": headline["tensor"], "roofline": headline["roofline"],
            "step_frac_hbm": headline["step_frac_hbm"], "cpu_baseline": cpu, "e2e": e2e,
            "configs": per_config, "decode": decode, "varlen": varlen, "gated_rmsnorm": norm,
            "backward": backward, "mimo_decode": mimo,
            "gpu_launches": K * headline["gpu_launches_per_step"], "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
