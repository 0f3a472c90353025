"""Seeded synthetic inputs for the Mamba-2 SSD layer core.

This module only draws random numbers; it holds none of the layer's
arithmetic.  The same draws feed both the CUDA library and the fp64 oracle, so
both see bit-identical (already rounded) values.

Shapes follow the Mamba-2 layer tables on the pages: headdim 64, d_state 128,
n_groups 8, conv kernel 4, chunk 128 ("Nemotron-H 스타일 Hybrid
Mamba-Transformer 3B 모델 구현 타당성 분석", tables 1.4 and 1.5, §2.6).

Recipe (fixed draw order, one ``torch.Generator`` on the CPU):
  x, z ~ N(0, 1); dt_raw ~ N(0, 1); B, C ~ N(0, 1) / sqrt(N)       (activations)
  dt_bias[h] = softplus^-1(dt0[h]),  dt0[h] = exp(U[ln 1e-3, ln 0.1])
  A[h] = -exp(U[ln 1, ln 16]); D = 1 (or U(0.5, 1.5) when ``random_D``)
  conv_w, conv_b ~ U(-0.5, 0.5)
  init_state ~ N(0, 0.1^2) fp32 when requested; init_conv_state ~ N(0, 1)
Activations are rounded to the activation dtype (bf16 round-to-nearest-even)
before anything else sees them; parameters and states stay fp32.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, asdict

import torch


@dataclass(frozen=True)
class Dims:
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    d_state: int
    ngroups: int
    chunk: int = 128
    d_conv: int = 4

    @property
    def d_inner(self) -> int:
        return self.nheads * self.headdim

    @property
    def conv_dim(self) -> int:
        return self.nheads * self.headdim + 2 * self.ngroups * self.d_state

    def as_dict(self) -> dict:
        return asdict(self)


# The five layer workloads: a tiny fp32 correctness case, three prefill
# shapes and one decode shape.
WORKLOADS = {
    "tiny_fp32": dict(dims=Dims(1, 256, 4, 64, 32, 1, 64), dtype=torch.float32, init_state=False,
                      desc="tiny fp32 prefill: B1 L256 H4 P64 N32 G1 Q64"),
    "nemotron_h_8b": dict(dims=Dims(1, 4096, 128, 64, 128, 8, 128), dtype=torch.bfloat16, init_state=False,
                          desc="Nemotron-H 8B Mamba-2 layer prefill: B1 L4096 H128 P64 N128 G8 Q128, bf16"),
    "nemotron3_nano": dict(dims=Dims(4, 8192, 64, 64, 128, 8, 128), dtype=torch.bfloat16, init_state=True,
                           desc="Nemotron 3 Nano Mamba-2 layer prefill: B4 L8192 H64 P64 N128 G8 Q128, bf16, "
                                "initial state ~ N(0, 0.1^2)"),
    "hybrid_3b": dict(dims=Dims(8, 4096, 40, 64, 128, 8, 128), dtype=torch.bfloat16, init_state=False,
                      desc="proposed 3B hybrid Mamba-2 layer prefill: B8 L4096 H40 P64 N128 G8 Q128, bf16"),
    "decode_nemotron_h_8b": dict(dims=Dims(256, 1, 128, 64, 128, 8, 128), dtype=torch.bfloat16, init_state=True,
                                 desc="decode step, 256 sequences, H128 P64 N128 G8, bf16 activations, "
                                      "fp32 state ~ N(0, 0.1^2), 64 consecutive steps"),
}
# seed = 43 + the workload's position in this list
WORKLOAD_ORDER = ["tiny_fp32", "nemotron_h_8b", "nemotron3_nano", "hybrid_3b", "decode_nemotron_h_8b"]


def seed_of(name: str) -> int:
    return 43 + WORKLOAD_ORDER.index(name)


def _uniform(g, shape, lo, hi):
    return torch.rand(shape, generator=g, dtype=torch.float32) * (hi - lo) + lo


def make_params(dims: Dims, g: torch.Generator, random_D: bool = False) -> dict:
    """Per-layer parameters (fp32), drawn after the activations."""
    H = dims.nheads
    dt0 = torch.exp(_uniform(g, (H,), math.log(1e-3), math.log(0.1)))
    # inverse of softplus at dt0: log(exp(dt0) - 1)
    dt_bias = torch.log(torch.expm1(dt0.double())).float()
    A = -torch.exp(_uniform(g, (H,), 0.0, math.log(16.0)))
    if random_D:
        D = _uniform(g, (H,), 0.5, 1.5)
    else:
        D = torch.ones(H, dtype=torch.float32)
    conv_w = _uniform(g, (dims.conv_dim, dims.d_conv), -0.5, 0.5)
    conv_b = _uniform(g, (dims.conv_dim,), -0.5, 0.5)
    return dict(A=A, D=D, dt_bias=dt_bias, conv_w=conv_w, conv_b=conv_b)


def make_prefill_inputs(dims: Dims, dtype=torch.bfloat16, seed: int = 43, init_state: bool = False,
                        init_conv_state: bool = False, random_D: bool = False) -> dict:
    """All inputs of one prefill call, on the CPU, already rounded to ``dtype``."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    Bt, L, H, P, N, G = dims.batch, dims.seqlen, dims.nheads, dims.headdim, dims.d_state, dims.ngroups
    x = torch.randn((Bt, L, H * P), generator=g)
    z = torch.randn((Bt, L, H * P), generator=g)
    dt = torch.randn((Bt, L, H), generator=g)
    Bm = torch.randn((Bt, L, G, N), generator=g) / math.sqrt(N)
    Cm = torch.randn((Bt, L, G, N), generator=g) / math.sqrt(N)
    out = dict(x=x.to(dtype), z=z.to(dtype), dt=dt.to(dtype), B=Bm.to(dtype), C=Cm.to(dtype))
    out.update(make_params(dims, g, random_D=random_D))
    out["init_state"] = (torch.randn((Bt, H, P, N), generator=g) * 0.1) if init_state else None
    out["init_conv_state"] = (torch.randn((Bt, dims.conv_dim, 3), generator=g).to(dtype)
                              if init_conv_state else None)
    return out


def make_backward_grads(dims: Dims, dtype=torch.bfloat16, seed: int = 53, d_final: bool = True) -> dict:
    """Incoming gradients of one prefill backward call, on the CPU: dy [B, L, H*P] ~ N(0, 1) rounded to
    ``dtype`` (the gradient of a loss with respect to y) and d_final [B, H, P, N] ~ N(0, 0.1^2) fp32 (the
    gradient with respect to final_state, present when the next segment's loss depends on it)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    Bt, L, H, P, N = dims.batch, dims.seqlen, dims.nheads, dims.headdim, dims.d_state
    dy = torch.randn((Bt, L, H * P), generator=g).to(dtype)
    df = torch.randn((Bt, H, P, N), generator=g) * 0.1
    return dict(dy=dy, d_final=df if d_final else None)


def varlen_lengths(nseq: int, lo: int, hi: int, seed: int) -> list:
    """``nseq`` sequence lengths drawn log-uniformly from [lo, hi] (a continuous-batching mix)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    u = torch.rand(nseq, generator=g, dtype=torch.float64)
    return [int(round(math.exp(math.log(lo) + float(v) * (math.log(hi) - math.log(lo))))) for v in u]


def make_varlen_inputs(dims: Dims, lengths, dtype=torch.bfloat16, seed: int = 43, init_state: bool = False,
                       init_conv_state: bool = False) -> tuple:
    """Inputs of one packed variable-length prefill: the sequences of ``lengths`` back to back
    (x/z [T, H*P], dt [T, H], B/C [T, G, N]; per-sequence initial states [nseq, ...]), drawn by
    the same recipe as ``make_prefill_inputs``; ``dims.batch`` / ``dims.seqlen`` are ignored.
    Returns (inputs, cu_seqlens as a list of nseq+1 offsets)."""
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    T, nseq = cu[-1], len(lengths)
    packed = make_prefill_inputs(Dims(1, T, dims.nheads, dims.headdim, dims.d_state, dims.ngroups, dims.chunk),
                                 dtype=dtype, seed=seed)
    out = {k: (v[0] if k in ("x", "z", "dt", "B", "C") else v) for k, v in packed.items()}
    g = torch.Generator(device="cpu").manual_seed(seed + 1000)
    out["init_state"] = (torch.randn((nseq, dims.nheads, dims.headdim, dims.d_state), generator=g) * 0.1
                         if init_state else None)
    out["init_conv_state"] = (torch.randn((nseq, dims.conv_dim, 3), generator=g).to(dtype)
                              if init_conv_state else None)
    return out, cu


def make_decode_inputs(dims: Dims, steps: int, dtype=torch.bfloat16, seed: int = 47,
                       random_D: bool = False) -> dict:
    """Initial states and ``steps`` rounds of fresh one-token inputs for decode."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    Bt, H, P, N, G = dims.batch, dims.nheads, dims.headdim, dims.d_state, dims.ngroups
    params = make_params(dims, g, random_D=random_D)
    ssm_state = torch.randn((Bt, H, P, N), generator=g) * 0.1
    conv_state = torch.randn((Bt, dims.conv_dim, 3), generator=g).to(dtype)
    per_step = []
    for _ in range(steps):
        x = torch.randn((Bt, H * P), generator=g)
        z = torch.randn((Bt, H * P), generator=g)
        dt = torch.randn((Bt, H), generator=g)
        Bm = torch.randn((Bt, G, N), generator=g) / math.sqrt(N)
        Cm = torch.randn((Bt, G, N), generator=g) / math.sqrt(N)
        per_step.append(dict(x=x.to(dtype), z=z.to(dtype), dt=dt.to(dtype), B=Bm.to(dtype), C=Cm.to(dtype)))
    return dict(params=params, ssm_state=ssm_state, conv_state=conv_state, steps=per_step)


def make_mimo_decode_inputs(dims: Dims, rank: int, steps: int, dtype=torch.bfloat16, seed: int = 59,
                            random_D: bool = False) -> dict:
    """Initial state and ``steps`` rounds of one-token inputs for the rank-``rank`` MIMO decode: x, z
    [B, H, R, P] ~ N(0, 1), dt [B, H] ~ N(0, 1), B, C [B, G, R, N] ~ N(0, 1)/sqrt(N), rounded to ``dtype``;
    fp32 state ~ N(0, 0.1^2); A, D, dt_bias as for the other workloads (the conv parameters are drawn too,
    so the draw order matches, but the MIMO step has no conv)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    Bt, H, P, N, G = dims.batch, dims.nheads, dims.headdim, dims.d_state, dims.ngroups
    params = make_params(dims, g, random_D=random_D)
    ssm_state = torch.randn((Bt, H, P, N), generator=g) * 0.1
    per_step = []
    for _ in range(steps):
        x = torch.randn((Bt, H, rank, P), generator=g)
        z = torch.randn((Bt, H, rank, P), generator=g)
        dt = torch.randn((Bt, H), generator=g)
        Bm = torch.randn((Bt, G, rank, N), generator=g) / math.sqrt(N)
        Cm = torch.randn((Bt, G, rank, N), generator=g) / math.sqrt(N)
        per_step.append(dict(x=x.to(dtype), z=z.to(dtype), dt=dt.to(dtype), B=Bm.to(dtype), C=Cm.to(dtype)))
    return dict(params=params, ssm_state=ssm_state, steps=per_step)


def workload(name: str, **overrides):
    """(dims, dtype, inputs) for one of the named workloads."""
    w = WORKLOADS[name]
    dims = w["dims"]
    if overrides:
        dims = Dims(**{**dims.as_dict(), **overrides})
    inp = make_prefill_inputs(dims, dtype=w["dtype"], seed=seed_of(name), init_state=w["init_state"])
    return dims, w["dtype"], inp
