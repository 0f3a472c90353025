"""GPU parity of ssd_prefill against the fp64 oracle (needs a B200)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_bf16_is_rounded, assert_close, dev_inputs, gpu_prefill, np64
from selective_state_space_43_b200 import ops
from selective_state_space_43_b200.synth import Dims, make_prefill_inputs, workload

pytestmark = pytest.mark.gpu


def run_both(dev, chunk):
    """(y32, y_native, final_state, conv_state): the fp32-y run, and the run in
    the activation dtype, which must agree bit for bit once y32 is rounded."""
    y, fs, cs = gpu_prefill(dev, chunk)
    if y.dtype == torch.float32:
        return y, y, fs, cs
    y32, fs32, cs32 = gpu_prefill(dev, chunk, y_dtype=torch.float32)
    assert_bf16_is_rounded(y, y32, "prefill y")
    assert torch.equal(fs, fs32) and torch.equal(cs, cs32)
    return y32, y, fs, cs


def _check_full(inp, chunk, tag):
    dev = dev_inputs(inp)
    y32, _, fs, cs = run_both(dev, chunk)
    ops.device_status()
    yo, fo, co = oracle.prefill(inp)
    r1 = assert_close(np64(y32), yo, f"{tag} y")
    r2 = assert_close(np64(fs), fo, f"{tag} final_state")
    assert np.array_equal(np64(cs), co), f"{tag} conv_state"
    return r1, r2


# Layer shapes of the pages at sizes the oracle finishes in seconds; several
# chunks plus a ragged tail, heads-per-group as in each model.
SMALL = {
    "nemotron_h_8b_shape": (Dims(1, 553, 32, 64, 128, 2, 128), torch.bfloat16, False),
    "nemotron3_nano_shape_init": (Dims(2, 300, 16, 64, 128, 8, 128), torch.bfloat16, True),
    "hybrid_3b_shape": (Dims(3, 257, 40, 64, 128, 8, 128), torch.bfloat16, False),
    "tiny_fp32_full": (Dims(1, 256, 4, 64, 32, 1, 64), torch.float32, False),
    "q64_ragged": (Dims(2, 300, 8, 64, 64, 2, 64), torch.bfloat16, True),
    "n16_per_head_groups": (Dims(1, 200, 4, 64, 16, 4, 128), torch.bfloat16, False),
    "n32_fp32_q128": (Dims(2, 140, 6, 64, 32, 3, 128), torch.float32, True),
    "n64_bf16": (Dims(1, 390, 8, 64, 64, 1, 128), torch.bfloat16, False),
    "n32_bf16_cuda_core": (Dims(1, 200, 8, 64, 32, 2, 128), torch.bfloat16, True),
}


@pytest.mark.parametrize("name", sorted(SMALL))
def test_prefill_small_matches_oracle(name):
    d, dt, init = SMALL[name]
    inp = make_prefill_inputs(d, dtype=dt, seed=101, init_state=init, init_conv_state=init, random_D=True)
    _check_full(inp, d.chunk, name)


@pytest.mark.parametrize("L", [0, 1, 2, 3, 5, 127, 128, 129])
@pytest.mark.parametrize("init", [False, True])
def test_prefill_edge_lengths(L, init):
    d = Dims(2, L, 16, 64, 128, 4, 128)
    inp = make_prefill_inputs(d, dtype=torch.bfloat16, seed=7 + L, init_state=init, init_conv_state=init)
    if L == 0:
        dev = dev_inputs(inp)
        y, fs, cs = gpu_prefill(dev, 128)
        _, fo, co = oracle.prefill(inp)
        want_fs = np64(inp["init_state"]) if init else np.zeros_like(fo)
        assert np.array_equal(np64(fs), want_fs)
        assert np.array_equal(np64(cs), co)
        return
    _check_full(inp, 128, f"L={L}")


def test_prefill_is_deterministic():
    d = Dims(1, 600, 16, 64, 128, 2, 128)
    inp = dev_inputs(make_prefill_inputs(d, dtype=torch.bfloat16, seed=5, init_state=True))
    a = [t.clone() for t in gpu_prefill(inp, 128)]
    b = gpu_prefill(inp, 128)
    for u, v in zip(a, b):
        assert torch.equal(u, v)


def test_final_state_may_overwrite_init_state():
    d = Dims(1, 300, 16, 64, 128, 2, 128)
    inp = make_prefill_inputs(d, dtype=torch.bfloat16, seed=12, init_state=True)
    dev = dev_inputs(inp)
    _, fs_ref, _ = gpu_prefill(dev, 128)
    st = dev["init_state"].clone()
    ops.prefill(dev["x"], dev["dt"], dev["B"], dev["C"], dev["z"], dev["A"], dev["D"], dev["dt_bias"],
                dev["conv_w"], dev["conv_b"], st, None, chunk=128, final_state=st)
    assert torch.equal(st, fs_ref)


def test_prefill_chunk_size_independence():
    # Q is a tiling parameter of the method: Q = 64 and Q = 128 agree within rounding.  The tensor-core
    # path works in 128-token chunks whatever Q is asked for (so its Q = 64 call is bit-equal to its
    # Q = 128 call); the CUDA-core path, fed the same values in fp32, scans in 64-token chunks.
    d = Dims(1, 700, 8, 64, 128, 2, 128)
    inp = dev_inputs(make_prefill_inputs(d, dtype=torch.bfloat16, seed=6, init_state=True))
    y1, f1, _ = gpu_prefill(inp, 128, y_dtype=torch.float32)
    y2, f2, _ = gpu_prefill(inp, 64, y_dtype=torch.float32)
    assert torch.equal(y1, y2) and torch.equal(f1, f2)
    inp32 = {k: (v.float() if v is not None and v.dtype == torch.bfloat16 else v) for k, v in inp.items()}
    y3, f3, _ = gpu_prefill(inp32, 64)
    assert_close(np64(y3), np64(y1), "y Q64 (CUDA cores) vs Q128 (tensor cores)", rel_tol=5e-3, abs_tol=2e-2)
    assert_close(np64(f3), np64(f1), "final_state Q64 vs Q128", rel_tol=5e-3, abs_tol=2e-2)


def test_prefill_split_sequence_continuation():
    d = Dims(2, 520, 16, 64, 128, 4, 128)
    inp = make_prefill_inputs(d, dtype=torch.bfloat16, seed=8, init_state=True, init_conv_state=True)
    dev = dev_inputs(inp)
    L1 = 259
    first = {k: (v[:, :L1].contiguous() if k in ("x", "z", "dt", "B", "C") else v) for k, v in dev.items()}
    second = {k: (v[:, L1:].contiguous() if k in ("x", "z", "dt", "B", "C") else v) for k, v in dev.items()}
    y1, f1, c1 = gpu_prefill(first, 128, y_dtype=torch.float32)
    second["init_state"], second["init_conv_state"] = f1, c1
    y2, f2, c2 = gpu_prefill(second, 128, y_dtype=torch.float32)
    yo, fo, co = oracle.prefill(inp)
    assert_close(np64(torch.cat([y1, y2], dim=1)), yo, "split y")
    assert_close(np64(f2), fo, "split final_state")
    assert np.array_equal(np64(c2), co)


def test_prefill_reports_small_workspace():
    import ctypes
    d = Dims(1, 256, 16, 64, 128, 2, 128)
    dims = ops.make_dims(d.batch, d.seqlen, d.nheads, d.headdim, d.d_state, d.ngroups, d.chunk)
    need = ops.prefill_workspace_bytes(dims, torch.bfloat16)
    if need == 0:
        pytest.skip("this shape takes a path without workspace")
    inp = dev_inputs(make_prefill_inputs(d, dtype=torch.bfloat16, seed=9))
    small = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    params = ops._params(inp["A"], inp["D"], inp["dt_bias"], inp["conv_w"], inp["conv_b"], d.nheads, d.conv_dim,
                         inp["x"].device)
    y = torch.empty_like(inp["x"])
    fs = torch.empty((d.batch, d.nheads, d.headdim, d.d_state), device="cuda")
    cs = torch.empty((d.batch, d.conv_dim, 3), device="cuda", dtype=torch.bfloat16)
    code = ops.lib().ssd_prefill(ctypes.byref(dims), ops.SSD_BF16, ctypes.byref(params),
                                 *[ops._ptr(inp[k]) for k in ("x", "dt", "B", "C", "z")], None, None,
                                 ops._ptr(y), ops._ptr(fs), ops._ptr(cs), ops._ptr(small), need - 16,
                                 ops._stream_ptr(inp["x"].device))
    assert code == 7


# Full-size workloads: every output of the GPU run is checked for finiteness;
# a sample of (sequence, head) pairs is recomputed by the oracle one by one.
FULL = ["tiny_fp32", "nemotron_h_8b", "nemotron3_nano", "hybrid_3b"]


@pytest.mark.parametrize("name", FULL)
def test_prefill_full_size_sampled(name):
    d, dt, inp = workload(name)
    dev = dev_inputs(inp)
    y, _, fs, cs = run_both(dev, d.chunk)
    ops.device_status()
    assert torch.isfinite(y).all() and torch.isfinite(fs).all()
    mask = np.zeros((d.batch, d.nheads), dtype=bool)
    hpg = d.nheads // d.ngroups
    picks = {(0, 0), (0, hpg - 1), (d.batch // 2, d.nheads // 2), (d.batch - 1, d.nheads - 1)}
    for b, h in picks:
        mask[b, h] = True
    yo, fo, co = oracle.prefill(inp, unit_mask=mask)
    P = d.headdim
    yg, fg = np64(y), np64(fs)
    for b, h in sorted(picks):
        assert_close(yg[b, :, h * P:(h + 1) * P], yo[b, :, h * P:(h + 1) * P], f"{name} y (b={b}, h={h})")
        assert_close(fg[b, h], fo[b, h], f"{name} final_state (b={b}, h={h})")
    assert np.array_equal(np64(cs), co)


def test_tensor_core_path_covers_d_state_64_and_chunk_64():
    # the 64-state and 64-token-chunk layers run on the tensor cores (chunks of 128 internally, the upper
    # 64 state channels zero for d_state 64); results agree with the oracle as for the other shapes
    for N, Q in ((64, 128), (64, 64), (128, 64)):
        assert ops.prefill_path(ops.make_dims(2, 300, 16, 64, N, 2, Q), torch.bfloat16) == 1, (N, Q)
    d = Dims(2, 300, 16, 64, 128, 2, 64)
    inp = make_prefill_inputs(d, dtype=torch.bfloat16, seed=103, init_state=True, init_conv_state=True)
    _check_full(inp, d.chunk, "n128_q64")


def test_layer_shapes_take_the_tensor_core_path():
    from selective_state_space_43_b200.synth import WORKLOADS
    for name in ("nemotron_h_8b", "nemotron3_nano", "hybrid_3b"):
        d = WORKLOADS[name]["dims"]
        dims = ops.make_dims(d.batch, d.seqlen, d.nheads, d.headdim, d.d_state, d.ngroups, d.chunk)
        assert ops.prefill_path(dims, torch.bfloat16) == 1, name


@pytest.mark.parametrize("d,dt", [(Dims(2, 300, 16, 64, 128, 2, 128), torch.bfloat16),
                                  (Dims(2, 140, 4, 64, 32, 1, 64), torch.float32)])
def test_prefill_reads_views_of_the_in_proj_output(d, dt):
    # x, z, dt, B, C as slices of one [Bt, L, z | x | B | C | dt] array (a Mamba-2 block's in_proj
    # output): the strided call must give exactly the contiguous call's results
    inp = make_prefill_inputs(d, dtype=dt, seed=111, init_state=True, init_conv_state=True)
    dev = dev_inputs(inp)
    HP, GN, H = d.nheads * d.headdim, d.ngroups * d.d_state, d.nheads
    zxbcdt = torch.empty((d.batch, d.seqlen, 2 * HP + 2 * GN + H), dtype=dt, device="cuda")
    views = {"z": zxbcdt[..., :HP], "x": zxbcdt[..., HP:2 * HP],
             "B": zxbcdt[..., 2 * HP:2 * HP + GN].unflatten(-1, (d.ngroups, d.d_state)),
             "C": zxbcdt[..., 2 * HP + GN:2 * HP + 2 * GN].unflatten(-1, (d.ngroups, d.d_state)),
             "dt": zxbcdt[..., 2 * HP + 2 * GN:]}
    for k, v in views.items():
        v.copy_(dev[k])
        assert not v.is_contiguous()
    ys, fss, css = gpu_prefill({**dev, **views}, d.chunk)
    yc, fsc, csc = gpu_prefill(dev, d.chunk)
    ops.device_status()
    assert torch.equal(ys, yc) and torch.equal(fss, fsc) and torch.equal(css, csc)


@pytest.mark.parametrize("norm_groups", [2, 1])
def test_gated_rmsnorm_after_prefill_matches_oracle(norm_groups):
    d = Dims(2, 300, 16, 64, 128, 2, 128)
    host = make_prefill_inputs(d, dtype=torch.bfloat16, seed=121, init_state=True)
    dev = dev_inputs(host)
    y32, y, _, _ = run_both(dev, d.chunk)
    w = torch.rand(d.nheads * d.headdim, generator=torch.Generator().manual_seed(7)) + 0.5
    wd = w.cuda()
    n32 = ops.gated_rmsnorm(y32, wd, norm_groups)
    ops.device_status()
    yo, _, _ = oracle.prefill(host)
    assert_close(np64(n32), oracle.gated_rmsnorm(yo, w.numpy(), norm_groups), "gated rmsnorm")
    # bf16 in and out: the same fp32 arithmetic on the bf16 values, rounded once at the end
    n16 = ops.gated_rmsnorm(y, wd, norm_groups)
    assert_bf16_is_rounded(n16, ops.gated_rmsnorm(y.float(), wd, norm_groups), "gated rmsnorm bf16")
    # in place
    y_copy = y.clone()
    ops.gated_rmsnorm(y_copy, wd, norm_groups, out=y_copy)
    assert torch.equal(y_copy, n16)


@pytest.mark.parametrize("groups", [1, 2, 4, 8])
def test_gated_rmsnorm_group_sizes(groups):
    # 4096 channels: groups of 4096 and 2048 take the two-read path, 1024 and 512 the register-held one
    g = torch.Generator().manual_seed(groups)
    y = torch.randn((37, 4096), generator=g) * 2.0
    w = torch.rand(4096, generator=g) + 0.5
    out = ops.gated_rmsnorm(y.cuda(), w.cuda(), groups)
    ops.device_status()
    assert_close(np64(out), oracle.gated_rmsnorm(y.double().numpy(), w.double().numpy(), groups),
                 f"rmsnorm, {groups} groups", rel_tol=1e-5, abs_tol=1e-4)
