"""Pins of the fp64 oracle against mathematics it does not share (CPU only).

Each test reaches a value the layer must produce by a route other than the
oracle's token loop: the SSD quadratic form, a closed form, a textbook or
library routine, or an invariant of the recurrence.
"""
import math

import numpy as np
import pytest
import torch
from scipy.signal import lfilter

import oracle
from pins import f64, fir_conv_silu, quadratic_form, rel_err, silu_lib, softplus_lib
from selective_state_space_43_b200.synth import Dims, WORKLOADS, make_decode_inputs, make_prefill_inputs


def tiny(seed=1, L=24, H=4, P=3, N=5, G=2, Bt=2, init_state=True, init_conv=True, dtype=torch.float32):
    d = Dims(Bt, L, H, P, N, G, 8)
    return d, make_prefill_inputs(d, dtype=dtype, seed=seed, init_state=init_state, init_conv_state=init_conv,
                                  random_D=True)


# --- conv + SiLU against numpy's correlate ------------------------------------------------------

@pytest.mark.parametrize("with_hist", [False, True])
def test_conv_silu_matches_library_fir(with_hist):
    rng = np.random.default_rng(3)
    seq = rng.standard_normal(50)
    hist = rng.standard_normal(3) if with_hist else None
    w = rng.uniform(-0.5, 0.5, 4)
    b = 0.3
    got = oracle.conv_silu(seq, hist, w, b)
    want = fir_conv_silu(seq, hist, w, b)
    assert np.max(np.abs(got - want)) < 1e-13


def test_conv_unit_impulse_picks_taps():
    # an impulse at t0 gives silu(b + w[k]) at t0 + 3 - k and silu(b) elsewhere
    w = np.array([0.1, -0.2, 0.3, 0.4])
    seq = np.zeros(10)
    seq[4] = 1.0
    got = oracle.conv_silu(seq, None, w, 0.05)
    for t in range(10):
        k = 4 + 3 - t
        pre = 0.05 + (w[k] if 0 <= k < 4 else 0.0)
        assert abs(got[t] - pre / (1 + math.exp(-pre))) < 1e-15


# --- the SSD quadratic form (brute force) ---------------------------------------------------------

@pytest.mark.parametrize("seed,init", [(1, True), (2, False)])
def test_prefill_matches_quadratic_form(seed, init):
    _, inp = tiny(seed=seed, init_state=init, init_conv=init)
    y, fs, _ = oracle.prefill(inp)
    yq, fq = quadratic_form(inp)
    assert rel_err(y, yq) < 1e-12
    assert rel_err(fs, fq) < 1e-12


def test_prefill_quadratic_form_bf16_inputs_groups_of_three():
    # bf16-rounded inputs, H/G = 3 heads per group, a different head->group map than H/G = 2
    _, inp = tiny(seed=5, L=17, H=6, P=2, N=3, G=2, Bt=1, dtype=torch.bfloat16)
    y, fs, _ = oracle.prefill(inp)
    yq, fq = quadratic_form(inp)
    assert rel_err(y, yq) < 1e-12
    assert rel_err(fs, fq) < 1e-12


# --- closed form for constant inputs ------------------------------------------------------------

def _const_inputs(L, P, N, dt_raw, A, xv, bv, cv, zv, D=1.0):
    inp = dict(
        x=np.full((1, L, P), xv), z=np.full((1, L, P), zv), dt=np.full((1, L, 1), dt_raw),
        B=np.full((1, L, 1, N), bv), C=np.full((1, L, 1, N), cv),
        A=np.array([A]), D=np.array([D]), dt_bias=np.array([0.0]),
        conv_w=np.tile(np.array([0.0, 0.0, 0.0, 1.0]), (P + 2 * N, 1)), conv_b=np.zeros(P + 2 * N),
        init_state=None, init_conv_state=None)
    return inp


@pytest.mark.parametrize("dt_raw,A", [(-1.2, -2.5), (0.8, -0.6), (35.0, -0.01)])
def test_closed_form_constant_inputs(dt_raw, A):
    L, P, N = 40, 3, 4
    xv, bv, cv, zv = 0.7, -0.4, 0.9, 0.3
    y, fs, _ = oracle.prefill(_const_inputs(L, P, N, dt_raw, A, xv, bv, cv, zv, D=0.5))
    dt = math.log1p(math.exp(dt_raw))
    a = math.exp(dt * A)
    ux, ub, uc = (v / (1 + math.exp(-v)) for v in (xv, bv, cv))
    gate = zv / (1 + math.exp(-zv))
    for t in range(L):
        geo = (1 - a ** (t + 1)) / (1 - a)
        want = (N * uc * ub * dt * ux * geo + 0.5 * ux) * gate
        assert abs(y[0, t, 0] - want) < 1e-13 * max(1.0, abs(want))
    want_state = dt * ux * ub * (1 - a ** L) / (1 - a)
    assert np.max(np.abs(fs - want_state)) < 1e-13


# --- special cases that reduce to textbook routines ---------------------------------------------

def test_A_zero_is_prefix_sum():
    _, inp = tiny(seed=7, init_state=False, init_conv=False)
    inp["A"] = torch.zeros_like(inp["A"])
    y, fs, _ = oracle.prefill(inp)
    Bt, L, HP = inp["x"].shape
    H = inp["A"].shape[0]
    P = HP // H
    G, N = inp["B"].shape[2:]
    from pins import post_conv
    for b in range(Bt):
        ux, uB, uC = post_conv(inp, b)
        dt = softplus_lib(f64(inp["dt"])[b] + f64(inp["dt_bias"])[None, :])
        for h in range(H):
            g = h // (H // G)
            xs = ux[:, h * P:(h + 1) * P]
            incr = (dt[:, h, None, None] * xs[:, :, None]) * uB[:, g, None, :]   # [L, P, N]
            S = np.cumsum(incr, axis=0)                                             # textbook prefix sum
            assert np.max(np.abs(fs[b, h] - S[-1])) < 1e-12
            yv = np.einsum("tpn,tn->tp", S, uC[:, g, :]) + f64(inp["D"])[h] * xs
            want = yv * silu_lib(f64(inp["z"])[b, :, h * P:(h + 1) * P])
            assert np.max(np.abs(y[b, :, h * P:(h + 1) * P] - want)) < 1e-12


def test_dt_to_zero_keeps_state_and_passes_skip():
    _, inp = tiny(seed=8)
    inp["dt"] = torch.full_like(inp["dt"], -1000.0)       # softplus -> exactly 0 in double
    y, fs, _ = oracle.prefill(inp)
    assert np.array_equal(fs, f64(inp["init_state"]))
    Bt, L, HP = inp["x"].shape
    H = inp["A"].shape[0]
    P = HP // H
    G = inp["B"].shape[2]
    from pins import post_conv
    for b in range(Bt):
        ux, _, uC = post_conv(inp, b)
        for h in range(H):
            g = h // (H // G)
            xs = ux[:, h * P:(h + 1) * P]
            yv = uC[:, g, :] @ f64(inp["init_state"])[b, h].T + f64(inp["D"])[h] * xs
            want = yv * silu_lib(f64(inp["z"])[b, :, h * P:(h + 1) * P])
            assert np.max(np.abs(y[b, :, h * P:(h + 1) * P] - want)) < 1e-13


def test_scalar_case_is_first_order_iir():
    # N = P = H = 1, constant dt, B, C; conv reduced to the identity tap, so u = silu(raw).
    rng = np.random.default_rng(11)
    L = 200
    xs = rng.standard_normal(L)
    inp = _const_inputs(L, 1, 1, -0.3, -1.7, 0.0, 0.8, -1.1, 2.0, D=0.25)
    inp["x"] = xs.reshape(1, L, 1)
    inp["z"] = np.full((1, L, 1), 40.0)                     # silu(40) = 40 - 1.7e-16
    y, _, _ = oracle.prefill(inp)
    dt = math.log1p(math.exp(-0.3))
    a = math.exp(dt * -1.7)
    ub, uc = silu_lib(0.8), silu_lib(-1.1)
    ux = silu_lib(xs)
    want = (lfilter([dt * ub * uc], [1.0, -a], ux) + 0.25 * ux) * silu_lib(40.0)
    assert np.max(np.abs(y[0, :, 0] - want)) < 1e-12


# --- invariants -----------------------------------------------------------------------------------

@pytest.mark.parametrize("init", [False, True])
def test_decode_steps_reproduce_prefill(init):
    d, inp = tiny(seed=21, L=19, init_state=init, init_conv=init)
    y, fs, cs = oracle.prefill(inp)
    Bt, L, HP = inp["x"].shape
    conv_state = (f64(inp["init_conv_state"]).copy() if init else np.zeros((Bt, d.conv_dim, 3)))
    ssm = (f64(inp["init_state"]).copy() if init else np.zeros((Bt, d.nheads, d.headdim, d.d_state)))
    params = {k: inp[k] for k in ("A", "D", "dt_bias", "conv_w", "conv_b")}
    for t in range(L):
        step = {k: f64(inp[k])[:, t] for k in ("x", "z", "dt", "B", "C")}
        yt = oracle.decode_step(step, params, conv_state, ssm)
        assert np.max(np.abs(yt - y[:, t])) < 1e-12
    assert np.max(np.abs(ssm - fs)) < 1e-12
    assert np.array_equal(conv_state, cs)


def test_split_sequence_equals_whole():
    d, inp = tiny(seed=22, L=30)
    y, fs, cs = oracle.prefill(inp)
    L1 = 11
    first = {k: (v[:, :L1] if k in ("x", "z", "dt", "B", "C") else v) for k, v in inp.items()}
    y1, fs1, cs1 = oracle.prefill(first)
    second = {k: (v[:, L1:] if k in ("x", "z", "dt", "B", "C") else v) for k, v in inp.items()}
    second["init_state"] = fs1
    second["init_conv_state"] = cs1
    y2, fs2, cs2 = oracle.prefill(second)
    assert np.max(np.abs(np.concatenate([y1, y2], axis=1) - y)) < 1e-12
    assert np.max(np.abs(fs2 - fs)) < 1e-12
    assert np.array_equal(cs2, cs)


@pytest.mark.parametrize("L", [1, 2, 3, 5])
@pytest.mark.parametrize("init", [False, True])
def test_conv_state_tail_short_sequences(L, init):
    d, inp = tiny(seed=23, L=L, init_state=False, init_conv=init)
    _, _, cs = oracle.prefill(inp)
    raw = np.concatenate([f64(inp["x"]), f64(inp["B"]).reshape(d.batch, L, -1),
                          f64(inp["C"]).reshape(d.batch, L, -1)], axis=2)        # [Bt, L, conv_dim]
    hist = f64(inp["init_conv_state"]) if init else np.zeros((d.batch, d.conv_dim, 3))
    full = np.concatenate([hist.transpose(0, 2, 1), raw], axis=1)              # tokens -3 .. L-1
    assert np.array_equal(cs, full[:, -3:, :].transpose(0, 2, 1))


def test_unit_mask_selects_pairs():
    _, inp = tiny(seed=24)
    y, fs, _ = oracle.prefill(inp)
    mask = np.zeros((2, 4), dtype=bool)
    mask[0, 1] = mask[1, 3] = True
    ym, fm, _ = oracle.prefill(inp, unit_mask=mask, nthreads=3)
    P = 3
    for b, h in [(0, 1), (1, 3)]:
        assert np.array_equal(ym[b, :, h * P:(h + 1) * P], y[b, :, h * P:(h + 1) * P])
        assert np.array_equal(fm[b, h], fs[b, h])
    assert np.isnan(ym[0, :, 0]).all()


def test_thread_count_does_not_change_results():
    _, inp = tiny(seed=25)
    a = oracle.prefill(inp, nthreads=1)
    b = oracle.prefill(inp, nthreads=5)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


# --- the input recipe -----------------------------------------------------------------------------

def test_synthetic_recipe_ranges():
    for name, w in WORKLOADS.items():
        d = w["dims"]
        small = Dims(1, 8, d.nheads, d.headdim, d.d_state, d.ngroups, d.chunk)
        inp = make_prefill_inputs(small, dtype=w["dtype"], seed=43)
        dt0 = softplus_lib(f64(inp["dt_bias"]))
        assert dt0.min() >= 1e-3 * (1 - 1e-6) and dt0.max() <= 0.1 * (1 + 1e-6), name
        A = f64(inp["A"])
        assert (A <= -1 + 1e-6).all() and (A >= -16 - 1e-5).all()
        assert inp["x"].dtype == w["dtype"]


def test_decode_inputs_deterministic():
    d = Dims(2, 1, 4, 64, 16, 2, 128)
    a = make_decode_inputs(d, steps=2, seed=9)
    b = make_decode_inputs(d, steps=2, seed=9)
    assert torch.equal(a["ssm_state"], b["ssm_state"])
    assert torch.equal(a["steps"][1]["x"], b["steps"][1]["x"])


# --- gated RMSNorm: closed forms and invariants -------------------------------------------------

def test_rmsnorm_hand_example():
    # one group [3, 4]: mean square 12.5, so out = [3, 4] / sqrt(12.5 + eps) * w
    y = np.array([[3.0, 4.0]])
    w = np.array([2.0, 0.5])
    out = oracle.gated_rmsnorm(y, w, 1, eps=0.5)
    np.testing.assert_allclose(out, [[3.0 * 2.0 / math.sqrt(13.0), 4.0 * 0.5 / math.sqrt(13.0)]], rtol=1e-15)


def test_rmsnorm_constant_group_and_group_independence():
    rng = np.random.default_rng(5)
    y = rng.standard_normal((3, 7, 64))
    y[:, :, 16:32] = -2.5                          # group 1 of 4 is constant: out = -2.5/sqrt(6.25 + eps) * w
    w = rng.uniform(0.5, 1.5, 64)
    out = oracle.gated_rmsnorm(y, w, 4, eps=1e-5)
    want = np.broadcast_to(-2.5 / math.sqrt(6.25 + 1e-5) * w[16:32], out[:, :, 16:32].shape)
    np.testing.assert_allclose(out[:, :, 16:32], want, rtol=1e-13)
    y2 = y.copy()
    y2[:, :, 48:] *= 10.0                          # another group changes: group 0 does not
    np.testing.assert_array_equal(oracle.gated_rmsnorm(y2, w, 4)[:, :, :16], out[:, :, :16])


def test_rmsnorm_output_has_unit_rms_and_is_scale_free():
    rng = np.random.default_rng(6)
    y = rng.standard_normal((5, 256)) * 3.0
    w = np.ones(256)
    out = oracle.gated_rmsnorm(y, w, 8, eps=0.0)
    ms = (out.reshape(5, 8, 32) ** 2).mean(axis=-1)
    np.testing.assert_allclose(ms, 1.0, rtol=1e-13)
    np.testing.assert_allclose(oracle.gated_rmsnorm(7.0 * y, w, 8, eps=0.0), out, rtol=1e-13)
    # one group over all channels is not the mean of the per-group norms
    assert not np.allclose(oracle.gated_rmsnorm(y, w, 1, eps=0.0), out)
