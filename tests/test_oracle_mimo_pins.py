"""Pins of the oracle's MIMO decode step against mathematics it does not share (CPU only).

* closed form over several steps, with numpy matrix products: S_T = (prod a) S_0 +
  sum_t (prod_{u>t} a_u) dt_t X_t^T B_t and y_t = (S_t C_t^T)^T + D X_t, gated;
* rank 1 with post-conv inputs equals the (separately pinned) Mamba-2 decode oracle with the conv
  reduced to the identity tap (w = [0, 0, 0, 1], b = 0, so its post-conv values are SiLU of the raw ones);
* permuting the R input/output slots permutes y and leaves the state unchanged;
* dt -> 0 leaves the state unchanged and reduces y to (S C_k + D x_k) silu(z_k).
"""
import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle
from pins import f64, silu_lib, softplus_lib
from selective_state_space_43_b200.synth import Dims, make_mimo_decode_inputs


def case(R=3, steps=4, Bt=2, H=4, G=2, P=5, N=6, seed=1):
    d = Dims(Bt, 1, H, P, N, G, 64)
    data = make_mimo_decode_inputs(d, R, steps, dtype=torch.float32, seed=seed, random_D=True)
    params = {k: f64(v) for k, v in data["params"].items()}
    steps_ = [{k: f64(v) for k, v in s.items()} for s in data["steps"]]
    return d, params, f64(data["ssm_state"]).copy(), steps_


@pytest.mark.parametrize("R", [1, 2, 4])
def test_closed_form_over_steps(R):
    d, prm, S0, steps = case(R=R, steps=5)
    S = S0.copy()
    ys = [oracle.mimo_decode_step(s, prm, S) for s in steps]
    H, G = d.nheads, d.ngroups
    for b in range(d.batch):
        for h in range(H):
            g = h // (H // G)
            dts = [softplus_lib(s["dt"][b, h] + prm["dt_bias"][h]) for s in steps]
            a = [np.exp(dt * prm["A"][h]) for dt in dts]
            for T in range(1, len(steps) + 1):
                St = np.prod(a[:T]) * S0[b, h]
                for t in range(T):
                    X, Bk = steps[t]["x"][b, h], steps[t]["B"][b, g]          # [R, P], [R, N]
                    St = St + np.prod(a[t + 1:T]) * dts[t] * (X.T @ Bk)
                s = steps[T - 1]
                y = ((St @ s["C"][b, g].T).T + prm["D"][h] * s["x"][b, h]) * silu_lib(s["z"][b, h])
                assert np.max(np.abs(ys[T - 1][b, h] - y)) < 1e-12 * max(1.0, np.max(np.abs(y)))
            assert np.max(np.abs(S[b, h] - St)) < 1e-12


def test_rank_one_is_the_mamba2_decode_without_conv():
    Bt, H, G, P, N = 2, 4, 2, 5, 6
    rng = np.random.default_rng(4)
    raw = dict(x=rng.standard_normal((Bt, H * P)), z=rng.standard_normal((Bt, H * P)),
               dt=rng.standard_normal((Bt, H)), B=rng.standard_normal((Bt, G, N)) / 3,
               C=rng.standard_normal((Bt, G, N)) / 3)
    conv_dim = H * P + 2 * G * N
    params = dict(A=-np.exp(rng.uniform(0, 2.7, H)), D=rng.uniform(0.5, 1.5, H), dt_bias=rng.uniform(-5, -1, H),
                  conv_w=np.tile([0.0, 0.0, 0.0, 1.0], (conv_dim, 1)), conv_b=np.zeros(conv_dim))
    S0 = rng.standard_normal((Bt, H, P, N)) * 0.1
    s_siso = S0.copy()
    y_siso = oracle.decode_step(raw, params, rng.standard_normal((Bt, conv_dim, 3)), s_siso)
    post = dict(x=(raw["x"] * expit(raw["x"])).reshape(Bt, H, 1, P), z=raw["z"].reshape(Bt, H, 1, P),
                dt=raw["dt"], B=(raw["B"] * expit(raw["B"]))[:, :, None, :],
                C=(raw["C"] * expit(raw["C"]))[:, :, None, :])
    s_mimo = S0.copy()
    y_mimo = oracle.mimo_decode_step(post, params, s_mimo)
    assert np.max(np.abs(y_mimo.reshape(Bt, H * P) - y_siso)) < 1e-12
    assert np.max(np.abs(s_mimo - s_siso)) < 1e-13


def test_slot_permutation():
    d, prm, S0, steps = case(R=4, steps=1, seed=3)
    s = steps[0]
    perm = [2, 0, 3, 1]
    ps = dict(s, x=s["x"][:, :, perm], z=s["z"][:, :, perm], B=s["B"][:, :, perm], C=s["C"][:, :, perm])
    S1, S2 = S0.copy(), S0.copy()
    y1 = oracle.mimo_decode_step(s, prm, S1)
    y2 = oracle.mimo_decode_step({k: np.ascontiguousarray(v) for k, v in ps.items()}, prm, S2)
    assert np.max(np.abs(S1 - S2)) < 1e-13
    assert np.max(np.abs(y1[:, :, perm] - y2)) < 1e-13


def test_vanishing_step_leaves_the_state():
    d, prm, S0, steps = case(R=2, steps=1, seed=5)
    s = dict(steps[0], dt=np.full_like(steps[0]["dt"], -60.0))
    prm = dict(prm, dt_bias=np.zeros_like(prm["dt_bias"]))
    S = S0.copy()
    y = oracle.mimo_decode_step(s, prm, S)
    assert np.max(np.abs(S - S0)) < 1e-20
    H, G = d.nheads, d.ngroups
    for b in range(d.batch):
        for h in range(H):
            g = h // (H // G)
            want = ((S0[b, h] @ s["C"][b, g].T).T + prm["D"][h] * s["x"][b, h]) * silu_lib(s["z"][b, h])
            assert np.max(np.abs(y[b, h] - want)) < 1e-13
