"""Pins of the oracle's backward (the gradients of the prefill) against mathematics it does not share.

The backward is the adjoint of the token-by-token recurrence.  It is pinned to the forward oracle
(itself pinned to the quadratic form, closed forms and library routines) by routes that do not
re-type the adjoint:

* central finite differences of the forward, along random directions in every input, and element by
  element for the per-head and per-channel parameters;
* exact identities of the forward's linear dependences: y and final_state are linear in the initial
  state, y is affine in D, so the loss's change between two values of those inputs equals the
  gradient's inner product with the difference, with no truncation error.
CPU only.
"""
import numpy as np
import pytest
import torch

import oracle
from pins import f64
from selective_state_space_43_b200.synth import Dims, make_backward_grads, make_prefill_inputs

KEYS = ("x", "dt", "B", "C", "z", "A", "D", "dt_bias", "conv_w", "conv_b", "init_state", "init_conv_state")


def case(seed=5, L=21, H=4, P=3, N=5, G=2, Bt=2, init=True, d_final=True):
    d = Dims(Bt, L, H, P, N, G, 8)
    inp = make_prefill_inputs(d, dtype=torch.float32, seed=seed, init_state=init, init_conv_state=init,
                              random_D=True)
    inp = {k: f64(v) for k, v in inp.items()}
    if not init:
        inp["init_state"] = np.zeros((Bt, H, P, N))
        inp["init_conv_state"] = np.zeros((Bt, d.conv_dim, 3))
    gr = make_backward_grads(d, dtype=torch.float32, seed=seed + 100, d_final=d_final)
    return inp, f64(gr["dy"]), f64(gr["d_final"])


def loss(inp, dy, df):
    y, fs, _ = oracle.prefill(inp, nthreads=1)
    v = float(np.sum(dy * y))
    if df is not None:
        v += float(np.sum(df * fs))
    return v


def perturbed(inp, key, delta):
    out = dict(inp)
    out[key] = inp[key] + delta
    return out


@pytest.mark.parametrize("init,d_final", [(True, True), (False, True), (True, False)])
def test_directional_finite_differences(init, d_final):
    inp, dy, df = case(init=init, d_final=d_final)
    grads = oracle.prefill_backward(inp, dy, df, nthreads=2)
    rng = np.random.default_rng(11)
    eps = 1e-5
    for key in KEYS:
        v = rng.standard_normal(inp[key].shape)
        fd = (loss(perturbed(inp, key, eps * v), dy, df) - loss(perturbed(inp, key, -eps * v), dy, df)) / (2 * eps)
        an = float(np.sum(grads[key] * v))
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(fd)), (key, fd, an)


def test_elementwise_finite_differences_of_parameters():
    inp, dy, df = case(seed=9, L=13)
    grads = oracle.prefill_backward(inp, dy, df, nthreads=1)
    eps = 1e-6
    for key in ("A", "D", "dt_bias", "conv_b", "conv_w"):
        flat = inp[key].reshape(-1)
        for i in range(flat.size):
            e = np.zeros(flat.size)
            e[i] = eps
            e = e.reshape(inp[key].shape)
            fd = (loss(perturbed(inp, key, e), dy, df) - loss(perturbed(inp, key, -e), dy, df)) / (2 * eps)
            an = grads[key].reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (key, i, fd, an)


def test_elementwise_finite_differences_of_activations():
    # every token of one sequence: checks the time indexing of dx, ddt, dB, dC, dz
    inp, dy, df = case(seed=4, L=11, Bt=1)
    grads = oracle.prefill_backward(inp, dy, df, nthreads=1)
    eps = 1e-6
    rng = np.random.default_rng(2)
    for key in ("x", "dt", "B", "C", "z"):
        for t in range(inp[key].shape[1]):
            e = np.zeros(inp[key].shape)
            e[0, t] = rng.standard_normal(e[0, t].shape) * eps
            fd = (loss(perturbed(inp, key, e), dy, df) - loss(perturbed(inp, key, -e), dy, df)) / 2
            an = float(np.sum(grads[key] * e))
            assert abs(fd - an) <= 1e-6 * max(eps, abs(fd)), (key, t, fd, an)


def test_initial_state_enters_linearly():
    # loss(S0) - loss(0) = <d_init_state, S0> exactly: y and final_state are linear in S0
    inp, dy, df = case(seed=7, L=40)
    grads = oracle.prefill_backward(inp, dy, df)
    zero = dict(inp)
    zero["init_state"] = np.zeros_like(inp["init_state"])
    diff = loss(inp, dy, df) - loss(zero, dy, df)
    an = float(np.sum(grads["init_state"] * inp["init_state"]))
    assert abs(diff - an) <= 1e-11 * max(1.0, abs(diff))
    # and the gradient does not depend on S0 itself
    g0 = oracle.prefill_backward(zero, dy, df)
    assert np.max(np.abs(g0["init_state"] - grads["init_state"])) < 1e-12


def test_D_enters_affinely():
    # y = (S C + D x) silu(z): loss(D) - loss(0) = <dD, D>, and dD is the same at D = 0
    inp, dy, df = case(seed=8, L=30)
    grads = oracle.prefill_backward(inp, dy, df)
    zero = dict(inp)
    zero["D"] = np.zeros_like(inp["D"])
    diff = loss(inp, dy, df) - loss(zero, dy, df)
    an = float(np.sum(grads["D"] * inp["D"]))
    assert abs(diff - an) <= 1e-11 * max(1.0, abs(diff))
    assert np.max(np.abs(oracle.prefill_backward(zero, dy, df)["D"] - grads["D"])) < 1e-12


def test_gradients_are_linear_in_the_incoming_gradients():
    inp, dy, df = case(seed=3, L=17)
    g1 = oracle.prefill_backward(inp, dy, None)
    g2 = oracle.prefill_backward(inp, np.zeros_like(dy), df)
    g12 = oracle.prefill_backward(inp, dy, df)
    for key in KEYS:
        assert np.max(np.abs(g1[key] + g2[key] - g12[key])) <= 1e-12 * max(1.0, np.max(np.abs(g12[key])))


def test_segment_recomputation_boundary():
    # 130 tokens cross two checkpoint segments; finite differences of the state-related inputs
    inp, dy, df = case(seed=12, L=130, H=2, G=1, P=2, N=3, Bt=1)
    grads = oracle.prefill_backward(inp, dy, df)
    rng = np.random.default_rng(5)
    eps = 1e-5
    for key in ("x", "dt", "B", "A", "init_state"):
        v = rng.standard_normal(inp[key].shape)
        fd = (loss(perturbed(inp, key, eps * v), dy, df) - loss(perturbed(inp, key, -eps * v), dy, df)) / (2 * eps)
        an = float(np.sum(grads[key] * v))
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(fd)), (key, fd, an)


def test_thread_count_does_not_change_the_result():
    inp, dy, df = case(seed=6, L=25, Bt=3)
    a = oracle.prefill_backward(inp, dy, df, nthreads=1)
    b = oracle.prefill_backward(inp, dy, df, nthreads=4)
    for key in KEYS:
        assert np.array_equal(a[key], b[key]), key
