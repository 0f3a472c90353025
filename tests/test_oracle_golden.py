"""Regression guard: the oracle still reproduces the stored tiny fixture,
written by tests/golden/make_golden.py from the oracle alone."""
import json
import os
import sys

import numpy as np

import oracle

sys.path.insert(0, os.path.join(os.path.dirname(__file__), "golden"))
import make_golden  # noqa: E402


def test_oracle_matches_stored_fixture():
    with open(os.path.join(os.path.dirname(__file__), "golden", "oracle_tiny.json")) as f:
        g = json.load(f)
    y, fs, cs = oracle.prefill(make_golden.inputs(), nthreads=1)
    assert np.max(np.abs(y.ravel() - np.array(g["y"]))) < 1e-14
    assert np.max(np.abs(fs.ravel() - np.array(g["final_state"]))) < 1e-14
    assert np.array_equal(cs.ravel(), np.array(g["conv_state"]))


def test_oracle_backward_and_mimo_match_stored_fixture():
    with open(os.path.join(os.path.dirname(__file__), "golden", "oracle_tiny_grads.json")) as f:
        g = json.load(f)
    gr = make_golden.grads_inputs()
    got = oracle.prefill_backward(make_golden.inputs(), gr["dy"], gr["d_final"], nthreads=1)
    for k, v in g["grads"].items():
        assert np.max(np.abs(got[k].ravel() - np.array(v))) <= 1e-13 * max(1.0, np.max(np.abs(v))), k
    ys, state = make_golden.mimo_outputs()
    for y, v in zip(ys, g["mimo_y"]):
        assert np.max(np.abs(y.ravel() - np.array(v))) < 1e-14
    assert np.max(np.abs(state.ravel() - np.array(g["mimo_state"]))) < 1e-14
