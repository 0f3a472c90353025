"""Writes oracle_tiny.json (the fp64 oracle's prefill on one tiny seeded input) and
oracle_tiny_grads.json (its backward on the same input, and two MIMO decode steps).

The stored values come from ``oracle/`` alone (this script calls nothing
else); they guard the oracle against unintended changes.  The oracle itself is
pinned to independent mathematics by tests/test_oracle_pins.py.
Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from selective_state_space_43_b200.synth import (Dims, make_backward_grads, make_mimo_decode_inputs,  # noqa: E402
                                                 make_prefill_inputs)

DIMS = Dims(1, 6, 2, 2, 3, 1, 8)
SEED = 1234


def inputs():
    return make_prefill_inputs(DIMS, dtype=torch.bfloat16, seed=SEED, init_state=True, init_conv_state=True,
                               random_D=True)


def grads_inputs():
    """dy and d_final of the backward fixture (bf16 dy, fp32 d_final)."""
    return make_backward_grads(DIMS, dtype=torch.bfloat16, seed=SEED + 1)


MIMO_DIMS = Dims(2, 1, 2, 2, 3, 1, 8)
MIMO_RANK = 2


def mimo_inputs():
    return make_mimo_decode_inputs(MIMO_DIMS, MIMO_RANK, 2, dtype=torch.bfloat16, seed=SEED + 2, random_D=True)


def mimo_outputs():
    data = mimo_inputs()
    state = data["ssm_state"].double().numpy().copy()
    ys = [oracle.mimo_decode_step(s, data["params"], state) for s in data["steps"]]
    return ys, state


if __name__ == "__main__":
    y, fs, cs = oracle.prefill(inputs(), nthreads=1)
    out = dict(dims=DIMS.as_dict(), seed=SEED, dtype="bf16", init_state=True, init_conv_state=True,
               random_D=True, y=y.ravel().tolist(), final_state=fs.ravel().tolist(),
               conv_state=cs.ravel().tolist())
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny.json"), "w") as f:
        json.dump(out, f, indent=0)

    gr = grads_inputs()
    g = oracle.prefill_backward(inputs(), gr["dy"], gr["d_final"], nthreads=1)
    ys, state = mimo_outputs()
    out = dict(dims=DIMS.as_dict(), seed=SEED, grads={k: v.ravel().tolist() for k, v in g.items()},
               mimo_dims=MIMO_DIMS.as_dict(), mimo_rank=MIMO_RANK, mimo_y=[y.ravel().tolist() for y in ys],
               mimo_state=state.ravel().tolist())
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny_grads.json"), "w") as f:
        json.dump(out, f, indent=0)
