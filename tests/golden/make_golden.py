"""Writes oracle_tiny.json: the fp64 oracle's output on one tiny seeded input.

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
from selective_state_space_43_b200.synth import Dims, make_prefill_inputs  # noqa: E402

DIMS = Dims(1, 6, 2, 2, 3, 1, 8)
SEED = 1234


def inputs():
    return make_prefill_inputs(DIMS, dtype=torch.bfloat16, seed=SEED, init_state=True, init_conv_state=True,
                               random_D=True)


if __name__ == "__main__":
    y, fs, cs = oracle.prefill(inputs(), nthreads=1)
    out = dict(dims=DIMS.as_dict(), seed=SEED, dtype="bf16", init_state=True, init_conv_state=True,
               random_D=True, y=y.ravel().tolist(), final_state=fs.ravel().tolist(),
               conv_state=cs.ravel().tolist())
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny.json"), "w") as f:
        json.dump(out, f, indent=0)
