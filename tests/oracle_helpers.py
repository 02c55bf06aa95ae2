"""Helpers shared by the oracle tests (test-side only)."""
import os

import numpy as np

import synth
from oracle import kimodo_oracle as ko

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

TINY = dict(d_model=32, n_heads=4, d_ff=64, n_layers=2, d_text=16)


def tiny_shapes():
    return synth.Dims(**TINY), ko.Shape(**TINY)


def tiny_params(seed=11, ln_identity=False):
    dims, shape = tiny_shapes()
    blob = synth.weight_blob(dims, seed=seed, ln_identity=ln_identity)
    return ko.unpack_weights(blob, shape)


def read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            k, v = (s.strip() for s in line.split("=", 1))
            vals[k] = float(v)
    return vals


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
