"""Regression snapshot of the oracle and the generator on the tiny workload.

tests/golden/tiny_oracle.json was written by tests/golden/make_golden.py,
which calls only the oracle and the seeded generator. It guards against
silent drift; the oracle's independent pins live in oracle_pins.py.
"""
import hashlib
import json
import os

import numpy as np

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "tiny_oracle.json")


def test_tiny_snapshot():
    with open(GOLDEN) as f:
        g = json.load(f)
    inp = workloads.make_inputs("tiny", seed=0)
    for n, h in g["inputs_sha256"].items():
        t = getattr(inp, n).contiguous().numpy().tobytes()
        assert hashlib.sha256(t).hexdigest() == h, f"generator drift in {n}"
    ref = oracle.reference_outputs(inp)
    w = inp.w
    np.testing.assert_allclose(ref["rstd_q"].reshape(w.T, w.Hq), g["rstd_q"], rtol=1e-13)
    np.testing.assert_allclose(ref["rstd_k"].reshape(w.T, w.Hkv), g["rstd_k"], rtol=1e-13)
    np.testing.assert_allclose(ref["dgamma_q"], g["dgamma_q"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(ref["dgamma_k"], g["dgamma_k"], rtol=1e-12, atol=1e-13)
    for name in ("q_out", "k_out", "dq", "dk"):
        a = ref[name].reshape(w.T, -1, w.D)
        for t in g["tokens"]:
            np.testing.assert_allclose(a[t], g[name][str(t)], rtol=1e-12, atol=1e-13)
        assert abs(float(np.sum(a)) - g[name + "_sum"]) < 1e-9
        assert abs(float(np.sum(a * a)) - g[name + "_sumsq"]) < 1e-9 * g[name + "_sumsq"]
