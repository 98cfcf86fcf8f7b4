"""Writes tests/golden/tiny_oracle.json from the CPU oracle alone.

The pages print no worked example for this op, so this fixture is not an
independent pin: it is a regression snapshot of the oracle (and of the seeded
generator) on the 32-token fp32 workload, seed 0. The oracle's independent
pins are in tests/oracle_pins.py. Regenerate only with a commit message that
names the passage, or the reading of it, that justifies the change.

Usage: python tests/golden/make_golden.py
"""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import workloads  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json")
KEEP_TOKENS = [0, 1, 17, 31]


def fingerprint(t) -> str:
    return hashlib.sha256(t.contiguous().numpy().tobytes()).hexdigest()


def main():
    inp = workloads.make_inputs("tiny", seed=0)
    ref = oracle.reference_outputs(inp)
    w = inp.w
    doc = {
        "what": "oracle outputs for workload 'tiny' (B=1 S=32 Hq=4 Hkv=2 D=16 "
                "R=16 theta=1e4 eps=1e-6 fp32), seed 0; regression snapshot",
        "inputs_sha256": {n: fingerprint(getattr(inp, n)) for n in
                          ("q", "k", "gamma_q", "gamma_k", "dq_out", "dk_out")},
        "tokens": KEEP_TOKENS,
        "rstd_q": ref["rstd_q"].reshape(w.T, w.Hq).tolist(),
        "rstd_k": ref["rstd_k"].reshape(w.T, w.Hkv).tolist(),
        "dgamma_q": ref["dgamma_q"].tolist(),
        "dgamma_k": ref["dgamma_k"].tolist(),
    }
    for name in ("q_out", "k_out", "dq", "dk"):
        a = ref[name].reshape(w.T, -1, w.D)
        doc[name] = {str(t): a[t].tolist() for t in KEEP_TOKENS}
        doc[name + "_sum"] = float(np.sum(a))
        doc[name + "_sumsq"] = float(np.sum(a * a))
    with open(OUT, "w") as f:
        json.dump(doc, f, indent=1)
    print("wrote", OUT)


if __name__ == "__main__":
    main()
