"""Write ``tiny_attention.json``: oracle outputs for two tiny seeded problems.

The pages print no worked example of Ring Self-Attention (no input/output values), so the
stored values here come from the fp64 oracle alone; they guard the oracle against silent
drift between commits. Run from the repository root: ``python tests/golden/make_golden.py``.
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import oracle  # noqa: E402
from sequence_ring_self_b200.inputs import make_inputs  # noqa: E402


def main():
    cases = []
    for causal in (False, True):
        x = make_inputs(1, 1, 8, 4, seed=0, dtype="f32")
        o, lse = oracle.forward(x.q, x.k, x.v, causal)
        dq, dk, dv = oracle.backward(x.q, x.k, x.v, x.do, causal)
        cases.append({
            "shape": [1, 1, 8, 4], "seed": 0, "dtype": "f32", "causal": causal,
            "O": o.ravel().tolist(), "lse": lse.ravel().tolist(),
            "dQ": dq.ravel().tolist(), "dK": dk.ravel().tolist(), "dV": dv.ravel().tolist(),
        })
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_attention.json")
    with open(out, "w") as f:
        json.dump({"source": "oracle/rsa_oracle.c via tests/golden/make_golden.py",
                   "cases": cases}, f, indent=0)
    print("wrote", out)


if __name__ == "__main__":
    main()
