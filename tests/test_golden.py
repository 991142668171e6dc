"""The oracle reproduces its stored outputs for the tiny seeded problems (drift guard)."""
import json
import os

import numpy as np

from sequence_ring_self_b200.inputs import make_inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_attention.json")


def test_oracle_matches_stored_outputs(orc):
    data = json.load(open(GOLDEN))
    for case in data["cases"]:
        B, H, L, d = case["shape"]
        x = make_inputs(B, H, L, d, seed=case["seed"], dtype=case["dtype"])
        o, lse = orc.forward(x.q, x.k, x.v, case["causal"])
        dq, dk, dv = orc.backward(x.q, x.k, x.v, x.do, case["causal"])
        for name, got in (("O", o), ("lse", lse), ("dQ", dq), ("dK", dk), ("dV", dv)):
            np.testing.assert_allclose(got.ravel(), np.array(case[name]), rtol=1e-13, atol=1e-15,
                                       err_msg=name)
