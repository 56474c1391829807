"""Regression check: the oracle still reproduces its frozen small-case output
(tests/golden/oracle_quant_small.json, written by tests/golden/make_golden.py)."""
import json
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_matches_frozen_fixture(orc):
    with open(os.path.join(HERE, "golden", "oracle_quant_small.json")) as f:
        gold = json.load(f)
    x = np.array([[int(t, 16) for t in row.split()] for row in gold["x_bf16_hex"]], dtype=np.uint16)
    for pow2 in (False, True):
        q, s = orc.quant_act_1x128(x, pow2)
        g = gold[f"act_pow2={int(pow2)}"]
        assert [" ".join(f"{v:02x}" for v in row) for row in q] == g["q_hex"]
        assert [[f"{int(v):08x}" for v in r.view(np.uint32)] for r in s] == g["s_f32_hex"]
