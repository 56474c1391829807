"""Write the oracle regression fixtures in this folder.  Calls only ``oracle`` and the
seeded generators; run ``python tests/golden/make_golden.py`` from the repo root.

The fixtures freeze the oracle's output on a small seeded case so that a later
change to its arithmetic shows up as a diff (and must name the passage that
justifies it).  They are not independent pins: those live in tests/test_oracle_*.py.
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle      # noqa: E402
import workloads   # noqa: E402


def main():
    rng = np.random.default_rng(20240501)
    x = workloads.normal_bf16(rng, (4, 256), 1.0, 0.01)
    w = workloads.normal_bf16(rng, (128, 256), 0.02)
    out = {"x_bf16_hex": [" ".join(f"{v:04x}" for v in row) for row in x]}
    for pow2 in (False, True):
        q, s = oracle.quant_act_1x128(x, pow2)
        out[f"act_pow2={int(pow2)}"] = {
            "q_hex": [" ".join(f"{v:02x}" for v in row) for row in q],
            "s_f32_hex": [[f"{int(v):08x}" for v in r.view(np.uint32)] for r in s],
        }
        qw, sw = oracle.quant_weight_128x128(w, pow2)
        out[f"weight_pow2={int(pow2)}"] = {
            "w_sha_rows": int(w.astype(np.uint64).sum()),
            "q_sum": int(qw.astype(np.uint64).sum()),
            "q_row0_hex": " ".join(f"{v:02x}" for v in qw[0]),
            "s_f32_hex": [[f"{int(v):08x}" for v in r.view(np.uint32)] for r in sw],
        }
    with open(os.path.join(HERE, "oracle_quant_small.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
