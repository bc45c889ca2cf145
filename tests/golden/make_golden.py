"""Writes oracle_small.json: oracle outputs on a small seeded unit.

Calls only ``oracle/`` and ``rkv_synth`` (the seeded inputs).  The pages
print no worked example, so this file is a regression record of the oracle
itself, not an independent pin: the pins live in tests/test_oracle_pins.py.
Re-run after any justified change to the oracle's arithmetic.
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from rkv_synth import Workload, bf16_bits, make_inputs  # noqa: E402

CASES = [
    # name, workload, redundancy mode
    ("mean_small", Workload("g", 1, 1, 2, 8, 128, (40,), buffer=24, seed=21), oracle.RED_MEAN),
    ("max_small", Workload("g", 1, 1, 2, 8, 128, (40,), buffer=24, seed=22), oracle.RED_MAX),
]


def compute():
    out = {}
    for name, w, mode in CASES:
        x = make_inputs(w)
        N = int(x["cur_len"][0])
        q = bf16_bits(x["Q"])[0, 0]
        k = bf16_bits(x["K"])[0, 0]
        G = w.n_q_heads // w.n_kv_heads
        heads = []
        for h in range(w.n_kv_heads):
            u = oracle.unit(q[h * G:(h + 1) * G], k[h], N, w.budget_of(0), w.mix_lambda,
                            red_mode=mode)
            heads.append({"kept": u["kept"].tolist(),
                          "I": [float(v) for v in u["I"]],
                          "r": [float(v) for v in u["r"]],
                          "Z": [float(v) for v in u["Z"]]})
        out[name] = {"N": N, "budget": w.budget_of(0), "window": w.window,
                     "lambda": w.mix_lambda, "mode": mode, "heads": heads}
    return out


if __name__ == "__main__":
    with open(os.path.join(HERE, "oracle_small.json"), "w") as f:
        json.dump(compute(), f, indent=1)
