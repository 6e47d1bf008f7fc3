"""Writes tests/golden/tiny_index.json from the fp64 oracle alone.

Run:  python tests/golden/make_golden.py
The stored values are a regression record of the oracle on the seeded
1024-token workload (S=1024, Hq=4, Hkv=2, d=128, b=128, gamma=0.9, tau=0.1);
the oracle's independent pins live in tests/test_oracle_pins.py.
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from dynamic_block_sparse_last_b200 import synth  # noqa: E402
from oracle import oracle as orc  # noqa: E402


def main():
    w = synth.WORKLOADS["tiny"]
    x = synth.make_inputs(w)
    P = orc.OracleProblem(x["q"], x["k"], x["v"], w.b)
    heads = []
    for h in range(w.Hq):
        out = P.build_index_head(h, w.gamma, w.tau)
        heads.append({"pattern": out["pattern"], "jsd": out["jsd"], "vhat": out["vhat"].tolist(),
                      "shat": out["shat"].tolist(), "rows": [list(map(int, r)) for r in out["rows"]]})
    doc = {"workload": "S=1024 Hq=4 Hkv=2 d=128 b=128 gamma=0.9 tau=0.1 seed=0",
           "writer": "tests/golden/make_golden.py (oracle only)", "heads": heads}
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_index.json"), "w") as f:
        json.dump(doc, f, indent=1)


if __name__ == "__main__":
    main()
