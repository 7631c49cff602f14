"""Writes tests/golden/tiny_oracle.json: a regression lock on the fp64 oracle
for the tiny workload (one 8x8 window, 1 head, d=32, r=8).

Calls only the oracle (``oracle/``) and the seeded input generator.  Run from
the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from rank_biased_window_b200.inputs import WORKLOADS, to_f64, workload_inputs  # noqa: E402


def main():
    wl = WORKLOADS["tiny"]
    x = {k: to_f64(v) for k, v in workload_inputs(wl).items()}
    o, lse = oracle.fwd(x["q"], x["k"], x["v"], x["u"], x["w"], wl.scale)
    rows = [0, 31, 63]
    out = {
        "what": "fp64 oracle forward on the tiny workload (seeded inputs), written by "
                "tests/golden/make_golden.py",
        "workload": wl.note,
        "lse": [float(t) for t in lse.reshape(-1)],
        "o_rows": {str(i): [float(t) for t in o.reshape(-1, wl.d)[i]] for i in rows},
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
