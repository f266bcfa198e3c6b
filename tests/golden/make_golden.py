"""Write tests/golden/tiny_oracle_snapshot.json from the oracle alone.

A regression snapshot of the oracle on the tiny workload (B=1, H=2, N=256,
d=64, fp16, seed 0): it makes any later change to the oracle's arithmetic
visible.  It calls nothing but ``oracle`` and the seeded input generator.
Run: python tests/golden/make_golden.py
"""

import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle as orc  # noqa: E402
from quantized_attention_06_b200.inputs import WORKLOADS, generate  # noqa: E402

ROWS = [0, 1, 63, 64, 127, 128, 200, 255]


def snapshot():
    w = WORKLOADS["tiny"]
    x = generate(w)
    heads = []
    for h in range(w.heads_q):
        r = orc.attention_head(x["q"][0, h], x["k"][0, h], x["v"][0, h])
        heads.append({
            "q8_sha256": hashlib.sha256(r["q8"].tobytes()).hexdigest(),
            "k8_sha256": hashlib.sha256(r["k8"].tobytes()).hexdigest(),
            "v8_sha256": hashlib.sha256(r["v8"].tobytes()).hexdigest(),
            "s_int_sha256": hashlib.sha256(r["s_int"].astype(np.int32).tobytes()).hexdigest(),
            "q_scale": [float(s) for s in r["q_scale"]],
            "k_scale": [float(s) for s in r["k_scale"]],
            "k_mean_first8": [float(s) for s in r["k_mean"][:8]],
            "rows": ROWS,
            "out_rows": [[float(v) for v in r["out"][i]] for i in ROWS],
            "lse_rows": [float(r["lse"][i]) for i in ROWS],
        })
    return {"workload": "tiny", "heads": heads}


if __name__ == "__main__":
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle_snapshot.json")
    with open(path, "w") as f:
        json.dump(snapshot(), f, indent=1)
    print("wrote", path)
