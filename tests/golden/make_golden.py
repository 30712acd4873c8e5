"""Write tests/golden/oracle_tiny.json and oracle_bwd_tiny.json from the fp64 oracle (and the seeded
inputs) only.

The pages print no worked numeric example for this recurrence, so this fixture is
a regression anchor of the oracle itself, not a value from the pages: it pins the
seeded generator plus the oracle against silent change. Run from the repo root:
    python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import dn_inputs as di  # noqa: E402
import oracle  # noqa: E402

SIZES = {"B": 1, "T": 6, "H": 2, "dk": 4, "dv": 4}
WORKLOAD = "fg2_osdn_long"

w = di.WORKLOADS[WORKLOAD].scaled(**SIZES)
x = di.make_inputs(w)
o, ST = oracle.fwd(**x)
out = {
    "what": "fp64 oracle on the seeded fg2_osdn_long recipe at tiny sizes (regression anchor)",
    "workload": WORKLOAD,
    "sizes": SIZES,
    "o_head": [float(v) for v in o.ravel()[:16]],
    "S_head": [float(v) for v in ST.ravel()[:16]],
    "o_norm": float(np.linalg.norm(o)),
    "S_norm": float(np.linalg.norm(ST)),
}
with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny.json"), "w") as f:
    json.dump(out, f, indent=1)
print("wrote oracle_tiny.json")

# the reverse mode on the same inputs, with the seeded cotangents of the same recipe
gb = di.make_bwd_inputs(w)
g = oracle.bwd(**x, dO=gb["dO"], dS_T=gb["dS_T"])
out = {
    "what": "fp64 oracle reverse mode on the seeded fg2_osdn_long recipe at tiny sizes (regression anchor)",
    "workload": WORKLOAD,
    "sizes": SIZES,
    "grad_head": {n: [float(v) for v in a.ravel()[:8]] for n, a in g.items() if a is not None},
    "grad_norm": {n: float(np.linalg.norm(a)) for n, a in g.items() if a is not None},
}
with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_bwd_tiny.json"), "w") as f:
    json.dump(out, f, indent=1)
print("wrote oracle_bwd_tiny.json")
