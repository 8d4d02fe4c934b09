"""Write tests/golden/oracle_small_case.json from the fp64 oracle.

The pages print no worked example of the layer, so this fixture is a
regression record, not an independent pin: it freezes the oracle's output on
one small seeded case (b=1, L=40, D=6, N=16, fp32 inputs, seed 11, CPU
generator) so that any later change to the oracle's arithmetic shows up.
Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from bidirectional_mamba_denoiser_b200 import workloads  # noqa: E402

CASE = {"batch": 1, "L": 40, "D": 6, "N": 16, "dtype": "fp32", "seed": 11}


def compute():
    inp, par = workloads.make_case(CASE["batch"], CASE["L"], CASE["D"], CASE["N"], CASE["dtype"], CASE["seed"])
    out, yf, yb = oracle.layer_fwd(inp, par, return_dirs=True)
    return out, yf, yb


def main():
    out, yf, yb = compute()
    rec = {
        "what": "fp64 oracle output of the bidirectional mixer layer on one seeded case",
        "case": CASE,
        "generator": "bidirectional_mamba_denoiser_b200.workloads.make_case (CPU torch.Generator)",
        "out": [float(v).hex() for v in out.ravel()],
        "y_fwd": [float(v).hex() for v in yf.ravel()],
        "y_rev": [float(v).hex() for v in yb.ravel()],
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small_case.json")
    with open(path, "w") as f:
        json.dump(rec, f, indent=0)
    print("wrote", path)


if __name__ == "__main__":
    main()
