"""Writes the oracle regression fixtures in this folder.

Run from the repository root:  python tests/golden/make_golden.py
Only the oracle computes the stored values; the inputs come from the seeded
generators.  The fixtures lock the oracle's output on two small cases so that
a later change to its arithmetic shows up as a failing test; such a change
must cite the passage of the pages (or the reading of it) that justifies it.
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from prng_seeded_decompress_b200 import inputs  # noqa: E402

CASES = [
    # name, rows, cols, (C, P), layer seed, activation seed
    ("oracle_c8p3_12x50", 12, 50, inputs.FORMAT_4BIT, 101, 201),
    ("oracle_c12p4_10x61", 10, 61, inputs.FORMAT_3BIT, 102, 202),
]


def case_values(rows, cols, cp, lseed, xseed):
    L = inputs.make_layer(rows, cols, *cp, seed=lseed)
    _, x = inputs.make_activations((cols,), "f16", xseed)
    W = oracle.decompress(L["fmt"], L["rec"], L["eplane"])
    y, ya = oracle.gemv(L["fmt"], L["rec"], L["eplane"], x)
    return {
        "fmt": L["fmt"],
        "W_row0": [float(v).hex() for v in W[0]],
        "W_sum": float(W.sum()).hex(),
        "y": [float(v).hex() for v in y],
        "yabs": [float(v).hex() for v in ya],
    }


def main():
    here = os.path.dirname(os.path.abspath(__file__))
    for name, rows, cols, cp, ls, xs in CASES:
        d = {"generated_by": "tests/golden/make_golden.py (oracle only)",
             "inputs": {"rows": rows, "cols": cols, "C": cp[0], "P": cp[1],
                        "layer_seed": ls, "x_seed": xs, "x_dtype": "f16"}}
        d.update(case_values(rows, cols, cp, ls, xs))
        with open(os.path.join(here, name + ".json"), "w") as fh:
            json.dump(d, fh, indent=1)
            fh.write("\n")


if __name__ == "__main__":
    main()
