"""Writes tq3_tie_counts.txt: for the TQ3 round-trip and KV-cache workloads, the number of
coefficients the oracle places within 1e-6 of a codebook boundary (the only places where an encoder
that rounds in another order may pick the neighbouring index), and the number of exact zeros among
them. Calls only the oracle and the seeded input recipes.

    python tests/golden/make_tq3_tie_counts.py
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from weight_quantization_b200 import inputs  # noqa: E402

WINDOW = 1e-6


def counts(x, is_bf16):
    xs, _, _, _ = oracle.tq3_encode_debug(x, inputs.tq3_sign_bits(), is_bf16=is_bf16)
    _, B = oracle.tq3_tables()
    near = np.zeros(xs.shape, bool)
    for b in B.astype(np.float64):
        near |= np.abs(xs.astype(np.float64) - b) < WINDOW
    return xs.shape[0], int(near.sum()), int((xs == 0).sum())


def main():
    oracle.lib()
    rows = [("tq3_roundtrip_fp32",) + counts(inputs.tq3_roundtrip(), False)]
    k, v = inputs.kv_cache()
    ck, cv = counts(k.reshape(-1, 128), True), counts(v.reshape(-1, 128), True)
    rows.append(("kv_cache_bf16", ck[0] + cv[0], ck[1] + cv[1], ck[2] + cv[2]))
    with open(os.path.join(HERE, "tq3_tie_counts.txt"), "w") as f:
        f.write("# Oracle counts on the seeded workloads (written by make_tq3_tie_counts.py from the oracle only).\n")
        f.write("# Page \"tq3_core.py\", tq3_quantize: xs = (fwht(s * x / norm)) / scale, bucketized against\n")
        f.write("# TQ3_BOUNDARIES. Columns: workload, vectors, coefficients with |xs - B_j| < 1e-6 for some j,\n")
        f.write("# coefficients with xs exactly 0 (a tie at the boundary 0.0, index 3 by searchsorted's rule).\n")
        for r in rows:
            f.write(" ".join(str(v) for v in r) + "\n")
    print(open(os.path.join(HERE, "tq3_tie_counts.txt")).read())


if __name__ == "__main__":
    main()
