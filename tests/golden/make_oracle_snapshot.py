"""Writes tiny_320_oracle_snapshot.npz: oracle outputs of the tiny workload on
a few seeded rows. Calls only the oracle and the seeded input generator."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import h3_inputs as hi  # noqa: E402
from oracle.h3_block import BlockOracle  # noqa: E402


def main():
    inp = hi.make_inputs("tiny_320")
    rows = hi.sample_rows(inp.layout, k=12, k_pad=2)
    lay = inp.layout
    r = BlockOracle(inp.dims, inp.weights).forward(inp.x, lay.tag, lay.tidx, lay.pos, inp.table, rows=rows)
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_320_oracle_snapshot.npz")
    np.savez(out, rows=rows, **{k: r[k] for k in ("h1", "q", "o", "x1", "a", "out")})
    print("wrote", out)


if __name__ == "__main__":
    main()
