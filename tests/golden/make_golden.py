"""Writes the stored expected values under tests/golden/. Calls only the oracle.

    python tests/golden/make_golden.py
"""

import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import features  # noqa: E402


def write_W(seed, m, d):
    W = features.draw_W(seed, m, d)
    path = os.path.join(HERE, f"W_seed{seed}_m{m}_d{d}.txt")
    with open(path, "w") as f:
        f.write(f"# oracle.features.draw_W(seed={seed}, m={m}, d={d}); fp64 hex, row-major, "
                f"{d} values per line\n")
        for row in W:
            f.write(" ".join(float(x).hex() for x in row) + "\n")


if __name__ == "__main__":
    write_W(1, 64, 64)
