"""Philox4x64-10, written from its published definition (Salmon, Moraes, Dror, Shaw,
"Parallel Random Numbers: As Easy as 1, 2, 3", SC'11, section 3: the Philox S-box built from a
64x64->128-bit multiply, 10 rounds, Weyl key schedule).

The pages give no generator; the build draws W from a counter-based generator so that the C++
library and this oracle produce bit-identical W from the same seed. Philox4x64-10 is chosen
because numpy ships an independent implementation of the same function, which pins this one
(``tests/test_oracle_features.py``).

Test infrastructure only (see ``oracle/__init__``).
"""

MASK64 = (1 << 64) - 1

# Round multipliers and Weyl constants of Philox4x64 (SC'11, table of Philox parameters).
PHILOX_M0 = 0xD2E7470EE14C6C93
PHILOX_M1 = 0xCA5A826395121157
PHILOX_W0 = 0x9E3779B97F4A7C15  # golden ratio
PHILOX_W1 = 0xBB67AE8584CAA73B  # sqrt(3) - 1


def philox4x64_10(counter, key):
    """One Philox4x64-10 block: 4 x uint64 counter, 2 x uint64 key -> 4 x uint64.

    Each round multiplies counter words 0 and 2 by the two multipliers, keeps the 128-bit
    products as (hi, lo), and permutes: (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0). The key is
    bumped by the Weyl constants between rounds.
    """
    c0, c1, c2, c3 = (int(x) & MASK64 for x in counter)
    k0, k1 = (int(x) & MASK64 for x in key)
    for _ in range(10):
        p0 = PHILOX_M0 * c0
        p1 = PHILOX_M1 * c2
        hi0, lo0 = p0 >> 64, p0 & MASK64
        hi1, lo1 = p1 >> 64, p1 & MASK64
        c0, c1, c2, c3 = (hi1 ^ c1 ^ k0), lo1, (hi0 ^ c3 ^ k1), lo0
        k0 = (k0 + PHILOX_W0) & MASK64
        k1 = (k1 + PHILOX_W1) & MASK64
    return c0, c1, c2, c3


def uniform_open01(x):
    """Map a uint64 to a double strictly inside (0, 1): ((x >> 11) + 0.5) * 2^-53.

    The top 53 bits give the mantissa; the half-ulp offset keeps 0 out, so log(u) is finite.
    """
    return ((int(x) >> 11) + 0.5) * (2.0 ** -53)
