"""Pins for the oracle's generator and feature draw (CPU only).

The generator is pinned to numpy's own Philox4x64-10 (an independent library implementation);
the Gaussian stream to the normal distribution (KS test, moments); W to the properties the pages
claim for positive orthogonal random features (orthogonal blocks, isotropic rows, chi(d) norms).
"""

import math
import os

import numpy as np
import pytest
from scipy import stats

from oracle import features, philox

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("counter,key", [
    ((0, 0, 0, 0), (0, 0)),
    ((10, 0, 0, 0), (5, 7)),
    ((3, 1, 0, 0), (2, 0)),
    ((2**64 - 2, 2**64 - 1, 2**63, 12345), (2**64 - 1, 2**62 + 3)),
    ((123456789, 4, 1, 0), (0xDEADBEEFCAFEF00D, 0)),
])
def test_philox_matches_numpy_library(counter, key):
    # numpy's Philox bumps the 256-bit counter before each block, so the block for counter c
    # is its first output when started at c - 1.
    c = sum(int(w) << (64 * i) for i, w in enumerate(counter))
    c_prev = (c - 1) % (1 << 256)
    prev_words = [(c_prev >> (64 * i)) & philox.MASK64 for i in range(4)]
    bg = np.random.Philox(counter=np.array(prev_words, dtype=np.uint64),
                          key=np.array(key, dtype=np.uint64))
    expected = [int(x) for x in bg.random_raw(4)]
    assert list(philox.philox4x64_10(counter, key)) == expected


def test_uniform_map_closed_form():
    assert philox.uniform_open01(0) == 2.0 ** -54
    assert philox.uniform_open01(2**64 - 1) == 1.0 - 2.0 ** -54
    assert philox.uniform_open01(1 << 63) == 0.5 + 2.0 ** -54
    assert 0.0 < philox.uniform_open01(2**11 - 1) < 1e-15


def test_gaussian_stream_is_standard_normal():
    g = np.concatenate([features.gaussians(seed, b, 0, 5000) for seed, b in ((1, 0), (2, 3))])
    assert stats.kstest(g, "norm").pvalue > 1e-3
    n = g.size
    assert abs(g.mean()) < 4.0 / math.sqrt(n)
    assert abs(g.var() - 1.0) < 4.0 * math.sqrt(2.0 / n)
    # pairs (cos, sin) share a radius but must be uncorrelated
    assert abs(np.corrcoef(g[0::2], g[1::2])[0, 1]) < 4.0 / math.sqrt(n / 2)


def test_gaussian_streams_are_distinct_and_prefix_stable():
    a = features.gaussians(7, 0, 0, 64)
    assert np.array_equal(features.gaussians(7, 0, 0, 10), a[:10])
    assert not np.array_equal(a, features.gaussians(7, 1, 0, 64))
    assert not np.array_equal(a, features.gaussians(7, 0, 1, 64))
    assert not np.array_equal(a, features.gaussians(8, 0, 0, 64))


@pytest.mark.parametrize("m,d", [(64, 64), (256, 64), (256, 128), (100, 32), (16, 64)])
def test_blocks_orthogonal_to_1e12(m, d):
    W = features.draw_W(3, m, d)
    assert W.shape == (m, d)
    for U in features.block_directions(W, d):
        err = np.abs(U @ U.T - np.eye(U.shape[0])).max()
        assert err <= 1e-12, err


def test_block_gram_is_diagonal():
    W = features.draw_W(9, 256, 64)
    for s in range(0, 256, 64):
        blk = W[s:s + 64]
        gram = blk @ blk.T
        off = gram - np.diag(np.diag(gram))
        assert np.abs(off).max() <= 1e-12 * np.abs(np.diag(gram)).max()


def test_truncated_last_block_is_prefix_of_full_block():
    W_full = features.draw_W(5, 128, 64)
    W_part = features.draw_W(5, 100, 64)
    assert np.array_equal(W_part, W_full[:100])


def test_row_norms_follow_chi_d():
    d = 64
    norms = np.concatenate([np.linalg.norm(features.draw_W(s, 128, d), axis=1) for s in range(8)])
    assert stats.kstest(norms, stats.chi(d).cdf).pvalue > 1e-3


def test_rows_are_isotropic_gaussian_marginally():
    # Each row of a block-orthogonal W is marginally N(0, I_d): E[w w^T] = I.
    d = 16
    rows = np.vstack([features.draw_W(s, 32, d) for s in range(300)])
    cov = rows.T @ rows / rows.shape[0]
    n = rows.shape[0]
    assert np.abs(cov - np.eye(d)).max() < 6.0 * math.sqrt(2.0 / n)
    assert np.abs(rows.mean(axis=0)).max() < 5.0 / math.sqrt(n)
    # a single coordinate is standard normal
    assert stats.kstest(rows[:, 3], "norm").pvalue > 1e-3


def test_golden_W_regression():
    """tests/golden/W_seed1_m64_d64.txt was written by tests/golden/make_golden.py (oracle only)."""
    path = os.path.join(GOLDEN, "W_seed1_m64_d64.txt")
    vals = []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                vals.extend(float.fromhex(t) for t in line.split())
    ref = np.array(vals).reshape(64, 64)
    assert np.array_equal(features.draw_W(1, 64, 64), ref)


def test_draw_rejects_bad_sizes():
    with pytest.raises(ValueError):
        features.draw_W(1, 0, 64)


def test_blocks_are_independent():
    # Separate d-row blocks come from separate Gaussian streams. For independent Haar-distributed
    # orthonormal blocks U0, U1 the product U0 U1^T is Haar on O(d), whose trace has mean 0 and
    # variance 1; blocks that shared their directions would give trace d. The chi norms of row i
    # in block 0 and row i in block 1 are independent draws (Pearson correlation ~ 0).
    d, n = 16, 300
    tr = np.empty(n)
    n0, n1 = [], []
    for s in range(n):
        W = features.draw_W(500 + s, 2 * d, d)
        U0, U1 = features.block_directions(W, d)
        tr[s] = np.trace(U0 @ U1.T)
        n0.append(np.linalg.norm(W[:d], axis=1))
        n1.append(np.linalg.norm(W[d:], axis=1))
    assert abs(tr.mean()) < 4.0 / math.sqrt(n)
    t2 = tr * tr
    assert abs(t2.mean() - 1.0) < 4.0 * t2.std(ddof=1) / math.sqrt(n)
    n0, n1 = np.concatenate(n0), np.concatenate(n1)
    assert abs(np.corrcoef(n0, n1)[0, 1]) < 4.0 / math.sqrt(n0.size)
