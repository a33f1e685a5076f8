"""Random feature draw for FAVOR+: Gaussian streams and the block-orthogonal matrix W.

What the pages fix ("Rethinking Attention with Performers", abstract; summary page
aipaper.jasonlin.tech, "Key contributions" and "Limitations"): the features are random,
positive and *orthogonal*; orthogonality holds inside blocks of at most d rows; the method
assumes isotropic (Gaussian) directions. What they leave open, and the reading taken:

* Blocks: ceil(m/d) independent d x d Gaussian blocks, each orthogonalised on its own; the last
  block is truncated to its first rows when d does not divide m.
* Orthogonalisation: modified Gram-Schmidt over the rows in index order, with one full
  re-orthogonalisation pass ("twice is enough"), so each block is orthonormal to ~1e-15.
* Row norms: each orthonormal row is rescaled by an independent chi(d) draw, sqrt(sum of d fresh
  squared Gaussians), so every row is marginally N(0, I_d) as in the iid estimator.
* Generator: Philox4x64-10 keyed by (seed, 0); Gaussian n of (block b, purpose p) comes from
  counter (n // 4, b, p, 0), outputs (x0, x1) -> Gaussians 4k, 4k+1 and (x2, x3) -> 4k+2, 4k+3,
  by Box-Muller: r = sqrt(-2 log u_a), g = (r cos(2 pi u_b), r sin(2 pi u_b)).
  Purpose 0 = the d x d block, purpose 1 = the chi norms.

Every floating-point step is a single IEEE operation in a fixed order (sequential sums, no fused
multiply-add), so the C++ library reproduces W bit for bit on the same host libm.

Test infrastructure only (see ``oracle/__init__``).
"""

import math

import numpy as np

from .philox import philox4x64_10, uniform_open01

PURPOSE_BLOCK = 0
PURPOSE_NORM = 1


def gaussians(seed, block, purpose, count):
    """``count`` standard normal doubles of stream (seed, block, purpose), in index order."""
    out = np.empty(count, dtype=np.float64)
    two_pi = 2.0 * math.pi
    n_calls = (count + 3) // 4
    for k in range(n_calls):
        x = philox4x64_10((k, block, purpose, 0), (seed, 0))
        for pair in range(2):
            ua = uniform_open01(x[2 * pair])
            ub = uniform_open01(x[2 * pair + 1])
            r = math.sqrt(-2.0 * math.log(ua))
            theta = two_pi * ub
            for j, g in enumerate((r * math.cos(theta), r * math.sin(theta))):
                idx = 4 * k + 2 * pair + j
                if idx < count:
                    out[idx] = g
    return out


def seq_dot(a, b):
    """Sequential left-to-right sum of a[k]*b[k] (products rounded, then added in order)."""
    return float(np.cumsum(np.multiply(a, b))[-1])


def orthonormal_rows(G):
    """Modified Gram-Schmidt with one re-orthogonalisation pass over the rows of G.

    Row i: v = G[i]; twice, for j < i in order: v = v - (U[j] . v) U[j]; then U[i] = v / |v|.
    """
    d = G.shape[0]
    U = np.zeros_like(G)
    for i in range(d):
        v = G[i].copy()
        for _ in range(2):
            for j in range(i):
                p = seq_dot(U[j], v)
                v = v - p * U[j]
        nrm = math.sqrt(seq_dot(v, v))
        U[i] = v / nrm
    return U


def chi_norms(seed, block, d):
    """d independent chi(d) draws: sqrt of the sequential sum of d fresh squared Gaussians."""
    g = gaussians(seed, block, PURPOSE_NORM, d * d).reshape(d, d)
    return np.array([math.sqrt(seq_dot(g[i], g[i])) for i in range(d)], dtype=np.float64)


def draw_W(seed, m, d):
    """Block-orthogonal positive-feature matrix W (m x d, fp64): rows n_i * u_i."""
    if m <= 0 or d <= 0:
        raise ValueError("m and d must be positive")
    rows = []
    n_blocks = (m + d - 1) // d
    for b in range(n_blocks):
        G = gaussians(seed, b, PURPOSE_BLOCK, d * d).reshape(d, d)
        U = orthonormal_rows(G)
        nrm = chi_norms(seed, b, d)
        rows.append(nrm[:, None] * U)
    return np.vstack(rows)[:m].copy()


def draw_W_iid(rng, m, d):
    """Unstructured estimator: m iid N(0, I_d) rows (the non-orthogonal baseline the claims of
    lower variance compare against)."""
    return rng.standard_normal((m, d))


def block_directions(W, d):
    """Unit directions of each d-row block of W (for orthogonality checks)."""
    m = W.shape[0]
    out = []
    for s in range(0, m, d):
        blk = W[s:s + d]
        out.append(blk / np.linalg.norm(blk, axis=1, keepdims=True))
    return out
