"""Pins for the oracle's generalised-attention (ReLU) and trigonometric-feature maps (CPU only).

Each map is checked against its kernel's closed form by Monte Carlo over independent Gaussian
feature draws (mean within 4 sigma, and the trigonometric estimator's closed-form variance), the
linear form against brute force on the explicit L x L matrix, and the variance comparison that
motivates positive features: where the softmax kernel is small the positive estimator's relative
variance stays bounded and the trigonometric one's does not. A planted-mistake check at the end
makes each pin earn its place.
"""

import importlib.util
import math
import sys

import numpy as np
import pytest

from oracle import kernels
from linear_attention_positive_b200.inputs import Workload, make_inputs

N_MC = 4000


def _pair(rng, d, dot):
    """Two vectors of norm about 1.2 with the given inner product."""
    x = rng.standard_normal(d)
    x *= 1.2 / np.linalg.norm(x)
    u = rng.standard_normal(d)
    u -= (u @ x) / (x @ x) * x
    u /= np.linalg.norm(u)
    a = dot / (x @ x)
    y = a * x + math.sqrt(max(1.44 - a * a * (x @ x), 0.0)) * u
    return x, y


def test_relu_features_estimate_the_arccos_kernel(K=kernels):
    rng = np.random.default_rng(3)
    d, m = 16, 8
    for dot in (-0.8, 0.2, 1.1):
        x, y = _pair(rng, d, dot)
        est = np.array([K.relu_features(x[None], W)[0] @ K.relu_features(y[None], W)[0]
                        for W in rng.standard_normal((N_MC, m, d))])
        ref = K.arccos1_kernel(x, y)
        assert abs(est.mean() - ref) <= 4 * est.std() / math.sqrt(N_MC), (dot, est.mean(), ref)
    # the kernel at x = y is half the second moment of w.x
    assert abs(K.arccos1_kernel(x, x) - 0.5 * (x @ x)) <= 1e-12


def test_trig_features_estimate_the_softmax_kernel_with_closed_form_variance(K=kernels):
    rng = np.random.default_rng(4)
    d, m = 16, 8
    for dot in (-0.8, 0.3, 1.2):
        x, y = _pair(rng, d, dot)
        est = np.array([K.trig_features(x[None], W)[0] @ K.trig_features(y[None], W)[0]
                        for W in rng.standard_normal((N_MC, m, d))])
        assert abs(est.mean() - math.exp(x @ y)) <= 4 * est.std() / math.sqrt(N_MC), dot
        u2 = float((x - y) @ (x - y))
        var = math.exp(x @ x + y @ y) * (1.0 - math.exp(-u2)) ** 2 / (2.0 * m)
        assert abs(est.var() / var - 1.0) <= 0.15, (dot, est.var(), var)


def test_positive_features_have_bounded_relative_variance_where_the_kernel_is_small():
    """Closed-form variances of one feature (iid w): positive exp(2xy)(exp|x+y|^2 - 1), trigonometric
    exp(|x|^2 + |y|^2)(1 - exp(-|x-y|^2))^2 / 2; divided by the squared kernel exp(2xy), the first
    stays bounded as x.y falls while the second grows without bound."""
    rel_pos, rel_trig = [], []
    for c in (0.0, -0.5, -0.9):
        x = np.array([1.5, 0.0])
        y = 1.5 * np.array([c, math.sqrt(1 - c * c)])
        k2 = math.exp(2 * (x @ y))
        rel_pos.append(k2 * (math.exp((x + y) @ (x + y)) - 1.0) / k2)
        rel_trig.append(math.exp(x @ x + y @ y) * (1.0 - math.exp(-((x - y) @ (x - y)))) ** 2 / 2.0 / k2)
    assert rel_pos == sorted(rel_pos, reverse=True)       # shrinks as the kernel shrinks
    assert rel_trig == sorted(rel_trig)                   # grows as the kernel shrinks
    assert rel_trig[-1] > 10 * rel_pos[-1]


@pytest.mark.parametrize("kind", ["relu", "trig"])
def test_linear_form_equals_brute_force(kind, K=kernels):
    w = Workload("t", 1, 1, 96, 16, 32, False, "f32", False, 1, 21)
    x = {k: v[0, 0].astype(np.float64) for k, v in make_inputs(w).items()}
    W = np.random.default_rng(5).standard_normal((32, 16))
    out = K.fwd_features(x["Q"], x["K"], x["V"], W, kind)
    ref = K.attention_brute_features(x["Q"], x["K"], x["V"], W, kind)
    assert np.abs(out - ref).max() <= 1e-10 * np.abs(ref).max()
    # a constant value column passes through unchanged
    V1 = np.tile(np.arange(16.0), (96, 1))
    assert np.abs(K.fwd_features(x["Q"], x["K"], V1, W, kind) - V1).max() <= 1e-9 * 16
    # the batched wrapper
    xb = {k: v.astype(np.float64) for k, v in make_inputs(w.with_(B=2, H=2)).items()}
    ob = K.fwd(xb["Q"], xb["K"], xb["V"], W, kind)
    assert np.array_equal(ob[1, 0], K.fwd_features(xb["Q"][1, 0], xb["K"][1, 0], xb["V"][1, 0], W, kind))


# ------------------------------------------------------------------ planted mistakes

MUTANTS = {
    "relu: no 1/sqrt(m)": ("np.maximum(X @ W.T, 0.0) / math.sqrt(W.shape[0])", "np.maximum(X @ W.T, 0.0)"),
    "relu: absolute value": ("np.maximum(X @ W.T, 0.0)", "np.abs(X @ W.T)"),
    "trig: norm factor exp(|x|^2)": ("np.exp(0.5 * np.sum(X * X", "np.exp(1.0 * np.sum(X * X"),
    "trig: cos only": ("np.concatenate([np.sin(P), np.cos(P)], axis=1)", "np.concatenate([np.cos(P), np.cos(P)], axis=1)"),
    "arccos: (pi + t)": ("(math.pi - t) * c", "(math.pi + t) * c"),
    "fwd: z from query features": ("z = Kp.T @ np.ones(K.shape[0])", "z = Qp.T @ np.ones(K.shape[0])"),
    "brute: column sums": ("A.sum(axis=1)[:, None]", "A.sum(axis=0)[:, None]"),
    "batched: b and h swapped": ("out[b, h] = fwd_features(Q[b, h], K[b, h], V[b, h], W, kind)",
                                 "out[b, h] = fwd_features(Q[h, b], K[h, b], V[h, b], W, kind)"),
}


def _mutant(edit):
    src = open(kernels.__file__).read()
    assert edit[0] in src, edit[0]
    spec = importlib.util.spec_from_loader("oracle_kernels_mutant", loader=None)
    mod = importlib.util.module_from_spec(spec)
    exec(compile(src.replace(edit[0], edit[1]), "oracle_kernels_mutant", "exec"), mod.__dict__)
    return mod


def _pins(K):
    return [
        lambda: test_relu_features_estimate_the_arccos_kernel(K),
        lambda: test_trig_features_estimate_the_softmax_kernel_with_closed_form_variance(K),
        lambda: test_linear_form_equals_brute_force("relu", K),
        lambda: test_linear_form_equals_brute_force("trig", K),
    ]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    K = _mutant(MUTANTS[name])
    failed = False
    for pin in _pins(K):
        try:
            with np.errstate(all="ignore"):
                pin()
        except (AssertionError, ValueError, IndexError, FloatingPointError):
            failed = True
            break
    assert failed, f"no pin fails with the planted mistake '{name}'"
