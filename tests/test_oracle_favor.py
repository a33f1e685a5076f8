"""Pins for the oracle's FAVOR+ forward and backward (CPU only).

Each check compares the oracle with something other than itself: brute force on the explicit
L x L matrix, the closed form exp(x.y) of the kernel it estimates (Monte-Carlo, 4 sigma), the
closed-form variance of the iid estimator, exact softmax attention as m grows, invariants that
hold for any positive feature map, and central finite differences for every gradient.
"""

import math

import numpy as np
import pytest

from oracle import favor, features
from linear_attention_positive_b200.inputs import WORKLOADS, make_inputs


def _head(w, b=0, h=0):
    x = make_inputs(w)
    return {k: v[b, h].astype(np.float64) for k, v in x.items()}


def _rms(a):
    return float(np.sqrt(np.mean(a * a)))


# ------------------------------------------------------------------ (a) brute force, (d) D-hat

@pytest.mark.parametrize("causal", [False, True])
def test_linear_form_equals_brute_force_config1(causal):
    w = WORKLOADS[1]
    x = _head(w)
    W = features.draw_W(w.w_seed, w.m, w.d)
    f = favor.fwd_causal if causal else favor.fwd_bidirectional
    out, den = f(x["Q"], x["K"], x["V"], W, return_den=True)
    ref, rowsum = favor.attention_brute(x["Q"], x["K"], x["V"], W, causal=causal)
    assert np.abs(out - ref).max() <= 1e-12 * _rms(ref)
    # (d): the normaliser D-hat equals the row sums of A'
    assert np.abs(den - rowsum).max() <= 1e-12 * np.abs(rowsum).max()


def test_causal_prefix_slice_equals_brute_force_L512():
    # The first 512 causal outputs depend only on the first 512 inputs (workload 3's slice).
    w = WORKLOADS[3].with_(B=1, H=1, L=512)
    x = _head(w)
    W = features.draw_W(w.w_seed, w.m, w.d)
    out = favor.fwd_causal(x["Q"], x["K"], x["V"], W)
    ref, _ = favor.attention_brute(x["Q"], x["K"], x["V"], W, causal=True)
    assert np.abs(out - ref).max() <= 1e-12 * _rms(ref)


def test_row_sampled_forms_match_full():
    rng = np.random.default_rng(0)
    L, d, m = 300, 16, 32
    Q, K, V = (rng.standard_normal((L, d)) * 0.5 for _ in range(3))
    W = features.draw_W(4, m, d)
    rows = [0, 1, 17, 128, 299]
    full_b = favor.fwd_bidirectional(Q, K, V, W)
    full_c = favor.fwd_causal(Q, K, V, W)
    assert np.allclose(favor.fwd_bidirectional_rows(Q, K, V, W, rows), full_b[rows], rtol=1e-12, atol=0)
    assert np.allclose(favor.fwd_causal_rows(Q, K, V, W, rows), full_c[rows], rtol=1e-12, atol=0)


# ------------------------------------------------------------------ (b) Monte-Carlo, variance

def _mc_estimates(x, y, draws):
    return np.array([favor.kernel_estimate(x, y, W) for W in draws])


def _xy(d):
    rng = np.random.default_rng(42)
    x = rng.standard_normal(d)
    y = rng.standard_normal(d)
    return 0.8 * x / np.linalg.norm(x), 0.6 * y / np.linalg.norm(y)


def test_mc_mean_matches_softmax_kernel_4sigma_orthogonal():
    d = m = 16
    x, y = _xy(d)
    N = 2000
    est = _mc_estimates(x, y, (features.draw_W(s, m, d) for s in range(N)))
    target = math.exp(x @ y)
    assert abs(est.mean() - target) <= 4.0 * est.std(ddof=1) / math.sqrt(N)
    assert (est > 0).all()  # positive features give positive estimates


def test_mc_mean_and_closed_form_variance_iid():
    d = m = 16
    x, y = _xy(d)
    N = 4000
    rng = np.random.default_rng(7)
    est = _mc_estimates(x, y, (features.draw_W_iid(rng, m, d) for _ in range(N)))
    target = math.exp(x @ y)
    assert abs(est.mean() - target) <= 4.0 * est.std(ddof=1) / math.sqrt(N)
    # Var[phi(x).phi(y)] = exp(2 x.y) (exp(|x+y|^2) - 1) / m for iid Gaussian rows
    var_cf = math.exp(2 * x @ y) * (math.exp(np.sum((x + y) ** 2)) - 1.0) / m
    c = est - est.mean()
    s2 = np.mean(c * c)
    se_s2 = math.sqrt(max(np.mean(c ** 4) - s2 ** 2, 0.0) / N)
    assert abs(s2 - var_cf) <= 4.0 * se_s2


def test_orthogonal_variance_not_above_iid():
    d = m = 16
    x, y = _xy(d)
    N = 3000
    rng = np.random.default_rng(11)
    ort = _mc_estimates(x, y, (features.draw_W(1000 + s, m, d) for s in range(N)))
    iid = _mc_estimates(x, y, (features.draw_W_iid(rng, m, d) for _ in range(N)))
    assert ort.var() < iid.var()


def test_error_vs_softmax_falls_as_m_grows():
    rng = np.random.default_rng(3)
    L, d = 64, 16
    errs = []
    for m in (16, 64, 256, 1024):
        e = []
        for s in range(6):
            Q, K, V = (rng.standard_normal((L, d)) * d ** -0.25 for _ in range(3))
            ref = favor.softmax_attention(Q, K, V)
            out = favor.fwd_bidirectional(Q, K, V, features.draw_W(50 + s, m, d))
            e.append(np.abs(out - ref).mean())
        errs.append(np.mean(e))
    assert all(a > b for a, b in zip(errs, errs[1:])), errs


def test_softmax_reference_matches_library_softmax():
    # The exact-softmax reference used above, against scipy's softmax row by row (causal rows
    # see keys 0..i only).
    from scipy.special import softmax

    rng = np.random.default_rng(5)
    L, d = 12, 6
    Q, K, V = (rng.standard_normal((L, d)) for _ in range(3))
    ref_b = softmax(Q @ K.T, axis=1) @ V
    ref_c = np.stack([softmax(K[: i + 1] @ Q[i]) @ V[: i + 1] for i in range(L)])
    assert np.allclose(favor.softmax_attention(Q, K, V), ref_b, rtol=1e-12, atol=1e-14)
    assert np.allclose(favor.softmax_attention(Q, K, V, causal=True), ref_c, rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------ invariants I1-I8

def _small(seed=0, L=40, d=8, m=24, scale=0.7):
    rng = np.random.default_rng(seed)
    Q, K, V, dO = (rng.standard_normal((L, d)) * scale for _ in range(4))
    return Q, K, V, dO, features.draw_W(seed + 1, m, d)


@pytest.mark.parametrize("causal", [False, True])
def test_I1_convex_combination_of_values(causal):
    Q, K, V, _, W = _small(1)
    out = (favor.fwd_causal if causal else favor.fwd_bidirectional)(Q, K, V, W)
    for i in range(len(Q)):
        vs = V[: i + 1] if causal else V
        assert (out[i] >= vs.min(axis=0) - 1e-12).all() and (out[i] <= vs.max(axis=0) + 1e-12).all()


@pytest.mark.parametrize("causal", [False, True])
def test_I2_constant_values_pass_through(causal):
    Q, K, V, _, W = _small(2)
    V[:] = np.array([0.5, -2.0, 3.0, 0.0, 1.0, 7.0, -1.0, 2.5])
    out = (favor.fwd_causal if causal else favor.fwd_bidirectional)(Q, K, V, W)
    assert np.allclose(out, V, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_I3_zero_features_give_key_norm_weighted_means(causal):
    Q, K, V, _, W = _small(3)
    W0 = np.zeros_like(W)
    out = (favor.fwd_causal if causal else favor.fwd_bidirectional)(Q, K, V, W0)
    wts = np.exp(-0.5 * np.sum(K * K, axis=1))
    if causal:
        ref = np.cumsum(wts[:, None] * V, axis=0) / np.cumsum(wts)[:, None]
    else:
        ref = np.broadcast_to((wts @ V) / wts.sum(), V.shape)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-14)
    out0 = favor.fwd_bidirectional(Q, np.zeros_like(K), V, W0)
    assert np.allclose(out0, V.mean(axis=0)[None, :], rtol=1e-12, atol=1e-14)


def test_I4_first_causal_output_is_first_value():
    Q, K, V, _, W = _small(4)
    assert np.allclose(favor.fwd_causal(Q, K, V, W)[0], V[0], rtol=1e-13, atol=0)


def test_I5_row_scaling_of_query_features_and_global_key_scaling_cancel():
    Q, K, V, _, W = _small(5)
    Qp, Kp = favor.phi(Q, W), favor.phi(K, W)

    def fa(Qp, Kp):  # D^-1 (Q'((K')^T V)) from given feature matrices
        return (Qp @ (Kp.T @ V)) / (Qp @ Kp.sum(axis=0))[:, None]

    base = fa(Qp, Kp)
    rng = np.random.default_rng(0)
    scaled = fa(Qp * rng.uniform(1e-3, 1e3, (len(Qp), 1)), Kp * 1e-7)
    assert np.allclose(base, scaled, rtol=1e-10, atol=0)
    assert np.allclose(base, favor.fwd_bidirectional(Q, K, V, W), rtol=1e-12, atol=0)


def test_I6_query_chain_term_vanishes_and_I7_value_gradients_sum_to_dO():
    for causal in (False, True):
        Q, K, V, dO, W = _small(6)
        f = favor.bwd_causal if causal else favor.bwd_bidirectional
        dQ, dK, dV, Qp, dQp, Kp, dKp = f(Q, K, V, W, dO, return_feature_grads=True)
        # I7: sum_j dV_j = sum_i dO_i
        assert np.allclose(dV.sum(axis=0), dO.sum(axis=0), rtol=1e-11, atol=1e-12)
        # I6: sum_r (phi(q_i) * dphi(q_i))_r = num_i.g_i + den_i s_i = 0 for every query
        P = Qp * dQp
        assert np.abs(P.sum(axis=1)).max() <= 1e-12 * np.abs(P).sum(axis=1).max()
        # ... while the key-side sum does not vanish (so dK keeps its -k * rowsum term)
        assert np.abs((Kp * dKp).sum(axis=1)).max() > 1e-3 * np.abs(Kp * dKp).sum(axis=1).max()


def test_I8_causal_prefix_property():
    Q, K, V, _, W = _small(8, L=50)
    full = favor.fwd_causal(Q, K, V, W)
    for ell in (1, 7, 33):
        assert np.allclose(favor.fwd_causal(Q[:ell], K[:ell], V[:ell], W), full[:ell], rtol=1e-13, atol=0)


# ------------------------------------------------------------------ gradients: finite differences

@pytest.mark.parametrize("causal", [False, True])
def test_gradients_match_central_finite_differences(causal):
    rng = np.random.default_rng(21 + causal)
    L, d, m = 7, 4, 10
    Q, K, V, dO = (rng.standard_normal((L, d)) * 0.6 for _ in range(4))
    W = features.draw_W_iid(rng, m, d)

    def loss(Q, K, V):
        return float(np.sum(dO * favor.attention_brute(Q, K, V, W, causal=causal)[0]))

    grads = (favor.bwd_causal if causal else favor.bwd_bidirectional)(Q, K, V, W, dO)
    h = 1e-6
    for idx, X in enumerate((Q, K, V)):
        num = np.zeros_like(X)
        for i in range(L):
            for j in range(d):
                args = [Q.copy(), K.copy(), V.copy()]
                args[idx][i, j] += h
                fp = loss(*args)
                args[idx][i, j] -= 2 * h
                fm = loss(*args)
                num[i, j] = (fp - fm) / (2 * h)
        assert np.abs(grads[idx] - num).max() <= 1e-6 * max(1.0, np.abs(num).max()), idx


def test_batched_wrappers_match_per_head():
    w = WORKLOADS[1].with_(B=2, H=2, L=32, d=8, m=16, backward=True)
    x = {k: v.astype(np.float64) for k, v in make_inputs(w).items()}
    W = features.draw_W(1, w.m, w.d)
    for causal in (False, True):
        out = favor.fwd(x["Q"], x["K"], x["V"], W, causal=causal)
        dQ, dK, dV = favor.bwd(x["Q"], x["K"], x["V"], W, x["dO"], causal=causal)
        f = favor.fwd_causal if causal else favor.fwd_bidirectional
        g = favor.bwd_causal if causal else favor.bwd_bidirectional
        assert np.array_equal(out[1, 0], f(x["Q"][1, 0], x["K"][1, 0], x["V"][1, 0], W))
        ref = g(x["Q"][0, 1], x["K"][0, 1], x["V"][0, 1], W, x["dO"][0, 1])
        assert np.array_equal(dK[0, 1], ref[1])


# ------------------------------------------------------------------ recurrent single-token step

def test_decode_steps_reproduce_brute_force_causal_rows():
    """Running the single-token step from the empty state over a sequence gives, at every step,
    the row of the explicit masked L x L attention; the carried state equals the explicit sums
    (K')^T V and (K')^T 1 over the tokens seen so far."""
    w = WORKLOADS[1].with_(L=48, d=16, m=32)
    x = _head(w)
    W = features.draw_W(3, w.m, w.d)
    ref, _ = favor.attention_brute(x["Q"], x["K"], x["V"], W, causal=True)
    S, z = np.zeros((w.m, w.d)), np.zeros(w.m)
    for t in range(w.L):
        o, S2, z2 = favor.decode_step(S, z, x["Q"][t], x["K"][t], x["V"][t], W)
        assert not np.shares_memory(S2, S)
        S, z = S2, z2
        assert np.abs(o - ref[t]).max() <= 1e-12 * np.abs(ref).max()
    Kp = favor.phi(x["K"], W)
    assert np.allclose(S, Kp.T @ x["V"], rtol=1e-12, atol=0)
    assert np.allclose(z, Kp.sum(axis=0), rtol=1e-12, atol=0)
