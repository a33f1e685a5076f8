"""The oracle's pins catch planted mistakes (CPU only).

Each case copies one oracle module with a single plausible mistake planted in its source (a
dropped term, a wrong sign, an off-by-one index, a transposed or swapped operand, a wrong stream
or constant), runs the oracle's pins against the copy and requires at least one of them to fail.
A mistake that passed every pin would leave that part of the oracle unchecked. The oracle's own
files are not touched: the copy is the module's source with one edit, executed as a new module
object, and the pin modules see it in place of the original for the duration of one case.

The pins run cheapest first and stop at the first failure; the case records which pin caught the
mistake. ``test_unchanged_copies_pass_the_pins`` runs the same machinery with no edit, so a
failure below is the planted mistake's and not the harness's.
"""

import inspect
import sys
import types

import numpy as np
import pytest

from oracle import favor, features, philox
from tests import test_oracle_favor as PF
from tests import test_oracle_features as PW

# Failures a planted mistake may cause: a wrong value (assertion), or shapes that no longer fit,
# an index out of range, a log of zero, a division by zero.
CAUGHT = (AssertionError, ValueError, IndexError, ZeroDivisionError, FloatingPointError, OverflowError)


def _copy(mod, edit=None, deps=None):
    """Execute ``mod``'s source, with ``edit = (old, new)`` applied once, as a new module.
    ``deps`` maps sibling module names (e.g. 'oracle.philox') to the objects its relative
    imports should bind while the copy is executed."""
    src = inspect.getsource(mod)
    if edit is not None:
        old, new = edit
        assert src.count(old) == 1, f"edit anchor not unique in {mod.__name__}: {old!r}"
        src = src.replace(old, new)
    m = types.ModuleType(mod.__name__)
    m.__package__ = "oracle"
    m.__file__ = mod.__file__
    saved = {}
    try:
        for name, obj in (deps or {}).items():
            saved[name] = sys.modules.get(name)
            sys.modules[name] = obj
        exec(compile(src, mod.__file__, "exec"), m.__dict__)
    finally:
        for name, obj in saved.items():
            if obj is None:
                del sys.modules[name]
            else:
                sys.modules[name] = obj
    return m


def _favor_pins():
    return [
        ("I4 first causal output", PF.test_I4_first_causal_output_is_first_value, ()),
        ("I2 constant values bidir", PF.test_I2_constant_values_pass_through, (False,)),
        ("I2 constant values causal", PF.test_I2_constant_values_pass_through, (True,)),
        ("I3 zero features bidir", PF.test_I3_zero_features_give_key_norm_weighted_means, (False,)),
        ("I3 zero features causal", PF.test_I3_zero_features_give_key_norm_weighted_means, (True,)),
        ("I1 convex bidir", PF.test_I1_convex_combination_of_values, (False,)),
        ("I1 convex causal", PF.test_I1_convex_combination_of_values, (True,)),
        ("brute force bidir", PF.test_linear_form_equals_brute_force_config1, (False,)),
        ("brute force causal", PF.test_linear_form_equals_brute_force_config1, (True,)),
        ("row-sampled forms", PF.test_row_sampled_forms_match_full, ()),
        ("I5 scaling cancels", PF.test_I5_row_scaling_of_query_features_and_global_key_scaling_cancel, ()),
        ("I6/I7 gradient sums", PF.test_I6_query_chain_term_vanishes_and_I7_value_gradients_sum_to_dO, ()),
        ("I8 causal prefix", PF.test_I8_causal_prefix_property, ()),
        ("batched wrappers", PF.test_batched_wrappers_match_per_head, ()),
        ("softmax vs library", PF.test_softmax_reference_matches_library_softmax, ()),
        ("finite differences bidir", PF.test_gradients_match_central_finite_differences, (False,)),
        ("finite differences causal", PF.test_gradients_match_central_finite_differences, (True,)),
        ("MC mean + variance iid", PF.test_mc_mean_and_closed_form_variance_iid, ()),
        ("causal L=512 brute force", PF.test_causal_prefix_slice_equals_brute_force_L512, ()),
        ("error falls with m", PF.test_error_vs_softmax_falls_as_m_grows, ()),
        ("MC mean orthogonal", PF.test_mc_mean_matches_softmax_kernel_4sigma_orthogonal, ()),
        ("orthogonal variance", PF.test_orthogonal_variance_not_above_iid, ()),
        ("decode steps vs brute force", PF.test_decode_steps_reproduce_brute_force_causal_rows, ()),
    ]


def _draw_pins():
    return [
        ("philox vs numpy", PW.test_philox_matches_numpy_library, ((10, 0, 0, 0), (5, 7))),
        ("philox vs numpy, wide words", PW.test_philox_matches_numpy_library,
         ((2**64 - 2, 2**64 - 1, 2**63, 12345), (2**64 - 1, 2**62 + 3))),
        ("uniform closed form", PW.test_uniform_map_closed_form, ()),
        ("bad sizes", PW.test_draw_rejects_bad_sizes, ()),
        ("streams distinct", PW.test_gaussian_streams_are_distinct_and_prefix_stable, ()),
        ("truncated block", PW.test_truncated_last_block_is_prefix_of_full_block, ()),
        ("orthogonal m=100 d=32", PW.test_blocks_orthogonal_to_1e12, (100, 32)),
        ("orthogonal m=256 d=64", PW.test_blocks_orthogonal_to_1e12, (256, 64)),
        ("block gram", PW.test_block_gram_is_diagonal, ()),
        ("gaussian stream", PW.test_gaussian_stream_is_standard_normal, ()),
        ("chi norms", PW.test_row_norms_follow_chi_d, ()),
        ("isotropic rows", PW.test_rows_are_isotropic_gaussian_marginally, ()),
        ("independent blocks", PW.test_blocks_are_independent, ()),
        ("MC mean + variance iid", PF.test_mc_mean_and_closed_form_variance_iid, ()),
        ("MC mean orthogonal", PF.test_mc_mean_matches_softmax_kernel_4sigma_orthogonal, ()),
        ("orthogonal variance", PF.test_orthogonal_variance_not_above_iid, ()),
        ("golden W", PW.test_golden_W_regression, ()),
    ]


def _first_failing(pins):
    for name, fn, args in pins:
        try:
            with np.errstate(all="ignore"):
                fn(*args)
        except CAUGHT:
            return name
    return None


def _install(monkeypatch, fav=None, feat=None, phil=None):
    if fav is not None:
        monkeypatch.setattr(PF, "favor", fav)
    if feat is not None:
        monkeypatch.setattr(PF, "features", feat)
        monkeypatch.setattr(PW, "features", feat)
    if phil is not None:
        monkeypatch.setattr(PW, "philox", phil)


# (old, new) edits of oracle/favor.py, each one plausible slip
FAVOR_MUTANTS = {
    "logit: + |x|^2/2": ("X @ W.T - 0.5 * np.sum", "X @ W.T + 0.5 * np.sum"),
    "logit: |x|^2 without 1/2": ("X @ W.T - 0.5 * np.sum", "X @ W.T - 1.0 * np.sum"),
    "logit: norm term dropped": ("return X @ W.T - 0.5 * np.sum(X * X, axis=1, keepdims=True)",
                                 "return X @ W.T"),
    "phi: exp(-u)": ("np.exp(feature_logits(X, W))", "np.exp(-feature_logits(X, W))"),
    "phi: 1/m for 1/sqrt(m)": ("/ math.sqrt(W.shape[0])", "/ W.shape[0]"),
    "kernel estimate: phi(x).phi(x)": ("[0] @ phi(y[None, :], W)[0]", "[0] @ phi(x[None, :], W)[0]"),
    "bidir: S from query features": ("S = Kp.T @ V                      #", "S = Qp.T @ V                      #"),
    "bidir: z from query features": ("z = Kp.T @ np.ones(K.shape[0])", "z = Qp.T @ np.ones(K.shape[0])"),
    "causal: strict mask (j < i)": (
        "        S += np.outer(Kp[i], V[i])\n        z += Kp[i]\n        den[i] = Qp[i] @ z\n"
        "        out[i] = (Qp[i] @ S) / den[i]\n",
        "        den[i] = Qp[i] @ z\n        out[i] = (Qp[i] @ S) / den[i]\n"
        "        S += np.outer(Kp[i], V[i])\n        z += Kp[i]\n"),
    "causal: z never updated": ("        z += Kp[i]\n        den[i] = Qp[i] @ z\n", "        den[i] = Qp[i] @ z\n"),
    "causal: value index off by one": ("S += np.outer(Kp[i], V[i])\n        z += Kp[i]\n        den[i]",
                                       "S += np.outer(Kp[i], V[i - 1])\n        z += Kp[i]\n        den[i]"),
    "brute: upper-triangular mask": ("A = np.tril(A)", "A = np.triu(A)"),
    "brute: column sums": ("D = A.sum(axis=1)", "D = A.sum(axis=0)"),
    "softmax: K Q^T": ("s = Q @ K.T", "s = K @ Q.T"),
    "batched fwd: b and h swapped": ("out[b, h] = f(Q[b, h], K[b, h], V[b, h], W)",
                                     "out[b, h] = f(Q[h, b], K[h, b], V[h, b], W)"),
    "batched bwd: dK and dV swapped": ("dQ[b, h], dK[b, h], dV[b, h] = f(", "dQ[b, h], dV[b, h], dK[b, h] = f("),
    "bwd bidir: sign of s": ("s = -np.sum(dO * out, axis=1) / den\n    dQp = g @ S.T",
                             "s = np.sum(dO * out, axis=1) / den\n    dQp = g @ S.T"),
    "bwd bidir: h term dropped": ("dKp = V @ G.T + h[None, :]", "dKp = V @ G.T"),
    "bwd bidir: dV from query features": ("dV = Kp @ G\n", "dV = Qp @ G\n"),
    "chain rule: -x rowsum dropped": ("return P @ W - X * P.sum(axis=1, keepdims=True)", "return P @ W"),
    "chain rule: sign of x rowsum": ("return P @ W - X * P.sum", "return P @ W + X * P.sum"),
    "bwd causal: suffix excludes j": (
        "        G += np.outer(Qp[j], g[j])\n        h += Qp[j] * s[j]\n"
        "        dV[j] = G.T @ Kp[j]\n        dKp[j] = G @ V[j] + h\n",
        "        dV[j] = G.T @ Kp[j]\n        dKp[j] = G @ V[j] + h\n"
        "        G += np.outer(Qp[j], g[j])\n        h += Qp[j] * s[j]\n"),
    "bwd causal: prefix excludes i": (
        "        S += np.outer(Kp[i], V[i])\n        z += Kp[i]\n        dQp[i] = S @ g[i] + z * s[i]\n",
        "        dQp[i] = S @ g[i] + z * s[i]\n        S += np.outer(Kp[i], V[i])\n        z += Kp[i]\n"),
    "causal rows: read one key early": ("while nxt < len(rows) and rows[nxt] == i:",
                                        "while nxt < len(rows) and rows[nxt] == i + 1:"),
    "bidir rows: first rows for requested": ("Qp = phi(Q[rows], W)\n    return", "Qp = phi(Q[:len(rows)], W)\n    return"),
    "decode: output before the state update": ("S = S + np.outer(pk, v)\n    z = z + pk\n    return (pq @ S) / (pq @ z), S, z",
                                               "out = (pq @ S) / (pq @ z)\n    S = S + np.outer(pk, v)\n    z = z + pk\n    return out, S, z"),
    "decode: key features for the query": ("pq = phi(q[None, :], W)[0]", "pq = phi(k[None, :], W)[0]"),
    "decode: normaliser left unchanged": ("    z = z + pk\n    return (pq @ S)", "    return (pq @ S)"),
}

FEATURE_MUTANTS = {
    "box-muller: radius sqrt(-log u)": ("r = math.sqrt(-2.0 * math.log(ua))", "r = math.sqrt(-math.log(ua))"),
    "box-muller: angle from the radius uniform": ("theta = two_pi * ub", "theta = two_pi * ua"),
    "stream: output index overlaps": ("idx = 4 * k + 2 * pair + j", "idx = 4 * k + pair + j"),
    "gram-schmidt: subtract raw rows": ("v = v - p * U[j]", "v = v - p * G[j]"),
    "gram-schmidt: no normalisation": ("U[i] = v / nrm", "U[i] = v"),
    "chi norms: d - 1 squares": ("math.sqrt(seq_dot(g[i], g[i]))", "math.sqrt(seq_dot(g[i][1:], g[i][1:]))"),
    "chi norms: squared norm": ("math.sqrt(seq_dot(g[i], g[i]))", "seq_dot(g[i], g[i])"),
    "chi norms: drawn from the direction stream": ("gaussians(seed, block, PURPOSE_NORM, d * d)",
                                                   "gaussians(seed, block, PURPOSE_BLOCK, d * d)"),
    "blocks: every block from stream 0": ("G = gaussians(seed, b, PURPOSE_BLOCK, d * d)",
                                          "G = gaussians(seed, 0, PURPOSE_BLOCK, d * d)"),
    "blocks: every block's norms from stream 0": ("nrm = chi_norms(seed, b, d)", "nrm = chi_norms(seed, 0, d)"),
    "truncation: last rows kept": ("return np.vstack(rows)[:m].copy()", "return np.vstack(rows)[-m:].copy()"),
}

PHILOX_MUTANTS = {
    "round: wrong key word": ("(hi0 ^ c3 ^ k1)", "(hi0 ^ c3 ^ k0)"),
    "round: words 1 and 3 swapped": ("(hi1 ^ c1 ^ k0), lo1, (hi0 ^ c3 ^ k1), lo0",
                                     "(hi1 ^ c3 ^ k0), lo1, (hi0 ^ c1 ^ k1), lo0"),
    "nine rounds": ("for _ in range(10):", "for _ in range(9):"),
    "key schedule: one Weyl constant": ("k1 = (k1 + PHILOX_W1)", "k1 = (k1 + PHILOX_W0)"),
    "multiplier typo": ("PHILOX_M1 = 0xCA5A826395121157", "PHILOX_M1 = 0xCA5A826395121175"),
    "uniform: half-ulp offset dropped": ("((int(x) >> 11) + 0.5)", "((int(x) >> 11) + 0.0)"),
    "uniform: 52-bit shift": ("((int(x) >> 11) + 0.5)", "((int(x) >> 12) + 0.5)"),
}


def test_unchanged_copies_pass_the_pins(monkeypatch):
    phil = _copy(philox)
    feat = _copy(features, deps={"oracle.philox": phil})
    _install(monkeypatch, fav=_copy(favor), feat=feat, phil=phil)
    cheap = {"MC mean orthogonal", "orthogonal variance"}
    pins = [p for p in _favor_pins() + _draw_pins() if p[0] not in cheap]
    assert _first_failing(pins) is None


@pytest.mark.parametrize("name", sorted(FAVOR_MUTANTS))
def test_favor_mistake_is_caught(name, monkeypatch):
    _install(monkeypatch, fav=_copy(favor, FAVOR_MUTANTS[name]))
    caught = _first_failing(_favor_pins())
    assert caught is not None, f"no pin fails with the planted mistake '{name}'"


@pytest.mark.parametrize("name", sorted(FEATURE_MUTANTS))
def test_feature_draw_mistake_is_caught(name, monkeypatch):
    feat = _copy(features, FEATURE_MUTANTS[name])
    _install(monkeypatch, feat=feat)
    caught = _first_failing(_draw_pins())
    assert caught is not None, f"no pin fails with the planted mistake '{name}'"


@pytest.mark.parametrize("name", sorted(PHILOX_MUTANTS))
def test_generator_mistake_is_caught(name, monkeypatch):
    phil = _copy(philox, PHILOX_MUTANTS[name])
    feat = _copy(features, deps={"oracle.philox": phil})
    _install(monkeypatch, feat=feat, phil=phil)
    caught = _first_failing(_draw_pins())
    assert caught is not None, f"no pin fails with the planted mistake '{name}'"
