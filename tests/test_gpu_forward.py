"""GPU parity of the forward pass through the C ABI against the fp64 oracle.

Tolerances (max |err| over all elements, relative to RMS of the oracle output): 1e-4 on the fp32
path, 2e-2 with bf16 inputs and fp32 accumulation.
"""

import numpy as np
import pytest

from linear_attention_positive_b200 import api
from linear_attention_positive_b200.inputs import WORKLOADS, Workload, make_inputs, round_to_bf16
from oracle import favor
from tests.helpers import features_for, rel_max_err, to_torch

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def run_fwd(w, x, Wr, device, causal, opts=None):
    Q, K, V = (to_torch(x[k], w.dtype, device) for k in "QKV")
    Wt = to_torch(Wr, w.dtype, device)
    out = api.fwd(Q, K, V, Wt, causal=causal, opts=opts)
    assert api.sync_status() == api.FAVOR_OK
    return out.double().cpu().numpy()


def oracle_fwd(x, W64, causal):
    X = {k: x[k].astype(np.float64) for k in "QKV"}
    return favor.fwd(X["Q"], X["K"], X["V"], W64, causal=causal)


def test_fp32_config1_against_brute_force(cuda_device):
    w = WORKLOADS[1]
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "f32")
    out = run_fwd(w, x, Wr, cuda_device, causal=False)
    ref, _ = favor.attention_brute(*(x[k][0, 0].astype(np.float64) for k in "QKV"), W64)
    assert rel_max_err(out[0, 0], ref) <= TOL["f32"]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,L,d,m", [(1, 2, 200, 64, 64), (2, 1, 131, 128, 96), (1, 1, 1, 64, 16)])
def test_fp32_shapes(cuda_device, causal, B, H, L, d, m):
    w = Workload("t", B, H, L, d, m, causal, "f32", False, 7, 70)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, m, d, "f32")
    out = run_fwd(w, x, Wr, cuda_device, causal)
    assert rel_max_err(out, oracle_fwd(x, W64, causal)) <= TOL["f32"]


BF16_SHAPES = [
    (1, 1, 128, 64, 256),    # one tile
    (1, 2, 1000, 64, 256),   # several tiles, ragged tail
    (1, 1, 2200, 64, 256),   # more than one split of tiles
    (2, 1, 777, 128, 256),   # d = 128, two passes over the value halves
    (1, 1, 300, 64, 128),    # one feature half
    (1, 3, 129, 64, 256),    # one row into the second tile
    (1, 1, 1, 64, 256),      # a single token
    (1, 1, 64, 128, 128),
]


@pytest.mark.parametrize("B,H,L,d,m", BF16_SHAPES)
def test_bf16_bidirectional_shapes(cuda_device, B, H, L, d, m):
    w = Workload("t", B, H, L, d, m, False, "bf16", False, 2, 20 + L)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, m, d, "bf16")
    out = run_fwd(w, x, Wr, cuda_device, causal=False)
    assert np.isfinite(out).all()
    assert rel_max_err(out, oracle_fwd(x, W64, False)) <= TOL["bf16"]


@pytest.mark.parametrize("d,m", [(64, 256), (128, 256), (128, 128), (64, 128)])
def test_bf16_bidirectional_ranges_crossing_heads(cuda_device, d, m):
    # 24 heads x 13 tiles = 312 tiles over at most 148 persistent CTAs (3 tiles each): most CTA
    # ranges end inside one head and start inside the next.
    w = Workload("t", 2, 12, 1600, d, m, False, "bf16", False, 2, 55)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, m, d, "bf16")
    out = run_fwd(w, x, Wr, cuda_device, causal=False)
    assert rel_max_err(out, oracle_fwd(x, W64, False)) <= TOL["bf16"]


def test_bf16_many_short_heads(cuda_device):
    # 300 one-tile heads over at most 148 CTAs: every CTA range holds several whole heads.
    w = Workload("t", 3, 100, 60, 64, 256, False, "bf16", False, 2, 56)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    out = run_fwd(w, x, Wr, cuda_device, causal=False)
    assert rel_max_err(out, oracle_fwd(x, W64, False)) <= TOL["bf16"]


def test_bf16_key_stabiliser_raised_within_a_range(cuda_device):
    # 300 key tiles of 64 tokens over at most 148 persistent CTAs (3 consecutive tiles each). Keys
    # k_j = a w_0 + noise with a = 0.2, 0.6, 1.0 on tiles 0, 1, 2 (mod 3): u_0 climbs by ~15 nats
    # inside every CTA's range, so the per-feature stabiliser set on a range's first tile is raised
    # on the next ones and the accumulated state rescaled. Queries lean towards w_0 as well, so
    # the feature that dominates the keys is not one the queries discount.
    w = Workload("t", 1, 1, 64 * 300, 64, 256, False, "bf16", False, 2, 58)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    w0 = W64[0].astype(np.float32)[None, :]
    a = np.array([0.2, 0.6, 1.0], dtype=np.float32)[(np.arange(w.L) // 64) % 3][:, None]
    x["K"][0, 0] = a * w0 + 0.3 * x["K"][0, 0]
    x["Q"][0, 0] = 0.1 * w0 + x["Q"][0, 0]
    x["K"] = round_to_bf16(x["K"])
    x["Q"] = round_to_bf16(x["Q"])
    K64 = x["K"][0, 0].astype(np.float64)
    u0 = K64 @ W64[0] - 0.5 * (K64 ** 2).sum(1)
    assert u0[128:192].max() - u0[:64].max() > 12.0  # nats: more than the 2^15 headroom of fp16
    out = run_fwd(w, x, Wr, cuda_device, causal=False)
    assert np.isfinite(out).all()
    assert rel_max_err(out, oracle_fwd(x, W64, False)) <= TOL["bf16"]


def test_bf16_key_stabiliser_raised_inside_a_wide_tile(cuda_device):
    # d = 64 runs on 128-token key tiles read in 32-token chunks. Keys k_j = a_q w_0 + noise with a_q
    # rising from 0.2 to 1.0 over 12 consecutive 32-token chunks (three tiles) and then falling back:
    # inside a CTA's range the stabiliser set on its first tile is raised in the middle of later
    # tiles, so chunks already stored with the old value are rescaled along with the state.
    L = 128 * 600
    w = Workload("t", 1, 1, L, 64, 256, False, "bf16", False, 2, 59)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    w0 = W64[0].astype(np.float32)[None, :]
    q = (np.arange(L) // 32) % 12
    a = (0.2 + 0.8 * q / 11.0).astype(np.float32)[:, None]
    x["K"][0, 0] = a * w0 + 0.3 * x["K"][0, 0]
    x["Q"][0, 0] = 0.1 * w0 + x["Q"][0, 0]
    x["K"] = round_to_bf16(x["K"])
    x["Q"] = round_to_bf16(x["Q"])
    K64 = x["K"][0, 0].astype(np.float64)
    u0 = K64 @ W64[0] - 0.5 * (K64 ** 2).sum(1)
    assert u0[352:384].max() - u0[:32].max() > 12.0  # nats: more than the 2^15 headroom of fp16
    out = run_fwd(w, x, Wr, cuda_device, causal=False)
    assert np.isfinite(out).all()
    assert rel_max_err(out, oracle_fwd(x, W64, False)) <= TOL["bf16"]


def test_bf16_value_tiles_of_very_different_magnitude(cuda_device):
    # One key tile's values near 3e4 and another's near 1e-5: the per-tile power-of-two scaling
    # of V keeps both inside fp16's normal range.
    w = Workload("t", 1, 1, 640, 64, 256, False, "bf16", False, 2, 57)
    x = make_inputs(w)
    x["V"][0, 0, :128] *= 3.0e4
    x["V"][0, 0, 256:384] *= 1.0e-5
    x["V"] = round_to_bf16(x["V"])
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    out = run_fwd(w, x, Wr, cuda_device, causal=False)
    assert np.isfinite(out).all()
    assert rel_max_err(out, oracle_fwd(x, W64, False)) <= TOL["bf16"]
    # the small tile alone: the same keys with every other value zeroed
    x2 = dict(x)
    x2["V"] = np.zeros_like(x["V"])
    x2["V"][0, 0, 256:384] = x["V"][0, 0, 256:384]
    out2 = run_fwd(w, x2, Wr, cuda_device, causal=False)
    assert rel_max_err(out2, oracle_fwd(x2, W64, False)) <= TOL["bf16"]


@pytest.mark.parametrize("d", [64, 128])
def test_bf16_bidirectional_values_beyond_range_are_reported(cuda_device, d):
    """The bidirectional key kernels scale each key tile's values by at most 2^-7 into fp16
    operands: values near 2^22 still give valid outputs, an entry of 2^23 (or a non-finite one) is
    reported as FAVOR_ERR_UNSUPPORTED instead of a silently wrong output."""
    w = Workload("t", 1, 1, 640, d, 256, False, "bf16", False, 2, 61)
    x = make_inputs(w)
    x["V"][0, 0, 128:256] *= 1.0e6
    x["V"] = round_to_bf16(x["V"])
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    out = run_fwd(w, x, Wr, cuda_device, causal=False)
    assert rel_max_err(out, oracle_fwd(x, W64, False)) <= TOL["bf16"]
    Q, K = (to_torch(x[k], w.dtype, cuda_device) for k in "QK")
    for bad in (np.inf, 2.0 ** 23):
        V = x["V"].copy()
        V[0, 0, 300, 3] = bad
        api.fwd(Q, K, to_torch(V, w.dtype, cuda_device), to_torch(Wr, w.dtype, cuda_device))
        assert api.sync_status() == api.FAVOR_ERR_UNSUPPORTED, bad
        assert api.sync_status() == api.FAVOR_OK


@pytest.mark.parametrize("split_tiles", [1, 3, 64])
def test_bf16_split_choice_does_not_change_result(cuda_device, split_tiles):
    w = Workload("t", 1, 2, 1500, 64, 256, False, "bf16", False, 2, 33)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    out = run_fwd(w, x, Wr, cuda_device, False, opts=api.make_opts(split_tiles=split_tiles))
    assert rel_max_err(out, oracle_fwd(x, W64, False)) <= TOL["bf16"]


def test_bf16_stabilisers_handle_large_logits(cuda_device):
    # Keys and queries large enough that unstabilised fp32 exponentials would overflow
    # (|w.k| up to ~150): the per-row and per-head maxima keep every feature in range.
    w = Workload("t", 1, 1, 512, 64, 256, False, "bf16", False, 2, 44)
    x = make_inputs(w)
    x["K"][0, 0, 100] *= 12.0
    x["Q"][0, 0, 7] *= 12.0
    # keep the inputs exactly representable in bf16, so kernel and oracle read the same values
    x["K"] = round_to_bf16(x["K"])
    x["Q"] = round_to_bf16(x["Q"])
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    out = run_fwd(w, x, Wr, cuda_device, False)
    assert np.isfinite(out).all()
    assert rel_max_err(out, oracle_fwd(x, W64, False)) <= TOL["bf16"]


def test_bf16_config2_full_size_sampled_rows(cuda_device):
    """Full bidirectional workload (B=8, H=8, L=4096, d=64, m=256) in the benchmark's launch
    configuration; every head is checked on 48 sampled rows (first, last, random)."""
    w = WORKLOADS[2]
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    out = run_fwd(w, x, Wr, cuda_device, False)
    assert np.isfinite(out).all()
    rng = np.random.default_rng(0)
    errs, refs = [], []
    for b in range(w.B):
        for h in range(w.H):
            rows = np.unique(np.concatenate([[0, w.L - 1], rng.integers(0, w.L, 46)]))
            X = {k: x[k][b, h].astype(np.float64) for k in "QKV"}
            ref = favor.fwd_bidirectional_rows(X["Q"], X["K"], X["V"], W64, rows)
            errs.append(np.abs(out[b, h, rows] - ref).max())
            refs.append(ref)
    rms = np.sqrt(np.mean(np.concatenate(refs) ** 2))
    assert max(errs) / rms <= TOL["bf16"]


CAUSAL_SHAPES = [
    (1, 1, 128, 64, 256),
    (1, 2, 1000, 64, 256),
    (1, 1, 2200, 64, 256),   # three segments of 8 tiles
    (2, 1, 700, 64, 128),
    (1, 1, 1, 64, 256),
    (1, 1, 520, 64, 256),    # just past the exact prefix
]


@pytest.mark.parametrize("B,H,L,d,m", CAUSAL_SHAPES)
def test_bf16_causal_shapes(cuda_device, B, H, L, d, m):
    w = Workload("t", B, H, L, d, m, True, "bf16", False, 3, 30 + L)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, m, d, "bf16")
    out = run_fwd(w, x, Wr, cuda_device, causal=True)
    assert np.isfinite(out).all()
    assert rel_max_err(out, oracle_fwd(x, W64, True)) <= TOL["bf16"]


@pytest.mark.parametrize("split_tiles", [1, 2, 5])
def test_bf16_causal_segment_choice(cuda_device, split_tiles):
    w = Workload("t", 1, 2, 1700, 64, 256, True, "bf16", False, 3, 37)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    out = run_fwd(w, x, Wr, cuda_device, True, opts=api.make_opts(split_tiles=split_tiles))
    assert rel_max_err(out, oracle_fwd(x, W64, True)) <= TOL["bf16"]


def test_bf16_causal_config3_prefix_slice_against_brute_force(cuda_device):
    """Full causal workload (B=4, H=8, L=8192); the first 512 outputs of every head depend only on
    the first 512 inputs and are checked against the explicit masked 512 x 512 matrix."""
    w = WORKLOADS[3]
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    out = run_fwd(w, x, Wr, cuda_device, True)
    assert np.isfinite(out).all()
    errs, refs = [], []
    for b in range(w.B):
        for h in range(w.H):
            X = {k: x[k][b, h, :512].astype(np.float64) for k in "QKV"}
            ref, _ = favor.attention_brute(X["Q"], X["K"], X["V"], W64, causal=True)
            errs.append(np.abs(out[b, h, :512] - ref).max())
            refs.append(ref)
    # every row of every head against the linear-form (prefix-sum) oracle, which also sets RMS(out)
    full_err, sq = [], 0.0
    for b in range(w.B):
        for h in range(w.H):
            ref = favor.fwd_causal(*(x[k][b, h].astype(np.float64) for k in "QKV"), W64)
            full_err.append(np.abs(out[b, h] - ref).max())
            sq += float(np.sum(ref * ref))
    rms = np.sqrt(sq / (w.B * w.H * w.L * w.d))
    assert max(errs) / rms <= TOL["bf16"]
    assert max(full_err) / rms <= TOL["bf16"]


def test_bf16_causal_config4_full_size_all_rows(cuda_device):
    """Long causal workload (B=1, H=16, L=65536, rotated 0.5-scaled inputs) in the benchmark's
    launch configuration, every row of every head against the fp64 prefix-sum oracle. (Rows just
    past the exact fp32 prefix carry the largest errors: there |out| is still ~40x RMS(out).)"""
    w = WORKLOADS[4]
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    out = run_fwd(w, x, Wr, cuda_device, True)
    assert np.isfinite(out).all()
    errs, sq = [], 0.0
    for h in range(w.H):
        ref = favor.fwd_causal(*(x[k][0, h].astype(np.float64) for k in "QKV"), W64)
        errs.append(np.abs(out[0, h] - ref).max())
        sq += float(np.sum(ref * ref))
    rms = np.sqrt(sq / (w.H * w.L * w.d))
    assert max(errs) / rms <= TOL["bf16"]


def test_bf16_causal_values_beyond_fp16_range(cuda_device):
    """The causal bf16 path feeds V to fp16 tensor-core operands; a segment (8 tiles of 128 keys)
    whose values exceed fp16's range is scaled by a power of two for the fp16 operands and the
    output scaled back. Segments of values up to ~1.2e6 and near 1e-4 beside ordinary ones, against
    the fp64 oracle. Entries from 2^23 on (beyond what the key side's per-tile scaling keeps in fp16)
    and non-finite ones are reported as FAVOR_ERR_UNSUPPORTED."""
    w = Workload("t", 1, 2, 3 * 1024 + 200, 64, 256, True, "bf16", False, 3, 41)
    x = make_inputs(w)
    x["V"][0, 0, 1024:2048] *= 3.0e5     # the second segment of head 0
    x["V"][0, 1, 2048:3072] *= 1.0e-4    # the third segment of head 1
    x["V"] = round_to_bf16(x["V"])
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    out = run_fwd(w, x, Wr, cuda_device, causal=True)
    assert np.isfinite(out).all()
    ref = oracle_fwd(x, W64, True)
    for h in range(2):  # each head against its own RMS: head 0's outputs after 1024 are ~1e6 larger
        assert rel_max_err(out[0, h], ref[0, h]) <= TOL["bf16"], h
    # one entry of 7e4 (past fp16's range; its segment shifted by 2^-2): finite, and the rows it
    # dominates within the fp16 operands' relative precision
    V = x["V"].copy()
    V[0, 1, 3100, 7] = 7.0e4
    x2 = dict(x, V=round_to_bf16(V))
    out2 = run_fwd(w, x2, Wr, cuda_device, causal=True)
    ref2 = oracle_fwd(x2, W64, True)
    assert np.isfinite(out2).all()
    assert np.abs(out2[0, 1, 3100:, 7] - ref2[0, 1, 3100:, 7]).max() <= 2e-3 * np.abs(ref2[0, 1, 3100:, 7]).max()
    Q, K = (to_torch(x[k], w.dtype, cuda_device) for k in "QK")
    for bad in (np.inf, 2.0 ** 23):
        V = x["V"].copy()
        V[0, 0, 600, 5] = bad
        api.fwd(Q, K, to_torch(V, w.dtype, cuda_device), to_torch(Wr, w.dtype, cuda_device), causal=True)
        assert api.sync_status() == api.FAVOR_ERR_UNSUPPORTED, bad
        assert api.sync_status() == api.FAVOR_OK  # the status word is cleared by the read


@pytest.mark.parametrize("poly_pct", [25, 50, 100, -1])
@pytest.mark.parametrize("causal,d", [(False, 64), (False, 128), (True, 64)])
def test_bf16_exponentials_on_the_fma_polynomial(cuda_device, poly_pct, causal, d):
    """favor_opts.exp_poly_pct moves a share of the feature exponentials from MUFU ex2 to the
    FMA-pipe polynomial (every kernel instantiates each share; -1 puts all of them on MUFU, 0 --
    the other tests -- takes the kernels' defaults); outputs stay within tolerance."""
    w = Workload("t", 1, 2, 1100, d, 256, causal, "bf16", False, 3 if causal else 2, 90 + abs(poly_pct))
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    out = run_fwd(w, x, Wr, cuda_device, causal, opts=api.make_opts(exp_poly_pct=poly_pct))
    assert np.isfinite(out).all()
    assert rel_max_err(out, oracle_fwd(x, W64, causal)) <= TOL["bf16"]
