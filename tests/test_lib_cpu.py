"""The C-ABI library on the CPU: it loads, exports every entry point include/favor.h declares,
draws W bit for bit like the oracle, sizes workspaces, and rejects bad arguments before any
launch (no compute call runs here)."""

import ctypes
import os
import re

import numpy as np
import pytest

from linear_attention_positive_b200 import api
from oracle import features

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_entry_points():
    with open(os.path.join(ROOT, "include", "favor.h")) as f:
        text = f.read()
    return re.findall(r"FAVOR_API\s+[^;(]*?\b(favor_\w+)\s*\(", text)


def test_exports_match_header(favor_lib):
    declared = header_entry_points()
    assert set(declared) >= set(api.EXPORTS)
    for name in declared:
        assert hasattr(favor_lib, name), name


@pytest.mark.parametrize("seed,m,d", [(1, 64, 64), (2, 256, 64), (5, 256, 128), (3, 100, 32),
                                      (2**64 - 1, 16, 64), (0, 1, 1)])
def test_draw_features_bit_exact_with_oracle(favor_lib, seed, m, d):
    assert np.array_equal(api.draw_features(seed, m, d), features.draw_W(seed, m, d))


def test_draw_features_matches_golden_fixture(favor_lib):
    vals = []
    with open(os.path.join(ROOT, "tests", "golden", "W_seed1_m64_d64.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                vals.extend(float.fromhex(t) for t in line.split())
    assert np.array_equal(api.draw_features(1, 64, 64), np.array(vals).reshape(64, 64))


def test_draw_features_rejects_bad_args(favor_lib):
    buf = (ctypes.c_double * 4)()
    assert favor_lib.favor_draw_features(1, 0, 4, buf) == api.FAVOR_ERR_INVALID_ARG
    assert favor_lib.favor_draw_features(1, 4, 0, buf) == api.FAVOR_ERR_INVALID_ARG
    assert favor_lib.favor_draw_features(1, 4, 4, None) == api.FAVOR_ERR_INVALID_ARG


def test_workspace_and_ctx_sizes(favor_lib):
    ok = api.make_shape(8, 8, 4096, 64, 256, api.FAVOR_BF16)
    assert api.workspace_size(ok) > 8 * 8 * 4096 * 4
    assert api.workspace_size(ok) % 256 == 0
    assert api.ctx_size(ok) >= 64 * (256 * 64 + 256) * 4
    f32 = api.make_shape(1, 1, 256, 64, 64, api.FAVOR_F32)
    assert api.workspace_size(f32) > 0 and api.workspace_size(f32, causal=True, backward=True) > 0
    # invalid or unsupported shapes size to zero
    for bad in (api.make_shape(0, 1, 256, 64, 64, 0), api.make_shape(1, 1, 256, 96, 64, 0),
                api.make_shape(1, 1, 256, 64, 192, api.FAVOR_BF16), api.make_shape(1, 1, 256, 64, 64, 7)):
        assert api.workspace_size(bad) == 0
    assert favor_lib.favor_workspace_size(None, 0, 0, None) == 0
    assert favor_lib.favor_workspace_size(ctypes.byref(ok), 2, 0, None) == 0


def test_fwd_bwd_argument_errors_return_before_launch(favor_lib):
    sh = api.make_shape(1, 1, 256, 64, 64, api.FAVOR_F32)
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    null = None
    fwd = favor_lib.favor_fwd
    assert fwd(None, p, p, p, p, 0, p, null, p, 1 << 20, null, null) == api.FAVOR_ERR_INVALID_ARG
    assert fwd(ctypes.byref(sh), null, p, p, p, 0, p, null, p, 1 << 20, null, null) == api.FAVOR_ERR_INVALID_ARG
    assert fwd(ctypes.byref(sh), p, p, p, p, 3, p, null, p, 1 << 20, null, null) == api.FAVOR_ERR_INVALID_ARG
    unaligned = ctypes.c_void_p(258)
    assert fwd(ctypes.byref(sh), unaligned, p, p, p, 0, p, null, p, 1 << 20, null, null) == api.FAVOR_ERR_INVALID_ARG
    assert fwd(ctypes.byref(sh), p, p, p, p, 0, p, null, null, 1 << 20, null, null) == api.FAVOR_ERR_WORKSPACE
    assert fwd(ctypes.byref(sh), p, p, p, p, 0, p, null, p, 16, null, null) == api.FAVOR_ERR_WORKSPACE
    odd = api.make_shape(1, 1, 256, 96, 64, api.FAVOR_F32)
    assert fwd(ctypes.byref(odd), p, p, p, p, 0, p, null, p, 1 << 20, null, null) == api.FAVOR_ERR_UNSUPPORTED
    bwd = favor_lib.favor_bwd
    assert bwd(ctypes.byref(sh), p, p, p, p, p, null, null, 0, p, p, p, p, 1 << 20, null, null) == api.FAVOR_ERR_INVALID_ARG
    assert bwd(ctypes.byref(sh), p, p, p, p, p, p, null, 0, p, p, p, p, 16, null, null) == api.FAVOR_ERR_WORKSPACE


def test_status_strings(favor_lib):
    for code in range(6):
        assert api.status_string(code).startswith("FAVOR_")
    assert "unknown" in api.status_string(99)


def test_causal_bf16_workspace_covers_its_parts(favor_lib):
    """The causal bf16 forward keeps, in the caller's workspace, the per-key -|k|^2/2 terms, the
    per-segment partial states and their exclusive prefixes ([m, d] + [m] fp32 per segment each)
    and the fp32 features of the exactly recomputed first tokens; shorter segments mean more of
    them. d = 128 has no causal bf16 forward (sized zero, refused before any launch)."""
    B, H, L, d = 1, 16, 65536, 64
    for m in (128, 256):
        sh = api.make_shape(B, H, L, d, m, api.FAVOR_BF16)
        n_seg = B * H * (((L + 127) // 128 + 7) // 8)        # default: 8 tiles of 128 per segment
        parts = (B * H * L * 4                                 # -|k|^2/2
                 + 2 * n_seg * m * (d + 1) * 4                 # partial states and prefixes
                 + 2 * B * H * m * 512 * 4)                    # exact-prefix features
        ws = api.workspace_size(sh, causal=True)
        assert ws >= parts and ws % 256 == 0
        short = api.workspace_size(sh, causal=True, opts=api.make_opts(split_tiles=2))
        assert short > ws
    tall = api.make_shape(1, 1, 1024, 128, 256, api.FAVOR_BF16)
    assert api.workspace_size(tall, causal=True) == 0
    assert api.workspace_size(tall, causal=False) > 0
    p = ctypes.c_void_p(256)
    assert favor_lib.favor_fwd(ctypes.byref(tall), p, p, p, p, 1, p, None, p, 1 << 30, None, None) == \
        api.FAVOR_ERR_UNSUPPORTED


def test_empty_inputs_are_refused_before_launch(favor_lib):
    """Empty tensors (B, H or L zero) are an argument error on every entry point, answered on the
    host before any CUDA call (the library documents L >= 1); their workspace and ctx sizes are 0."""
    p = ctypes.c_void_p(256)
    null = None
    for dims in ((1, 1, 0), (0, 1, 256), (1, 0, 256)):
        for dt in (api.FAVOR_F32, api.FAVOR_BF16):
            sh = api.make_shape(*dims, 64, 128, dt)
            assert api.workspace_size(sh) == 0 and api.workspace_size(sh, True, True) == 0
            assert favor_lib.favor_ctx_size(ctypes.byref(sh), 0) == 0
            for causal in (0, 1):
                assert favor_lib.favor_fwd(ctypes.byref(sh), p, p, p, p, causal, p, null, p, 1 << 20, null,
                                           null) == api.FAVOR_ERR_INVALID_ARG
                assert favor_lib.favor_bwd(ctypes.byref(sh), p, p, p, p, p, p, null, causal, p, p, p, p, 1 << 20,
                                           null, null) == api.FAVOR_ERR_INVALID_ARG
            if dt == api.FAVOR_BF16:
                assert favor_lib.favor_fwd_static_scratch(ctypes.byref(sh), p, p, p, p, p,
                                                          null) == api.FAVOR_ERR_INVALID_ARG


def test_decode_state_size_and_argument_errors(favor_lib):
    """favor_decode_step answers argument errors on the host before any CUDA call."""
    for d, m in ((64, 256), (128, 128), (64, 32)):
        sh = api.make_shape(2, 3, 1, d, m, api.FAVOR_BF16)
        assert favor_lib.favor_decode_state_size(ctypes.byref(sh)) == 2 * 3 * (d * m + 2 * m) * 4
    for d, m in ((96, 256), (64, 48), (64, 512)):
        sh = api.make_shape(1, 1, 1, d, m, api.FAVOR_BF16)
        assert favor_lib.favor_decode_state_size(ctypes.byref(sh)) == 0
    p, null = ctypes.c_void_p(256), None
    ok = api.make_shape(1, 2, 1, 64, 256, api.FAVOR_BF16)
    two = api.make_shape(1, 2, 2, 64, 256, api.FAVOR_BF16)
    assert favor_lib.favor_decode_step(ctypes.byref(two), p, p, p, p, p, p, null) == api.FAVOR_ERR_INVALID_ARG
    assert favor_lib.favor_decode_step(ctypes.byref(ok), null, p, p, p, p, p, null) == api.FAVOR_ERR_INVALID_ARG
    assert favor_lib.favor_decode_step(ctypes.byref(ok), p, p, p, p, ctypes.c_void_p(260), p, null) == \
        api.FAVOR_ERR_INVALID_ARG
    odd = api.make_shape(1, 2, 1, 64, 48, api.FAVOR_BF16)
    assert favor_lib.favor_decode_step(ctypes.byref(odd), p, p, p, p, p, p, null) == api.FAVOR_ERR_UNSUPPORTED


def test_bounded_wait_selftest_rejects_limits_on_the_host(favor_lib):
    assert favor_lib.favor_selftest_bounded_wait(0, None) == api.FAVOR_ERR_INVALID_ARG
    assert favor_lib.favor_selftest_bounded_wait(1000001, None) == api.FAVOR_ERR_INVALID_ARG


def test_bf16_bidirectional_backward_requires_the_forward_context(favor_lib):
    sh = api.make_shape(1, 2, 300, 64, 256, api.FAVOR_BF16)
    ws = api.workspace_size(sh, causal=False, backward=True)
    assert ws > 0 and ws % 256 == 0
    p = ctypes.c_void_p(256)
    assert favor_lib.favor_bwd(ctypes.byref(sh), p, p, p, p, p, p, None, 0, p, p, p, p, ws, None, None) == \
        api.FAVOR_ERR_WORKSPACE


def test_feature_map_workspace_and_refusals(favor_lib):
    """Other feature maps are built for the bf16 bidirectional forward only; elsewhere the sizes are
    zero and the calls refuse before any launch."""
    sh = api.make_shape(1, 2, 1000, 64, 256, api.FAVOR_BF16)
    relu, trig = api.make_opts(feature_map=api.FAVOR_MAP_RELU), api.make_opts(feature_map=api.FAVOR_MAP_TRIG)
    wr, wt = api.workspace_size(sh, opts=relu), api.workspace_size(sh, opts=trig)
    assert 0 < wr < wt and wr % 256 == 0  # the trigonometric map carries 2m features
    assert api.workspace_size(sh, causal=True, opts=relu) == 0
    assert api.workspace_size(sh, backward=True, opts=trig) == 0
    f32 = api.make_shape(1, 2, 1000, 64, 256, api.FAVOR_F32)
    assert api.workspace_size(f32, opts=relu) == 0
    bad = api.make_opts(feature_map=7)
    assert api.workspace_size(sh, opts=bad) == 0
    p = ctypes.c_void_p(256)
    assert favor_lib.favor_fwd(ctypes.byref(sh), p, p, p, p, 1, p, None, p, 1 << 30, ctypes.byref(relu), None) == \
        api.FAVOR_ERR_UNSUPPORTED
    assert favor_lib.favor_fwd(ctypes.byref(sh), p, p, p, p, 0, p, None, p, 1 << 30, ctypes.byref(bad), None) == \
        api.FAVOR_ERR_UNSUPPORTED
    assert favor_lib.favor_bwd(ctypes.byref(sh), p, p, p, p, p, p, p, 0, p, p, p, p, 1 << 30, ctypes.byref(relu),
                               None) == api.FAVOR_ERR_UNSUPPORTED
