"""GPU parity of the backward (dQ, dK, dV with W fixed) through the C ABI against the fp64
oracle's chain-rule gradients (themselves pinned by finite differences). Tolerances as for the
forward: 1e-4 * RMS on the fp32 path, 2e-2 * RMS with bf16 inputs, per gradient tensor.

The bf16 backward (both masks) runs the split-precision tensor-core passes and needs the context
of a bf16 forward on the same inputs."""

import numpy as np
import pytest

from linear_attention_positive_b200 import api
from linear_attention_positive_b200.inputs import WORKLOADS, Workload, make_inputs
from oracle import favor
from tests.helpers import features_for, rel_max_err, to_torch

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def run_fwd_bwd(w, x, Wr, device, causal):
    T = {k: to_torch(x[k], w.dtype, device) for k in x}
    Wt = to_torch(Wr, w.dtype, device)
    shape = api.make_shape(w.B, w.H, w.L, w.d, w.m, api.FAVOR_BF16 if w.dtype == "bf16" else api.FAVOR_F32)
    import torch

    ctx = torch.empty(max(api.ctx_size(shape, causal), 256), dtype=torch.uint8, device=device)
    out = api.fwd(T["Q"], T["K"], T["V"], Wt, causal=causal, ctx=ctx if w.dtype == "bf16" else None)
    grads = api.bwd(T["Q"], T["K"], T["V"], Wt, out, T["dO"], ctx=ctx, causal=causal)
    assert api.sync_status() == api.FAVOR_OK
    return out.double().cpu().numpy(), [g.double().cpu().numpy() for g in grads]


def oracle_grads(x, W64, causal):
    X = {k: x[k].astype(np.float64) for k in x}
    return favor.bwd(X["Q"], X["K"], X["V"], W64, X["dO"], causal=causal)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,L,d,m", [(1, 2, 150, 64, 64), (1, 1, 97, 128, 32)])
def test_fp32_backward(cuda_device, causal, B, H, L, d, m):
    w = Workload("t", B, H, L, d, m, causal, "f32", True, 4, 60 + L)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, m, d, "f32")
    _, grads = run_fwd_bwd(w, x, Wr, cuda_device, causal)
    for g, r in zip(grads, oracle_grads(x, W64, causal)):
        assert rel_max_err(g, r) <= TOL["f32"]


@pytest.mark.parametrize("causal", [False, True])
def test_bf16_backward_small(cuda_device, causal):
    w = Workload("t", 1, 2, 300, 64, 256, causal, "bf16", True, 5, 77)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    _, grads = run_fwd_bwd(w, x, Wr, cuda_device, causal)
    for g, r in zip(grads, oracle_grads(x, W64, causal)):
        assert rel_max_err(g, r) <= TOL["bf16"]


BIDIR_SHAPES = [
    (1, 1, 1, 64, 256),      # a single token
    (1, 1, 64, 128, 128),    # one 64-token tile, one feature tile
    (2, 3, 1000, 64, 256),   # ragged tail, six heads
    (1, 2, 777, 128, 256),   # d = 128, ragged
    (2, 1, 4100, 64, 128),   # several token splits of the state sums
    (1, 1, 300, 128, 128),
]


@pytest.mark.parametrize("B,H,L,d,m", BIDIR_SHAPES)
def test_bf16_bidirectional_backward_shapes(cuda_device, B, H, L, d, m):
    w = Workload("t", B, H, L, d, m, False, "bf16", True, 5, 30 + L)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, m, d, "bf16")
    _, grads = run_fwd_bwd(w, x, Wr, cuda_device, False)
    for name, g, r in zip(("dQ", "dK", "dV"), grads, oracle_grads(x, W64, False)):
        assert np.isfinite(g).all(), name
        if L == 1 and name != "dV":
            # one key: the output is that key's value whatever the query and the key, so dQ and dK
            # are exactly zero (the reference is rounding noise); bound them by the upstream scale
            assert np.abs(g).max() <= 1e-3 * np.sqrt(np.mean(x["dO"].astype(np.float64) ** 2)), name
            continue
        assert rel_max_err(g, r) <= TOL["bf16"], name


def test_bf16_backward_config5_slice_L1024(cuda_device):
    """Workload 5's shape (B=2, H=8, d=128, m=256) on its first 1024 rows as a separate problem."""
    w = WORKLOADS[5]
    x = {k: v[:, :, :1024].copy() for k, v in make_inputs(w).items()}
    ws = w.with_(L=1024)
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    out, grads = run_fwd_bwd(ws, x, Wr, cuda_device, False)
    X = {k: x[k].astype(np.float64) for k in x}
    assert rel_max_err(out, favor.fwd(X["Q"], X["K"], X["V"], W64)) <= TOL["bf16"]
    for g, r in zip(grads, oracle_grads(x, W64, False)):
        assert rel_max_err(g, r) <= TOL["bf16"]


def test_bf16_backward_config5_full_length(cuda_device):
    """Workload 5 at its full size (B=2, H=8, L=16384, d=128, m=256), in the launch configuration
    the benchmark times: every gradient element of two heads against the fp64 oracle (run on those
    heads alone: heads are independent), and all outputs finite."""
    w = WORKLOADS[5]
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    _, grads = run_fwd_bwd(w, x, Wr, cuda_device, False)
    for g in grads:
        assert np.isfinite(g).all()
    for b, h in ((0, 0), (1, 7)):
        X = {k: x[k][b, h].astype(np.float64) for k in x}
        ref = favor.bwd_bidirectional(X["Q"], X["K"], X["V"], W64, X["dO"])
        for name, g, r in zip(("dQ", "dK", "dV"), grads, ref):
            assert rel_max_err(g[b, h], r) <= TOL["bf16"], (name, b, h)


def test_bf16_bidirectional_backward_needs_context(cuda_device):
    import torch

    w = Workload("t", 1, 1, 128, 64, 256, False, "bf16", True, 5, 3)
    x = make_inputs(w)
    Wr, _ = features_for(w.w_seed, w.m, w.d, "bf16")
    T = {k: to_torch(x[k], "bf16", cuda_device) for k in x}
    Wt = to_torch(Wr, "bf16", cuda_device)
    out = api.fwd(T["Q"], T["K"], T["V"], Wt)
    with pytest.raises(api.FavorError) as ei:
        api.bwd(T["Q"], T["K"], T["V"], Wt, out, T["dO"], ctx=None)
    assert ei.value.status == api.FAVOR_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert api.sync_status() == api.FAVOR_OK


CAUSAL_SHAPES = [
    (1, 1, 1, 64, 256),      # a single token
    (1, 1, 128, 64, 256),    # one chunk
    (1, 2, 300, 64, 256),    # ragged last chunk
    (2, 1, 1000, 64, 128),   # several chunks, one feature tile
    (1, 1, 2200, 64, 256),
]


@pytest.mark.parametrize("B,H,L,d,m", CAUSAL_SHAPES)
def test_bf16_causal_backward_shapes(cuda_device, B, H, L, d, m):
    w = Workload("t", B, H, L, d, m, True, "bf16", True, 3, 40 + L)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, m, d, "bf16")
    _, grads = run_fwd_bwd(w, x, Wr, cuda_device, True)
    for name, g, r in zip(("dQ", "dK", "dV"), grads, oracle_grads(x, W64, True)):
        assert np.isfinite(g).all(), name
        if L == 1 and name != "dV":  # exactly zero, as above
            assert np.abs(g).max() <= 1e-3 * np.sqrt(np.mean(x["dO"].astype(np.float64) ** 2)), name
            continue
        assert rel_max_err(g, r) <= TOL["bf16"], name


def test_bf16_causal_backward_long(cuda_device):
    """Causal gradients over 32 chunks (L = 4096, two heads) against the oracle's prefix / suffix
    recurrences: the between-chunk prefix and suffix state images carry most of the sums."""
    w = Workload("t", 1, 2, 4096, 64, 256, True, "bf16", True, 3, 13)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    _, grads = run_fwd_bwd(w, x, Wr, cuda_device, True)
    for name, g, r in zip(("dQ", "dK", "dV"), grads, oracle_grads(x, W64, True)):
        assert np.isfinite(g).all(), name
        assert rel_max_err(g, r) <= TOL["bf16"], name
