"""GPU parity of the backward (dQ, dK, dV with W fixed) through the C ABI against the fp64
oracle's chain-rule gradients (themselves pinned by finite differences). Tolerances as for the
forward: 1e-4 * RMS on the fp32 path, 2e-2 * RMS with bf16 inputs, per gradient tensor."""

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
