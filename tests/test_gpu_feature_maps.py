"""GPU parity of the bidirectional forward with the other feature maps favor_opts.feature_map
selects, through the C ABI, against the fp64 oracle (oracle.kernels): generalised attention with
ReLU features and FAVOR's trigonometric softmax features. Tolerance 2e-2 * RMS(out) (bf16 inputs).

The trigonometric normaliser sums terms of both signs; on unit-variance inputs it crosses zero for
some rows and no finite precision reproduces those outputs, which is the instability the positive
features remove. Its checks use 0.5-scaled inputs (the long-sequence workload's distribution),
where the normaliser stays well away from zero."""

import numpy as np
import pytest

from linear_attention_positive_b200 import api
from linear_attention_positive_b200.inputs import Workload, make_inputs
from oracle import kernels
from tests.helpers import features_for, rel_max_err, to_torch

pytestmark = pytest.mark.gpu

MAPS = {"relu": api.FAVOR_MAP_RELU, "trig": api.FAVOR_MAP_TRIG}
SHAPES = [
    (1, 1, 1, 64, 256),
    (1, 2, 1000, 64, 256),
    (2, 1, 777, 128, 128),
    (1, 1, 4100, 64, 256),
    (2, 3, 130, 128, 256),
]


@pytest.mark.parametrize("kind", ["relu", "trig"])
@pytest.mark.parametrize("B,H,L,d,m", SHAPES)
def test_feature_map_forward_matches_oracle(cuda_device, kind, B, H, L, d, m):
    scale = 0.5 if kind == "trig" else 1.0
    w = Workload("t", B, H, L, d, m, False, "bf16", False, 2, 50 + L, scale=scale)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, m, d, "bf16")
    Q, K, V = (to_torch(x[k], "bf16", cuda_device) for k in "QKV")
    out = api.fwd(Q, K, V, to_torch(Wr, "bf16", cuda_device), opts=api.make_opts(feature_map=MAPS[kind]))
    assert api.sync_status() == api.FAVOR_OK
    out = out.double().cpu().numpy()
    assert np.isfinite(out).all()
    X = {k: x[k].astype(np.float64) for k in "QKV"}
    assert rel_max_err(out, kernels.fwd(X["Q"], X["K"], X["V"], W64, kind)) <= 2e-2


def test_feature_maps_are_refused_where_not_built(cuda_device):
    w = Workload("t", 1, 1, 128, 64, 256, True, "bf16", True, 2, 3)
    x = make_inputs(w)
    Wr, _ = features_for(w.w_seed, w.m, w.d, "bf16")
    T = {k: to_torch(x[k], "bf16", cuda_device) for k in x}
    Wt = to_torch(Wr, "bf16", cuda_device)
    relu = api.make_opts(feature_map=api.FAVOR_MAP_RELU)
    with pytest.raises(api.FavorError) as ei:
        api.fwd(T["Q"], T["K"], T["V"], Wt, causal=True, opts=relu, workspace=api._alloc_bytes(1 << 20, cuda_device))
    assert ei.value.status == api.FAVOR_ERR_UNSUPPORTED
    out = api.fwd(T["Q"], T["K"], T["V"], Wt)
    with pytest.raises(api.FavorError) as ei:
        api.bwd(T["Q"], T["K"], T["V"], Wt, out, T["dO"], opts=relu, workspace=api._alloc_bytes(1 << 20, cuda_device))
    assert ei.value.status == api.FAVOR_ERR_UNSUPPORTED
    import torch

    torch.cuda.synchronize()
    assert api.sync_status() == api.FAVOR_OK
