"""favor_fwd_static_scratch: the forward entry point for callers that cannot allocate device
memory (code inside another allocator's callback, or processes whose device memory a
framework's caching allocator has fully reserved). It takes no workspace and uses the library's
own fixed device array; here it is checked through the C ABI against favor_fwd, which takes a
caller-provided workspace, on two calls in a row with different inputs (so stale contents of the
shared array would show). This file is collected last on purpose."""

import ctypes

import numpy as np
import pytest

from linear_attention_positive_b200 import api
from linear_attention_positive_b200.inputs import Workload, make_inputs
from tests.helpers import features_for, rel_max_err, to_torch

pytestmark = pytest.mark.gpu


def _inputs(seed, device, B=2, H=4, L=1500):
    w = Workload("t", B, H, L, 64, 256, False, "bf16", False, 2, seed)
    x = make_inputs(w)
    Wr, _ = features_for(w.w_seed, w.m, w.d, "bf16")
    return [to_torch(x[k], "bf16", device) for k in "QKV"] + [to_torch(Wr, "bf16", device)]


def test_static_scratch_matches_workspace_entry_point(cuda_device):
    for seed in (101, 202):
        Q, K, V, W = _inputs(seed, cuda_device)
        ref = api.fwd(Q, K, V, W).double().cpu().numpy()
        out = api.fwd_static_scratch(Q, K, V, W)
        assert api.sync_status() == api.FAVOR_OK
        out = out.double().cpu().numpy()
        assert np.isfinite(out).all()
        assert rel_max_err(out, ref) <= 2e-2


def test_static_scratch_rejects_shapes_beyond_its_size(cuda_device):
    lib = api.library()
    big = api.make_shape(64, 64, 4096, 64, 256, api.FAVOR_BF16)
    assert api.workspace_size(big) > api.STATIC_SCRATCH_BYTES
    p = ctypes.c_void_p(256)  # never dereferenced: the size check comes first
    assert lib.favor_fwd_static_scratch(ctypes.byref(big), p, p, p, p, p, None) == api.FAVOR_ERR_WORKSPACE
    f32 = api.make_shape(1, 1, 128, 64, 256, api.FAVOR_F32)
    assert lib.favor_fwd_static_scratch(ctypes.byref(f32), p, p, p, p, p, None) == api.FAVOR_ERR_UNSUPPORTED
