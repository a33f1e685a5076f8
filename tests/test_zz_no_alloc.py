"""favor_fwd_static_scratch: the forward entry point for callers that cannot allocate device
memory (code inside another allocator's callback, where a nested cudaMalloc would recurse, or a
process whose device memory a framework's caching allocator has fully reserved). It takes no
workspace and uses the library's own fixed device array.

Checked through the C ABI against favor_fwd, which takes a caller-provided workspace: the two run
the same deterministic kernels, so their outputs must be bit-identical, on two calls in a row
with different inputs (stale contents of the shared array would show). One call is also checked
against the fp64 oracle. This file is collected last on purpose."""

import ctypes

import numpy as np
import pytest

from linear_attention_positive_b200 import api
from linear_attention_positive_b200.inputs import Workload, make_inputs
from oracle import favor
from tests.helpers import features_for, rel_max_err, to_torch

pytestmark = pytest.mark.gpu


def _case(seed, device, B=2, H=4, L=1500):
    w = Workload("t", B, H, L, 64, 256, False, "bf16", False, 2, seed)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    dev = [to_torch(x[k], "bf16", device) for k in "QKV"] + [to_torch(Wr, "bf16", device)]
    return x, W64, dev


def test_static_scratch_matches_workspace_entry_point(cuda_device):
    for seed in (101, 202):
        x, W64, (Q, K, V, W) = _case(seed, cuda_device)
        ref = api.fwd(Q, K, V, W).cpu().numpy()
        out = api.fwd_static_scratch(Q, K, V, W)
        assert api.sync_status() == api.FAVOR_OK
        out = out.cpu().numpy()
        assert np.isfinite(out).all()
        assert np.array_equal(out, ref), "static-scratch output differs from favor_fwd's"
        if seed == 101:
            X = {k: x[k].astype(np.float64) for k in "QKV"}
            assert rel_max_err(out, favor.fwd(X["Q"], X["K"], X["V"], W64)) <= 2e-2


def test_static_scratch_rejects_shapes_beyond_its_size(cuda_device):
    import torch

    lib = api.library()
    big = api.make_shape(64, 64, 4096, 64, 256, api.FAVOR_BF16)
    assert api.workspace_size(big) > api.STATIC_SCRATCH_BYTES
    # real (small) device buffers: the call must refuse on the shape alone, before any launch
    buf = torch.zeros(4096, dtype=torch.uint8, device=cuda_device)
    p = ctypes.c_void_p(buf.data_ptr())
    assert lib.favor_fwd_static_scratch(ctypes.byref(big), p, p, p, p, p, None) == api.FAVOR_ERR_WORKSPACE
    f32 = api.make_shape(1, 1, 128, 64, 256, api.FAVOR_F32)
    assert lib.favor_fwd_static_scratch(ctypes.byref(f32), p, p, p, p, p, None) == api.FAVOR_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert api.sync_status() == api.FAVOR_OK
