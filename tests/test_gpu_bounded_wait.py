"""Failure reporting of the device-side bounded waits, tested without a GPU fault.

Every kernel waits on shared-memory barriers through one bounded wait; a wait that runs out
records FAVOR_ERR_TIMEOUT in the device status word, the kernel frees its tensor memory and
returns. favor_selftest_bounded_wait runs that wait on a barrier nothing arrives on, with a limit
of a few microseconds: the status must come back as FAVOR_ERR_TIMEOUT (once: reading clears it),
and the context must stay usable for a normal call that still matches the oracle."""

import numpy as np
import pytest

from linear_attention_positive_b200 import api
from linear_attention_positive_b200.inputs import Workload, make_inputs
from oracle import favor
from tests.helpers import features_for, rel_max_err, to_torch

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_reports_timeout_and_leaves_context_usable(cuda_device):
    assert api.sync_status() == api.FAVOR_OK
    api.selftest_bounded_wait(5)
    assert api.sync_status() == api.FAVOR_ERR_TIMEOUT
    assert api.sync_status() == api.FAVOR_OK  # cleared by the read

    w = Workload("t", 1, 2, 500, 64, 256, False, "bf16", False, 2, 5)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    Q, K, V = (to_torch(x[k], "bf16", cuda_device) for k in "QKV")
    out = api.fwd(Q, K, V, to_torch(Wr, "bf16", cuda_device))
    assert api.sync_status() == api.FAVOR_OK
    X = {k: x[k].astype(np.float64) for k in "QKV"}
    assert rel_max_err(out.double().cpu().numpy(), favor.fwd(X["Q"], X["K"], X["V"], W64)) <= 2e-2


def test_selftest_rejects_limits_out_of_range(cuda_device):
    lib = api.library()
    assert lib.favor_selftest_bounded_wait(0, None) == api.FAVOR_ERR_INVALID_ARG
    assert lib.favor_selftest_bounded_wait(2000000, None) == api.FAVOR_ERR_INVALID_ARG
