"""GPU parity of the sequence-parallel forward (favor_sp_state / favor_sp_output) through the C
ABI: the tokens of every head are cut into runs as ranks would hold them, the runs' partial states
are summed on the device (the all-reduce of a multi-GPU run), and the outputs of every run are
checked against the fp64 oracle on the whole sequence (2e-2 * RMS, bf16 inputs). This GPU runs the
ranks one after another; the cross-rank exchange itself is tested on CPU with gloo
(tests/test_sequence_parallel_ranks.py)."""

import numpy as np
import pytest

from linear_attention_positive_b200 import api
from linear_attention_positive_b200.inputs import WORKLOADS, Workload, make_inputs
from oracle import favor
from tests.helpers import features_for, rel_max_err, to_torch

pytestmark = pytest.mark.gpu


def run_split(x, Wr, cuts, device):
    import torch

    Wt = to_torch(Wr, "bf16", device)
    T = {k: to_torch(x[k], "bf16", device) for k in "QKV"}
    states = [api.sp_state(T["K"][:, :, a:b].contiguous(), T["V"][:, :, a:b].contiguous(), Wt)
              for a, b in zip(cuts[:-1], cuts[1:])]
    total = torch.stack(states).sum(dim=0)
    outs = [api.sp_output(T["Q"][:, :, a:b].contiguous(), Wt, total) for a, b in zip(cuts[:-1], cuts[1:])]
    assert api.sync_status() == api.FAVOR_OK
    return torch.cat(outs, dim=2).double().cpu().numpy(), total


@pytest.mark.parametrize("B,H,L,d,m,cuts", [
    (1, 2, 1000, 64, 256, [0, 1000]),
    (1, 2, 1000, 64, 256, [0, 300, 1000]),
    (2, 1, 777, 128, 128, [0, 100, 101, 777]),
    (1, 3, 2500, 64, 256, [0, 640, 1280, 1920, 2500]),
])
def test_runs_summed_match_the_whole_sequence(cuda_device, B, H, L, d, m, cuts):
    w = Workload("t", B, H, L, d, m, False, "bf16", False, 2, 60 + L)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, m, d, "bf16")
    out, total = run_split(x, Wr, cuts, cuda_device)
    X = {k: x[k].astype(np.float64) for k in "QKV"}
    assert np.isfinite(out).all()
    assert rel_max_err(out, favor.fwd(X["Q"], X["K"], X["V"], W64)) <= 2e-2
    # the total state against its definition: exp(-c_r) sqrt(m) (K')^T [V | 1]
    c = 0.5 * np.sum(W64 * W64, axis=1) - 40.0
    st = total.double().cpu().numpy().reshape(B * H, m, d + 64)
    Kp = favor.phi(X["K"][0, 0], W64) * np.sqrt(m) * np.exp(-c)[None, :]
    ref = np.concatenate([Kp.T @ X["V"][0, 0], Kp.sum(axis=0)[:, None]], axis=1)
    assert np.abs(st[0, :, :d + 1] - ref).max() <= 1e-4 * np.abs(ref).max()
    assert np.abs(st[:, :, d + 1:]).max() == 0.0


def test_workload2_in_eight_runs(cuda_device):
    """Workload 2 (B=8, H=8, L=4096) cut into eight runs of 512 tokens, as eight ranks would hold
    it; 48 sampled rows of every head against the oracle."""
    w = WORKLOADS[2]
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    out, _ = run_split(x, Wr, list(range(0, 4097, 512)), cuda_device)
    rng = np.random.default_rng(1)
    errs, refs = [], []
    for b in range(w.B):
        for h in range(w.H):
            rows = np.unique(np.concatenate([[0, w.L - 1], rng.integers(0, w.L, 46)]))
            X = {k: x[k][b, h].astype(np.float64) for k in "QKV"}
            ref = favor.fwd_bidirectional_rows(X["Q"], X["K"], X["V"], W64, rows)
            errs.append(np.abs(out[b, h, rows] - ref).max())
            refs.append(ref)
    assert max(errs) / np.sqrt(np.mean(np.concatenate(refs) ** 2)) <= 2e-2
