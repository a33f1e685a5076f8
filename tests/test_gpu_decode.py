"""GPU parity of the recurrent single-token step (favor_decode_step) through the C ABI.

Feeding a sequence one token per call from the empty (all-zero) state must reproduce the rows of
the masked FA-part: checked against the fp64 oracle's recurrence (oracle.favor.decode_step, pinned
against brute force on the explicit masked matrix) and against the GPU's own causal forward. The
step computes in fp32 for either input dtype, so the fp32 bound 1e-4 * RMS(out) applies."""

import numpy as np
import pytest

from linear_attention_positive_b200 import api
from linear_attention_positive_b200.inputs import Workload, make_inputs, round_to_bf16
from oracle import favor
from tests.helpers import features_for, rel_max_err, to_torch

pytestmark = pytest.mark.gpu

TOL = 1e-4


def run_decode(x, Wr, dtype, device):
    import torch

    B, H, L, d = x["Q"].shape
    T = {k: to_torch(x[k], dtype, device) for k in "QKV"}
    Wt = to_torch(Wr, dtype, device)
    state = api.decode_state(B, H, d, Wr.shape[0], device)
    outs = []
    for t in range(L):
        outs.append(api.decode_step(T["Q"][:, :, t].contiguous(), T["K"][:, :, t].contiguous(),
                                    T["V"][:, :, t].contiguous(), Wt, state))
    assert api.sync_status() == api.FAVOR_OK
    return torch.stack(outs, dim=2).double().cpu().numpy(), state


def oracle_decode(x, W64):
    B, H, L, d = x["Q"].shape
    out = np.empty((B, H, L, d))
    states = {}
    for b in range(B):
        for h in range(H):
            S, z = np.zeros((W64.shape[0], d)), np.zeros(W64.shape[0])
            X = {k: x[k][b, h].astype(np.float64) for k in "QKV"}
            for t in range(L):
                out[b, h, t], S, z = favor.decode_step(S, z, X["Q"][t], X["K"][t], X["V"][t], W64)
            states[(b, h)] = (S, z)
    return out, states


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,H,L,d,m", [(2, 3, 200, 64, 256), (1, 2, 150, 128, 128), (1, 1, 40, 64, 32)])
def test_decode_steps_match_oracle(cuda_device, dtype, B, H, L, d, m):
    w = Workload("t", B, H, L, d, m, True, dtype, False, 3, 70 + L)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, m, d, dtype)
    out, state = run_decode(x, Wr, dtype, cuda_device)
    ref, states = oracle_decode(x, W64)
    assert np.isfinite(out).all()
    assert rel_max_err(out, ref) <= TOL
    # the carried state: exp(D_r) S'[c][r] = sqrt(m) S[r][c] and exp(D_r) z'[r] = sqrt(m) z[r]
    st = state.double().cpu().numpy().reshape(B * H, d * m + 2 * m)
    for b in range(B):
        for h in range(H):
            row = st[b * H + h]
            Sp, zp, Dl = row[: d * m].reshape(d, m), row[d * m: d * m + m], row[d * m + m:]
            S_ref, z_ref = states[(b, h)]
            S_gpu = (np.exp(Dl)[None, :] * Sp).T / np.sqrt(m)
            z_gpu = np.exp(Dl) * zp / np.sqrt(m)
            assert np.abs(S_gpu - S_ref).max() <= 1e-4 * np.abs(S_ref).max()
            assert np.abs(z_gpu - z_ref).max() <= 1e-4 * np.abs(z_ref).max()


def test_decode_matches_causal_forward_rows(cuda_device):
    """Token-by-token decoding against the GPU's own chunked causal forward on the same inputs."""
    w = Workload("t", 1, 2, 640, 64, 256, True, "bf16", False, 3, 12)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "bf16")
    out, _ = run_decode(x, Wr, "bf16", cuda_device)
    T = {k: to_torch(x[k], "bf16", cuda_device) for k in "QKV"}
    fwd = api.fwd(T["Q"], T["K"], T["V"], to_torch(Wr, "bf16", cuda_device), causal=True)
    assert api.sync_status() == api.FAVOR_OK
    ref = favor.fwd(*(x[k].astype(np.float64) for k in "QKV"), W64, causal=True)
    assert rel_max_err(out, ref) <= TOL
    assert rel_max_err(fwd.double().cpu().numpy(), ref) <= 2e-2


def test_decode_key_logits_far_above_earlier_ones(cuda_device):
    """Keys whose logits jump by ~24 nats over earlier ones raise the per-feature stabilisers and
    rescale the carried rows; nothing overflows and the outputs still match."""
    w = Workload("t", 1, 1, 64, 64, 128, True, "f32", False, 3, 5)
    x = make_inputs(w)
    Wr, W64 = features_for(w.w_seed, w.m, w.d, "f32")
    w0 = W64[0].astype(np.float32)
    x["K"][0, 0, 40:] += w0[None, :]
    x["Q"][0, 0] += 0.2 * w0[None, :]
    K64 = x["K"][0, 0].astype(np.float64)
    u0 = K64 @ W64[0] - 0.5 * (K64 ** 2).sum(1)
    assert u0[40:].max() - u0[:40].max() > 20.0
    out, _ = run_decode(x, Wr, "f32", cuda_device)
    ref, _ = oracle_decode(x, W64)
    assert np.isfinite(out).all()
    assert rel_max_err(out, ref) <= TOL
