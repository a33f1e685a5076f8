"""The exchange of the sequence-parallel forward on CPU (gloo, world size 2): each rank holds a
contiguous run of every head's tokens, computes the partial state of its keys, the partial states
are summed by one all-reduce, and each rank answers its own queries from the total.

The rank-local compute here is a host stand-in written from the oracle's definitions with the
state contract of favor_sp_state / favor_sp_output (state = sum_j exp(u_r(k_j) - c_r) [v_j | 1],
c_r = |w_r|^2/2 - 40), so the test runs without a GPU; the GPU test of the same split
(tests/test_gpu_sequence_parallel.py) runs the library's kernels. No rank's compute waits on
another's: the only cross-rank step is the all-reduce."""

import os
import socket
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _offsets(W):
    return 0.5 * np.sum(W * W, axis=1) - 40.0


def host_state(K, V, W):
    """The favor_sp_state contract on the host: [B*H, m, d+64] float64."""
    from oracle import favor

    K, V = K.numpy(), V.numpy()
    B, H, L, d = K.shape
    m = W.shape[0]
    c = _offsets(W)
    out = np.zeros((B * H, m, d + 64))
    for b in range(B):
        for h in range(H):
            phi = np.exp(favor.feature_logits(K[b, h], W) - c[None, :])
            out[b * H + h, :, :d] = phi.T @ V[b, h]
            out[b * H + h, :, d] = phi.sum(axis=0)
    return torch.from_numpy(out)


def host_output(Q, W, state):
    Q, S = Q.numpy(), state.numpy()
    B, H, L, d = Q.shape
    c = _offsets(W)
    out = np.empty((B, H, L, d))
    for b in range(B):
        for h in range(H):
            u = Q[b, h] @ W.T + c[None, :]
            p = np.exp(u - u.max(axis=1, keepdims=True))
            nd = p @ S[b * H + h]
            out[b, h] = nd[:, :d] / nd[:, d:d + 1]
    return torch.from_numpy(out)


def _rank_main(rank, world, port, cuts, q):
    import torch.distributed as dist

    from linear_attention_positive_b200 import api
    from linear_attention_positive_b200.inputs import Workload, make_inputs
    from oracle import features

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = Workload("t", 1, 2, 300, 16, 32, False, "f32", False, 4, 9)
        x = make_inputs(w)
        W = features.draw_W(w.w_seed, w.m, w.d)
        lo, hi = cuts[rank], cuts[rank + 1]
        run = {k: torch.from_numpy(x[k][:, :, lo:hi].astype(np.float64)) for k in "QKV"}
        out = api.sp_forward(run["Q"], run["K"], run["V"], W, state_fn=host_state, output_fn=host_output)
        q.put((rank, out.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_partial_states_summed_across_two_ranks_give_the_full_attention():
    from linear_attention_positive_b200.inputs import Workload, make_inputs
    from oracle import favor, features

    cuts = [0, 113, 300]  # uneven runs
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, cuts, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    got = np.concatenate([results[0], results[1]], axis=2)
    w = Workload("t", 1, 2, 300, 16, 32, False, "f32", False, 4, 9)
    x = make_inputs(w)
    W = features.draw_W(w.w_seed, w.m, w.d)
    ref = favor.fwd(*(x[k].astype(np.float64) for k in "QKV"), W)
    assert np.abs(got - ref).max() <= 1e-10 * np.abs(ref).max()
