"""Shared test helpers: device placement of the seeded inputs and error metrics. No method
arithmetic lives here."""

import functools

import numpy as np

from linear_attention_positive_b200 import api
from linear_attention_positive_b200.inputs import round_to_bf16
from oracle import features as oracle_features


def rel_max_err(a, ref):
    """max |a - ref| / RMS(ref), over all elements."""
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(np.asarray(a, dtype=np.float64) - ref).max() / np.sqrt(np.mean(ref * ref)))


@functools.lru_cache(maxsize=None)
def _oracle_W(w_seed, m, d):
    return oracle_features.draw_W(w_seed, m, d)


def features_for(w_seed, m, d, dtype):
    """(W for the kernels, W for the oracle).

    The kernels get the library's own draw (favor_draw_features), rounded to the compute dtype;
    the oracle gets the oracle's draw (oracle.features.draw_W), rounded the same way. The two
    draws are asserted bit-identical first, so the oracle side never takes an input from the
    library."""
    W_lib = api.draw_features(w_seed, m, d)
    W_orc = _oracle_W(w_seed, m, d)
    assert np.array_equal(W_lib, W_orc), "library and oracle feature draws differ"

    def rounded(W):
        return round_to_bf16(W.astype(np.float32)) if dtype == "bf16" else W.astype(np.float32)

    return rounded(W_lib), rounded(W_orc).astype(np.float64)


def to_torch(arr, dtype, device):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32))
    t = t.to(torch.bfloat16) if dtype == "bf16" else t
    return t.to(device).contiguous()
