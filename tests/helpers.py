"""Shared test helpers: device placement of the seeded inputs and error metrics. No method
arithmetic lives here."""

import numpy as np

from linear_attention_positive_b200 import api
from linear_attention_positive_b200.inputs import round_to_bf16


def rel_max_err(a, ref):
    """max |a - ref| / RMS(ref), over all elements."""
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(np.asarray(a, dtype=np.float64) - ref).max() / np.sqrt(np.mean(ref * ref)))


def features_for(w_seed, m, d, dtype):
    """W drawn by the library, rounded to the compute dtype, and the exact fp64 values the kernels
    read (what the oracle must consume)."""
    W64 = api.draw_features(w_seed, m, d)
    Wr = round_to_bf16(W64.astype(np.float32)) if dtype == "bf16" else W64.astype(np.float32)
    return Wr, Wr.astype(np.float64)


def to_torch(arr, dtype, device):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32))
    t = t.to(torch.bfloat16) if dtype == "bf16" else t
    return t.to(device).contiguous()
