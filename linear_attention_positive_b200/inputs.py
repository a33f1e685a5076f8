"""Seeded synthetic inputs for the FAVOR+ workloads (shared by the tests, the bench and smoke).

This module draws random numbers and rounds them to the storage precision; it holds none of the
method's arithmetic. Both the CUDA path and the fp64 oracle consume exactly the arrays made here.

Workloads (no dataset is present; all inputs are synthetic with the shapes of the long-sequence
workloads the Performer pages describe):

1. ``bidir-fp32-L256``: B=1, H=1, L=256, d=64, m=64, fp32. Q, K, V iid N(0,1); Q, K scaled by
   d^-1/4. W seed 1, data seed 11.
2. ``bidir-bf16-L4096``: B=8, H=8, L=4096, d=64, m=256, bf16. Same distribution. W seed 2,
   data seed 12.
3. ``causal-bf16-L8192``: B=4, H=8, L=8192, d=64, m=256, bf16 causal. W seed 3, data seed 13.
4. ``causal-bf16-L65536-protein``: B=1, H=16, L=65536, d=64, m=256, bf16 causal. Each head's
   Q, K, V rows are 0.5 * N(0, I) rotated by a seeded Haar-random orthogonal R_h (protein-shaped
   long sequences stand-in); Q, K then scaled by d^-1/4. W seed 4, data seed 14.
5. ``bidir-bf16-L16384-d128-fwdbwd``: B=2, H=8, L=16384, d=128, m=256, bf16 forward + backward;
   upstream gradient dO iid N(0,1). W seed 5, data seed 15.

Two more shapes measure the other feature maps (not among the method's five configurations):

6. ``bidir-bf16-L4096-relu``: workload 2's shape and inputs, generalised attention with ReLU
   features.
7. ``bidir-bf16-L4096-trig``: workload 2's shape, trigonometric features, inputs 0.5 * N(0, 1)
   (with unit-variance inputs the trigonometric normaliser crosses zero). Data seed 17.
8. ``bidir-bf16-L4096-seqpar``: workload 2 through the sequence-parallel calls (partial state,
   then outputs from the state) on one GPU.
"""

from dataclasses import dataclass, replace

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    d: int
    m: int
    causal: bool
    dtype: str          # "f32" or "bf16": storage / compute-input dtype
    backward: bool
    w_seed: int
    data_seed: int
    scale: float = 1.0  # std of the Gaussian rows before the d^-1/4 scaling of Q and K
    rotated: bool = False
    feature_map: str = "positive"  # "positive", "relu" or "trig"
    sequence_parallel: bool = False  # through the state / output calls of the sequence-parallel path

    @property
    def tokens(self):
        return self.B * self.H * self.L

    def with_(self, **kw):
        return replace(self, **kw)


WORKLOADS = {
    1: Workload("bidir-fp32-L256", 1, 1, 256, 64, 64, False, "f32", False, 1, 11),
    2: Workload("bidir-bf16-L4096", 8, 8, 4096, 64, 256, False, "bf16", False, 2, 12),
    3: Workload("causal-bf16-L8192", 4, 8, 8192, 64, 256, True, "bf16", False, 3, 13),
    4: Workload("causal-bf16-L65536-protein", 1, 16, 65536, 64, 256, True, "bf16", False, 4, 14,
                scale=0.5, rotated=True),
    5: Workload("bidir-bf16-L16384-d128-fwdbwd", 2, 8, 16384, 128, 256, False, "bf16", True, 5, 15),
    6: Workload("bidir-bf16-L4096-relu", 8, 8, 4096, 64, 256, False, "bf16", False, 2, 12, feature_map="relu"),
    7: Workload("bidir-bf16-L4096-trig", 8, 8, 4096, 64, 256, False, "bf16", False, 2, 17, scale=0.5,
                feature_map="trig"),
    8: Workload("bidir-bf16-L4096-seqpar", 8, 8, 4096, 64, 256, False, "bf16", False, 2, 12,
                sequence_parallel=True),
}


def round_to_bf16(x):
    """Round float32 values to the nearest bf16 (ties to even); returns float32 holding them."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    bias = 0x7FFF + ((bits >> 16) & 1)
    out = ((bits + bias) & 0xFFFF0000).astype(np.uint32)
    return out.view(np.float32)


def haar_orthogonal(rng, d):
    """A Haar-distributed d x d orthogonal matrix: QR of a Gaussian matrix with the sign of
    R's diagonal folded into Q."""
    g = rng.standard_normal((d, d))
    q, r = np.linalg.qr(g)
    return q * np.sign(np.diag(r))[None, :]


def make_inputs(w: Workload, with_grad=None):
    """Seeded Q, K, V (and dO when the workload has a backward) as float32 arrays [B,H,L,d]
    whose values are exactly representable in the workload's dtype."""
    rng = np.random.default_rng(w.data_seed)
    shape = (w.B, w.H, w.L, w.d)
    out = {}
    for name in ("Q", "K", "V"):
        out[name] = rng.standard_normal(shape, dtype=np.float32)
    if w.rotated:
        for h in range(w.H):
            R = haar_orthogonal(rng, w.d).astype(np.float32)
            for name in ("Q", "K", "V"):
                out[name][:, h] = out[name][:, h] @ R.T
    if w.scale != 1.0:
        for name in ("Q", "K", "V"):
            out[name] *= np.float32(w.scale)
    qk = np.float32(w.d ** -0.25)
    out["Q"] *= qk
    out["K"] *= qk
    if with_grad if with_grad is not None else w.backward:
        out["dO"] = rng.standard_normal(shape, dtype=np.float32)
    if w.dtype == "bf16":
        for k in list(out):
            out[k] = round_to_bf16(out[k])
    return out


def small_case(w: Workload, L=None, B=None, H=None):
    """A reduced copy of a workload (same d, m, dtype, seeds) for oracle-sized checks."""
    return w.with_(L=L or w.L, B=B or w.B, H=H or w.H)
