"""Random-feature attention with feature maps other than the positive softmax features, in plain
fp64 numpy: the generalised (kernelizable) attention and the trigonometric softmax features.

What the pages fix: FAVOR+ "can be also used to efficiently model kernelizable attention
mechanisms beyond softmax" ("Rethinking Attention with Performers", abstract; the summary page
aipaper.jasonlin.tech, "Key contributions": attention extended beyond softmax to other kernelizable
mechanisms), and the Performer line of work moved "from the so-called FAVOR, to FAVOR+"
("Random Features for Efficient Attention Approximation", thesis abstract), the "+" being the
positive features that give lower variance (summary page, "Key contributions"). The pages print
neither map; the readings taken:

* Generalised attention: a kernel K(x, y) = E_w[f(w.x) f(w.y)] estimated by phi(x) = f(W x)/sqrt(m),
  here with f = ReLU (a non-negative f keeps the normaliser D positive, as the softmax features
  do). With w ~ N(0, I) its expectation is the degree-1 arc-cosine kernel
  |x| |y| (sin t + (pi - t) cos t) / (2 pi), t the angle between x and y.
* FAVOR's trigonometric features for the softmax kernel: phi(x) = exp(|x|^2/2)/sqrt(m)
  [sin(W x), cos(W x)] (2m features); phi(x).phi(y) = exp((|x|^2 + |y|^2)/2) mean_r cos(w_r.(x - y)),
  whose expectation is exp(x.y). Unlike the positive features it can be negative, so D can be too.

Attention with either map is the FA-part of "Fast Attention Via Positive Orthogonal Random
Features" (codewithpapers.app/method/favor) with Q' = phi(Q), K' = phi(K):
out = D^-1 (Q' ((K')^T V)), D = diag(Q' ((K')^T 1_L)).

Test infrastructure only (see ``oracle/__init__``).
"""

import math

import numpy as np


def relu_features(X, W):
    """phi(x) = max(W x, 0) / sqrt(m), row-wise (L x m)."""
    return np.maximum(X @ W.T, 0.0) / math.sqrt(W.shape[0])


def trig_features(X, W):
    """phi(x) = exp(|x|^2 / 2) / sqrt(m) [sin(W x), cos(W x)], row-wise (L x 2m)."""
    P = X @ W.T
    scale = np.exp(0.5 * np.sum(X * X, axis=1, keepdims=True)) / math.sqrt(W.shape[0])
    return scale * np.concatenate([np.sin(P), np.cos(P)], axis=1)


FEATURES = {"relu": relu_features, "trig": trig_features}


def arccos1_kernel(x, y):
    """Degree-1 arc-cosine kernel: E_{w ~ N(0, I)}[max(w.x, 0) max(w.y, 0)]."""
    nx, ny = float(np.linalg.norm(x)), float(np.linalg.norm(y))
    c = float(np.clip(x @ y / (nx * ny), -1.0, 1.0))
    t = math.acos(c)
    return nx * ny * (math.sin(t) + (math.pi - t) * c) / (2.0 * math.pi)


def fwd_features(Q, K, V, W, kind):
    """Bidirectional FA-part with the feature map ``kind`` ("relu" or "trig"); one head."""
    f = FEATURES[kind]
    Qp, Kp = f(Q, W), f(K, W)
    S = Kp.T @ V
    z = Kp.T @ np.ones(K.shape[0])
    return (Qp @ S) / (Qp @ z)[:, None]


def attention_brute_features(Q, K, V, W, kind):
    """Explicit L x L definition with the feature map ``kind``: A'(i, j) = phi(q_i).phi(k_j), rows
    normalised by their sums, applied to V."""
    f = FEATURES[kind]
    A = f(Q, W) @ f(K, W).T
    return (A @ V) / A.sum(axis=1)[:, None]


def fwd(Q, K, V, W, kind):
    """Batched over [B, H, L, d] arrays (W shared by all heads)."""
    B, H = Q.shape[:2]
    out = np.empty(Q.shape[:3] + (V.shape[3],))
    for b in range(B):
        for h in range(H):
            out[b, h] = fwd_features(Q[b, h], K[b, h], V[b, h], W, kind)
    return out
