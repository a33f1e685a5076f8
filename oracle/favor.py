"""FAVOR+ attention in plain fp64 numpy: the definitions, written out.

Notation (per batch-head): Q, K, V in R^{L x d}, W in R^{m x d}.

* Feature map (positive random features; the formula is the reading taken, the pages only say
  the features are positive and estimate the softmax kernel):
  u(x) = W x - |x|^2 / 2,  phi(x) = exp(u(x)) / sqrt(m).
  With w ~ N(0, I): E[exp(w.x - |x|^2/2) exp(w.y - |y|^2/2)] = exp(x.y), the softmax kernel
  ("Fast Attention Via Positive Orthogonal Random Features", codewithpapers.app/method/favor,
  the identity K(x,y) = E[phi(x)^T phi(y)]).
* Bidirectional FA-part (same page, the equation for Att<->): Q' = phi(Q), K' = phi(K),
  out = D^-1 (Q' ((K')^T V)),  D = diag(Q' ((K')^T 1_L)). The page prints the normaliser as
  diag(Q'((K')1_L)), which does not type-check (K' is L x r); the reading taken is (K')^T 1_L,
  the one that matches the output equation.
* Causal (masked) variant ("Random Features for Efficient Attention Approximation", abstract:
  masked self-attention): out_i = sum_{j<=i} (phi(q_i).phi(k_j)) v_j / sum_{j<=i} phi(q_i).phi(k_j),
  i.e. prefix sums S_i = sum_{j<=i} phi(k_j) v_j^T, z_i = sum_{j<=i} phi(k_j). The mask keeps
  the diagonal (j <= i).
* Backward with W fixed (not on the pages; derived by the chain rule from the definitions above,
  and pinned by finite differences in the tests): with g_i = dO_i / den_i and
  s_i = -(dO_i . out_i) / den_i,
    dphi(q_i) = S_(i) g_i + z_(i) s_i,
    dv_j = G_(j)^T phi(k_j),  dphi(k_j) = G_(j) v_j + h_(j),
    G = sum_i phi(q_i) g_i^T,  h = sum_i phi(q_i) s_i  (causal: sums over i >= j),
    dx = W^T (phi(x) * dphi(x)) - x * sum_r (phi(x) * dphi(x))_r   (since d phi_r/dx = phi_r (w_r - x)).

No stabiliser is used here: fp64 exp covers |u| < 700.

Test infrastructure only (see ``oracle/__init__``).
"""

import math

import numpy as np


def feature_logits(X, W):
    """u(x) = W x - |x|^2/2 for every row x of X (L x m)."""
    return X @ W.T - 0.5 * np.sum(X * X, axis=1, keepdims=True)


def phi(X, W):
    """Positive random features phi(x) = exp(W x - |x|^2/2) / sqrt(m), row-wise (L x m)."""
    return np.exp(feature_logits(X, W)) / math.sqrt(W.shape[0])


def kernel_estimate(x, y, W):
    """phi(x)^T phi(y): the random-feature estimate of the softmax kernel exp(x.y)."""
    return float(phi(x[None, :], W)[0] @ phi(y[None, :], W)[0])


# --------------------------------------------------------------------------------------------
# Forward
# --------------------------------------------------------------------------------------------

def fwd_bidirectional(Q, K, V, W, return_den=False):
    """FA-part: out = D^-1 (Q'((K')^T V)), D = diag(Q'((K')^T 1_L)); one head, fp64."""
    Qp = phi(Q, W)
    Kp = phi(K, W)
    S = Kp.T @ V                      # (K')^T V, m x d
    z = Kp.T @ np.ones(K.shape[0])    # (K')^T 1_L, m
    num = Qp @ S
    den = Qp @ z                      # diagonal of D
    out = num / den[:, None]
    return (out, den) if return_den else out


def fwd_causal(Q, K, V, W, return_den=False):
    """Masked FA-part by the prefix-sum recurrence S_i = S_{i-1} + phi(k_i) v_i^T,
    z_i = z_{i-1} + phi(k_i), out_i = phi(q_i)^T S_i / phi(q_i)^T z_i; one head, fp64."""
    Qp = phi(Q, W)
    Kp = phi(K, W)
    L, d = V.shape
    m = W.shape[0]
    S = np.zeros((m, d))
    z = np.zeros(m)
    out = np.empty((L, d))
    den = np.empty(L)
    for i in range(L):
        S += np.outer(Kp[i], V[i])
        z += Kp[i]
        den[i] = Qp[i] @ z
        out[i] = (Qp[i] @ S) / den[i]
    return (out, den) if return_den else out


def attention_brute(Q, K, V, W, causal=False):
    """Explicit L x L definition: A'(i,j) = phi(q_i).phi(k_j) (masked j <= i if causal),
    rows normalised by their sums, applied to V. Returns (out, row_sums)."""
    A = phi(Q, W) @ phi(K, W).T
    if causal:
        A = np.tril(A)
    D = A.sum(axis=1)
    return (A @ V) / D[:, None], D


def softmax_attention(Q, K, V, causal=False):
    """Exact softmax attention softmax(Q K^T) V (inputs already carry the d^-1/4 scaling)."""
    s = Q @ K.T
    if causal:
        s = np.where(np.tril(np.ones_like(s, dtype=bool)), s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return (p @ V) / p.sum(axis=1, keepdims=True)


def fwd(Q, K, V, W, causal=False):
    """Batched forward over [B, H, L, d] arrays (W shared by all heads)."""
    f = fwd_causal if causal else fwd_bidirectional
    B, H = Q.shape[:2]
    out = np.empty(Q.shape[:3] + (V.shape[3],))
    for b in range(B):
        for h in range(H):
            out[b, h] = f(Q[b, h], K[b, h], V[b, h], W)
    return out


# --------------------------------------------------------------------------------------------
# Backward (W fixed)
# --------------------------------------------------------------------------------------------

def _input_grad(X, Xp, dXp, W):
    """Chain rule through phi: dX = (phi * dphi) W - X * rowsum(phi * dphi)."""
    P = Xp * dXp
    return P @ W - X * P.sum(axis=1, keepdims=True)


def bwd_bidirectional(Q, K, V, W, dO, return_feature_grads=False):
    """Gradients (dQ, dK, dV) of sum(dO * out) for the bidirectional FA-part; one head.
    With ``return_feature_grads`` also (phi(Q), dphi(Q), phi(K), dphi(K))."""
    Qp = phi(Q, W)
    Kp = phi(K, W)
    S = Kp.T @ V
    z = Kp.sum(axis=0)
    num = Qp @ S
    den = Qp @ z
    out = num / den[:, None]
    g = dO / den[:, None]
    s = -np.sum(dO * out, axis=1) / den
    dQp = g @ S.T + s[:, None] * z[None, :]
    G = Qp.T @ g
    h = Qp.T @ s
    dV = Kp @ G
    dKp = V @ G.T + h[None, :]
    grads = (_input_grad(Q, Qp, dQp, W), _input_grad(K, Kp, dKp, W), dV)
    return grads + (Qp, dQp, Kp, dKp) if return_feature_grads else grads


def bwd_causal(Q, K, V, W, dO, return_feature_grads=False):
    """Gradients (dQ, dK, dV) for the causal FA-part, by a forward prefix recurrence for
    (S_i, z_i) and a reverse suffix recurrence for (G_j, h_j); one head.
    With ``return_feature_grads`` also (phi(Q), dphi(Q), phi(K), dphi(K))."""
    Qp = phi(Q, W)
    Kp = phi(K, W)
    L, d = V.shape
    m = W.shape[0]
    out, den = fwd_causal(Q, K, V, W, return_den=True)
    g = dO / den[:, None]
    s = -np.sum(dO * out, axis=1) / den
    dQp = np.empty((L, m))
    S = np.zeros((m, d))
    z = np.zeros(m)
    for i in range(L):
        S += np.outer(Kp[i], V[i])
        z += Kp[i]
        dQp[i] = S @ g[i] + z * s[i]
    dKp = np.empty((L, m))
    dV = np.empty((L, d))
    G = np.zeros((m, d))
    h = np.zeros(m)
    for j in range(L - 1, -1, -1):
        G += np.outer(Qp[j], g[j])
        h += Qp[j] * s[j]
        dV[j] = G.T @ Kp[j]
        dKp[j] = G @ V[j] + h
    grads = (_input_grad(Q, Qp, dQp, W), _input_grad(K, Kp, dKp, W), dV)
    return grads + (Qp, dQp, Kp, dKp) if return_feature_grads else grads


def bwd(Q, K, V, W, dO, causal=False):
    """Batched backward over [B, H, L, d] arrays."""
    f = bwd_causal if causal else bwd_bidirectional
    dQ = np.empty_like(Q)
    dK = np.empty_like(K)
    dV = np.empty_like(V)
    B, H = Q.shape[:2]
    for b in range(B):
        for h in range(H):
            dQ[b, h], dK[b, h], dV[b, h] = f(Q[b, h], K[b, h], V[b, h], W, dO[b, h])
    return dQ, dK, dV


# --------------------------------------------------------------------------------------------
# Recurrent single-token step (causal decoding)
# --------------------------------------------------------------------------------------------

def decode_step(S, z, q, k, v, W):
    """One step of the masked FA-part's prefix-sum recurrence for a new token t with query q,
    key k and value v (one head): S_t = S_{t-1} + phi(k) v^T, z_t = z_{t-1} + phi(k),
    out_t = phi(q)^T S_t / phi(q)^T z_t. The empty state is S = 0 (m x d), z = 0 (m).
    Returns (out_t, S_t, z_t); the inputs are not modified."""
    pk = phi(k[None, :], W)[0]
    pq = phi(q[None, :], W)[0]
    S = S + np.outer(pk, v)
    z = z + pk
    return (pq @ S) / (pq @ z), S, z


# --------------------------------------------------------------------------------------------
# Row-sampled evaluation for full-size parity checks
# --------------------------------------------------------------------------------------------

def fwd_bidirectional_rows(Q, K, V, W, rows):
    """Outputs of the bidirectional FA-part at the query rows ``rows`` only (full key sums)."""
    Kp = phi(K, W)
    S = Kp.T @ V
    z = Kp.sum(axis=0)
    Qp = phi(Q[rows], W)
    return (Qp @ S) / (Qp @ z)[:, None]


def fwd_causal_rows(Q, K, V, W, rows):
    """Causal outputs at the (sorted) query rows ``rows``; the prefix sums are accumulated in
    key order with the same recurrence as ``fwd_causal`` and read out at each requested row."""
    rows = np.asarray(sorted(rows))
    Kp = phi(K, W)
    Qp = phi(Q[rows], W)
    m = W.shape[0]
    d = V.shape[1]
    S = np.zeros((m, d))
    z = np.zeros(m)
    out = np.empty((len(rows), d))
    nxt = 0
    for i in range(int(rows[-1]) + 1):
        S += np.outer(Kp[i], V[i])
        z += Kp[i]
        while nxt < len(rows) and rows[nxt] == i:
            out[nxt] = (Qp[nxt] @ S) / (Qp[nxt] @ z)
            nxt += 1
    return out
