"""Chunk-wise restatement of the gated delta rule, fp64 (pins the chunk algebra).

TEST INFRASTRUCTURE ONLY: never imported by the product path.

The recurrence of "Super Apriel: One Checkpoint, Many Speeds", §2A (GDN:
scalar gate; KDA: channel-wise gate), S_t = S_{t-1} Diag(a_t)(I - b_t k_t k_t^T)
+ b_t v_t k_t^T, o_t = S_t q_t, can be unrolled over a chunk of C tokens that
starts from a state S0.  With decay(t, j) = prod_{s=j+1..t} Diag(a_s) (empty
product = I) and Gamma_t = decay(t, -1) = prod_{s<=t} Diag(a_s):

    S_t = S0 Gamma_t + sum_{j<=t} u_j k_j^T decay(t, j)                (1)

Substituting (1) for S_{t-1} in u_t = b_t (v_t - S_{t-1} Diag(a_t) k_t) gives
a unit lower-triangular system for the rows u_t of U (C x d_v):

    (I + A) U = Diag(b) (V - Kt S0^T),   A[t,j] = b_t k_t^T decay(t,j) k_j  (j < t)
                                          Kt[t]  = Gamma_t k_t

and then, from (1),

    O     = Qt S0^T + P U,               P[t,j] = q_t^T decay(t,j) k_j     (j <= t)
                                          Qt[t]  = Gamma_t q_t
    S_end = S0 Gamma_{C-1} + sum_j u_j (decay(C-1, j) k_j)^T.

Everything here is fp64 with explicit pairwise decay products (no logarithms,
so gates equal to zero are exact).  This is a second, independent statement of
the same result as ``oracle.recurrent``; the tests require the two to agree to
rounding (about 1e-12 relative).
"""

import numpy as np


def _pairwise_decay(a):
    """a: [L, d] gates of one chunk -> D [L, L, d] with D[t, j] = prod_{s=j+1..t} a_s
    for j <= t and 0 above the diagonal."""
    L, d = a.shape
    D = np.zeros((L, L, d))
    for t in range(L):
        D[t, t] = 1.0
        for j in range(t - 1, -1, -1):
            D[t, j] = D[t, j + 1] * a[j + 1]
    return D


def _chunk(q, k, v, a, b, S0):
    """One chunk of one (batch, head).  q, k [L, dk]; v [L, dv]; a [L, dk]
    (scalar gates already broadcast); b [L]; S0 [dv, dk]."""
    L = q.shape[0]
    D = _pairwise_decay(a)                                   # [L, L, dk]
    gamma = np.cumprod(a, axis=0)                            # Gamma_t, [L, dk]
    A = np.einsum('tc,tjc,jc->tj', k, D, k) * b[:, None]
    A = np.tril(A, -1)
    P = np.tril(np.einsum('tc,tjc,jc->tj', q, D, k))
    Kt = gamma * k
    Qt = gamma * q
    rhs = b[:, None] * (v - Kt @ S0.T)
    U = np.linalg.solve(np.eye(L) + A, rhs)
    O = Qt @ S0.T + P @ U
    S_end = S0 * gamma[L - 1][None, :] + U.T @ (D[L - 1] * k)
    return O, S_end


def chunked_gated_delta_rule(q, k, v, alpha, beta, s0=None, chunk=64):
    """Same arguments and results as ``oracle.recurrent.gated_delta_rule``, computed
    chunk by chunk (the last chunk may be shorter than ``chunk``)."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    alpha = np.asarray(alpha, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if alpha.ndim == 3:
        alpha = np.broadcast_to(alpha[..., None], (B, T, H, dk))
    S = np.zeros((B, H, dv, dk)) if s0 is None else np.array(s0, dtype=np.float64)
    o = np.empty((B, T, H, dv))
    for bi in range(B):
        for h in range(H):
            Sh = S[bi, h]
            for t0 in range(0, T, chunk):
                sl = slice(t0, min(T, t0 + chunk))
                O, Sh = _chunk(q[bi, sl, h], k[bi, sl, h], v[bi, sl, h],
                               alpha[bi, sl, h], beta[bi, sl, h], Sh)
                o[bi, sl, h] = O
            S[bi, h] = Sh
    return o, S
