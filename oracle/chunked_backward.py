"""Chunk-wise restatement of the gated delta rule's gradient, fp64.

TEST INFRASTRUCTURE ONLY: never imported by the product path.

"Super Apriel: One Checkpoint, Many Speeds", §2B trains the mixers of §2A, so their
gradient is needed; backward.py takes it token by token.  This module takes the same
gradient from the chunk algebra of chunked.py instead, differentiating its lines (not
the recurrence).  For a chunk of L tokens entering with state S0 (decay(t, j) =
prod_{s=j+1..t} Diag(a_s), Gamma_t = decay(t, -1), M = (I + A)^{-1}):

    R = V - Kt S0^T,   U = M Diag(b) R,
    O = Qt S0^T + P U, S_end = S0 Gamma_{L-1} + U^T Kh,   Kh[j] = decay(L-1, j) k_j.

Given dO and dS_end = dL/dS_end, line by line in reverse:

    dU   = P^T dO + Kh dS_end^T                 dP  = dO U^T      (kept on j <= t)
    dKh  = U dS_end                             dQt = dO S0
    dRb  = M^T dU,  dR = Diag(b) dRb            dV  = dR
    dM   = dU (Diag(b) R)^T,  dA = -M^T dM M^T  (kept on j < t)
    dKt  = -dR S0
    dS0  = dS_end Gamma_{L-1} + dO^T Qt - dR^T Kt
    dbeta_t = dRb_t . R_t + sum_j dA[t, j] A0[t, j]      (A = Diag(b) A0)

and dq, dk from the Gram A0, P, Qt, Kt and Kh.  dS0 is the dS_end of the chunk
before, so the state gradient chains backward through the chunks as the state chains
forward; in the transposed form with U^T, the chain of one chunk is three products,
Y = (dS_end K^ + dO^T P) T and dS0 = dS_end Gamma_{L-1} + dO^T Qt - Y Kt, with
T = M Diag(b), K^ = Kh^T and dV = Y^T: the forward carry's shape with the roles of
Kt and Kh exchanged.

Every gate enters through some decay(t, j), j = -1 .. t.  With W[t, j] = dL/ddecay(t, j)
(per channel), dL/da_s = sum_{j < s <= t} W[t, j] decay(t, s) decay(s - 1, j), the
product of the other factors: nothing is divided, so gates equal to zero are exact.
The scalar gate's gradient sums that over the channels.

Pinned in tests/test_oracle_chunked_backward.py against backward.py (itself pinned by
finite differences) to rounding, on ragged chunks, zero gates and zero betas.
"""

import numpy as np


def _decay_table(a):
    """a [L, d] -> E [L, L + 1, d] with E[t, j + 1] = decay(t, j) for j = -1 .. t
    (decay(t, t) = 1) and zero for j > t."""
    L, d = a.shape
    E = np.zeros((L, L + 1, d))
    for t in range(L):
        E[t, t + 1] = 1.0
        for j in range(t - 1, -2, -1):
            E[t, j + 1] = E[t, j + 2] * a[j + 1]
    return E


def _chunk_forward(k, v, a, b, S0):
    """The chunk's forward quantities that its gradient reuses."""
    L = k.shape[0]
    E = _decay_table(a)
    D = E[:, 1:, :]                                   # decay(t, j), [L, L, d]
    gamma = E[:, 0, :]                                # Gamma_t
    A0 = np.tril(np.einsum('tc,tjc,jc->tj', k, D, k), -1)
    M = np.linalg.inv(np.eye(L) + b[:, None] * A0)
    Kt = gamma * k
    R = v - Kt @ S0.T
    U = M @ (b[:, None] * R)
    Kh = E[L - 1, 1:, :] * k
    return E, D, gamma, A0, M, Kt, R, U, Kh


def _chunk_backward(q, k, v, a, b, S0, dO, dS_end):
    """Gradients of one chunk of one (batch, head): q, k [L, dk]; v, dO [L, dv];
    a [L, dk] (scalar gates broadcast); b [L]; S0, dS_end [dv, dk].
    Returns dq, dk, dv, da [L, dk] (per channel), db [L], dS0."""
    L = q.shape[0]
    E, D, gamma, A0, M, Kt, R, U, Kh = _chunk_forward(k, v, a, b, S0)
    P = np.tril(np.einsum('tc,tjc,jc->tj', q, D, k))
    Qt = gamma * q

    dU = P.T @ dO + Kh @ dS_end.T
    dP = np.tril(dO @ U.T)
    dKh = U @ dS_end
    dQt = dO @ S0
    dRb = M.T @ dU
    dR = b[:, None] * dRb
    dM = dU @ (b[:, None] * R).T
    dA = np.tril(-M.T @ dM @ M.T, -1)
    dKt = -dR @ S0
    dS0 = dS_end * gamma[L - 1][None, :] + dO.T @ Qt - dR.T @ Kt
    db = (dRb * R).sum(1) + (dA * A0).sum(1)
    dA0 = dA * b[:, None]

    # q and k through the Gram, P, Qt, Kt and Kh
    dq = np.einsum('tj,tjc,jc->tc', dP, D, k) + dQt * gamma
    dk = (np.einsum('tj,tjc,jc->tc', dA0, D, k) + np.einsum('tj,tjc,tc->jc', dA0, D, k)
          + np.einsum('tj,tjc,tc->jc', dP, D, q) + dKt * gamma + dKh * E[L - 1, 1:, :])

    # W[t, j + 1] = dL/ddecay(t, j), j = -1 .. t
    W = np.zeros_like(E)
    W[:, 1:, :] += np.einsum('tj,tc,jc->tjc', dA0, k, k)
    W[:, 1:, :] += np.einsum('tj,tc,jc->tjc', dP, q, k)
    W[:, 0, :] += dKt * k + dQt * q
    W[L - 1, 1:, :] += dKh * k
    W[L - 1, 0, :] += (dS_end * S0).sum(0)
    da = np.zeros_like(a)
    for s in range(L):
        # decay(s - 1, j) for j = -1 .. s - 1 (the empty product when s = 0)
        right = E[s - 1, :s + 1, :] if s > 0 else np.ones((1, a.shape[1]))
        for t in range(s, L):
            da[s] += E[t, s + 1] * (W[t, :s + 1, :] * right).sum(0)
    return dq, dk, dR, da, db, dS0


def chunked_gated_delta_rule_backward(q, k, v, alpha, beta, s0, do, ds_final=None,
                                      chunk=64):
    """Same arguments and results as ``oracle.backward.gated_delta_rule_backward``,
    computed chunk by chunk (the last chunk may be shorter than ``chunk``): a forward
    walk keeps the state entering every chunk, a reverse walk chains dL/dS through
    the chunks and forms each chunk's gradients from its entering state."""
    q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
    alpha = np.asarray(alpha, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    per_channel = alpha.ndim == 4
    a_full = alpha if per_channel else np.broadcast_to(alpha[..., None], (B, T, H, dk))
    S = np.zeros((B, H, dv, dk)) if s0 is None else np.array(s0, dtype=np.float64)
    dS = np.zeros((B, H, dv, dk)) if ds_final is None else np.array(ds_final,
                                                                     dtype=np.float64)
    dq, dkk, dvv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dal, dbe = np.zeros_like(alpha), np.zeros_like(beta)
    starts = list(range(0, T, chunk))
    for bi in range(B):
        for h in range(H):
            # forward: the state entering every chunk
            entering = []
            Sh = S[bi, h]
            for t0 in starts:
                sl = slice(t0, min(T, t0 + chunk))
                entering.append(Sh)
                *_, U, Kh = _chunk_forward(k[bi, sl, h], v[bi, sl, h], a_full[bi, sl, h],
                                           beta[bi, sl, h], Sh)
                gamma_last = np.prod(a_full[bi, sl, h], axis=0)
                Sh = Sh * gamma_last[None, :] + U.T @ Kh
            # reverse: dL/dS chained from the last chunk to the first
            dSh = dS[bi, h]
            for n in range(len(starts) - 1, -1, -1):
                sl = slice(starts[n], min(T, starts[n] + chunk))
                gq, gk, gv, ga, gb, dSh = _chunk_backward(
                    q[bi, sl, h], k[bi, sl, h], v[bi, sl, h], a_full[bi, sl, h],
                    beta[bi, sl, h], entering[n], do[bi, sl, h], dSh)
                dq[bi, sl, h], dkk[bi, sl, h], dvv[bi, sl, h] = gq, gk, gv
                dal[bi, sl, h] = ga if per_channel else ga.sum(-1)
                dbe[bi, sl, h] = gb
            dS[bi, h] = dSh
    return dq, dkk, dvv, dal, dbe, dS
