"""The gated delta rule, token by token, in fp64 (the oracle proper).

TEST INFRASTRUCTURE ONLY: never imported by the product path.

Follows "Super Apriel: One Checkpoint, Many Speeds", §2A (Mixer Vocabulary):
GDN = delta rule with a scalar gate, KDA = delta rule with a channel-wise gate.
The recurrence written out (the published gated delta rule) is

    S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
    o_t = S_t q_t

Expanding the product with S~ = S_{t-1} Diag(alpha_t):

    S_t = S~ - beta_t (S~ k_t) k_t^T + beta_t v_t k_t^T
        = S~ + u_t k_t^T,        u_t = beta_t (v_t - S~ k_t)

which is exactly the same matrix (an identity of the definition, no
approximation), so the loop below applies a rank-one update per token instead
of forming the d_k x d_k matrix (I - beta k k^T).

Conventions (readings of the pages, which give no layout):
  * S is d_v x d_k ("S q" is a d_v vector, "v k^T" is d_v x d_k), stored
    [B, H, d_v, d_k] with k contiguous.
  * the gate is applied before the delta correction, as the product is written
    (Diag(alpha) sits to the left of (I - beta k k^T)).
  * no scaling of q; o_t reads the state after the token's own update.
"""

import numpy as np


def _as_f64(x):
    return np.asarray(x, dtype=np.float64)


def gated_delta_rule(q, k, v, alpha, beta, s0=None):
    """Run the recurrence over T tokens for every (batch, head).

    Arguments (any float dtype; all upcast to fp64 exactly):
      q, k   [B, T, H, d_k]
      v      [B, T, H, d_v]
      alpha  [B, T, H] (GDN, one gate per head and token) or
             [B, T, H, d_k] (KDA, one gate per key channel)
      beta   [B, T, H]
      s0     [B, H, d_v, d_k] initial state, or None for zeros

    Returns (o [B, T, H, d_v], s_final [B, H, d_v, d_k]) in fp64.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    alpha, beta = _as_f64(alpha), _as_f64(beta)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != (B, T, H, dk) or v.shape != (B, T, H, dv):
        raise ValueError("q, k, v shapes disagree")
    per_channel = alpha.ndim == 4
    if per_channel and alpha.shape != (B, T, H, dk):
        raise ValueError("per-channel alpha must be [B, T, H, d_k]")
    if not per_channel and alpha.shape != (B, T, H):
        raise ValueError("scalar alpha must be [B, T, H]")
    if beta.shape != (B, T, H):
        raise ValueError("beta must be [B, T, H]")
    S = np.zeros((B, H, dv, dk)) if s0 is None else _as_f64(s0).copy()
    if S.shape != (B, H, dv, dk):
        raise ValueError("s0 must be [B, H, d_v, d_k]")
    o = np.empty((B, T, H, dv))
    for t in range(T):
        if per_channel:
            # S Diag(alpha): column c of S (key channel c) scaled by alpha_c
            St = S * alpha[:, t, :, None, :]
        else:
            St = S * alpha[:, t, :, None, None]
        kt = k[:, t]                                   # [B, H, dk]
        pred = np.matmul(St, kt[..., None])[..., 0]    # S~ k_t   [B, H, dv]
        u = beta[:, t, :, None] * (v[:, t] - pred)     # [B, H, dv]
        S = St + u[..., :, None] * kt[..., None, :]
        o[:, t] = np.matmul(S, q[:, t][..., None])[..., 0]
    return o, S


def decode_step(q, k, v, alpha, beta, state):
    """One token for each of N sequences: the recurrence with T = 1.

      q, k [N, H, d_k]; v [N, H, d_v]; alpha [N, H] or [N, H, d_k];
      beta [N, H]; state [N, H, d_v, d_k].
    Returns (o [N, H, d_v], new_state) in fp64; the input state is not modified.
    """
    o, s = gated_delta_rule(_as_f64(q)[:, None], _as_f64(k)[:, None],
                            _as_f64(v)[:, None], _as_f64(alpha)[:, None],
                            _as_f64(beta)[:, None], state)
    return o[:, 0], s


def verify_steps(q, k, v, alpha, beta, state):
    """K tokens per sequence from a carried state, keeping the state after each token.

    "Super Apriel: One Checkpoint, Many Speeds", §2D and §4 (speculative decoding):
    the all-GDN placement drafts tokens for the all-FA placement to verify, so a
    recurrent mixer must be able to resume from any of K tokens.  By definition the
    snapshot after token t is the state the recurrence reaches after the first t
    tokens, and the outputs are those of the same run.

      q, k [N, K, H, d_k]; v [N, K, H, d_v]; alpha [N, K, H] or [N, K, H, d_k];
      beta [N, K, H]; state [N, H, d_v, d_k] (not modified).
    Returns (o [N, K, H, d_v], snapshots [K, N, H, d_v, d_k]) in fp64.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    alpha, beta = _as_f64(alpha), _as_f64(beta)
    K = q.shape[1]
    S = _as_f64(state)
    outs, snaps = [], []
    for t in range(K):
        o, S = gated_delta_rule(q[:, t:t + 1], k[:, t:t + 1], v[:, t:t + 1],
                                alpha[:, t:t + 1], beta[:, t:t + 1], S)
        outs.append(o[:, 0])
        snaps.append(S)
    return np.stack(outs, axis=1), np.stack(snaps, axis=0)


def prefill_varlen(q, k, v, alpha, beta, cu_seqlens, state, slots=None):
    """Sequences of different lengths packed along the token axis, each run from (and
    back into) its own slot of a state pool.

    "Super Apriel: One Checkpoint, Many Speeds", §2D (serving) and §4 (context-length
    scaling): prompts of many lengths are prefilled together and each keeps its state.
    Sequence i is tokens cu_seqlens[i] .. cu_seqlens[i+1]-1 and runs the recurrence
    from state[slots[i]] (slot i when slots is None); nothing crosses a boundary.

      q, k [total, H, d_k]; v [total, H, d_v]; alpha [total, H] or [total, H, d_k];
      beta [total, H]; state [nslots, H, d_v, d_k] (not modified).
    Returns (o [total, H, d_v], new_state [nslots, H, d_v, d_k]) in fp64.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    alpha, beta = _as_f64(alpha), _as_f64(beta)
    cu = [int(x) for x in cu_seqlens]
    pool = _as_f64(state).copy()
    o = np.zeros(v.shape)
    for i in range(len(cu) - 1):
        a, b = cu[i], cu[i + 1]
        slot = i if slots is None else int(slots[i])
        if b == a:
            continue
        oi, si = gated_delta_rule(q[None, a:b], k[None, a:b], v[None, a:b], alpha[None, a:b],
                                  beta[None, a:b], pool[slot][None])
        o[a:b] = oi[0]
        pool[slot] = si[0]
    return o, pool
