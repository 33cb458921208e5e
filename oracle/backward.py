"""Gradients of the gated delta rule, token by token in reverse, in fp64.

TEST INFRASTRUCTURE ONLY: never imported by the product path.

"Super Apriel: One Checkpoint, Many Speeds", §2B (Training Recipe): the mixers are
trained, by stochastic distillation (S1) and then supervised fine-tuning (S2), so
the mixer's gradient with respect to its inputs and its initial state is needed.
The pages give the forward recurrence only (§2A; the one in recurrent.py); the
backward below is that recurrence differentiated by hand, step by step, with
nothing reassociated:

  forward, token t:   S~  = S_{t-1} Diag(alpha_t)
                      r_t = v_t - S~ k_t               (the residual)
                      u_t = beta_t r_t
                      S_t = S~ + u_t k_t^T
                      o_t = S_t q_t

  reverse, token t (dS = dL/dS_t, arriving from token t + 1 or the final state):
                      dS   += do_t q_t^T               and dq_t = S_t^T do_t
                      du    = dS k_t,   dk_t = dS^T u_t (the rank-one update)
                      dv_t  = beta_t du,  dbeta_t = du . r_t
                      dS~   = dS - beta_t du k_t^T,  dk_t -= beta_t S~^T du
                      dalpha_t[c] = sum_r S_{t-1}[r, c] dS~[r, c]
                                    (summed over c as well for the scalar gate)
                      dS    = dS~ Diag(alpha_t)        (now dL/dS_{t-1})

and ds0 is dS after token 1.  The gradient is taken with respect to alpha itself
(not log alpha), and the loss is sum_t <do_t, o_t> + <ds_final, S_T>.
"""

import numpy as np


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def gated_delta_rule_backward(q, k, v, alpha, beta, s0, do, ds_final=None):
    """Gradients of L = sum_t <do_t, o_t> + <ds_final, S_T> for the recurrence of
    recurrent.gated_delta_rule.

    Arguments as there (q, k [B,T,H,d_k]; v [B,T,H,d_v]; alpha [B,T,H] or
    [B,T,H,d_k]; beta [B,T,H]; s0 [B,H,d_v,d_k] or None), plus
      do        [B, T, H, d_v]   dL/do
      ds_final  [B, H, d_v, d_k] dL/dS_T, or None for zeros

    Returns (dq, dk, dv, dalpha, dbeta, ds0) in fp64, shaped like q, k, v, alpha,
    beta and the state.
    """
    q, k, v, alpha, beta, do = map(_f64, (q, k, v, alpha, beta, do))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    per_channel = alpha.ndim == 4
    S = np.zeros((B, H, dv, dk)) if s0 is None else _f64(s0).copy()
    # forward, keeping every state S_0 .. S_T (small cases only)
    states = [S]
    for t in range(T):
        a = alpha[:, t, :, None, :] if per_channel else alpha[:, t, :, None, None]
        St = S * a
        r = v[:, t] - np.einsum("bhrc,bhc->bhr", St, k[:, t])
        S = St + (beta[:, t, :, None] * r)[..., :, None] * k[:, t][..., None, :]
        states.append(S)
    dq = np.zeros_like(q)
    dkk = np.zeros_like(k)
    dvv = np.zeros_like(v)
    dal = np.zeros_like(alpha)
    dbe = np.zeros_like(beta)
    dS = np.zeros((B, H, dv, dk)) if ds_final is None else _f64(ds_final).copy()
    for t in range(T - 1, -1, -1):
        Sprev, St_ = states[t], states[t + 1]
        a = alpha[:, t, :, None, :] if per_channel else alpha[:, t, :, None, None]
        Sdec = Sprev * a                                           # S~
        kt, qt, bt = k[:, t], q[:, t], beta[:, t, :, None]
        r = v[:, t] - np.einsum("bhrc,bhc->bhr", Sdec, kt)
        u = bt * r
        # o_t = S_t q_t
        dS = dS + do[:, t][..., :, None] * qt[..., None, :]
        dq[:, t] = np.einsum("bhrc,bhr->bhc", St_, do[:, t])
        # S_t = S~ + u k^T
        du = np.einsum("bhrc,bhc->bhr", dS, kt)
        dkk[:, t] = np.einsum("bhrc,bhr->bhc", dS, u)
        # u = beta (v - S~ k)
        dvv[:, t] = bt * du
        dbe[:, t] = np.einsum("bhr,bhr->bh", du, r)
        dSdec = dS - (bt * du)[..., :, None] * kt[..., None, :]
        dkk[:, t] -= np.einsum("bhrc,bhr->bhc", Sdec, bt * du)
        # S~ = S_{t-1} Diag(alpha)
        g = np.einsum("bhrc,bhrc->bhc", Sprev, dSdec)
        dal[:, t] = g if per_channel else g.sum(-1)
        dS = dSdec * a
    return dq, dkk, dvv, dal, dbe, dS
