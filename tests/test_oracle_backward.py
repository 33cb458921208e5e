"""Pins for the fp64 backward oracle (oracle/backward.py).

The pages give the forward recurrence only ("Super Apriel: One Checkpoint, Many
Speeds", §2A) and say that the mixers are trained (§2B), so the gradient is fixed by
the mathematics: central finite differences of the forward oracle on tiny cases
(every input element, both mixers, with an entering state and a final-state
gradient), and closed forms for the identity gates (alpha = 1, beta = 0).  Planted
mistakes in a copy of the backward (below) must fail the finite-difference pin.
"""

import numpy as np
import pytest

from oracle import gated_delta_rule, gated_delta_rule_backward


def _case(kda, B=2, T=6, H=2, dk=4, dv=3, seed=7):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    alpha = rng.uniform(0.3, 1.0, size=(B, T, H, dk) if kda else (B, T, H))
    beta = rng.uniform(0.1, 1.0, size=(B, T, H))
    s0 = rng.standard_normal((B, H, dv, dk))
    do = rng.standard_normal((B, T, H, dv))
    dsf = rng.standard_normal((B, H, dv, dk))
    return [q, k, v, alpha, beta, s0], do, dsf


def _loss(args, do, dsf):
    o, s = gated_delta_rule(*args)
    return float((o * do).sum() + (s * dsf).sum())


def _finite_differences(args, do, dsf, h=1e-6):
    grads = []
    for i, x in enumerate(args):
        g = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = x[idx]
            x[idx] = old + h
            lp = _loss(args, do, dsf)
            x[idx] = old - h
            lm = _loss(args, do, dsf)
            x[idx] = old
            g[idx] = (lp - lm) / (2 * h)
        grads.append(g)
    return grads


def _fd_pin(backward, kda):
    args, do, dsf = _case(kda)
    fd = _finite_differences(args, do, dsf)
    got = backward(*args, do, dsf)
    # order: dq, dk, dv, dalpha, dbeta, ds0  vs  args q, k, v, alpha, beta, s0
    return all(np.allclose(g, f, rtol=1e-6, atol=1e-7) for g, f in zip(got, fd))


@pytest.mark.parametrize("kda", [False, True])
def test_backward_matches_finite_differences(kda):
    assert _fd_pin(gated_delta_rule_backward, kda)


@pytest.mark.parametrize("kda", [False, True])
def test_backward_without_final_state_gradient(kda):
    """ds_final = None is a zero final-state gradient; s0 = None is a zero state."""
    args, do, _ = _case(kda, seed=3)
    a = gated_delta_rule_backward(*args, do, None)
    b = gated_delta_rule_backward(*args, do, np.zeros_like(args[5]))
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    args[5] = None
    fd_args = list(args)
    fd_args[5] = np.zeros((2, 2, 3, 4))
    fd = _finite_differences(fd_args, do, np.zeros((2, 2, 3, 4)))
    got = gated_delta_rule_backward(*args, do, None)
    assert all(np.allclose(g, f, rtol=1e-6, atol=1e-7) for g, f in zip(got, fd))


def test_identity_gates_closed_form():
    """alpha = 1, beta = 0: S_t = S0 for every t and o_t = S0 q_t, so
    dq_t = S0^T do_t, dk = dv = 0, ds0 = ds_final + sum_t do_t q_t^T, and with
    G_t = ds_final + sum_{s >= t} do_s q_s^T:  dbeta_t = (G_t k_t) . (v_t - S0 k_t),
    dalpha_t = <S0, G_t> (GDN)."""
    args, do, dsf = _case(False, seed=11)
    q, k, v, alpha, beta, s0 = args
    alpha[:] = 1.0
    beta[:] = 0.0
    dq, dk, dv, dal, dbe, ds0 = gated_delta_rule_backward(*args, do, dsf)
    T = q.shape[1]
    assert np.allclose(dq, np.einsum("bhrc,bthr->bthc", s0, do), atol=1e-12)
    assert np.abs(dk).max() == 0 and np.abs(dv).max() == 0
    assert np.allclose(ds0, dsf + np.einsum("bthr,bthc->bhrc", do, q), atol=1e-12)
    for t in range(T):
        G = dsf + np.einsum("bthr,bthc->bhrc", do[:, t:], q[:, t:])
        r = v[:, t] - np.einsum("bhrc,bhc->bhr", s0, k[:, t])
        assert np.allclose(dbe[:, t], np.einsum("bhr,bhr->bh",
                                                np.einsum("bhrc,bhc->bhr", G, k[:, t]), r),
                           atol=1e-12)
        assert np.allclose(dal[:, t], np.einsum("bhrc,bhrc->bh", s0, G), atol=1e-12)


# ---------------------------------------------------------------------------------------
# planted mistakes: a copy of the backward with one plausible slip each
# ---------------------------------------------------------------------------------------

MUTANTS = ["no_beta_term_in_dk", "output_grad_after_du", "dalpha_from_new_state",
           "no_decay_on_ds", "dbeta_without_residual_sign"]


def _mutant_backward(kind):
    def run(q, k, v, alpha, beta, s0, do, ds_final=None):
        per_channel = alpha.ndim == 4
        B, T, H, dk = q.shape
        S = s0.copy()
        states = [S]
        for t in range(T):
            a = alpha[:, t, :, None, :] if per_channel else alpha[:, t, :, None, None]
            St = S * a
            r = v[:, t] - np.einsum("bhrc,bhc->bhr", St, k[:, t])
            S = St + (beta[:, t, :, None] * r)[..., :, None] * k[:, t][..., None, :]
            states.append(S)
        dq, dkk, dvv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
        dal, dbe = np.zeros_like(alpha), np.zeros_like(beta)
        dS = ds_final.copy()
        for t in range(T - 1, -1, -1):
            Sprev, Snew = states[t], states[t + 1]
            a = alpha[:, t, :, None, :] if per_channel else alpha[:, t, :, None, None]
            Sdec = Sprev * a
            kt, qt, bt = k[:, t], q[:, t], beta[:, t, :, None]
            r = v[:, t] - np.einsum("bhrc,bhc->bhr", Sdec, kt)
            u = bt * r
            if kind != "output_grad_after_du":
                dS = dS + do[:, t][..., :, None] * qt[..., None, :]
            dq[:, t] = np.einsum("bhrc,bhr->bhc", Snew, do[:, t])
            du = np.einsum("bhrc,bhc->bhr", dS, kt)
            dkk[:, t] = np.einsum("bhrc,bhr->bhc", dS, u)
            if kind == "output_grad_after_du":
                dS = dS + do[:, t][..., :, None] * qt[..., None, :]
            dvv[:, t] = bt * du
            dbe[:, t] = np.einsum("bhr,bhr->bh", du, -r if kind == "dbeta_without_residual_sign" else r)
            dSdec = dS - (bt * du)[..., :, None] * kt[..., None, :]
            if kind != "no_beta_term_in_dk":
                dkk[:, t] -= np.einsum("bhrc,bhr->bhc", Sdec, bt * du)
            src = Snew if kind == "dalpha_from_new_state" else Sprev
            g = np.einsum("bhrc,bhrc->bhc", src, dSdec)
            dal[:, t] = g if per_channel else g.sum(-1)
            dS = dSdec if kind == "no_decay_on_ds" else dSdec * a
        return dq, dkk, dvv, dal, dbe, dS
    return run


def test_mutant_copy_is_faithful():
    """With no mistake planted the copy equals the oracle."""
    for kda in (False, True):
        args, do, dsf = _case(kda, seed=5)
        a = _mutant_backward("none")(*args, do, dsf)
        b = gated_delta_rule_backward(*args, do, dsf)
        assert all(np.allclose(x, y, rtol=0, atol=1e-13) for x, y in zip(a, b))


@pytest.mark.parametrize("kind", MUTANTS)
def test_finite_differences_catch_planted_mistake(kind):
    assert not (_fd_pin(_mutant_backward(kind), False) and _fd_pin(_mutant_backward(kind), True))
