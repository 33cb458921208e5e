"""Pins for the chunk-wise gradient (oracle/chunked_backward.py).

It must reproduce the token-by-token backward (oracle/backward.py, pinned by finite
differences of the forward) to rounding on both mixers, with chunks that split the
sequence raggedly, one-token chunks and a single chunk, gates and betas equal to zero,
and with or without an entering state and a final-state gradient.  The three-product
form of the reverse chain stated in its header is checked against its per-chunk
result, and planted mistakes in a copy of the chunk gradient must fail.
"""

import numpy as np
import pytest

import oracle.chunked_backward as cbw
from oracle import gated_delta_rule_backward


def _case(kda, B=2, T=11, H=2, dk=5, dv=3, seed=3, zeros=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    alpha = rng.uniform(0.3, 1.0, size=(B, T, H, dk) if kda else (B, T, H))
    beta = rng.uniform(0.1, 1.0, size=(B, T, H))
    if zeros:
        alpha[0, 3] = 0.0          # a gate that forgets everything
        alpha[1, 7, 1] = 0.0
        beta[1, 5] = 0.0           # a token that writes nothing
    s0 = rng.standard_normal((B, H, dv, dk))
    do = rng.standard_normal((B, T, H, dv))
    dsf = rng.standard_normal((B, H, dv, dk))
    return q, k, v, alpha, beta, s0, do, dsf


def _rel(got, ref):
    return max(float(np.abs(g - r).max()) / max(1.0, float(np.abs(r).max()))
               for g, r in zip(got, ref))


@pytest.mark.parametrize("kda", [False, True])
@pytest.mark.parametrize("chunk", [1, 4, 5, 64])
def test_matches_token_backward(kda, chunk):
    q, k, v, alpha, beta, s0, do, dsf = _case(kda)
    ref = gated_delta_rule_backward(q, k, v, alpha, beta, s0, do, dsf)
    got = cbw.chunked_gated_delta_rule_backward(q, k, v, alpha, beta, s0, do, dsf,
                                                chunk=chunk)
    assert _rel(got, ref) < 1e-12


@pytest.mark.parametrize("kda", [False, True])
def test_no_state_no_final_gradient(kda):
    q, k, v, alpha, beta, _, do, _ = _case(kda, seed=11)
    ref = gated_delta_rule_backward(q, k, v, alpha, beta, None, do, None)
    got = cbw.chunked_gated_delta_rule_backward(q, k, v, alpha, beta, None, do, None,
                                                chunk=4)
    assert _rel(got, ref) < 1e-12


@pytest.mark.parametrize("kda", [False, True])
def test_reverse_chain_three_products(kda):
    # one chunk: Y = (dS_end K^ + dO^T P) T is dV^T and
    # dS0 = dS_end Gamma_last + dO^T Qt - Y Kt, with T = (I + A)^{-1} Diag(b), K^ = Kh^T
    q, k, v, alpha, beta, s0, do, dsf = _case(kda, B=1, T=6, H=1, seed=5, zeros=False)
    a = alpha[0, :, 0] if kda else np.broadcast_to(alpha[0, :, 0, None], (6, 5))
    qc, kc, vc, bc = q[0, :, 0], k[0, :, 0], v[0, :, 0], beta[0, :, 0]
    S0, dO, dS_end = s0[0, 0], do[0, :, 0], dsf[0, 0]
    E, D, gamma, A0, M, Kt, R, U, Kh = cbw._chunk_forward(kc, vc, a, bc, S0)
    P = np.tril(np.einsum('tc,tjc,jc->tj', qc, D, kc))
    Tm = M @ np.diag(bc)
    Y = (dS_end @ Kh.T + dO.T @ P) @ Tm
    dS0 = dS_end * gamma[-1][None, :] + dO.T @ (gamma * qc) - Y @ Kt
    _, _, gv, _, _, gS0 = cbw._chunk_backward(qc, kc, vc, a, bc, S0, dO, dS_end)
    assert np.allclose(Y.T, gv, rtol=1e-13, atol=1e-13)
    assert np.allclose(dS0, gS0, rtol=1e-13, atol=1e-13)


def _planted(monkeypatch, mistake):
    """A copy of the chunk gradient with one plausible mistake."""
    good = cbw._chunk_backward

    def bad(q, k, v, a, b, S0, dO, dS_end):
        dq, dk, dv, da, db, dS0 = good(q, k, v, a, b, S0, dO, dS_end)
        E, D, gamma, A0, M, Kt, R, U, Kh = cbw._chunk_forward(k, v, a, b, S0)
        if mistake == "dU without the final-state term":
            dU_missing = Kh @ dS_end.T
            dv = dv - b[:, None] * (M.T @ dU_missing)
        elif mistake == "dS0 without the decay":
            dS0 = dS0 - dS_end * gamma[-1][None, :] + dS_end
        elif mistake == "beta gradient without the Gram term":
            dU = np.tril(np.einsum('tc,tjc,jc->tj', q, D, k)).T @ dO + Kh @ dS_end.T
            db = ((M.T @ dU) * R).sum(1)
        elif mistake == "gate gradient off by one token":
            da = np.roll(da, 1, axis=0)
        return dq, dk, dv, da, db, dS0

    monkeypatch.setattr(cbw, "_chunk_backward", bad)


@pytest.mark.parametrize("mistake", ["dU without the final-state term",
                                     "dS0 without the decay",
                                     "beta gradient without the Gram term",
                                     "gate gradient off by one token"])
def test_planted_mistakes_fail(monkeypatch, mistake):
    q, k, v, alpha, beta, s0, do, dsf = _case(True, zeros=False)
    ref = gated_delta_rule_backward(q, k, v, alpha, beta, s0, do, dsf)
    _planted(monkeypatch, mistake)
    got = cbw.chunked_gated_delta_rule_backward(q, k, v, alpha, beta, s0, do, dsf, chunk=4)
    assert _rel(got, ref) > 1e-6
