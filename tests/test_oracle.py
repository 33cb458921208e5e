"""Pins for the fp64 oracle, checked against what the definition fixes.

The mixer is the gated delta rule named in "Super Apriel: One Checkpoint, Many
Speeds", §2A (GDN: scalar gate per head and token; KDA: channel-wise gate):
S_t = S_{t-1} Diag(a_t)(I - b_t k_t k_t^T) + b_t v_t k_t^T, o_t = S_t q_t.
The pages print no worked example, no closed form and no error bound, so each
pin below is fixed by the mathematics instead: a hand-worked case (golden file),
exact rational brute force of the literal matrix product, invariants and special
cases.  Every pin is also run against planted mistakes (mutants of the
recurrence, below) to show that a plausible slip fails at least one of them.
"""

import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import gated_delta_rule, decode_step, chunked_gated_delta_rule

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def _rand_case(B=2, T=9, H=3, dk=4, dv=3, kda=True, unit_k=True, s0=True, rng=RNG,
               alpha_range=(0.2, 1.0)):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    shape = (B, T, H, dk) if kda else (B, T, H)
    alpha = rng.uniform(*alpha_range, size=shape)
    beta = rng.uniform(0.1, 1.0, size=(B, T, H))
    S0 = rng.standard_normal((B, H, dv, dk)) if s0 else None
    return q, k, v, alpha, beta, S0


# --------------------------------------------------------------------------------------
# pins, written against an implementation so that mutants can be run through them too
# --------------------------------------------------------------------------------------

def pin_hand_case(impl):
    with open(os.path.join(GOLDEN, "hand_case_d2.json")) as f:
        g = json.load(f)
    inp = g["inputs"]
    q = np.array(inp["q"])[None, :, None]
    k = np.array(inp["k"])[None, :, None]
    v = np.array(inp["v"])[None, :, None]
    beta = np.array(inp["beta"])[None, :, None]
    ok = True
    for mix, alpha in (("gdn", np.array(inp["alpha_gdn"])[None, :, None]),
                       ("kda", np.array(inp["alpha_kda"])[None, :, None])):
        o, s = impl(q, k, v, alpha, beta, None)
        ok &= np.allclose(o[0, :, 0], g[mix]["o"], rtol=0, atol=1e-14)
        ok &= np.allclose(s[0, 0], g[mix]["s_final"], rtol=0, atol=1e-14)
    return bool(ok)


def _frac_matmul(A, B):
    return [[sum((A[i][x] * B[x][j] for x in range(len(B))), Fraction(0))
             for j in range(len(B[0]))] for i in range(len(A))]


def _literal_rule_exact(q, k, v, a, b, S0):
    """The literal definition, S Diag(a)(I - b k k^T) + b v k^T, in exact rationals
    for one (batch, head): q, k [T][dk], v [T][dv], a [T][dk], b [T], S0 [dv][dk]."""
    T, dk, dv = len(q), len(q[0]), len(v[0])
    S = [row[:] for row in S0]
    outs = []
    for t in range(T):
        diag_a = [[a[t][i] if i == j else Fraction(0) for j in range(dk)] for i in range(dk)]
        proj = [[(Fraction(1) if i == j else Fraction(0)) - b[t] * k[t][i] * k[t][j]
                 for j in range(dk)] for i in range(dk)]
        S = _frac_matmul(_frac_matmul(S, diag_a), proj)
        S = [[S[i][j] + b[t] * v[t][i] * k[t][j] for j in range(dk)] for i in range(dv)]
        outs.append([sum((S[i][j] * q[t][j] for j in range(dk)), Fraction(0))
                     for i in range(dv)])
    return outs, S


def pin_rational_bruteforce(impl):
    """Dyadic inputs (exact in binary floating point), d_k != d_v, non-zero S0, both
    gate kinds; the implementation must match exact rational arithmetic."""
    rng = np.random.default_rng(77)
    B, T, H, dk, dv = 1, 5, 2, 3, 2
    ok = True
    for kda in (False, True):
        qn = rng.integers(-8, 9, size=(B, T, H, dk)) / 8
        kn = rng.integers(-8, 9, size=(B, T, H, dk)) / 8
        vn = rng.integers(-8, 9, size=(B, T, H, dv)) / 8
        an = rng.integers(0, 5, size=(B, T, H, dk) if kda else (B, T, H)) / 4
        bn = rng.integers(1, 5, size=(B, T, H)) / 4
        sn = rng.integers(-4, 5, size=(B, H, dv, dk)) / 4
        o, s = impl(qn, kn, vn, an, bn, sn)
        for h in range(H):
            F_ = lambda x: Fraction(x).limit_denominator(64)  # noqa: E731
            q = [[F_(x) for x in qn[0, t, h]] for t in range(T)]
            k = [[F_(x) for x in kn[0, t, h]] for t in range(T)]
            v = [[F_(x) for x in vn[0, t, h]] for t in range(T)]
            if kda:
                a = [[F_(x) for x in an[0, t, h]] for t in range(T)]
            else:
                a = [[F_(an[0, t, h])] * dk for t in range(T)]
            b = [F_(bn[0, t, h]) for t in range(T)]
            S0 = [[F_(x) for x in row] for row in sn[0, h]]
            outs, S = _literal_rule_exact(q, k, v, a, b, S0)
            ref_o = np.array([[float(x) for x in row] for row in outs])
            ref_s = np.array([[float(x) for x in row] for row in S])
            scale = max(1.0, np.abs(ref_o).max(), np.abs(ref_s).max())
            ok &= np.abs(o[0, :, h] - ref_o).max() <= 1e-13 * scale
            ok &= np.abs(s[0, h] - ref_s).max() <= 1e-13 * scale
    return bool(ok)


def pin_identity(impl):
    """alpha = 1, beta = 0: the state never changes and o_t = S0 q_t."""
    q, k, v, alpha, beta, S0 = _rand_case(kda=True, rng=np.random.default_rng(3))
    alpha[:] = 1.0
    beta[:] = 0.0
    o, s = impl(q, k, v, alpha, beta, S0)
    ref = np.einsum("bhvk,bthk->bthv", S0, q)
    return bool(np.allclose(s, S0, rtol=0, atol=0) and np.allclose(o, ref, rtol=1e-14, atol=1e-14))


def pin_readback(impl):
    """beta = 1 and |k_t| = 1: whatever the gates, S_t k_t = v_t; with q_t = k_t the
    output reads v_t back exactly."""
    ok = True
    for kda in (False, True):
        q, k, v, alpha, beta, S0 = _rand_case(kda=kda, rng=np.random.default_rng(5))
        beta[:] = 1.0
        o, s = impl(k, k, v, alpha, beta, S0)
        ok &= np.allclose(o, v, rtol=0, atol=1e-12)
        ok &= np.allclose(np.einsum("bhvk,bhk->bhv", s, k[:, -1]), v[:, -1], atol=1e-12)
    return bool(ok)


def pin_alpha0_beta1(impl):
    """alpha = 0 forgets everything; beta = 1 then writes exactly v_t k_t^T."""
    q, k, v, alpha, beta, S0 = _rand_case(kda=True, rng=np.random.default_rng(6))
    alpha[:] = 0.0
    beta[:] = 1.0
    o, s = impl(q, k, v, alpha, beta, S0)
    ref_s = np.einsum("bhv,bhk->bhvk", v[:, -1], k[:, -1])
    ref_o = v * np.einsum("bthk,bthk->bth", k, q)[..., None]
    return bool(np.allclose(s, ref_s, atol=1e-14) and np.allclose(o, ref_o, atol=1e-13))


def pin_pure_decay(impl):
    """beta = 0: S_t = S0 Diag(prod_{s<=t} alpha_s) and o_t = S_t q_t (closed form)."""
    q, k, v, alpha, beta, S0 = _rand_case(kda=True, rng=np.random.default_rng(7))
    beta[:] = 0.0
    o, s = impl(q, k, v, alpha, beta, S0)
    cp = np.cumprod(alpha, axis=1)                           # [B, T, H, dk]
    ref_o = np.einsum("bhvk,bthk,bthk->bthv", S0, cp, q)
    ref_s = S0 * cp[:, -1][:, :, None, :]
    return bool(np.allclose(o, ref_o, rtol=1e-12, atol=1e-13) and
                np.allclose(s, ref_s, rtol=1e-12, atol=1e-14))


def pin_kda_equal_gates_is_gdn(impl):
    q, k, v, alpha, beta, S0 = _rand_case(kda=False, rng=np.random.default_rng(8))
    o1, s1 = impl(q, k, v, alpha, beta, S0)
    o2, s2 = impl(q, k, v, np.repeat(alpha[..., None], q.shape[-1], axis=-1), beta, S0)
    return bool(np.allclose(o1, o2, rtol=1e-14, atol=1e-14) and
                np.allclose(s1, s2, rtol=1e-14, atol=1e-14))


def pin_channel_permutation(impl):
    """KDA: permuting the key channels of q, k, alpha and the columns of S0 together
    leaves o unchanged and permutes the columns of the final state."""
    q, k, v, alpha, beta, S0 = _rand_case(kda=True, dk=5, dv=3, rng=np.random.default_rng(9))
    perm = np.array([3, 0, 4, 1, 2])
    o1, s1 = impl(q, k, v, alpha, beta, S0)
    o2, s2 = impl(q[..., perm], k[..., perm], v, alpha[..., perm], beta, S0[..., perm])
    return bool(np.allclose(o1, o2, rtol=1e-12, atol=1e-13) and
                np.allclose(s1[..., perm], s2, rtol=1e-12, atol=1e-13))


def pin_rotation_gdn(impl):
    """GDN: an orthogonal change of key basis R (q -> Rq, k -> Rk, S0 -> S0 R^T)
    leaves o unchanged and maps the final state to S R^T."""
    q, k, v, alpha, beta, S0 = _rand_case(kda=False, dk=4, dv=3, rng=np.random.default_rng(10))
    R, _ = np.linalg.qr(np.random.default_rng(11).standard_normal((4, 4)))
    o1, s1 = impl(q, k, v, alpha, beta, S0)
    o2, s2 = impl(q @ R.T, k @ R.T, v, alpha, beta, S0 @ R.T)
    return bool(np.allclose(o1, o2, rtol=1e-12, atol=1e-12) and
                np.allclose(s1 @ R.T, s2, rtol=1e-12, atol=1e-12))


def pin_linearity(impl):
    """For fixed q, k, gates and beta the map (S0, V) -> (O, S_T) is linear."""
    rng = np.random.default_rng(12)
    q, k, v1, alpha, beta, S1 = _rand_case(kda=True, rng=rng)
    v2 = rng.standard_normal(v1.shape)
    S2 = rng.standard_normal(S1.shape)
    c = -1.75
    oa, sa = impl(q, k, v1, alpha, beta, S1)
    ob, sb = impl(q, k, v2, alpha, beta, S2)
    oc, sc = impl(q, k, v1 + c * v2, alpha, beta, S1 + c * S2)
    return bool(np.allclose(oc, oa + c * ob, rtol=1e-12, atol=1e-12) and
                np.allclose(sc, sa + c * sb, rtol=1e-12, atol=1e-12))


PINS = [pin_hand_case, pin_rational_bruteforce, pin_identity, pin_readback,
        pin_alpha0_beta1, pin_pure_decay, pin_kda_equal_gates_is_gdn,
        pin_channel_permutation, pin_rotation_gdn, pin_linearity]


def _oracle(q, k, v, alpha, beta, s0):
    return gated_delta_rule(q, k, v, alpha, beta, s0)


def _chunked16(q, k, v, alpha, beta, s0):
    return chunked_gated_delta_rule(q, k, v, alpha, beta, s0, chunk=4)


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    assert pin(_oracle)


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_chunked_restatement_pin(pin):
    assert pin(_chunked16)


# --------------------------------------------------------------------------------------
# planted mistakes: each mutant is the recurrence with one plausible slip
# --------------------------------------------------------------------------------------

def _mutant(kind):
    def run(q, k, v, alpha, beta, s0):
        q, k, v, alpha, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, alpha, beta))
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        a4 = alpha if alpha.ndim == 4 else np.broadcast_to(alpha[..., None], (B, T, H, dk))
        S = np.zeros((B, H, dv, dk)) if s0 is None else np.array(s0, dtype=np.float64)
        o = np.empty((B, T, H, dv))
        for t in range(T):
            a = a4[:, t]
            kt, vt, bt = k[:, t], v[:, t], beta[:, t][..., None]
            if kind == "gate_on_rows" and dk == dv:
                St = S * a[..., :, None]
            elif kind == "gate_after_update":
                St = S
            elif kind == "gate_not_applied":
                St = S
            else:
                St = S * a[..., None, :]
            if kind == "transposed_read" and dk == dv:
                pred = np.einsum("bhvk,bhv->bhk", St, kt)
            elif kind == "pred_from_old_state":
                pred = np.einsum("bhvk,bhk->bhv", S, kt)
            else:
                pred = np.einsum("bhvk,bhk->bhv", St, kt)
            if kind == "beta_on_v_only":
                u = bt * vt - pred
            else:
                u = bt * (vt - pred)
            sign = -1.0 if kind == "sign_flip" else 1.0
            S_new = St + sign * u[..., :, None] * kt[..., None, :]
            if kind == "gate_after_update":
                S_new = S_new * a[..., None, :]
            if kind == "output_before_update":
                o[:, t] = np.einsum("bhvk,bhk->bhv", St, q[:, t])
            else:
                o[:, t] = np.einsum("bhvk,bhk->bhv", S_new, q[:, t])
            S = S_new
        return o, S
    return run


MUTANTS = ["gate_on_rows", "gate_after_update", "gate_not_applied", "transposed_read",
           "pred_from_old_state", "beta_on_v_only", "sign_flip", "output_before_update"]


def test_mutant_harness_is_faithful():
    """With no mistake planted the mutant harness is the recurrence itself."""
    assert all(pin(_mutant("none")) for pin in PINS)


@pytest.mark.parametrize("kind", MUTANTS)
def test_pins_catch_planted_mistake(kind):
    failed = [pin.__name__ for pin in PINS if not pin(_mutant(kind))]
    assert failed, f"no pin caught the planted mistake {kind!r}"


# --------------------------------------------------------------------------------------
# chunk algebra and state carry
# --------------------------------------------------------------------------------------

@pytest.mark.parametrize("kda", [False, True])
@pytest.mark.parametrize("T,chunk", [(64, 64), (200, 64), (200, 16), (37, 8), (1, 64)])
@pytest.mark.parametrize("gates", ["mixed", "slow", "zeros"])
def test_chunked_equals_sequential(kda, T, chunk, gates):
    rng = np.random.default_rng(T * 7 + chunk + kda)
    q, k, v, alpha, beta, S0 = _rand_case(B=1, T=T, H=2, dk=8, dv=6, kda=kda, rng=rng)
    if gates == "slow":
        alpha = 0.995 + 0.005 * rng.random(alpha.shape)
    elif gates == "zeros":
        alpha[:, ::5] = 0.0
    o1, s1 = gated_delta_rule(q, k, v, alpha, beta, S0)
    o2, s2 = chunked_gated_delta_rule(q, k, v, alpha, beta, S0, chunk=chunk)
    assert np.linalg.norm(o1 - o2) <= 1e-12 * np.linalg.norm(o1)
    assert np.linalg.norm(s1 - s2) <= 1e-12 * np.linalg.norm(s1)


@pytest.mark.parametrize("kda", [False, True])
def test_split_composition(kda):
    """run(T1) then run(T2 from that state) equals run(T1 + T2)."""
    q, k, v, alpha, beta, S0 = _rand_case(B=2, T=23, H=2, kda=kda, rng=np.random.default_rng(21))
    o, s = gated_delta_rule(q, k, v, alpha, beta, S0)
    t1 = 10
    oa, sa = gated_delta_rule(q[:, :t1], k[:, :t1], v[:, :t1], alpha[:, :t1], beta[:, :t1], S0)
    ob, sb = gated_delta_rule(q[:, t1:], k[:, t1:], v[:, t1:], alpha[:, t1:], beta[:, t1:], sa)
    assert np.allclose(np.concatenate([oa, ob], axis=1), o, rtol=1e-14, atol=1e-14)
    assert np.allclose(sb, s, rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("kda", [False, True])
def test_decode_steps_equal_prefill(kda):
    """Feeding tokens one at a time through decode_step equals one prefill."""
    q, k, v, alpha, beta, S0 = _rand_case(B=3, T=6, H=2, kda=kda, rng=np.random.default_rng(22))
    o, s = gated_delta_rule(q, k, v, alpha, beta, S0)
    st = S0
    for t in range(q.shape[1]):
        ot, st = decode_step(q[:, t], k[:, t], v[:, t], alpha[:, t], beta[:, t], st)
        assert np.allclose(ot, o[:, t], rtol=1e-14, atol=1e-14)
    assert np.allclose(st, s, rtol=1e-14, atol=1e-14)


def test_state_size_independent_of_length():
    """The state is a fixed d_v x d_k matrix per head whatever the prefix length."""
    for T in (1, 10, 100):
        q, k, v, alpha, beta, S0 = _rand_case(B=1, T=T, H=2, dk=4, dv=3,
                                              rng=np.random.default_rng(T))
        _, s = gated_delta_rule(q, k, v, alpha, beta, S0)
        assert s.shape == (1, 2, 3, 4)


def test_decode_does_not_modify_input_state():
    q, k, v, alpha, beta, S0 = _rand_case(B=2, T=1, H=2, rng=np.random.default_rng(23))
    keep = S0.copy()
    decode_step(q[:, 0], k[:, 0], v[:, 0], alpha[:, 0], beta[:, 0], S0)
    assert np.array_equal(S0, keep)


# --------------------------------------------------------------------------------------
# verify_steps: K tokens from a carried state with the state after each token

from oracle import verify_steps  # noqa: E402


def _verify_case(kda, N=2, K=5, H=3, dk=4, dv=3, seed=31, **kw):
    q, k, v, alpha, beta, S0 = _rand_case(B=N, T=K, H=H, dk=dk, dv=dv, kda=kda,
                                          rng=np.random.default_rng(seed), **kw)
    return q, k, v, alpha, beta, S0


@pytest.mark.parametrize("kda", [False, True])
def test_verify_snapshots_match_the_chunked_restatement(kda):
    """Snapshot t is the state after the first t+1 tokens, and the outputs are those
    of the same run: checked against the independent chunk-wise code."""
    q, k, v, alpha, beta, S0 = _verify_case(kda)
    o, snaps = verify_steps(q, k, v, alpha, beta, S0)
    assert o.shape == (2, 5, 3, 3) and snaps.shape == (5, 2, 3, 3, 4)
    for t in range(q.shape[1]):
        oc, sc = chunked_gated_delta_rule(q[:, :t + 1], k[:, :t + 1], v[:, :t + 1],
                                          alpha[:, :t + 1], beta[:, :t + 1], S0, chunk=4)
        assert np.allclose(snaps[t], sc, rtol=1e-12, atol=1e-12)
        assert np.allclose(o[:, :t + 1], oc, rtol=1e-12, atol=1e-12)


def test_verify_identity_gates_keep_the_state():
    """alpha = 1, beta = 0: every snapshot is S0 and o_t = S0 q_t exactly."""
    q, k, v, alpha, beta, S0 = _verify_case(True)
    alpha = np.ones_like(alpha)
    beta = np.zeros_like(beta)
    o, snaps = verify_steps(q, k, v, alpha, beta, S0)
    for t in range(q.shape[1]):
        assert np.array_equal(snaps[t], S0)
        assert np.allclose(o[:, t], np.einsum("nhvk,nhk->nhv", S0, q[:, t]), rtol=0, atol=1e-14)


@pytest.mark.parametrize("kda", [False, True])
def test_verify_read_back_after_every_token(kda):
    """beta = 1 and unit k: the state after token t maps k_t to v_t, whatever the gates."""
    q, k, v, alpha, beta, S0 = _verify_case(kda, seed=32)
    beta = np.ones_like(beta)
    _, snaps = verify_steps(q, k, v, alpha, beta, S0)
    for t in range(q.shape[1]):
        assert np.allclose(np.einsum("nhvk,nhk->nhv", snaps[t], k[:, t]), v[:, t], atol=1e-12)


def test_verify_pins_catch_an_off_by_one_snapshot():
    """A planted mistake (recording the state before each token instead of after it)
    fails the read-back pin."""
    q, k, v, alpha, beta, S0 = _verify_case(False, seed=33)
    beta = np.ones_like(beta)
    _, snaps = verify_steps(q, k, v, alpha, beta, S0)
    wrong = np.concatenate([S0[None], snaps[:-1]], axis=0)
    ok = all(np.allclose(np.einsum("nhvk,nhk->nhv", wrong[t], k[:, t]), v[:, t], atol=1e-12)
             for t in range(q.shape[1]))
    assert not ok


def test_verify_leaves_the_input_state():
    q, k, v, alpha, beta, S0 = _verify_case(True, seed=34)
    keep = S0.copy()
    verify_steps(q, k, v, alpha, beta, S0)
    assert np.array_equal(S0, keep)


# --------------------------------------------------------------------------------------
# prefill_varlen: packed sequences of different lengths with a pool of state slots

from oracle import prefill_varlen  # noqa: E402


def _varlen_case(kda, lens, H=2, dk=4, dv=3, nslots=None, seed=41):
    rng = np.random.default_rng(seed)
    total = sum(lens)
    q = rng.standard_normal((total, H, dk))
    k = rng.standard_normal((total, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((total, H, dv))
    alpha = rng.uniform(0.2, 1.0, size=(total, H, dk) if kda else (total, H))
    beta = rng.uniform(0.1, 1.0, size=(total, H))
    pool = rng.standard_normal((nslots or len(lens), H, dv, dk))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    return q, k, v, alpha, beta, cu, pool


@pytest.mark.parametrize("kda", [False, True])
def test_varlen_equal_lengths_is_the_batched_call(kda):
    """nseq sequences of T tokens each, slot i: the same as one [nseq, T] batch."""
    q, k, v, alpha, beta, cu, pool = _varlen_case(kda, [5, 5, 5])
    o, new = prefill_varlen(q, k, v, alpha, beta, cu, pool)
    sh = lambda x: x.reshape((3, 5) + x.shape[1:])  # noqa: E731
    ob, sb = gated_delta_rule(sh(q), sh(k), sh(v), sh(alpha), sh(beta), pool)
    assert np.allclose(o, ob.reshape(o.shape), rtol=1e-14, atol=1e-14)
    assert np.allclose(new, sb, rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("kda", [False, True])
def test_varlen_ragged_matches_the_chunked_restatement(kda):
    """Ragged lengths (including an empty sequence) and permuted slots, against the
    independent chunk-wise code run sequence by sequence."""
    lens = [7, 0, 1, 12, 4]
    slots = [5, 0, 2, 1, 3]
    q, k, v, alpha, beta, cu, pool = _varlen_case(kda, lens, nslots=7, seed=42)
    o, new = prefill_varlen(q, k, v, alpha, beta, cu, pool, slots)
    for i, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        s = slots[i]
        if a == b:
            assert np.array_equal(new[s], pool[s])
            continue
        oc, sc = chunked_gated_delta_rule(q[None, a:b], k[None, a:b], v[None, a:b],
                                          alpha[None, a:b], beta[None, a:b], pool[s][None],
                                          chunk=4)
        assert np.allclose(o[a:b], oc[0], rtol=1e-12, atol=1e-12)
        assert np.allclose(new[s], sc[0], rtol=1e-12, atol=1e-12)
    for s in (4, 6):                       # slots no sequence uses are left alone
        assert np.array_equal(new[s], pool[s])


def test_varlen_sequences_do_not_leak_into_each_other():
    """Changing one sequence's tokens changes no other sequence's outputs or state."""
    q, k, v, alpha, beta, cu, pool = _varlen_case(True, [6, 9, 3], seed=43)
    o1, s1 = prefill_varlen(q, k, v, alpha, beta, cu, pool)
    v2 = v.copy()
    v2[6:15] += 1.0                        # sequence 1 only
    o2, s2 = prefill_varlen(q, k, v2, alpha, beta, cu, pool)
    assert np.array_equal(o1[:6], o2[:6]) and np.array_equal(o1[15:], o2[15:])
    assert np.array_equal(s1[0], s2[0]) and np.array_equal(s1[2], s2[2])
    assert not np.allclose(s1[1], s2[1])
