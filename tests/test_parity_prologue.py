"""GPU fused prologue (raw q, k L2-normalised in the kernels; the gate formed from its
logit) vs the oracle: oracle.apply_prologue on the same raw inputs, then the fp64
recurrence.  Through the C ABI's *_ex entry points (via the ctypes binding)."""

import numpy as np
import pytest
import torch

from oracle import apply_prologue, gated_delta_rule, prefill_varlen, verify_steps
from _util import check_elem, rel_err, slice_errs, to_np

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-3}
BOTH = 3   # PROLOGUE_L2NORM_QK | PROLOGUE_GATE_LOGIT


def raw_inputs(mixer, lead, H, dk, dv, dtype, seed, state=True):
    """q, k ~ N(0,1) times a log-normal scale per vector (not normalised), v ~ N(0,1),
    beta = sigmoid(N(0,1)), gate logits x = N(0,1) + 2 (the workload gates are
    exp(-softplus(x)) of exactly this), s0 ~ 0.02 N(0,1)."""
    g = torch.Generator().manual_seed(seed)
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    lead = tuple(lead)
    sc = lambda: torch.exp(torch.randn(lead + (H, 1), generator=g))  # noqa: E731
    q = (torch.randn(lead + (H, dk), generator=g) * sc()).to(td)
    k = (torch.randn(lead + (H, dk), generator=g) * sc()).to(td)
    v = torch.randn(lead + (H, dv), generator=g).to(td)
    beta = torch.sigmoid(torch.randn(lead + (H,), generator=g))
    x = torch.randn(lead + ((H, dk) if mixer == "kda" else (H,)), generator=g) + 2.0
    return dict(q=q, k=k, v=v, beta=beta, alpha=x)


def cls_of(mixer, dtype, dk, dv):
    """Precision class of the prefill kernel these parameters select (tests/_util.py);
    with bf16 inputs the CUDA-core paths read q, k that both sides normalised and
    rounded to bf16 on their own, so they take the "pro" bound."""
    import gated_delta_rule_79_b200 as g
    if dtype == "f32":
        return "f32"
    return ("tc" if g.prefill_path(dk, dv, torch.bfloat16, mixer == "kda") == "tensor-core"
            else "pro")


def prepared(x, dtype, flags):
    q, k, a = apply_prologue(x["q"].double().numpy(), x["k"].double().numpy(),
                             x["alpha"].double().numpy(), l2norm=bool(flags & 1),
                             gate_logit=bool(flags & 2), bf16=(dtype == "bf16"))
    return q, k, x["v"].double().numpy(), a, x["beta"].double().numpy()


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("bf16", 128, 32), ("bf16", 64, 64),
                                         ("f32", 128, 128), ("f32", 32, 64)])
@pytest.mark.parametrize("flags", [BOTH, 1, 2])
def test_prefill(mixer, dtype, dk, dv, flags):
    import gated_delta_rule_79_b200 as g
    B, T, H = 2, 200, 3
    x = raw_inputs(mixer, (B, T), H, dk, dv, dtype, seed=dk + dv + flags)
    if not flags & 1:   # the kernel then takes q, k as given: hand it normalised ones
        x["q"] = torch.from_numpy(prepared(x, dtype, 1)[0]).to(x["q"].dtype)
        x["k"] = torch.from_numpy(prepared(x, dtype, 1)[1]).to(x["k"].dtype)
    if not flags & 2:   # ... and the gate itself, not its logit
        x["alpha"] = torch.from_numpy(prepared(x, dtype, 2)[3]).float()
    s0 = 0.02 * torch.randn((B, H, dv, dk), generator=torch.Generator().manual_seed(1))
    fn = g.kda_prefill if mixer == "kda" else g.gdn_prefill
    t = {k_: v_.cuda() for k_, v_ in x.items()}
    o, s = fn(t["q"], t["k"], t["v"], t["alpha"], t["beta"], s0.cuda(), out_dtype=torch.float32,
              prologue=flags)
    torch.cuda.synchronize()
    o_ref, s_ref = gated_delta_rule(*prepared(x, dtype, flags), s0.double().numpy())
    eo, es = rel_err(to_np(o), o_ref), rel_err(to_np(s), s_ref)
    print(f"{mixer} {dtype} {dk}x{dv} flags={flags}: o {eo:.2e} s {es:.2e}")
    assert eo <= TOL[dtype] and es <= TOL[dtype]
    cls = cls_of(mixer, dtype, dk, dv)
    if cls == "pro" and not flags & 1:
        cls = "cc"      # q, k given normalised: nothing is rounded on either side
    check_elem(to_np(o), o_ref, cls, axes=(0, 2), label="o")
    check_elem(to_np(s), s_ref, cls, axes=(0, 1), label="s")


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
def test_prefill_small_workspace_runs_the_cuda_core_kernel(mixer):
    """With only the status word as workspace the prologue runs in the CUDA-core kernel
    (the single-kernel tensor-core fallbacks do not carry it)."""
    import gated_delta_rule_79_b200 as g
    x = raw_inputs(mixer, (1, 130), 2, 128, 128, "bf16", seed=4)
    fn = g.kda_prefill if mixer == "kda" else g.gdn_prefill
    t = {k_: v_.cuda() for k_, v_ in x.items()}
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    o, s = fn(t["q"], t["k"], t["v"], t["alpha"], t["beta"], None, out_dtype=torch.float32,
              workspace=ws, prologue=BOTH)
    torch.cuda.synchronize()
    g.workspace_status(ws)
    o_ref, s_ref = gated_delta_rule(*prepared(x, "bf16", BOTH), None)
    assert rel_err(to_np(o), o_ref) <= TOL["bf16"] and rel_err(to_np(s), s_ref) <= TOL["bf16"]
    check_elem(to_np(o), o_ref, "pro", axes=(0, 2), label="o")
    check_elem(to_np(s), s_ref, "pro", axes=(0, 1), label="s")


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 64, 32)])
def test_decode(mixer, dtype, dk, dv):
    import gated_delta_rule_79_b200 as g
    N, H = 6, 3
    x = raw_inputs(mixer, (N,), H, dk, dv, dtype, seed=dk + 7)
    state = 0.02 * torch.randn((N, H, dv, dk), generator=torch.Generator().manual_seed(2))
    st = state.cuda()
    fn = g.kda_decode if mixer == "kda" else g.gdn_decode
    t = {k_: v_.cuda() for k_, v_ in x.items()}
    o = fn(t["q"], t["k"], t["v"], t["alpha"], t["beta"], st, out_dtype=torch.float32,
           prologue=BOTH)
    torch.cuda.synchronize()
    q, k, v, a, b = prepared(x, dtype, BOTH)
    o_ref, s_ref = gated_delta_rule(q[:, None], k[:, None], v[:, None], a[:, None], b[:, None],
                                    state.double().numpy())
    assert rel_err(to_np(o), o_ref[:, 0]) <= TOL[dtype]
    assert rel_err(to_np(st), s_ref) <= TOL[dtype]
    cls = "f32" if dtype == "f32" else "pro"
    check_elem(to_np(o), o_ref[:, 0], cls, axes=(0, 1), label="o")
    check_elem(to_np(st), s_ref, cls, axes=(0, 1), label="s")


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
def test_verify(mixer):
    import gated_delta_rule_79_b200 as g
    N, K, H = 4, 3, 2
    x = raw_inputs(mixer, (N, K), H, 128, 64, "bf16", seed=9)
    state = 0.02 * torch.randn((N, H, 64, 128), generator=torch.Generator().manual_seed(3))
    fn = g.kda_verify if mixer == "kda" else g.gdn_verify
    t = {k_: v_.cuda() for k_, v_ in x.items()}
    o, snaps = fn(t["q"], t["k"], t["v"], t["alpha"], t["beta"], state.cuda(),
                  out_dtype=torch.float32, prologue=BOTH)
    torch.cuda.synchronize()
    o_ref, s_ref = verify_steps(*prepared(x, "bf16", BOTH), state.double().numpy())
    assert slice_errs(to_np(o), o_ref, axes=(0, 2)) <= TOL["bf16"]
    assert max(rel_err(to_np(snaps[i]), s_ref[i]) for i in range(K)) <= TOL["bf16"]
    check_elem(to_np(o), o_ref, "pro", axes=(0, 2), label="o")
    for i in range(K):
        check_elem(to_np(snaps[i]), s_ref[i], "pro", axes=(0, 1), label=f"snapshot {i}")


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
def test_varlen(mixer):
    import gated_delta_rule_79_b200 as g
    lens = [70, 0, 1, 129, 64]
    H, dv = 2, 128
    total = sum(lens)
    x = raw_inputs(mixer, (total,), H, 128, dv, "bf16", seed=12)
    pool0 = 0.02 * torch.randn((5, H, dv, 128), generator=torch.Generator().manual_seed(5))
    pool = pool0.cuda()
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    fn = g.kda_prefill_varlen if mixer == "kda" else g.gdn_prefill_varlen
    t = {k_: v_.cuda() for k_, v_ in x.items()}
    o = fn(t["q"], t["k"], t["v"], t["alpha"], t["beta"], cu.cuda(), pool,
           out_dtype=torch.float32, prologue=BOTH)
    torch.cuda.synchronize()
    o_ref, p_ref = prefill_varlen(*prepared(x, "bf16", BOTH), cu.numpy(), pool0.double().numpy())
    assert rel_err(to_np(o), o_ref) <= TOL["bf16"]
    assert rel_err(to_np(pool), p_ref) <= TOL["bf16"]
    check_elem(to_np(o), o_ref, "tc", axes=(1,), label="o")
    check_elem(to_np(pool), p_ref, "tc", axes=(0, 1), label="pool")


def test_unknown_flags_are_rejected():
    import gated_delta_rule_79_b200 as g
    x = raw_inputs("gdn", (1, 8), 1, 64, 64, "bf16", seed=1)
    t = {k_: v_.cuda() for k_, v_ in x.items()}
    with pytest.raises(g.GdrError) as e:
        g.gdn_prefill(t["q"], t["k"], t["v"], t["alpha"], t["beta"], None, prologue=4)
    assert e.value.status == g.GDR_ERR_INVALID_ARG


@pytest.mark.parametrize("name", ["gdn_prefill_prologue", "kda_prefill_prologue"])
def test_full_workload_sampled(name):
    """The full 32-head, 4096-token prologue workload in one call (the bench's
    configuration); sampled heads are redrawn on the CPU and checked."""
    import gated_delta_rule_79_b200 as g
    from synth import WORKLOADS, device_inputs, slice_inputs
    w = WORKLOADS[name]
    dev = torch.device("cuda")
    x = device_inputs(w, dev, seed=5)
    picks = [3, 30]
    parts = {}
    for h in picks:
        p = slice_inputs(w, 0, h, seed=5)
        for key in ("q", "k", "v", "beta", "alpha"):
            x[key][0, :, h] = p[key].to(dev)
        parts[h] = p
    fn = g.kda_prefill if w.mixer == "kda" else g.gdn_prefill
    o, s = fn(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["s0"], prologue=w.prologue)
    torch.cuda.synchronize()
    for h in picks:
        p = parts[h]
        q, k, a = apply_prologue(p["q"].double().numpy(), p["k"].double().numpy(),
                                 p["alpha"].double().numpy(), bf16=True)
        col = lambda z: z[None, :, None]  # noqa: E731
        o_ref, s_ref = gated_delta_rule(col(q), col(k), col(p["v"].double().numpy()), col(a),
                                        col(p["beta"].double().numpy()), None)
        eo = rel_err(to_np(o[0, :, h]), o_ref[0, :, 0])
        es = rel_err(to_np(s[0, h]), s_ref[0, 0])
        print(f"{name} head {h}: o {eo:.2e} s {es:.2e}")
        assert eo <= TOL["bf16"] and es <= TOL["bf16"]
        check_elem(to_np(o[0, :, h]), o_ref[0, :, 0], "tc", bf16_out=o.dtype == torch.bfloat16,
                   label=f"head {h} o")
        check_elem(to_np(s[0, h]), s_ref[0, 0], "tc", label=f"head {h} s")
