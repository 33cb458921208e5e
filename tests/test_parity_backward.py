"""GPU gradients (gdn_backward / kda_backward) vs the fp64 backward oracle, through the
C ABI (via the ctypes binding): dq, dk, dv, dalpha, dbeta and ds0 element by element,
normwise.  Inputs as bf16 are upcast exactly on both sides, so the only difference is
the kernel's fp32 arithmetic."""

import numpy as np
import pytest
import torch

from oracle import gated_delta_rule_backward
from synth import WORKLOADS, Workload, device_inputs, make_inputs, slice_inputs
from _util import check_elem, rel_err, to_np

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-3}
NAMES = ("dq", "dk", "dv", "dalpha", "dbeta", "ds0")


def _grads_in(x, seed, do_dtype=torch.float32, final=True):
    g = torch.Generator().manual_seed(seed)
    B, T, H, _ = x["q"].shape
    dv, dk = x["v"].shape[-1], x["q"].shape[-1]
    do = torch.randn((B, T, H, dv), generator=g).to(do_dtype)
    dsf = torch.randn((B, H, dv, dk), generator=g) if final else None
    return do, dsf


def _run(mixer, x, do, dsf):
    import gated_delta_rule_79_b200 as gg
    fn = gg.kda_backward if mixer == "kda" else gg.gdn_backward
    t = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
    out = fn(t["q"], t["k"], t["v"], t["alpha"], t["beta"], t["s0"], do.cuda(),
             None if dsf is None else dsf.cuda())
    torch.cuda.synchronize()
    return [to_np(o) for o in out]


def _ref(x, do, dsf):
    args = [x[k].double().numpy() for k in ("q", "k", "v", "alpha", "beta")]
    s0 = None if x["s0"] is None else x["s0"].double().numpy()
    return gated_delta_rule_backward(*args, s0, do.double().numpy(),
                                     None if dsf is None else dsf.double().numpy())


# per-(batch, head) slicing of each gradient for the element-wise bound: the token
# tensors [B, T, H, ...] over (0, 2), ds0 [B, H, d_v, d_k] over (0, 1)
AXES = ((0, 2), (0, 2), (0, 2), (0, 2), (0, 2), (0, 1))


def _check(got, ref, tol, label, axes=AXES):
    errs = {n: rel_err(a, b) for n, a, b in zip(NAMES, got, ref)}
    print(label, " ".join(f"{n} {e:.1e}" for n, e in errs.items()))
    assert all(e <= tol for e in errs.values()), errs
    for n, a, b, ax in zip(NAMES, got, ref, axes):
        check_elem(a, b, "cc", axes=ax, label=f"{label} {n}")


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 64), (128, 128), (64, 128), (128, 32)])
@pytest.mark.parametrize("T", [1, 65, 200])
def test_small_shapes(mixer, dtype, dk, dv, T):
    w = Workload("bw", mixer, 2, 2, T, dk, dv, dtype, "randn")
    x = make_inputs(w, seed=T + dk + dv)
    do, dsf = _grads_in(x, seed=T)
    _check(_run(mixer, x, do, dsf), _ref(x, do, dsf), TOL[dtype],
           f"{mixer} {dtype} {dk}x{dv} T={T}")


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
@pytest.mark.parametrize("gates", ["slow", "one", "zero_some"])
def test_stress_gates(mixer, gates):
    """Gates that keep the state alive across chunks (and zero gates)."""
    w = Workload("bws", mixer, 1, 3, 300, 128, 128, "bf16", "randn")
    x = make_inputs(w, seed=5, gates=gates)
    do, dsf = _grads_in(x, seed=6, do_dtype=torch.bfloat16)
    _check(_run(mixer, x, do, dsf), _ref(x, do, dsf), TOL["bf16"], f"{mixer} gates={gates}")


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
def test_no_state_no_final_gradient(mixer):
    w = Workload("bw0", mixer, 2, 2, 70, 64, 64, "bf16", "zeros")
    x = make_inputs(w, seed=2)
    do, _ = _grads_in(x, seed=4, final=False)
    _check(_run(mixer, x, do, None), _ref(x, do, None), TOL["bf16"], f"{mixer} no state")


def test_zero_tokens_pass_the_final_gradient_through():
    import gated_delta_rule_79_b200 as gg
    dev = torch.device("cuda")
    q = torch.zeros((2, 0, 3, 64), dtype=torch.bfloat16, device=dev)
    a = torch.zeros((2, 0, 3), device=dev)
    do = torch.zeros((2, 0, 3, 64), device=dev)
    dsf = torch.randn((2, 3, 64, 64), device=dev)
    out = gg.gdn_backward(q, q, q, a, a, None, do, dsf)
    torch.cuda.synchronize()
    assert torch.equal(out[5], dsf)
    out = gg.gdn_backward(q, q, q, a, a, None, do, None)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out[5]) == 0


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
def test_deterministic(mixer):
    """No atomics: two calls give the same bits."""
    w = Workload("bwd", mixer, 1, 4, 130, 128, 128, "bf16", "randn")
    x = make_inputs(w, seed=9)
    do, dsf = _grads_in(x, seed=10)
    a = _run(mixer, x, do, dsf)
    b = _run(mixer, x, do, dsf)
    assert all(np.array_equal(u, v) for u, v in zip(a, b))


@pytest.mark.parametrize("name", ["gdn_prefill", "kda_prefill"])
def test_full_workload_sampled(name):
    """The full 32-head, 4096-token workload in one call; sampled heads are redrawn on
    the CPU and checked (all six gradients of those heads)."""
    import gated_delta_rule_79_b200 as gg
    w = WORKLOADS[name]
    dev = torch.device("cuda")
    x = device_inputs(w, dev, seed=3)
    gen = torch.Generator(device=dev).manual_seed(4)
    do = torch.randn((w.B, w.T, w.H, w.dv), generator=gen, device=dev).to(torch.bfloat16)
    dsf = torch.randn((w.B, w.H, w.dv, w.dk), generator=gen, device=dev)
    picks = [0, 21]
    ref_in = {}
    for h in picks:
        p = slice_inputs(w, 0, h, seed=3)
        for key in ("q", "k", "v", "beta", "alpha"):
            x[key][0, :, h] = p[key].to(dev)
        ref_in[h] = p
    fn = gg.kda_backward if w.mixer == "kda" else gg.gdn_backward
    out = fn(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["s0"], do, dsf)
    torch.cuda.synchronize()
    for h in picks:
        p = ref_in[h]
        args = [p[key].double().numpy()[None, :, None] for key in ("q", "k", "v", "alpha", "beta")]
        s0 = None if x["s0"] is None else x["s0"][0, h].double().cpu().numpy()[None, None]
        ref = gated_delta_rule_backward(*args, s0, to_np(do[0, :, h])[None, :, None],
                                        to_np(dsf[0, h])[None, None])
        got = [to_np(out[0][0, :, h]), to_np(out[1][0, :, h]), to_np(out[2][0, :, h]),
               to_np(out[3][0, :, h]), to_np(out[4][0, :, h]), to_np(out[5][0, h])]
        ref = [r[0, :, 0] if i < 5 else r[0, 0] for i, r in enumerate(ref)]
        _check(got, ref, TOL["bf16"], f"{name} head {h}", axes=((),) * 6)


def test_rejects_unsupported_and_missing_workspace():
    import gated_delta_rule_79_b200 as gg
    w = Workload("bwx", "gdn", 1, 1, 10, 96, 64, "f32", "randn")
    dev = torch.device("cuda")
    q = torch.zeros((1, 10, 1, 96), device=dev)
    v = torch.zeros((1, 10, 1, 64), device=dev)
    a = torch.ones((1, 10, 1), device=dev)
    with pytest.raises(gg.GdrError) as e:
        gg.gdn_backward(q, q, v, a, a, None, v)
    assert e.value.status == gg.GDR_ERR_UNSUPPORTED
    q = torch.zeros((1, 10, 1, 64), device=dev)
    with pytest.raises(gg.GdrError) as e:
        gg.gdn_backward(q, q, v, a, a, None, v,
                        workspace=torch.empty(16, dtype=torch.uint8, device=dev))
    assert e.value.status == gg.GDR_ERR_INVALID_ARG
    del w
