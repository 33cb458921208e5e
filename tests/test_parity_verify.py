"""GPU multi-token verify (K tokens from a carried state, the state after each token
kept) vs the fp64 oracle, through the C ABI (via the ctypes binding)."""

import numpy as np
import pytest
import torch

from oracle import verify_steps
from synth import WORKLOADS, Workload, device_inputs, make_inputs, slice_inputs
from _util import check_elem, rel_err, slice_errs, to_np

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-3}


def _fn(mixer):
    import gated_delta_rule_79_b200 as g
    return g.kda_verify if mixer == "kda" else g.gdn_verify


def _ref(x):
    return verify_steps(*[x[k].double().numpy() for k in ("q", "k", "v", "alpha", "beta")],
                        x["s0"].double().numpy())


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 32), (32, 128)])
@pytest.mark.parametrize("K", [1, 3, 16])
def test_verify_snapshots(mixer, dtype, dk, dv, K):
    """Outputs (fp32) and every snapshot; the input state is left unchanged."""
    w = Workload("ver", mixer, 5, 3, K, dk, dv, dtype, "randn")
    x = make_inputs(w, seed=K + dk)
    dev = torch.device("cuda")
    t = {k: v.to(dev) for k, v in x.items()}
    keep = t["s0"].clone()
    o, snaps = _fn(mixer)(t["q"], t["k"], t["v"], t["alpha"], t["beta"], t["s0"],
                          out_dtype=torch.float32)
    torch.cuda.synchronize()
    o_ref, s_ref = _ref(x)
    eo = slice_errs(to_np(o), o_ref, axes=(0, 2))
    es = max(slice_errs(to_np(snaps[i]), s_ref[i], axes=(0, 1)) for i in range(K))
    print(f"{mixer} {dtype} {dk}x{dv} K={K}: o {eo:.2e} snapshots {es:.2e}")
    assert eo <= TOL[dtype] and es <= TOL[dtype]
    check_elem(to_np(o), o_ref, "cc", axes=(0, 2), label="o")
    for i in range(K):
        check_elem(to_np(snaps[i]), s_ref[i], "cc", axes=(0, 1), label=f"snapshot {i}")
    assert torch.equal(t["s0"], keep)


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
@pytest.mark.parametrize("K", [2, 7])
def test_verify_in_place(mixer, K):
    """Without a snapshot buffer the state is advanced in place by the K tokens."""
    w = Workload("ver", mixer, 4, 2, K, 128, 64, "bf16", "randn")
    x = make_inputs(w, seed=40 + K)
    dev = torch.device("cuda")
    t = {k: v.to(dev) for k, v in x.items()}
    o, snaps = _fn(mixer)(t["q"], t["k"], t["v"], t["alpha"], t["beta"], t["s0"],
                          snapshots=False)
    torch.cuda.synchronize()
    assert snaps is None and o.dtype == torch.bfloat16
    o_ref, s_ref = _ref(x)
    assert rel_err(to_np(o), o_ref) <= TOL["bf16"]
    assert rel_err(to_np(t["s0"]), s_ref[-1]) <= TOL["bf16"]
    check_elem(to_np(o), o_ref, "cc", axes=(0, 2), bf16_out=True, label="o")
    check_elem(to_np(t["s0"]), s_ref[-1], "cc", axes=(0, 1), label="state")


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
def test_verify_workload_sampled(mixer):
    """256 sequences x 32 heads, d = 128, K = 4 at full size; sampled (sequence, head)
    chains are drawn on the CPU and checked (outputs and all snapshots)."""
    w = WORKLOADS[f"verify_{mixer}"]
    dev = torch.device("cuda")
    full = device_inputs(w, dev, seed=9)
    picks = [(0, 0), (77, 13), (255, 31)]
    parts = [slice_inputs(w, n, h) for n, h in picks]
    for (n, h), p in zip(picks, parts):
        for key in ("q", "k", "v", "beta", "alpha"):
            full[key][n, :, h] = p[key].to(dev)
        full["s0"][n, h] = p["s0"].to(dev)
    o, snaps = _fn(mixer)(full["q"], full["k"], full["v"], full["alpha"], full["beta"],
                          full["s0"])
    torch.cuda.synchronize()
    for (n, h), p in zip(picks, parts):
        args = [p[k].double().numpy()[None, :, None] for k in ("q", "k", "v", "alpha", "beta")]
        o_ref, s_ref = verify_steps(*args, p["s0"].double().numpy()[None, None])
        eo = rel_err(to_np(o[n, :, h]), o_ref[0, :, 0])
        es = rel_err(to_np(snaps[:, n, h]), s_ref[:, 0, 0])
        print(f"{mixer} verify ({n}, {h}): o {eo:.2e} snapshots {es:.2e}")
        assert eo <= TOL["bf16"] and es <= TOL["bf16"]
        check_elem(to_np(o[n, :, h]), o_ref[0, :, 0], "cc", bf16_out=o.dtype == torch.bfloat16,
                   label=f"({n}, {h}) o")
        for i in range(w.T):
            check_elem(to_np(snaps[i, n, h]), s_ref[i, 0, 0], "cc", label=f"({n}, {h}) snap {i}")


def test_verify_rejects_bad_token_counts():
    import gated_delta_rule_79_b200 as g
    w = Workload("ver", "gdn", 2, 2, 17, 64, 64, "bf16", "randn")
    x = {k: v.cuda() for k, v in make_inputs(w, seed=1).items()}
    with pytest.raises(g.GdrError) as e:
        g.gdn_verify(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["s0"])
    assert e.value.status == g.GDR_ERR_UNSUPPORTED


def test_verify_empty_batch():
    import gated_delta_rule_79_b200 as g
    w = Workload("ver", "kda", 0, 2, 3, 64, 64, "bf16", "randn")
    dev = torch.device("cuda")
    q = torch.zeros((0, 3, 2, 64), dtype=torch.bfloat16, device=dev)
    a = torch.zeros((0, 3, 2, 64), device=dev)
    b = torch.zeros((0, 3, 2), device=dev)
    s = torch.zeros((0, 2, 64, 64), device=dev)
    o, snaps = g.kda_verify(q, q, q, a, b, s)
    assert o.shape == (0, 3, 2, 64) and snaps.shape == (3, 0, 2, 64, 64)
    del w
