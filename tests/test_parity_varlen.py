"""GPU packed variable-length prefill vs the fp64 oracle, through the C ABI (via the
ctypes binding): sequences of different lengths packed along the tokens, each run
from and back into its own slot of a state pool."""

import numpy as np
import pytest
import torch

from oracle import prefill_varlen
from synth import Workload, make_inputs
from _util import check_elem, rel_err, to_np

pytestmark = pytest.mark.gpu

TOL = 2e-3


def _packed(mixer, lens, H, dv, seed):
    """Each sequence drawn as its own slice of the workload recipe, then packed."""
    parts = [make_inputs(Workload("vl", mixer, 1, H, max(n, 1), 128, dv, "bf16", "randn"),
                         seed=seed + i) for i, n in enumerate(lens)]
    cat = lambda key: torch.cat([p[key][0, :n] for p, n in zip(parts, lens)])  # noqa: E731
    x = {key: cat(key) for key in ("q", "k", "v", "alpha", "beta")}
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    return x, cu


def _ref(x, cu, pool, slots):
    return prefill_varlen(*[x[k].double().numpy() for k in ("q", "k", "v", "alpha", "beta")],
                          cu.numpy(), pool.double().numpy(),
                          None if slots is None else slots.numpy())


def _run(mixer, x, cu, pool, slots, out_dtype=None):
    import gated_delta_rule_79_b200 as g
    fn = g.kda_prefill_varlen if mixer == "kda" else g.gdn_prefill_varlen
    d = {k: v.cuda() for k, v in x.items()}
    o = fn(d["q"], d["k"], d["v"], d["alpha"], d["beta"], cu.cuda(), pool,
           slots=None if slots is None else slots.cuda(), out_dtype=out_dtype)
    torch.cuda.synchronize()
    return o


@pytest.mark.parametrize("carry", ["chain", "rows", "sliced"])
@pytest.mark.parametrize("mixer", ["gdn", "kda"])
@pytest.mark.parametrize("dv", [128, 32])
def test_varlen_ragged(mixer, dv, carry, monkeypatch):
    """Lengths across the chunk edges (and an empty sequence), permuted slots in a pool
    with unused slots; outputs in fp32 and every slot checked, through either carry."""
    monkeypatch.setenv("GDR_CARRY", carry)
    lens = [70, 0, 1, 64, 129, 13, 200, 63]
    H = 3
    x, cu = _packed(mixer, lens, H, dv, seed=5)
    gen = torch.Generator().manual_seed(3)
    pool0 = 0.02 * torch.randn((11, H, dv, 128), generator=gen)
    slots = torch.tensor([4, 9, 0, 2, 7, 1, 10, 5], dtype=torch.int32)
    pool = pool0.cuda()
    o = _run(mixer, x, cu, pool, slots, out_dtype=torch.float32)
    o_ref, p_ref = _ref(x, cu, pool0, slots)
    for i in range(len(lens)):
        a, b = int(cu[i]), int(cu[i + 1])
        if b > a:
            eo = rel_err(to_np(o[a:b]), o_ref[a:b])
            assert eo <= TOL, (i, eo)
            check_elem(to_np(o[a:b]), o_ref[a:b], "tc", axes=(1,), label=f"sequence {i} o")
    for s in range(pool.shape[0]):
        es = rel_err(to_np(pool[s]), p_ref[s])
        assert es <= TOL, (s, es)
    check_elem(to_np(pool), p_ref, "tc", axes=(0, 1), label="pool")
    print(f"{mixer} dv={dv}: o {rel_err(to_np(o), o_ref):.2e} pool {rel_err(to_np(pool), p_ref):.2e}")


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
def test_varlen_equal_lengths_match_the_dense_call_bitwise(mixer):
    """Three sequences of 200 tokens packed: bit for bit what the dense [3, 200] call
    computes (the same chunks run through the same kernels)."""
    import gated_delta_rule_79_b200 as g
    w = Workload("vd", mixer, 3, 2, 200, 128, 128, "bf16", "randn")
    x = {k: v.cuda() for k, v in make_inputs(w, seed=8).items()}
    fn = g.kda_prefill if mixer == "kda" else g.gdn_prefill
    o_d, s_d = fn(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["s0"])
    flat = lambda t: t.reshape((600,) + t.shape[2:]).contiguous()  # noqa: E731
    pool = x["s0"].clone()
    cu = torch.tensor([0, 200, 400, 600], dtype=torch.int32, device="cuda")
    fv = g.kda_prefill_varlen if mixer == "kda" else g.gdn_prefill_varlen
    o_v = fv(flat(x["q"]), flat(x["k"]), flat(x["v"]), flat(x["alpha"]), flat(x["beta"]), cu,
             pool)
    torch.cuda.synchronize()
    assert torch.equal(o_v, flat(o_d))
    assert torch.equal(pool, s_d)


def test_varlen_bad_offsets_are_reported_and_nothing_runs():
    import gated_delta_rule_79_b200 as g
    x, cu = _packed("gdn", [10, 20], 2, 64, seed=9)
    bad = torch.tensor([0, 25, 20], dtype=torch.int32)       # decreasing pair
    pool = torch.randn((2, 2, 64, 128), device="cuda")
    keep = pool.clone()
    d = {k: v.cuda() for k, v in x.items()}
    need = g.lib.gdr_prefill_varlen_workspace_bytes(2, 30, 2, 128, 64, 0)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    g.gdn_prefill_varlen(d["q"], d["k"], d["v"], d["alpha"], d["beta"], bad.cuda(), pool,
                         workspace=ws)
    with pytest.raises(g.GdrError) as e:
        g.workspace_status(ws)
    assert e.value.status == g.GDR_ERR_INVALID_ARG
    assert torch.equal(pool, keep)
    # the same workspace then serves a good call
    g.gdn_prefill_varlen(d["q"], d["k"], d["v"], d["alpha"], d["beta"], cu.cuda(), pool,
                         workspace=ws)
    g.workspace_status(ws)


def test_varlen_rejects_unsupported_shapes():
    import gated_delta_rule_79_b200 as g
    x, cu = _packed("gdn", [5], 1, 64, seed=1)
    d = {k: v.cuda() for k, v in x.items()}
    pool = torch.zeros((1, 1, 64, 128), device="cuda")
    with pytest.raises(g.GdrError) as e:
        g.gdn_prefill_varlen(d["q"].float(), d["k"].float(), d["v"].float(), d["alpha"],
                             d["beta"], cu.cuda(), pool)
    assert e.value.status == g.GDR_ERR_UNSUPPORTED
