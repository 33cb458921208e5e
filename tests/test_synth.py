"""The seeded input generator: determinism, shapes, dtypes and the workload recipe."""

import torch

from synth import WORKLOADS, make_inputs, slice_inputs


def test_slices_are_deterministic_and_distinct():
    w = WORKLOADS["gdn_seq_f32"]
    a = slice_inputs(w, 0, 0)
    b = slice_inputs(w, 0, 0)
    c = slice_inputs(w, 0, 1)
    for key in ("q", "k", "v", "beta", "alpha"):
        assert torch.equal(a[key], b[key])
        assert not torch.equal(a[key], c[key])


def test_recipe_properties():
    w = WORKLOADS["kda_prefill"].with_(T=256, H=2)
    x = make_inputs(w)
    assert x["q"].shape == (1, 256, 2, 128) and x["q"].dtype == torch.bfloat16
    assert x["alpha"].shape == (1, 256, 2, 128) and x["alpha"].dtype == torch.float32
    n = x["k"].float().norm(dim=-1)
    assert torch.allclose(n, torch.ones_like(n), atol=1e-2)     # unit rows before bf16 rounding
    assert (x["alpha"] > 0).all() and (x["alpha"] < 1).all()
    assert (x["beta"] > 0).all() and (x["beta"] < 1).all()
    # exp(-softplus(N(0,1)+2)): mean log-gate near -2.2
    assert -2.4 < torch.log(x["alpha"]).mean().item() < -2.0
    assert x["s0"] is None


def test_decode_layout_and_state():
    w = WORKLOADS["decode_gdn"].with_(B=3, H=2, T=5)
    x = make_inputs(w)
    assert x["q"].shape == (5, 3, 2, 128)        # [steps, N, H, dk]
    assert x["alpha"].shape == (5, 3, 2)
    assert x["s0"].shape == (3, 2, 128, 128)
    assert abs(x["s0"].std().item() - 0.02) < 1e-3
    one = slice_inputs(w, 1, 1)
    assert torch.equal(x["q"][:, 1, 1], one["q"])


def test_stress_gates():
    w = WORKLOADS["gdn_seq_f32"]
    slow = slice_inputs(w, 0, 0, gates="slow")["alpha"]
    assert slow.min() > 0.9
    z = slice_inputs(w, 0, 0, gates="zero_some")["alpha"]
    assert (z[::7] == 0).all() and (z[1::7] > 0).all()
