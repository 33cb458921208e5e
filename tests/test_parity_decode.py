"""GPU decode vs the fp64 oracle, through the C ABI (via the ctypes binding)."""

import numpy as np
import pytest
import torch

from oracle import decode_step
from synth import WORKLOADS, Workload, device_inputs, make_inputs, slice_inputs
from _util import check_elem, rel_err, to_np

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-3}


def _fn(mixer):
    import gated_delta_rule_79_b200 as g
    return g.kda_decode if mixer == "kda" else g.gdn_decode


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 64), (128, 128), (128, 64), (32, 128)])
@pytest.mark.parametrize("out", ["same", "f32"])
def test_decode_small(mixer, dtype, dk, dv, out):
    w = Workload("dec", mixer, 5, 3, 7, dk, dv, dtype, "randn", decode=True)
    x = make_inputs(w, seed=dk + dv)
    dev = torch.device("cuda")
    state = x["s0"].to(dev).clone()
    ref = x["s0"].double().numpy()
    out_dtype = torch.float32 if out == "f32" else None
    for t in range(w.T):
        args = [x[k][t] for k in ("q", "k", "v", "alpha", "beta")]
        o = _fn(mixer)(*[a.to(dev) for a in args], state, out_dtype=out_dtype)
        o_ref, ref = decode_step(*[a.double().numpy() for a in args], ref)
        torch.cuda.synchronize()
        tol = TOL[dtype] if (out == "f32" or dtype == "f32") else TOL["bf16"]
        assert rel_err(to_np(o), o_ref) <= tol
        check_elem(to_np(o), o_ref, "cc", axes=(0, 1), bf16_out=o.dtype == torch.bfloat16,
                   label=f"step {t} o")
    es = rel_err(to_np(state), ref)
    print(f"{mixer} {dtype} {dk}x{dv}: state err {es:.2e}")
    assert es <= TOL[dtype]
    check_elem(to_np(state), ref, "cc", axes=(0, 1), label="state")


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
def test_decode_workload_sampled(mixer):
    """256 sequences x 32 heads, d=128, 512 steps, launched at full size; sampled
    (sequence, head) chains are drawn on the CPU and followed by the oracle over
    all 512 steps (outputs of every step and the final state)."""
    w = WORKLOADS[f"decode_{mixer}"]
    dev = torch.device("cuda")
    full = device_inputs(w, dev, seed=7)
    picks = [(0, 0), (100, 5), (255, 31)]
    parts = [slice_inputs(w, n, h) for n, h in picks]
    for (n, h), p in zip(picks, parts):
        for key in ("q", "k", "v", "beta", "alpha"):
            full[key][:, n, h] = p[key].to(dev)
        full["s0"][n, h] = p["s0"].to(dev)
    state = full["s0"]
    outs = []
    for t in range(w.T):
        o = _fn(mixer)(full["q"][t], full["k"][t], full["v"][t], full["alpha"][t],
                       full["beta"][t], state)
        outs.append(torch.stack([o[n, h] for n, h in picks]).float())
    torch.cuda.synchronize()
    outs = torch.stack(outs, 1).double().cpu().numpy()          # [n, steps, dv]
    ref = np.stack([p["s0"].double().numpy() for p in parts])[:, None]
    o_ref = []
    for t in range(w.T):
        args = [np.stack([p[key][t].double().numpy() for p in parts])[:, None]
                for key in ("q", "k", "v", "alpha", "beta")]
        o_t, ref = decode_step(*args, ref)
        o_ref.append(o_t[:, 0])
    o_ref = np.stack(o_ref, 1)
    for i, (n, h) in enumerate(picks):
        eo = rel_err(outs[i], o_ref[i])
        es = rel_err(to_np(state[n, h]), ref[i, 0])
        print(f"decode {mixer} {(n, h)}: o {eo:.2e} s {es:.2e}")
        assert eo <= TOL["bf16"] and es <= TOL["bf16"]
        check_elem(outs[i], o_ref[i], "cc", bf16_out=True, label=f"{(n, h)} o")
        check_elem(to_np(state[n, h]), ref[i, 0], "cc", label=f"{(n, h)} s")


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
def test_decode_in_bounds(mixer):
    w = Workload("dec", mixer, 4, 3, 1, 128, 128, "bf16", "randn", decode=True)
    x = {k: v.cuda() for k, v in make_inputs(w).items()}
    n_s = 4 * 3 * 128 * 128
    n_o = 4 * 3 * 128
    sbuf = torch.full((n_s + 1024,), 5.0, device="cuda")
    sbuf[:n_s] = x["s0"].flatten()
    obuf = torch.full((n_o + 1024,), -3.0, device="cuda")
    _fn(mixer)(x["q"][0], x["k"][0], x["v"][0], x["alpha"][0], x["beta"][0],
               sbuf[:n_s].view(4, 3, 128, 128), o=obuf[:n_o].view(4, 3, 128),
               out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert (sbuf[n_s:] == 5.0).all() and (obuf[n_o:] == -3.0).all()
