"""GPU prefill vs the fp64 oracle, through the C ABI (via the ctypes binding).

Bar: normwise relative error <= 2e-3 for bf16 inputs and <= 1e-5 for fp32
inputs, on the outputs and on the final state, for the whole tensor and for
every (batch, head) slice; and every element within the element-wise bound of
its precision class (tests/_util.py).
"""

import numpy as np
import pytest
import torch

from oracle import gated_delta_rule
from synth import WORKLOADS, Workload, device_inputs, make_inputs, slice_inputs
from _util import bf16_round_floor, check_elem, rel_err, slice_errs, to_np

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-3}


def gpu_prefill(mixer, x, out_dtype=None, workspace=None):
    import gated_delta_rule_79_b200 as g
    fn = g.kda_prefill if mixer == "kda" else g.gdn_prefill
    t = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
    o, s = fn(t["q"], t["k"], t["v"], t["alpha"], t["beta"], t["s0"], out_dtype=out_dtype,
              workspace=workspace)
    torch.cuda.synchronize()
    return to_np(o), to_np(s)


def ref_prefill(x):
    s0 = None if x["s0"] is None else x["s0"].double().numpy()
    args = [x[k].double().numpy() for k in ("q", "k", "v", "alpha", "beta")]
    return gated_delta_rule(*args, s0)


def path_cls(mixer, dtype, dk=128, dv=128):
    """Precision class of the prefill that serves these parameters: fp32 inputs go to
    the CUDA-core kernel (1e-5), bf16 inputs to the tensor-core kernels when d_k = 128
    and to the CUDA-core kernel otherwise."""
    import gated_delta_rule_79_b200 as g
    if dtype == "f32":
        return "f32"
    tdt = torch.bfloat16
    return "tc" if g.prefill_path(dk, dv, tdt, mixer == "kda") == "tensor-core" else "cc"


def check(o, s, o_ref, s_ref, tol, label="", cls="tc", bf16_out=False):
    eo, es = rel_err(o, o_ref), rel_err(s, s_ref)
    eo_h = slice_errs(o, o_ref, axes=(0, 2))      # per (batch, head) over (T, d_v)
    es_h = slice_errs(s, s_ref, axes=(0, 1))
    print(f"{label} o {eo:.2e} (worst head {eo_h:.2e})  s {es:.2e} (worst head {es_h:.2e})")
    assert eo <= tol and eo_h <= tol, (eo, eo_h)
    assert es <= tol and es_h <= tol, (es, es_h)
    check_elem(o, o_ref, cls, axes=(0, 2), bf16_out=bf16_out, label=f"{label} o")
    check_elem(s, s_ref, cls, axes=(0, 1), label=f"{label} s")


def test_gdn_sequential_f32_workload():
    """B=1 H=2 T=64 d=32, fp32 inputs, zero state: 1e-5."""
    w = WORKLOADS["gdn_seq_f32"]
    x = make_inputs(w)
    o, s = gpu_prefill("gdn", x)
    o_ref, s_ref = ref_prefill(x)
    check(o, s, o_ref, s_ref, TOL["f32"], w.name, cls="f32")


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 64), (128, 128), (64, 128), (128, 32)])
@pytest.mark.parametrize("T", [1, 65, 200])
def test_small_shapes(mixer, dtype, dk, dv, T):
    """Outputs in fp32 so that the check measures the kernel's arithmetic (a bf16
    output adds a rounding floor of about 1.7e-3 that is noisy on small slices)."""
    w = Workload("small", mixer, 2, 2, T, dk, dv, dtype, "randn")
    x = make_inputs(w, seed=T + dk)
    o, s = gpu_prefill(mixer, x, out_dtype=torch.float32)
    o_ref, s_ref = ref_prefill(x)
    check(o, s, o_ref, s_ref, TOL[dtype], f"{mixer} {dtype} {dk}x{dv} T={T}",
          cls=path_cls(mixer, dtype, dk, dv))


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("gates", ["slow", "one", "zero_some"])
def test_stress_gates(mixer, dtype, gates):
    """Gates that make the carry between chunks matter (the workload gates decay by
    about e^-140 per chunk, which would hide a broken carry)."""
    w = Workload("stress", mixer, 1, 3, 300, 128, 128, dtype, "randn")
    x = make_inputs(w, seed=5, gates=gates)
    o, s = gpu_prefill(mixer, x, out_dtype=torch.float32)
    o_ref, s_ref = ref_prefill(x)
    check(o, s, o_ref, s_ref, TOL[dtype], f"{mixer} {dtype} gates={gates}",
          cls=path_cls(mixer, dtype))


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
@pytest.mark.parametrize("gates", ["workload", "slow", "zero_some"])
@pytest.mark.parametrize("T", [77, 200])
def test_single_kernel_path(mixer, gates, T):
    """With a workspace that holds only the status word, bf16 d=128 prefill runs the
    single-kernel tensor-core kernels instead of the two-kernel ones."""
    import gated_delta_rule_79_b200 as g
    w = Workload("single", mixer, 2, 2, T, 128, 128, "bf16", "randn")
    x = make_inputs(w, seed=T + 3, gates=gates)
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    o, s = gpu_prefill(mixer, x, out_dtype=torch.float32, workspace=ws)
    g.workspace_status(ws)
    o_ref, s_ref = ref_prefill(x)
    check(o, s, o_ref, s_ref, TOL["bf16"], f"single-kernel {mixer} gates={gates} T={T}")


@pytest.mark.parametrize("T", [63, 64, 127, 128, 129])
def test_chunk_boundaries(T):
    w = Workload("edges", "kda", 1, 2, T, 128, 128, "bf16", "randn")
    x = make_inputs(w, seed=T, gates="slow")
    o, s = gpu_prefill("kda", x, out_dtype=torch.float32)
    o_ref, s_ref = ref_prefill(x)
    check(o, s, o_ref, s_ref, TOL["bf16"], f"T={T}")


@pytest.mark.parametrize("name", ["gdn_prefill", "kda_prefill"])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_full_workload(name, out):
    """The full B=1 H=32 T=4096 d=128 bf16 workloads, every head against the oracle.
    Outputs are checked both as bf16 (which carries the bf16 rounding floor) and
    as fp32."""
    w = WORKLOADS[name]
    x = make_inputs(w)
    o, s = gpu_prefill(w.mixer, x, out_dtype=torch.bfloat16 if out == "bf16" else torch.float32)
    o_ref, s_ref = ref_prefill(x)
    if out == "bf16":
        print(f"bf16 rounding floor of o: {bf16_round_floor(o_ref):.2e}")
    check(o, s, o_ref, s_ref, TOL["bf16"], f"{name} out={out}", bf16_out=out == "bf16")


def test_kda_long_context_sampled():
    """B=4 H=32 T=65536 with a carried N(0, 0.02) state, launched at full size; a
    sample of (batch, head) chains is drawn on the CPU and checked against the
    oracle over all 65536 tokens (every chain is independent of the others)."""
    w = WORKLOADS["kda_long"]
    dev = torch.device("cuda")
    full = device_inputs(w, dev, seed=99)
    picks = [(0, 0), (1, 17), (3, 31)]
    parts = [slice_inputs(w, b, h) for b, h in picks]
    for (b, h), p in zip(picks, parts):
        for key in ("q", "k", "v", "beta", "alpha"):
            full[key][b, :, h] = p[key].to(dev)
        full["s0"][b, h] = p["s0"].to(dev)
    import gated_delta_rule_79_b200 as g
    o, s = g.kda_prefill(full["q"], full["k"], full["v"], full["alpha"], full["beta"],
                         full["s0"])
    torch.cuda.synchronize()
    # the sampled chains as an oracle batch: [n, T, 1, ...] and s0 [n, 1, dv, dk]
    def col(key):
        return torch.stack([p[key] for p in parts])[:, :, None].double().numpy()
    s0 = torch.stack([p["s0"] for p in parts])[:, None].double().numpy()
    o_ref, s_ref = gated_delta_rule(col("q"), col("k"), col("v"), col("alpha"), col("beta"), s0)
    for i, (b, h) in enumerate(picks):
        eo = rel_err(to_np(o[b, :, h]), o_ref[i, :, 0])
        es = rel_err(to_np(s[b, h]), s_ref[i, 0])
        print(f"kda_long slice {(b, h)}: o {eo:.2e} s {es:.2e}")
        assert eo <= TOL["bf16"] and es <= TOL["bf16"]
        check_elem(to_np(o[b, :, h]), o_ref[i, :, 0], "tc", bf16_out=o.dtype == torch.bfloat16,
                   label=f"kda_long {(b, h)} o")
        check_elem(to_np(s[b, h]), s_ref[i, 0], "tc", label=f"kda_long {(b, h)} s")


def test_empty_and_state_passthrough():
    import gated_delta_rule_79_b200 as g
    w = Workload("t0", "gdn", 2, 2, 0, 64, 64, "bf16", "randn")
    dev = torch.device("cuda")
    q = torch.zeros((2, 0, 2, 64), dtype=torch.bfloat16, device=dev)
    a = torch.zeros((2, 0, 2), device=dev)
    s0 = torch.randn((2, 2, 64, 64), device=dev)
    o, s = g.gdn_prefill(q, q, q, a, a, s0)
    torch.cuda.synchronize()
    assert o.shape == (2, 0, 2, 64) and torch.equal(s, s0)
    o, s = g.gdn_prefill(q, q, q, a, a, None)
    torch.cuda.synchronize()
    assert torch.count_nonzero(s) == 0
    del w


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
def test_outputs_stay_in_bounds(mixer):
    """Canaries after the output and state buffers are untouched."""
    import gated_delta_rule_79_b200 as g
    w = Workload("canary", mixer, 1, 3, 130, 128, 128, "bf16", "randn")
    x = {k: (v.cuda() if v is not None else None) for k, v in make_inputs(w, seed=3).items()}
    n_o = 1 * 130 * 3 * 128
    n_s = 1 * 3 * 128 * 128
    obuf = torch.full((n_o + 4096,), 12345.0, dtype=torch.bfloat16, device="cuda")
    sbuf = torch.full((n_s + 4096,), -777.0, device="cuda")
    fn = g.kda_prefill if mixer == "kda" else g.gdn_prefill
    fn(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["s0"],
       o=obuf[:n_o].view(1, 130, 3, 128), s_final=sbuf[:n_s].view(1, 3, 128, 128))
    torch.cuda.synchronize()
    assert (obuf[n_o:] == 12345.0).all()
    assert (sbuf[n_s:] == -777.0).all()
    assert torch.isfinite(obuf[:n_o].float()).all()


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
def test_in_place_state_carry(mixer):
    """s_final may alias s0."""
    import gated_delta_rule_79_b200 as g
    w = Workload("alias", mixer, 2, 2, 150, 128, 128, "bf16", "randn")
    x = make_inputs(w, seed=4)
    o_ref, s_ref = ref_prefill(x)
    t = {k: v.cuda() for k, v in x.items()}
    fn = g.kda_prefill if mixer == "kda" else g.gdn_prefill
    state = t["s0"].clone()
    o, s = fn(t["q"], t["k"], t["v"], t["alpha"], t["beta"], state, s_final=state)
    torch.cuda.synchronize()
    assert s.data_ptr() == state.data_ptr()
    check(to_np(o), to_np(state), o_ref, s_ref, TOL["bf16"], "alias",
          bf16_out=o.dtype == torch.bfloat16)


@pytest.mark.parametrize("dv", [128, 64])
def test_kda_carry_with_64_value_columns(dv, monkeypatch):
    """With enough (sequence, head) chains the value-sliced carry takes 64 value columns
    per CTA (two slices sharing each chunk's operands): 3 x 50 heads run that way."""
    monkeypatch.setenv("GDR_CARRY", "sliced")
    w = Workload("wide", "kda", 3, 50, 130, 128, dv, "bf16", "randn")
    x = make_inputs(w, seed=77)
    o, s = gpu_prefill("kda", x, out_dtype=torch.float32)
    o_ref, s_ref = ref_prefill(x)
    check(o, s, o_ref, s_ref, TOL["bf16"], f"kda 64-column carry dv={dv}")


@pytest.mark.parametrize("carry", ["chain", "rows", "sliced"])
@pytest.mark.parametrize("mixer", ["gdn", "kda"])
@pytest.mark.parametrize("dv", [128, 64, 32])
@pytest.mark.parametrize("gates", ["slow", "zero_some"])
def test_both_carries(carry, mixer, dv, gates, monkeypatch):
    """Each state carry, forced (the chained and the per-head ones run all value rows of
    a head in one CTA, the value-sliced one spreads them): a ragged tail, an entering
    state, gates that make the carry matter."""
    monkeypatch.setenv("GDR_CARRY", carry)
    w = Workload("carry", mixer, 2, 3, 200, 128, dv, "bf16", "randn")
    x = make_inputs(w, seed=dv + 11, gates=gates)
    o, s = gpu_prefill(mixer, x, out_dtype=torch.float32)
    o_ref, s_ref = ref_prefill(x)
    check(o, s, o_ref, s_ref, TOL["bf16"], f"{carry} carry {mixer} dv={dv} gates={gates}")


@pytest.mark.parametrize("carry", ["chain", "rows", "sliced"])
@pytest.mark.parametrize("mixer", ["gdn", "kda"])
def test_both_carries_bf16_out_in_place(carry, mixer, monkeypatch):
    """bf16 outputs and the final state written over the entering one."""
    import gated_delta_rule_79_b200 as g
    monkeypatch.setenv("GDR_CARRY", carry)
    w = Workload("carry16", mixer, 3, 2, 129, 128, 128, "bf16", "randn")
    x = make_inputs(w, seed=21, gates="slow")
    o_ref, s_ref = ref_prefill(x)
    t = {k: v.cuda() for k, v in x.items()}
    fn = g.kda_prefill if mixer == "kda" else g.gdn_prefill
    state = t["s0"].clone()
    o, s = fn(t["q"], t["k"], t["v"], t["alpha"], t["beta"], state, s_final=state)
    torch.cuda.synchronize()
    assert o.dtype == torch.bfloat16
    check(to_np(o), to_np(state), o_ref, s_ref, TOL["bf16"], f"{carry} carry bf16 in place",
          bf16_out=True)


def test_more_chains_than_sms():
    """40 sequences x 4 heads = 160 chains, more than the SMs: the chained carry runs
    them in a second wave; checked against the oracle on sampled chains."""
    w = Workload("many", "gdn", 40, 4, 96, 128, 128, "bf16", "randn")
    x = make_inputs(w, seed=31, gates="slow")
    o, s = gpu_prefill("gdn", x, out_dtype=torch.float32)
    picks = [0, 17, 39]
    sub = {k: (v[picks] if v is not None else None) for k, v in x.items()}
    o_ref, s_ref = ref_prefill(sub)
    check(o[picks], s[picks], o_ref, s_ref, TOL["bf16"], "many chains")



@pytest.mark.parametrize("B,H,T,dv", [(1, 4, 200, 128), (2, 3, 129, 64), (1, 1, 64, 32),
                                      (1, 37, 130, 128), (3, 1, 1000, 128)])
@pytest.mark.parametrize("init", [True, False])
def test_gdn_prefill_chain_counts(B, H, T, dv, init):
    """GDN on the value-sliced carry: ragged tails, one chunk, exactly as many
    (sequence, head, 32-column slice) chains as 148 SMs hold, long chains, with and
    without an entering state."""
    w = Workload("chains", "gdn", B, H, T, 128, dv, "bf16", "randn")
    x = make_inputs(w, seed=B * 100 + H + T, gates="slow")
    if not init:
        x["s0"] = None
    o, s = gpu_prefill("gdn", x, out_dtype=torch.float32)
    o_ref, s_ref = ref_prefill(x)
    check(o, s, o_ref, s_ref, TOL["bf16"], f"B={B} H={H} T={T} dv={dv}")


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
def test_prefill_bf16_out_repeated(mixer):
    """bf16 outputs, the final state over the entering one, and the same workspace for
    several calls in a row."""
    import gated_delta_rule_79_b200 as g
    w = Workload("rep16", mixer, 1, 8, 300, 128, 128, "bf16", "randn")
    x = make_inputs(w, seed=5, gates="slow")
    t = {k: v.cuda() for k, v in x.items()}
    fn = g.kda_prefill if mixer == "kda" else g.gdn_prefill
    ws, _ = g.prefill_workspace(1, 300, 8, 128, 128, mixer == "kda", torch.device("cuda"))
    s_ref = x["s0"].double().numpy()
    state = t["s0"].clone()
    for it in range(3):
        o, _ = fn(t["q"], t["k"], t["v"], t["alpha"], t["beta"], state, s_final=state,
                  workspace=ws)
        torch.cuda.synchronize()
        g.workspace_status(ws)
        args = [x[k].double().numpy() for k in ("q", "k", "v", "alpha", "beta")]
        o_ref, s_ref = gated_delta_rule(*args, s_ref)
        check(to_np(o), to_np(state), o_ref, s_ref, TOL["bf16"], f"{mixer} bf16 call {it}",
              bf16_out=o.dtype == torch.bfloat16)
        s_ref = to_np(state).astype(np.float64)
