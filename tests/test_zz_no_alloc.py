"""gdn_prefill_noalloc, the prefill entry point for callers that cannot allocate
device memory (serving loops that must not stall the device with cudaMalloc or
cudaFree, embedders whose device memory belongs to another allocator).  It uses
the library's static device scratch instead of a caller workspace.  On two calls in
a row its results must match gdn_prefill's (the entry point with a workspace) and
the fp64 oracle's, within the tolerances the other parity tests use; a bounded wait
that gives up must stay on record until gdr_noalloc_status reads it.  This file is
collected last so that a run stopping at the first failure has run every other test
before it."""

import ctypes
import os

import pytest
import torch

from oracle import gated_delta_rule
from synth import Workload, make_inputs
from _util import check_elem, rel_err, to_np

pytestmark = pytest.mark.gpu

TOL = 2e-3   # the bf16-input parity tolerance used throughout the tests


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _noalloc(g, x, o, s, dk=128):
    B, T, H, _ = x["q"].shape
    dv = x["v"].shape[-1]
    return g.lib.gdn_prefill_noalloc(_ptr(x["q"]), _ptr(x["k"]), _ptr(x["v"]), _ptr(x["alpha"]),
                                     _ptr(x["beta"]), _ptr(x["s0"]), _ptr(o), _ptr(s), B, T, H,
                                     dk, dv, g.GDR_BF16, g.GDR_F32, g.CHUNK, _stream())


def test_noalloc_matches_workspace_entry_point_and_oracle_on_two_calls():
    import gated_delta_rule_79_b200 as g
    w = Workload("noalloc", "gdn", 2, 3, 200, 128, 128, "bf16", "randn")
    xc = make_inputs(w, seed=21, gates="slow")
    x = {k: v.cuda() for k, v in xc.items()}
    assert g.prefill_path(128, 128, torch.bfloat16, False) == "tensor-core"
    o_ws, s_ws = g.gdn_prefill(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["s0"],
                               out_dtype=torch.float32)
    torch.cuda.synchronize()
    o_ref, s_ref = gated_delta_rule(*[xc[k].double().numpy()
                                      for k in ("q", "k", "v", "alpha", "beta")],
                                    xc["s0"].double().numpy())
    for call in range(2):
        o = torch.full_like(o_ws, float("nan"))
        s = torch.full_like(s_ws, float("nan"))
        status = _noalloc(g, x, o, s)
        assert status == g.GDR_OK, g.lib.gdr_last_error().decode()
        torch.cuda.synchronize()
        assert g.lib.gdr_noalloc_status(_stream()) == g.GDR_OK
        # against the entry point with a workspace
        assert rel_err(to_np(o), to_np(o_ws)) <= TOL
        assert rel_err(to_np(s), to_np(s_ws)) <= TOL
        # against the oracle, normwise and element by element
        assert rel_err(to_np(o), o_ref) <= TOL and rel_err(to_np(s), s_ref) <= TOL
        check_elem(to_np(o), o_ref, "tc", axes=(0, 2), label=f"call {call} o")
        check_elem(to_np(s), s_ref, "tc", axes=(0, 1), label=f"call {call} s")


def test_noalloc_rejects_what_gdn_prefill_rejects():
    import gated_delta_rule_79_b200 as g
    w = Workload("noalloc_bad", "gdn", 1, 1, 8, 128, 128, "bf16", "zeros")
    x = {k: (v.cuda() if v is not None else None) for k, v in make_inputs(w).items()}
    o = torch.empty((1, 8, 1, 128), device="cuda")
    assert _noalloc(g, x, o, None, dk=48) == g.GDR_ERR_UNSUPPORTED
    assert "d_k=48" in g.lib.gdr_last_error().decode()


def test_noalloc_rejects_sizes_beyond_what_the_library_indexes():
    """Checked on the host before anything is enqueued (no pointer is read)."""
    import gated_delta_rule_79_b200 as g
    dummy = torch.zeros(16, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    st = g.lib.gdn_prefill_noalloc(p, p, p, p, p, None, p, None, 1 << 30, 1 << 30, 1 << 30,
                                   128, 128, g.GDR_BF16, g.GDR_F32, g.CHUNK, _stream())
    assert st == g.GDR_ERR_INVALID_ARG
    assert "gdn_prefill_noalloc" in g.lib.gdr_last_error().decode()


def test_noalloc_keeps_a_timeout_on_record_until_queried():
    """GDR_SPIN_LIMIT=0 makes the kernel's first bounded wait give up at once (no fault,
    no hang: the work completes and is drained).  The status survives later calls and
    is reported once by gdr_noalloc_status, after which calls run normally."""
    import gated_delta_rule_79_b200 as g
    w = Workload("noalloc_fi", "gdn", 1, 2, 100, 128, 128, "bf16", "randn")
    x = {k: v.cuda() for k, v in make_inputs(w, seed=11).items()}
    o = torch.empty((1, 100, 2, 128), device="cuda")
    s = torch.empty((1, 2, 128, 128), device="cuda")
    assert g.lib.gdr_noalloc_status(_stream()) == g.GDR_OK
    old = os.environ.get("GDR_SPIN_LIMIT")
    os.environ["GDR_SPIN_LIMIT"] = "0"
    try:
        assert _noalloc(g, x, o, s) == g.GDR_OK
    finally:
        if old is None:
            del os.environ["GDR_SPIN_LIMIT"]
        else:
            os.environ["GDR_SPIN_LIMIT"] = old
    assert _noalloc(g, x, o, s) == g.GDR_OK          # a normal call does not clear the record
    assert g.lib.gdr_noalloc_status(_stream()) == g.GDR_ERR_TIMEOUT
    assert g.lib.gdr_noalloc_status(_stream()) == g.GDR_OK
    assert _noalloc(g, x, o, s) == g.GDR_OK
    assert g.lib.gdr_noalloc_status(_stream()) == g.GDR_OK
    assert torch.isfinite(o).all() and torch.isfinite(s).all()
