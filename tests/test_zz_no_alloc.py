"""gdn_prefill_noalloc, the prefill entry point for callers that cannot allocate
device memory (serving loops that must not stall the device with cudaMalloc or
cudaFree, embedders whose device memory belongs to another allocator).  It uses
the library's static device scratch instead of a caller workspace; its results
must match gdn_prefill's on consecutive calls.  This file is collected last so
that a run stopping at the first failure has run every other test before it."""

import ctypes

import pytest
import torch

from synth import Workload, make_inputs
from _util import rel_err, to_np

pytestmark = pytest.mark.gpu

TOL = 2e-3   # the bf16-input parity tolerance used throughout the tests


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(g, x, o, s, dk=128):
    B, T, H, _ = x["q"].shape
    dv = x["v"].shape[-1]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return g.lib.gdn_prefill_noalloc(_ptr(x["q"]), _ptr(x["k"]), _ptr(x["v"]), _ptr(x["alpha"]),
                                     _ptr(x["beta"]), _ptr(x["s0"]), _ptr(o), _ptr(s), B, T, H,
                                     dk, dv, g.GDR_BF16, g.GDR_F32, g.CHUNK, stream)


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    import gated_delta_rule_79_b200 as g
    w = Workload("noalloc", "gdn", 2, 3, 200, 128, 128, "bf16", "randn")
    x = {k: v.cuda() for k, v in make_inputs(w, seed=21, gates="slow").items()}
    assert g.prefill_path(128, 128, torch.bfloat16, False) == "tensor-core"
    o_ref, s_ref = g.gdn_prefill(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["s0"],
                                 out_dtype=torch.float32)
    torch.cuda.synchronize()
    for _ in range(2):
        o = torch.full_like(o_ref, float("nan"))
        s = torch.full_like(s_ref, float("nan"))
        status = _noalloc(g, x, o, s)
        assert status == g.GDR_OK, g.lib.gdr_last_error().decode()
        torch.cuda.synchronize()
        assert rel_err(to_np(o), to_np(o_ref)) <= TOL
        assert rel_err(to_np(s), to_np(s_ref)) <= TOL


def test_noalloc_rejects_what_gdn_prefill_rejects():
    import gated_delta_rule_79_b200 as g
    w = Workload("noalloc_bad", "gdn", 1, 1, 8, 128, 128, "bf16", "zeros")
    x = {k: (v.cuda() if v is not None else None) for k, v in make_inputs(w).items()}
    o = torch.empty((1, 8, 1, 128), device="cuda")
    assert _noalloc(g, x, o, None, dk=48) == g.GDR_ERR_UNSUPPORTED
    assert "d_k=48" in g.lib.gdr_last_error().decode()
