"""Failure detection without a GPU fault: the tensor-core prefill bounds every wait
on the tensor cores.  Setting GDR_SPIN_LIMIT=0 makes the first wait give up at
once (the MMA itself completes normally and is drained), so the kernel records
GDR_ERR_TIMEOUT in the workspace status word and ends cleanly; the host reads it
with gdr_workspace_status, and the next call runs normally."""

import os

import pytest
import torch

from synth import Workload, make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
@pytest.mark.parametrize("path", ["single-kernel", "two-kernel chain", "two-kernel rows",
                                  "two-kernel sliced"])
def test_bounded_wait_reports_timeout_and_recovers(mixer, path, monkeypatch):
    import gated_delta_rule_79_b200 as g
    if path.startswith("two-kernel"):
        monkeypatch.setenv("GDR_CARRY", path.split()[1])
    kda = mixer == "kda"
    w = Workload("fi", mixer, 1, 2, 100, 128, 128, "bf16", "randn")
    x = {k: v.cuda() for k, v in make_inputs(w, seed=11).items()}
    assert g.prefill_path(128, 128, torch.bfloat16, kda) == "tensor-core"
    fn = g.kda_prefill if kda else g.gdn_prefill
    full = g.lib.gdr_prefill_workspace_bytes(1, 100, 2, 128, 128, int(kda))
    ws = torch.zeros(4096 if path == "single-kernel" else full, dtype=torch.uint8, device="cuda")
    old = os.environ.get("GDR_SPIN_LIMIT")
    os.environ["GDR_SPIN_LIMIT"] = "0"
    try:
        fn(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["s0"], workspace=ws)
        with pytest.raises(g.GdrError) as e:
            g.workspace_status(ws)
        assert e.value.status == g.GDR_ERR_TIMEOUT
    finally:
        if old is None:
            del os.environ["GDR_SPIN_LIMIT"]
        else:
            os.environ["GDR_SPIN_LIMIT"] = old
    # the status word was cleared and the context is healthy
    o, s = fn(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["s0"], workspace=ws)
    g.workspace_status(ws)
    assert torch.isfinite(o.float()).all() and torch.isfinite(s).all()
