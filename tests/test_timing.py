"""The per-kernel timing aid of the C ABI (gdr_timing_start / gdr_timing_stop), which
bench.py uses to split a prefill call's time among its kernels."""

import pytest
import torch

from synth import Workload, make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
def test_timing_counts_kernels_and_calls(mixer):
    import gated_delta_rule_79_b200 as g
    kda = mixer == "kda"
    fn = g.kda_prefill if kda else g.gdn_prefill
    w = Workload("tm", mixer, 1, 2, 300, 128, 128, "bf16", "randn")
    x = {k: v.cuda() for k, v in make_inputs(w, seed=2).items()}
    args = (x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["s0"])
    full = g.lib.gdr_prefill_workspace_bytes(1, 300, 2, 128, 128, int(kda))
    big = torch.zeros(full, dtype=torch.uint8, device="cuda")
    small = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    fn(*args, workspace=big)                       # warm-up outside the record
    g.timing_start()
    for _ in range(3):
        fn(*args, workspace=big)
    ms, calls = g.timing_stop()
    assert calls == 3 and len(ms) == 2 and all(m > 0 for m in ms)
    g.timing_start()
    fn(*args, workspace=small)                     # the single-kernel path
    ms1, calls1 = g.timing_stop()
    assert calls1 == 1 and len(ms1) == 1 and ms1[0] > 0
    fn(*args, workspace=big)                       # recording is off again
    assert g.timing_stop() == ([], 0)
