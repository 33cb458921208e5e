"""Resumption through the state (the state is the checkpoint of a sequence):
prefill(T1) then prefill(T2) from its state equals prefill(T1 + T2), and
prefill(T) followed by n decode steps equals prefill(T + n)."""

import pytest
import torch

from synth import Workload, make_inputs
from _util import rel_err, to_np

pytestmark = pytest.mark.gpu


def _g():
    import gated_delta_rule_79_b200 as g
    return g


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
@pytest.mark.parametrize("t1", [64, 100])
def test_split_prefill(mixer, t1):
    g = _g()
    w = Workload("split", mixer, 2, 2, 230, 128, 128, "bf16", "randn")
    x = {k: v.cuda() for k, v in make_inputs(w, seed=8, gates="slow").items()}
    fn = g.kda_prefill if mixer == "kda" else g.gdn_prefill
    o, s = fn(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["s0"], out_dtype=torch.float32)
    part = lambda key, a, b: x[key][:, a:b].contiguous()  # noqa: E731
    oa, sa = fn(*[part(k, 0, t1) for k in ("q", "k", "v", "alpha", "beta")], x["s0"],
                out_dtype=torch.float32)
    ob, sb = fn(*[part(k, t1, 230) for k in ("q", "k", "v", "alpha", "beta")], sa,
                out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert rel_err(to_np(torch.cat([oa, ob], 1)), to_np(o)) <= 2e-3
    assert rel_err(to_np(sb), to_np(s)) <= 2e-3


@pytest.mark.parametrize("mixer", ["gdn", "kda"])
def test_prefill_then_decode(mixer):
    g = _g()
    T, n = 130, 5
    w = Workload("pd", mixer, 3, 2, T + n, 128, 128, "bf16", "randn")
    x = {k: v.cuda() for k, v in make_inputs(w, seed=9, gates="slow").items()}
    pf = g.kda_prefill if mixer == "kda" else g.gdn_prefill
    dec = g.kda_decode if mixer == "kda" else g.gdn_decode
    o_all, s_all = pf(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["s0"],
                      out_dtype=torch.float32)
    sl = lambda key: x[key][:, :T].contiguous()  # noqa: E731
    _, state = pf(*[sl(k) for k in ("q", "k", "v", "alpha", "beta")], x["s0"])
    for t in range(T, T + n):
        step = [x[k][:, t].contiguous() for k in ("q", "k", "v", "alpha", "beta")]
        o = dec(*step, state, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert rel_err(to_np(o), to_np(o_all[:, t])) <= 2e-3
    assert rel_err(to_np(state), to_np(s_all)) <= 2e-3
