"""The GDR_CHECKS debug build (libgdr_checks.so): the same kernels with device-side
index checks that record a status bit and skip the access instead of faulting.

test_small_parity_suite_with_checks runs the small-shape parity tests of prefill,
packed prefill, decode and verify in a child process that loads the checks build,
with a fixture that asserts, after every test, that no check fired
(gdr_check_status == GDR_OK).  test_bad_slot_is_recorded_not_faulted, run the same way,
hands a packed prefill a negative state slot from the host: the carry's check records
bit 2 and skips that sequence's state, the other sequences come out right, and the
status reads clean afterwards.  The tests marked `checks_build` run only inside that
child process."""

import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from _util import rel_err, to_np

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
IN_CHECKS = os.environ.get("GDR_LIBRARY") == "checks"

SMALL = ["tests/test_parity_prefill.py::test_small_shapes",
         "tests/test_parity_prefill.py::test_gdn_prefill_chain_counts",
         "tests/test_parity_prefill.py::test_both_carries",
         "tests/test_parity_varlen.py::test_varlen_ragged",
         "tests/test_parity_decode.py::test_decode_small",
         "tests/test_parity_verify.py::test_verify_snapshots"]


def _child(args):
    env = dict(os.environ, GDR_LIBRARY="checks")
    env.pop("GDR_ELEM_LOG", None)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        *args], cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    print(r.stdout[-3000:], r.stderr[-2000:])
    return r.returncode


@pytest.mark.skipif(IN_CHECKS, reason="the parent runs the child")
def test_small_parity_suite_with_checks():
    assert _child(SMALL) == 0


@pytest.mark.skipif(IN_CHECKS, reason="the parent runs the child")
def test_bad_slot_is_recorded_not_faulted():
    assert _child(["tests/test_checks_build.py::test_negative_slot_in_checks_build"]) == 0


@pytest.mark.skipif(not IN_CHECKS, reason="runs in the child process on libgdr_checks.so")
def test_negative_slot_in_checks_build():
    import gated_delta_rule_79_b200 as g
    from oracle import prefill_varlen
    from synth import Workload, make_inputs
    stream = None
    assert g.lib.gdr_check_status(stream) == g.GDR_OK      # the checks build is loaded
    lens = [70, 33, 129]
    H, dv = 2, 128
    parts = [make_inputs(Workload("cb", "gdn", 1, H, n, 128, dv, "bf16", "randn"), seed=3 + i)
             for i, n in enumerate(lens)]
    x = {key: torch.cat([p[key][0] for p in parts]) for key in ("q", "k", "v", "alpha", "beta")}
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    pool0 = 0.02 * torch.randn((4, H, dv, 128), generator=torch.Generator().manual_seed(2))
    slots = torch.tensor([2, -1, 0], dtype=torch.int32)    # sequence 1 has a bad slot
    pool = pool0.cuda()
    d = {k: v.cuda() for k, v in x.items()}
    o = g.gdn_prefill_varlen(d["q"], d["k"], d["v"], d["alpha"], d["beta"], cu.cuda(), pool,
                             slots=slots.cuda(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    with pytest.raises(g.GdrError) as e:
        g.check_status()
    assert e.value.status == g.GDR_ERR_INVALID_ARG and "0x2" in str(e.value)
    g.check_status()                                        # read and cleared
    # the good sequences against the oracle (sequence 1 alone, from a zero state, as the
    # carry ran it without its slot)
    good = torch.tensor([2, 3, 0], dtype=torch.int32)       # slot 3 stands in for the bad one
    o_ref, p_ref = prefill_varlen(*[x[k].double().numpy() for k in ("q", "k", "v", "alpha",
                                                                    "beta")],
                                  cu.numpy(), np.concatenate([pool0.double().numpy()[:3],
                                                              np.zeros((1, H, dv, 128))]),
                                  good.numpy())
    assert rel_err(to_np(o), o_ref) <= 2e-3
    for s in (0, 2):
        assert rel_err(to_np(pool[s]), p_ref[s]) <= 2e-3
    assert torch.equal(pool[1], pool0[1].cuda()) and torch.equal(pool[3], pool0[3].cuda())
