"""The C-ABI library: it loads, exports every symbol include/gdr.h declares, and
rejects bad arguments on the host (these calls return before any CUDA work, so
they run without a GPU)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"GDR_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)
    return names


@pytest.fixture(scope="module")
def g():
    import gated_delta_rule_79_b200 as pkg
    return pkg


def test_header_declares_the_entry_points():
    names = _declared_symbols()
    for required in ("gdn_prefill", "kda_prefill", "gdn_decode", "kda_decode",
                     "gdr_prefill_workspace_bytes", "gdr_last_error"):
        assert required in names


def test_library_exports_every_declared_symbol(g):
    lib = ctypes.CDLL(g.LIB_PATH)
    for name in _declared_symbols():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert set(_declared_symbols()) <= set(g.EXPORTS) | {"gdr_version"}


def test_version_and_workspace(g):
    assert g.lib.gdr_version() >= 100
    n = g.lib.gdr_prefill_workspace_bytes(1, 4096, 32, 128, 128, 0)
    assert n >= 256
    assert g.lib.gdr_prefill_workspace_bytes(-1, 1, 1, 128, 128, 0) == 0


def _prefill(g, fn, **kw):
    a = dict(q=1 << 20, k=1 << 20, v=1 << 20, alpha=1 << 20, beta=1 << 20, s0=None, o=1 << 20,
             s_final=None, B=1, T=8, H=1, dk=64, dv=64, i=1, oo=1, chunk=64, ws=1 << 20,
             nws=4096, stream=None)
    a.update(kw)
    f = getattr(g.lib, fn)
    return f(a["q"], a["k"], a["v"], a["alpha"], a["beta"], a["s0"], a["o"], a["s_final"],
             a["B"], a["T"], a["H"], a["dk"], a["dv"], a["i"], a["oo"], a["chunk"], a["ws"],
             a["nws"], a["stream"])


@pytest.mark.parametrize("fn", ["gdn_prefill", "kda_prefill"])
def test_prefill_rejects_bad_arguments(g, fn):
    assert _prefill(g, fn, dk=48) == g.GDR_ERR_UNSUPPORTED
    assert "d_k=48" in g.lib.gdr_last_error().decode()
    assert _prefill(g, fn, dv=256) == g.GDR_ERR_UNSUPPORTED
    assert _prefill(g, fn, chunk=32) == g.GDR_ERR_UNSUPPORTED
    assert _prefill(g, fn, B=-1) == g.GDR_ERR_INVALID_ARG
    assert _prefill(g, fn, i=7) == g.GDR_ERR_INVALID_ARG
    assert _prefill(g, fn, ws=None) == g.GDR_ERR_INVALID_ARG
    assert _prefill(g, fn, nws=16) == g.GDR_ERR_INVALID_ARG
    assert _prefill(g, fn, ws=(1 << 20) + 16) == g.GDR_ERR_INVALID_ARG   # not 256-aligned
    assert _prefill(g, fn, q=None) == g.GDR_ERR_INVALID_ARG
    assert "q is NULL" in g.lib.gdr_last_error().decode()
    assert _prefill(g, fn, v=(1 << 20) + 8) == g.GDR_ERR_INVALID_ARG     # misaligned
    # empty batches are valid and enqueue nothing
    assert _prefill(g, fn, B=0) == g.GDR_OK
    assert _prefill(g, fn, H=0) == g.GDR_OK
    assert g.lib.gdr_last_error().decode() == ""


@pytest.mark.parametrize("fn", ["gdn_decode", "kda_decode"])
def test_decode_rejects_bad_arguments(g, fn):
    f = getattr(g.lib, fn)
    P = 1 << 20

    def call(**kw):
        a = dict(q=P, k=P, v=P, alpha=P, beta=P, state=P, o=P, N=4, H=2, dk=128, dv=128,
                 i=1, oo=1)
        a.update(kw)
        return f(a["q"], a["k"], a["v"], a["alpha"], a["beta"], a["state"], a["o"], a["N"],
                 a["H"], a["dk"], a["dv"], a["i"], a["oo"], None)
    assert call(dk=16) == g.GDR_ERR_UNSUPPORTED
    assert call(N=-2) == g.GDR_ERR_INVALID_ARG
    assert call(state=None) == g.GDR_ERR_INVALID_ARG
    assert call(alpha=P + 4) == g.GDR_ERR_INVALID_ARG
    assert call(oo=3) == g.GDR_ERR_INVALID_ARG
    assert call(N=0) == g.GDR_OK


def test_public_names_resolve():
    """Every name the package advertises resolves to the binding."""
    import gated_delta_rule_79_b200 as g
    for name in g.__all__:
        assert getattr(g, name) is not None, name


@pytest.mark.parametrize("fn", ["gdn_verify", "kda_verify"])
def test_verify_rejects_bad_arguments(g, fn):
    f, fx = getattr(g.lib, fn), getattr(g.lib, fn + "_ex")
    P = 1 << 20

    def call(ex=None, **kw):
        a = dict(q=P, k=P, v=P, alpha=P, beta=P, state=P, snaps=P, o=P, N=4, K=3, H=2,
                 dk=128, dv=64, i=1, oo=1)
        a.update(kw)
        args = (a["q"], a["k"], a["v"], a["alpha"], a["beta"], a["state"], a["snaps"], a["o"],
                a["N"], a["K"], a["H"], a["dk"], a["dv"], a["i"], a["oo"], None)
        return f(*args) if ex is None else fx(*args, ex)
    assert call(K=0) == g.GDR_ERR_UNSUPPORTED
    assert call(K=17) == g.GDR_ERR_UNSUPPORTED
    assert call(dk=48) == g.GDR_ERR_UNSUPPORTED
    assert call(N=-1) == g.GDR_ERR_INVALID_ARG
    assert call(state=None) == g.GDR_ERR_INVALID_ARG
    assert call(snaps=P + 4) == g.GDR_ERR_INVALID_ARG
    assert call(oo=3) == g.GDR_ERR_INVALID_ARG
    assert call(ex=4) == g.GDR_ERR_INVALID_ARG
    assert "prologue" in g.lib.gdr_last_error().decode()
    assert call(N=0) == g.GDR_OK


@pytest.mark.parametrize("fn", ["gdn_prefill_varlen", "kda_prefill_varlen"])
def test_varlen_rejects_bad_arguments(g, fn):
    f, fx = getattr(g.lib, fn), getattr(g.lib, fn + "_ex")
    P = 1 << 20

    def call(ex=None, **kw):
        a = dict(q=P, k=P, v=P, alpha=P, beta=P, cu=P, slots=None, state=P, o=P, nseq=3,
                 total=100, H=2, dk=128, dv=128, i=g.GDR_BF16, oo=1, chunk=64, ws=P,
                 nws=1 << 30)
        a.update(kw)
        args = (a["q"], a["k"], a["v"], a["alpha"], a["beta"], a["cu"], a["slots"], a["state"],
                a["o"], a["nseq"], a["total"], a["H"], a["dk"], a["dv"], a["i"], a["oo"],
                a["chunk"], a["ws"], a["nws"], None)
        return f(*args) if ex is None else fx(*args, ex)
    assert call(chunk=32) == g.GDR_ERR_UNSUPPORTED
    assert call(dk=64) == g.GDR_ERR_UNSUPPORTED
    assert call(i=g.GDR_F32) == g.GDR_ERR_UNSUPPORTED
    assert call(nseq=-1) == g.GDR_ERR_INVALID_ARG
    assert call(cu=None) == g.GDR_ERR_INVALID_ARG
    assert call(cu=P + 2) == g.GDR_ERR_INVALID_ARG
    assert call(ws=None) == g.GDR_ERR_INVALID_ARG
    assert call(nws=256) == g.GDR_ERR_INVALID_ARG
    assert call(ex=8) == g.GDR_ERR_INVALID_ARG
    assert call(nseq=0) == g.GDR_OK


@pytest.mark.parametrize("fn", ["gdn_backward", "kda_backward"])
def test_backward_rejects_bad_arguments(g, fn):
    f = getattr(g.lib, fn)
    P = 1 << 20

    def call(**kw):
        a = dict(q=P, k=P, v=P, alpha=P, beta=P, s0=None, dO=P, dsf=None, dq=P, dk_out=P,
                 dv_out=P, dalpha=P, dbeta=P, ds0=P, B=2, T=100, H=2, dk=128, dv=128,
                 i=1, do=1, ws=P, nws=1 << 30)
        a.update(kw)
        return f(a["q"], a["k"], a["v"], a["alpha"], a["beta"], a["s0"], a["dO"], a["dsf"],
                 a["dq"], a["dk_out"], a["dv_out"], a["dalpha"], a["dbeta"], a["ds0"], a["B"],
                 a["T"], a["H"], a["dk"], a["dv"], a["i"], a["do"], a["ws"], a["nws"], None)
    assert call(dk=48) == g.GDR_ERR_UNSUPPORTED
    assert call(B=-1) == g.GDR_ERR_INVALID_ARG
    assert call(i=7) == g.GDR_ERR_INVALID_ARG
    assert call(dq=None) == g.GDR_ERR_INVALID_ARG
    assert call(ds0=None) == g.GDR_ERR_INVALID_ARG
    assert call(dO=P + 8) == g.GDR_ERR_INVALID_ARG
    assert call(ws=None) == g.GDR_ERR_INVALID_ARG
    assert call(B=0) == g.GDR_OK


def test_checks_build_exports_the_same_symbols(g):
    """The debug twin (device-side index checks) is built beside the product library and
    exports every declared symbol too."""
    path = os.path.join(os.path.dirname(g.LIB_PATH), "libgdr_checks.so")
    assert os.path.exists(path), "libgdr_checks.so missing: build with --checks"
    lib = ctypes.CDLL(path)
    for name in _declared_symbols():
        assert hasattr(lib, name), f"{name} not exported by libgdr_checks.so"


def test_product_build_has_no_device_checks(g):
    """gdr_check_status answers GDR_ERR_UNSUPPORTED in the product build, without a CUDA
    call (so this runs on a machine with no GPU)."""
    if os.environ.get("GDR_LIBRARY") == "checks":
        pytest.skip("the checks build is loaded")
    assert g.lib.gdr_check_status(None) == g.GDR_ERR_UNSUPPORTED
    assert "GDR_CHECKS" in g.lib.gdr_last_error().decode()
