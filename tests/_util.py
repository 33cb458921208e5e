"""Shared helpers for the parity tests: run the CUDA path on CPU-drawn inputs and
compare with the oracle, normwise and element by element.

Normwise: ||x - ref||_2 / ||ref||_2 over the whole tensor and over every (batch, head)
slice, against the bar of the precision class (2e-3 for bf16 inputs, 1e-5 for fp32).

Element-wise: every element must satisfy

    |x - ref| <= tol_e * (|ref| + rms(ref over its (batch, head) slice))

so that one wrong element (a bad lane, a stale token row) cannot hide under a norm
taken over half a million elements.  The rms term keeps elements near zero from
demanding a relative accuracy no rounding model gives them.  The bounds per precision
class (ELEM_TOL) follow from the arithmetic of the path:

* ``tc``: bf16 inputs through the tensor-core kernels, whose state-dependent operands
  are rounded to tf32 (unit 2^-11).  The normwise error is 3-6e-4; an element's error
  is a sum of many such roundings, and its largest value over ~1e6 elements sits a
  few standard deviations out, so 8e-3 (16 tf32 units) bounds it with margin.
* ``cc``: fp32 arithmetic on the CUDA cores (decode, verify, the CUDA-core prefill,
  the backward) on bf16 or fp32 inputs: normwise ~1e-6.  The chunk-local cumulative
  log gate G is held in fp32, so a decay e^{G_t - G_j} is off by up to |G| 2^-24
  relative; the stress gates (alpha = 0, floored at e^-30) drive |G| to several hundred
  within a chunk, i.e. ~3e-5 per factor.  Bound 1e-4 per element.
* ``f32``: fp32 inputs through the CUDA-core prefill, held to the 1e-5 normwise bar:
  the same fp32 arithmetic as ``cc``, bound 1e-4.
* ``pro``: the fused prologue on bf16 inputs through the CUDA-core kernels.  Both
  sides normalise q and k and round them to bf16 on their own, so a rounding decision
  may differ by one bf16 unit (at most 2^-7 of that element of q or k); that element
  enters an output through one term of a d_k-term product, which bounds its effect
  near 2^-7 / sqrt(d_k) of the output scale; 2e-3 with the fp32 arithmetic on top.
* A bf16 output adds at most half a bf16 unit, 2^-8 of |x|, on top (``bf16_out``).

When GDR_ELEM_LOG names a file, every check appends its measured worst ratio there
(one JSON object per line) so the bounds can be compared with the errors the kernels
actually make.
"""

import json
import os

import numpy as np
import torch

NORM_TOL = {"f32": 1e-5, "bf16": 2e-3}
ELEM_TOL = {"tc": 8e-3, "cc": 1e-4, "f32": 1e-4, "pro": 2e-3}
BF16_HALF_UNIT = 2.0 ** -8


def rel_err(x, ref):
    """Normwise relative error ||x - ref||_2 / ||ref||_2 (0 if both are 0)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    n = np.linalg.norm(ref)
    d = np.linalg.norm(x - ref)
    return d / n if n > 0 else d


def _slices(a, axes):
    """View of `a` as [n_slices, slice_elements], slicing over `axes`."""
    a = np.asarray(a, dtype=np.float64)
    if not axes:
        return a.reshape(1, -1)
    n = int(np.prod([a.shape[i] for i in axes]))
    return np.moveaxis(a, axes, range(len(axes))).reshape(n, -1)


def slice_errs(x, ref, axes):
    """Max over slices of the normwise relative error, slicing over ``axes``
    (the remaining axes form one slice)."""
    xs, rs = _slices(x, axes), _slices(ref, axes)
    out = 0.0
    for a, b in zip(xs, rs):
        out = max(out, rel_err(a, b))
    return out


def elem_err(x, ref, axes=()):
    """Largest |x - ref| / (|ref| + rms(ref over the element's slice)), slicing over
    ``axes`` (empty: the whole tensor is one slice).  Returns (ratio, flat index)."""
    xs, rs = _slices(x, axes), _slices(ref, axes)
    if rs.size == 0:
        return 0.0, None
    rms = np.sqrt(np.mean(rs * rs, axis=1, keepdims=True))
    den = np.abs(rs) + rms
    num = np.abs(xs - rs)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(den > 0, num / np.where(den > 0, den, 1.0), np.where(num > 0, np.inf, 0.0))
    i = int(np.argmax(ratio))
    return float(ratio.flat[i]), i


def elem_tol(cls, bf16_out=False):
    """Element-wise bound of precision class `cls`, plus half a bf16 unit when the
    output was rounded to bf16."""
    return ELEM_TOL[cls] + (BF16_HALF_UNIT if bf16_out else 0.0)


def check_elem(x, ref, cls, axes=(), bf16_out=False, label=""):
    """Assert the element-wise bound of `cls` on x against ref (see the module doc)."""
    tol = elem_tol(cls, bf16_out)
    r, i = elem_err(x, ref, axes)
    path = os.environ.get("GDR_ELEM_LOG")
    if path:
        test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
        with open(path, "a") as f:
            f.write(json.dumps({"test": test, "label": label, "cls": cls,
                                "bf16_out": bool(bf16_out), "ratio": r, "tol": tol}) + "\n")
    assert r <= tol, (f"{label}: element {i} off by {r:.3e} of (|ref| + slice rms), "
                      f"bound {tol:.3e}")
    return r


def is_bf16(t):
    return getattr(t, "dtype", None) == torch.bfloat16


def to_np(t):
    return t.detach().to("cpu", torch.float64).numpy()


def bf16_round_floor(ref):
    """Normwise error of merely rounding the exact result to bf16: the floor any
    bf16 output carries."""
    r = torch.from_numpy(np.asarray(ref)).to(torch.bfloat16).to(torch.float64).numpy()
    return rel_err(r, ref)
