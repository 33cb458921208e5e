"""Shared helpers for the parity tests: run the CUDA path on CPU-drawn inputs and
compare with the oracle using the normwise relative error."""

import numpy as np
import torch


def rel_err(x, ref):
    """Normwise relative error ||x - ref||_2 / ||ref||_2 (0 if both are 0)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    n = np.linalg.norm(ref)
    d = np.linalg.norm(x - ref)
    return d / n if n > 0 else d


def slice_errs(x, ref, axes):
    """Max over slices of the normwise relative error, slicing over ``axes``
    (the remaining axes form one slice)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    other = tuple(i for i in range(x.ndim) if i not in axes)
    xs = np.moveaxis(x, axes, range(len(axes))).reshape(
        int(np.prod([x.shape[a] for a in axes])), -1)
    rs = np.moveaxis(ref, axes, range(len(axes))).reshape(xs.shape[0], -1)
    del other
    out = 0.0
    for a, b in zip(xs, rs):
        out = max(out, rel_err(a, b))
    return out


def to_np(t):
    return t.detach().to("cpu", torch.float64).numpy()


def bf16_round_floor(ref):
    """Normwise error of merely rounding the exact result to bf16: the floor any
    bf16 output carries."""
    r = torch.from_numpy(np.asarray(ref)).to(torch.bfloat16).to(torch.float64).numpy()
    return rel_err(r, ref)
