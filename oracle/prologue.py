"""The mixer's input prologue in fp64: L2-normalised q, k and the gate from its logit.

TEST INFRASTRUCTURE ONLY: never imported by the product path.

"Super Apriel: One Checkpoint, Many Speeds" names the GDN and KDA mixers (§2A) but
leaves the projections around the recurrence unspecified.  The configurations the
kernels are measured on draw q and k as L2-normalised vectors per (token, head) and
the gates as alpha = exp(-softplus(x)) of a pre-activation x; the fused prologue takes
the raw q, k and x and forms those inside the kernels.  Readings taken where the pages
are silent:

  * q_hat = q / sqrt(sum(q^2) + eps) with eps = 1e-6 (a zero vector stays zero), the same
    for k, over the d_k channels of one (token, head);
  * with bf16 inputs the normalised vectors are rounded to bf16 (round to nearest even),
    as a bf16 tensor would hold them before the mixer;
  * softplus(x) = log(1 + e^x), alpha = exp(-softplus(x)) = 1 / (1 + e^x).
"""

import numpy as np
import torch

L2NORM_EPS = 1e-6


def l2_normalise(x, eps=L2NORM_EPS):
    """x / sqrt(sum of squares over the last axis + eps), in fp64."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt((x * x).sum(axis=-1, keepdims=True) + eps)


def softplus(x):
    """log(1 + e^x) in fp64, without overflow for large |x|."""
    x = np.asarray(x, dtype=np.float64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def gate_from_logit(x):
    """alpha = exp(-softplus(x))."""
    return np.exp(-softplus(x))


def round_bf16(x):
    """Round fp64 values to the nearest bf16 (ties to even), returned as fp64."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64)).to(torch.float32)
    return t.to(torch.bfloat16).to(torch.float64).numpy()


def apply_prologue(q, k, alpha, l2norm=True, gate_logit=True, bf16=False):
    """The inputs the recurrence sees: (q_hat, k_hat, alpha) from raw q, k and, with
    gate_logit, the gate pre-activation in `alpha`.  Flags off pass the tensor through."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    if l2norm:
        q, k = l2_normalise(q), l2_normalise(k)
        if bf16:
            q, k = round_bf16(q), round_bf16(k)
    a = gate_from_logit(alpha) if gate_logit else np.asarray(alpha, dtype=np.float64)
    return q, k, a
