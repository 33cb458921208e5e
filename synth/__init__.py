"""Seeded synthetic inputs for the GDN / KDA workloads.

This module is shared by the tests, the oracle side and the GPU side.  It holds
no arithmetic of the method itself: it only draws random tensors with the
distributions of the workloads and rounds them to the input dtype.

Workloads (all inputs synthetic; the pages publish no dataset for the mixer):

  gdn_seq_f32   GDN, B=1 H=2 T=64 d_k=d_v=32, fp32 inputs, zero initial state
  gdn_prefill   GDN, B=1 H=32 T=4096 d=128, bf16 q/k/v, zero initial state
  kda_prefill   KDA, same shapes, per-channel gates
  decode        N=256 sequences x H=32, d=128, 512 one-token steps, bf16
                q/k/v, fp32 state ~ 0.02 N(0,1); GDN and KDA gates
  kda_long      KDA, B=4 H=32 T=65536 d=128, bf16, state ~ 0.02 N(0,1)
  verify_gdn    N=256 sequences x H=32, d=128, K=4 tokens from a carried state
  verify_kda    ~ 0.02 N(0,1), bf16 q/k/v; GDN and KDA gates (B = N, T = K)
  gdn_varlen    64 prompts packed along the tokens, H=32, d=128, bf16, each from its
  kda_varlen    own slot of a state pool ~ 0.02 N(0,1); lengths from varlen_lengths
  gdn_backward  the gradients of the gdn_prefill / kda_prefill shapes; dL/do ~ N(0,1)
  kda_backward  (bf16) and dL/dS_T ~ N(0,1) (fp32), drawn after the inputs
  *_prologue    gdn_prefill, kda_prefill and decode_gdn with the raw inputs of the fused
                prologue: q, k not normalised and the gate logits x in place of alpha

Recipe per (batch b, head h) slice, one ``torch.Generator`` (CPU) seeded with
``slice_seed(seed, b, h)``, drawing in this fixed order:

  q [T, d_k] ~ N(0,1), then divided by its L2 norm over d_k (fp32), then cast
  k [T, d_k] ~ N(0,1), same normalisation and cast
  v [T, d_v] ~ N(0,1), cast
  beta [T]           = sigmoid(N(0,1))                           (fp32)
  alpha [T] (GDN) or [T, d_k] (KDA) = exp(-softplus(N(0,1) + 2)) (fp32)
  s0 [d_v, d_k]      = 0.02 N(0,1) when the workload has a non-zero state

Prologue workloads draw, in the same order, q and k as N(0,1) times exp(N(0,1)) (one
scale per vector, drawn after the vector) instead of unit vectors, and the gate logits
x = N(0,1) + 2 instead of alpha = exp(-softplus(x)).

Stress gate recipes (not part of the workloads; used by tests so that the
inter-chunk carry matters): "slow" = exp(-softplus(N(0,1) - 5)) (about 0.993),
"one" = 1, "zero_some" = the workload gates with every 7th token set to 0.

For decode the "T" axis of a slice is the step axis: slice (n, h) holds the
inputs of sequence n, head h for every step.
"""

from dataclasses import dataclass, replace
import math

import torch
import torch.nn.functional as F


@dataclass(frozen=True)
class Workload:
    name: str
    mixer: str          # "gdn" or "kda"
    B: int              # batch (sequences for decode)
    H: int
    T: int              # tokens (decode: steps)
    dk: int
    dv: int
    dtype: str          # "f32" or "bf16" for q, k, v
    state: str          # "zeros" or "randn"
    decode: bool = False
    verify: bool = False  # K tokens (the T axis) from a carried state, snapshots kept
    varlen: bool = False  # B sequences of varlen_lengths(w) tokens packed (T: median)
    backward: bool = False  # the gradients of the prefill of these shapes
    prologue: int = 0       # fused-prologue flags: raw q, k and gate logits are drawn

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw):
        return replace(self, **kw)


WORKLOADS = {
    "gdn_seq_f32": Workload("gdn_seq_f32", "gdn", 1, 2, 64, 32, 32, "f32", "zeros"),
    "gdn_prefill": Workload("gdn_prefill", "gdn", 1, 32, 4096, 128, 128, "bf16", "zeros"),
    "kda_prefill": Workload("kda_prefill", "kda", 1, 32, 4096, 128, 128, "bf16", "zeros"),
    "decode_gdn": Workload("decode_gdn", "gdn", 256, 32, 512, 128, 128, "bf16", "randn", True),
    "decode_kda": Workload("decode_kda", "kda", 256, 32, 512, 128, 128, "bf16", "randn", True),
    "kda_long": Workload("kda_long", "kda", 4, 32, 65536, 128, 128, "bf16", "randn"),
    # kda_long's batch, heads and entering state over 4096 tokens: the same kernels and
    # per-chunk traffic (128 chains take the per-head carry) in 1/16 of the memory, for
    # ncu captures that must stay small
    "kda_long_t4096": Workload("kda_long_t4096", "kda", 4, 32, 4096, 128, 128, "bf16", "randn"),
    "verify_gdn": Workload("verify_gdn", "gdn", 256, 32, 4, 128, 128, "bf16", "randn",
                           verify=True),
    "verify_kda": Workload("verify_kda", "kda", 256, 32, 4, 128, 128, "bf16", "randn",
                           verify=True),
    "gdn_varlen": Workload("gdn_varlen", "gdn", 64, 32, 256, 128, 128, "bf16", "randn",
                           varlen=True),
    "kda_varlen": Workload("kda_varlen", "kda", 64, 32, 256, 128, 128, "bf16", "randn",
                           varlen=True),
    "gdn_backward": Workload("gdn_backward", "gdn", 1, 32, 4096, 128, 128, "bf16", "zeros",
                             backward=True),
    "gdn_prefill_prologue": Workload("gdn_prefill_prologue", "gdn", 1, 32, 4096, 128, 128, "bf16",
                                     "zeros", prologue=3),
    "kda_prefill_prologue": Workload("kda_prefill_prologue", "kda", 1, 32, 4096, 128, 128, "bf16",
                                     "zeros", prologue=3),
    "decode_gdn_prologue": Workload("decode_gdn_prologue", "gdn", 256, 32, 512, 128, 128, "bf16",
                                    "randn", True, prologue=3),
    "kda_backward": Workload("kda_backward", "kda", 1, 32, 4096, 128, 128, "bf16", "zeros",
                             backward=True),
}


def varlen_lengths(w: Workload, seed: int = 0):
    """Prompt lengths of a packed workload: log-normal around the median w.T
    (sigma 0.8), rounded, clipped to [1, 16 w.T], drawn from a seeded CPU generator."""
    g = torch.Generator().manual_seed(1_000_003 * seed + 17)
    x = torch.randn(w.B, generator=g, dtype=torch.float64)
    lens = torch.exp(math.log(w.T) + 0.8 * x).round().clamp(1, 16 * w.T).to(torch.int64)
    return [int(n) for n in lens]


def slice_seed(seed, b, h):
    """Deterministic 63-bit seed for slice (b, h) of a workload drawn with ``seed``."""
    return ((seed * 1_000_003 + b) * 1_000_003 + h) % (2 ** 63 - 1)


def _unit_rows(x):
    return x / x.norm(dim=-1, keepdim=True)


def _gates(gen, shape, gates):
    x = torch.randn(shape, generator=gen, dtype=torch.float32)
    if gates == "slow":
        return torch.exp(-F.softplus(x - 5.0))
    a = torch.exp(-F.softplus(x + 2.0))
    if gates == "one":
        return torch.ones_like(a)
    if gates == "zero_some":
        a[::7] = 0.0
        return a
    if gates != "workload":
        raise ValueError(f"unknown gate recipe {gates!r}")
    return a


def slice_inputs(w: Workload, b: int, h: int, seed: int = 0, gates: str = "workload"):
    """Inputs of slice (b, h): dict of CPU tensors q, k [T, dk] and v [T, dv] in the
    workload dtype; beta [T], alpha [T] or [T, dk] and s0 [dv, dk] (or None) in fp32."""
    g = torch.Generator().manual_seed(slice_seed(seed, b, h))
    T, dk, dv = w.T, w.dk, w.dv
    if w.prologue:
        def vec():
            x = torch.randn((T, dk), generator=g)
            return (x * torch.exp(torch.randn((T, 1), generator=g))).to(w.torch_dtype)
        q, k = vec(), vec()
        v = torch.randn((T, dv), generator=g).to(w.torch_dtype)
        beta = torch.sigmoid(torch.randn((T,), generator=g))
        alpha = torch.randn((T, dk) if w.mixer == "kda" else (T,), generator=g) + 2.0
        s0 = 0.02 * torch.randn((dv, dk), generator=g) if w.state == "randn" else None
        return dict(q=q, k=k, v=v, beta=beta, alpha=alpha, s0=s0)
    q = _unit_rows(torch.randn((T, dk), generator=g)).to(w.torch_dtype)
    k = _unit_rows(torch.randn((T, dk), generator=g)).to(w.torch_dtype)
    v = torch.randn((T, dv), generator=g).to(w.torch_dtype)
    beta = torch.sigmoid(torch.randn((T,), generator=g))
    alpha = _gates(g, (T, dk) if w.mixer == "kda" else (T,), gates)
    s0 = 0.02 * torch.randn((dv, dk), generator=g) if w.state == "randn" else None
    return dict(q=q, k=k, v=v, beta=beta, alpha=alpha, s0=s0)


def make_inputs(w: Workload, seed: int = 0, gates: str = "workload"):
    """Full input tensors on the CPU, assembled from the per-slice draws.

    Prefill layout: q, k [B, T, H, dk]; v [B, T, H, dv]; beta [B, T, H];
    alpha [B, T, H] (GDN) or [B, T, H, dk] (KDA); s0 [B, H, dv, dk] or None.
    Decode layout: the same with B -> N and T -> steps, permuted to
    [steps, N, H, ...] so that step s reads x[s]; s0 [N, H, dv, dk].
    """
    B, T, H = w.B, w.T, w.H
    parts = [[slice_inputs(w, b, h, seed, gates) for h in range(H)] for b in range(B)]

    def stack(key):
        if parts[0][0][key] is None:
            return None
        return torch.stack([torch.stack([parts[b][h][key] for h in range(H)], dim=1)
                            for b in range(B)])          # [B, T, H, ...]

    out = {key: stack(key) for key in ("q", "k", "v", "beta", "alpha")}
    s0 = None
    if parts[0][0]["s0"] is not None:
        s0 = torch.stack([torch.stack([parts[b][h]["s0"] for h in range(H)])
                          for b in range(B)])
    out["s0"] = s0
    if w.decode:
        for key in ("q", "k", "v", "beta", "alpha"):
            out[key] = out[key].transpose(0, 1).contiguous()   # [steps, N, H, ...]
    return out


def device_inputs(w: Workload, device, seed: int = 0, dtype_override=None):
    """Inputs with the same distributions drawn directly on ``device`` (used by the
    benchmark, where only the distribution matters; values differ from
    ``make_inputs``).  Same layouts as ``make_inputs``."""
    g = torch.Generator(device=device).manual_seed(seed)
    dt = dtype_override or w.torch_dtype
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
    lead = (T, B, H) if w.decode else (B, T, H)

    def unit(shape):
        x = torch.randn(shape, generator=g, device=device)
        if w.prologue:
            scale = torch.exp(torch.randn(shape[:-1] + (1,), generator=g, device=device))
            return (x * scale).to(dt)
        return (x / x.norm(dim=-1, keepdim=True)).to(dt)

    q = unit(lead + (dk,))
    k = unit(lead + (dk,))
    v = torch.randn(lead + (dv,), generator=g, device=device).to(dt)
    beta = torch.sigmoid(torch.randn(lead, generator=g, device=device))
    ashape = lead + (dk,) if w.mixer == "kda" else lead
    logit = torch.randn(ashape, generator=g, device=device) + 2.0
    alpha = logit if w.prologue else torch.exp(-F.softplus(logit))
    s0 = None
    if w.state == "randn":
        s0 = 0.02 * torch.randn((B, H, dv, dk), generator=g, device=device)
    return dict(q=q, k=k, v=v, beta=beta, alpha=alpha, s0=s0)


def tokens(w: Workload):
    """Tokens processed by one pass of the workload (prefill: B*T; decode: N*steps;
    packed: the sum of the lengths)."""
    if w.varlen:
        return sum(varlen_lengths(w))
    return w.B * w.T


def chunk_count(w: Workload, chunk=64):
    return w.B * w.H * math.ceil(w.T / chunk)
