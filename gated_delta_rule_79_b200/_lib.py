"""ctypes binding of libgdr (include/gdr.h): argument marshalling only.

Every function here checks tensor devices, dtypes, shapes and contiguity,
allocates outputs with torch (device memory is torch's job), and passes raw
pointers plus the current CUDA stream to the C ABI.  All arithmetic of the
method runs in the library's CUDA kernels; there is no fallback.  Importing this
module raises if libgdr.so has not been built.
"""

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# GDR_LIBRARY=checks loads the debug build with device-side index checks
# (libgdr_checks.so, see build.py) instead of the product library.
LIB_PATH = os.path.join(_HERE, "libgdr_checks.so" if os.environ.get("GDR_LIBRARY") == "checks"
                        else "libgdr.so")

GDR_OK, GDR_ERR_INVALID_ARG, GDR_ERR_UNSUPPORTED, GDR_ERR_CUDA, GDR_ERR_TIMEOUT = range(5)
GDR_F32, GDR_BF16 = 0, 1
CHUNK = 64

EXPORTS = ["gdr_version", "gdr_last_error", "gdr_prefill_workspace_bytes", "gdn_prefill",
           "kda_prefill", "gdn_decode", "kda_decode", "gdr_workspace_status",
           "gdr_prefill_path", "gdn_prefill_noalloc", "gdr_noalloc_status", "gdr_check_status",
           "gdr_timing_start", "gdr_timing_stop",
           "gdn_verify", "kda_verify", "gdr_prefill_varlen_workspace_bytes",
           "gdn_prefill_varlen", "kda_prefill_varlen", "gdr_backward_workspace_bytes",
           "gdn_backward", "kda_backward", "gdn_prefill_ex", "kda_prefill_ex", "gdn_decode_ex",
           "kda_decode_ex", "gdn_verify_ex", "kda_verify_ex", "gdn_prefill_varlen_ex",
           "kda_prefill_varlen_ex"]

# fused prologue flags of the *_ex entry points (prologue= keyword below)
PROLOGUE_L2NORM_QK = 1   # q, k raw: L2-normalised per (token, head) inside the kernels
PROLOGUE_GATE_LOGIT = 2  # alpha holds x: the gate is exp(-softplus(x))


class GdrError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"[gdr status {status}] {message}")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m gated_delta_rule_79_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, fp, i, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.gdr_version.restype = i
    lib.gdr_version.argtypes = []
    lib.gdr_last_error.restype = ctypes.c_char_p
    lib.gdr_last_error.argtypes = []
    lib.gdr_prefill_workspace_bytes.restype = sz
    lib.gdr_prefill_workspace_bytes.argtypes = [i, i, i, i, i, i]
    for name in ("gdn_prefill", "kda_prefill"):
        f = getattr(lib, name)
        f.restype = i
        f.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, i, i, i, i, i, i, i, i, vp, sz, vp]
    for name in ("gdn_decode", "kda_decode"):
        f = getattr(lib, name)
        f.restype = i
        f.argtypes = [vp, vp, vp, fp, fp, fp, vp, i, i, i, i, i, i, vp]
    for name in ("gdn_verify", "kda_verify"):
        f = getattr(lib, name)
        f.restype = i
        f.argtypes = [vp, vp, vp, fp, fp, fp, fp, vp, i, i, i, i, i, i, i, vp]
    lib.gdr_prefill_varlen_workspace_bytes.restype = sz
    lib.gdr_prefill_varlen_workspace_bytes.argtypes = [i, i, i, i, i, i]
    for name in ("gdn_prefill_varlen", "kda_prefill_varlen"):
        f = getattr(lib, name)
        f.restype = i
        f.argtypes = [vp, vp, vp, fp, fp, vp, vp, fp, vp, i, i, i, i, i, i, i, i, vp, sz, vp]
    for name in ("gdn_prefill", "kda_prefill", "gdn_decode", "kda_decode", "gdn_verify",
                 "kda_verify", "gdn_prefill_varlen", "kda_prefill_varlen"):
        f = getattr(lib, name + "_ex")
        f.restype = i
        f.argtypes = list(getattr(lib, name).argtypes) + [ctypes.c_uint]
    lib.gdr_backward_workspace_bytes.restype = sz
    lib.gdr_backward_workspace_bytes.argtypes = [i, i, i, i, i, i]
    for name in ("gdn_backward", "kda_backward"):
        f = getattr(lib, name)
        f.restype = i
        f.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, fp, fp, fp, fp, fp, fp,
                      i, i, i, i, i, i, i, vp, sz, vp]
    lib.gdn_prefill_noalloc.restype = i
    lib.gdn_prefill_noalloc.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, i, i, i, i, i, i, i, i, vp]
    lib.gdr_noalloc_status.restype = i
    lib.gdr_noalloc_status.argtypes = [vp]
    lib.gdr_check_status.restype = i
    lib.gdr_check_status.argtypes = [vp]
    lib.gdr_prefill_path.restype = i
    lib.gdr_prefill_path.argtypes = [i, i, i, i]
    lib.gdr_workspace_status.restype = i
    lib.gdr_workspace_status.argtypes = [vp, sz, vp]
    lib.gdr_timing_start.restype = i
    lib.gdr_timing_start.argtypes = []
    lib.gdr_timing_stop.restype = i
    lib.gdr_timing_stop.argtypes = [ctypes.POINTER(ctypes.c_float), i, ctypes.POINTER(i)]
    return lib


lib = _load()


def _check(status):
    if status != GDR_OK:
        raise GdrError(status, lib.gdr_last_error().decode())


def _pick(name, prologue):
    """The plain entry point, or its fused-prologue variant with the flags appended."""
    if prologue:
        return getattr(lib, name + "_ex"), (int(prologue),)
    return getattr(lib, name), ()


def _code(dtype):
    if dtype == torch.float32:
        return GDR_F32
    if dtype == torch.bfloat16:
        return GDR_BF16
    raise TypeError(f"unsupported dtype {dtype} (float32 or bfloat16)")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device, stream):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, shape, dtype=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


_ws_lock = threading.Lock()
_ws_cache = {}


def prefill_workspace(B, T, H, dk, dv, kda, device, stream=None):
    """Zero-initialised device workspace for a prefill call, cached per
    (device, stream) and grown on demand.  Returns (tensor, nbytes)."""
    need = lib.gdr_prefill_workspace_bytes(B, T, H, dk, dv, int(kda))
    if need == 0:
        raise GdrError(GDR_ERR_INVALID_ARG, "invalid prefill sizes")
    s = stream if stream is not None else torch.cuda.current_stream(device)
    key = (device, s.cuda_stream)
    with _ws_lock:
        buf = _ws_cache.get(key)
        if buf is None or buf.numel() < need:
            with torch.cuda.stream(s):
                buf = torch.zeros(max(need, 1 << 12), dtype=torch.uint8, device=device)
            _ws_cache[key] = buf
    return buf, buf.numel()


def _prefill(kda, q, k, v, alpha, beta, s0, out_dtype, o, s_final, chunk, stream, workspace,
             prologue=0):
    if q.dim() != 4:
        raise ValueError("q must be [B, T, H, d_k]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (there is no CPU path)")
    dt = q.dtype
    _need(q, "q", (B, T, H, dk), dt, dev)
    _need(k, "k", (B, T, H, dk), dt, dev)
    _need(v, "v", (B, T, H, dv), dt, dev)
    _need(alpha, "alpha", (B, T, H, dk) if kda else (B, T, H), torch.float32, dev)
    _need(beta, "beta", (B, T, H), torch.float32, dev)
    if s0 is not None:
        _need(s0, "s0", (B, H, dv, dk), torch.float32, dev)
    out_dtype = out_dtype or dt
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=out_dtype, device=dev)
    _need(o, "o", (B, T, H, dv), out_dtype, dev)
    if s_final is None:
        s_final = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    elif s_final is not False:
        _need(s_final, "s_final", (B, H, dv, dk), torch.float32, dev)
    sf = None if s_final is False else s_final
    if workspace is None:
        ws, nws = prefill_workspace(B, T, H, dk, dv, kda, dev, stream)
    else:
        ws, nws = workspace, workspace.numel() * workspace.element_size()
    fn, extra = _pick("kda_prefill" if kda else "gdn_prefill", prologue)
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(s0), _ptr(o), _ptr(sf),
              B, T, H, dk, dv, _code(dt), _code(out_dtype), chunk, _ptr(ws), nws,
              _stream(dev, stream), *extra))
    return o, sf


def gdn_prefill(q, k, v, alpha, beta, s0=None, *, out_dtype=None, o=None, s_final=None,
                chunk=CHUNK, stream=None, workspace=None, prologue=0):
    """Gated DeltaNet chunked prefill (scalar gate alpha [B, T, H]).

    q, k [B, T, H, d_k] and v [B, T, H, d_v] in float32 or bfloat16; alpha, beta
    float32; s0 [B, H, d_v, d_k] float32 or None.  Returns (o, s_final); pass
    s_final=False to skip writing the final state, or s_final=s0 to carry in place.
    prologue: PROLOGUE_* flags (raw q, k normalised in the kernel; alpha given as the
    gate pre-activation x, alpha = exp(-softplus(x))).
    """
    return _prefill(False, q, k, v, alpha, beta, s0, out_dtype, o, s_final, chunk, stream,
                    workspace, prologue)


def kda_prefill(q, k, v, alpha, beta, s0=None, *, out_dtype=None, o=None, s_final=None,
                chunk=CHUNK, stream=None, workspace=None, prologue=0):
    """Kimi Delta Attention chunked prefill (per-channel gate alpha [B, T, H, d_k]);
    otherwise as ``gdn_prefill``."""
    return _prefill(True, q, k, v, alpha, beta, s0, out_dtype, o, s_final, chunk, stream,
                    workspace, prologue)


def _decode(kda, q, k, v, alpha, beta, state, out_dtype, o, stream, prologue=0):
    if q.dim() != 3:
        raise ValueError("q must be [N, H, d_k]")
    N, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (there is no CPU path)")
    dt = q.dtype
    _need(q, "q", (N, H, dk), dt, dev)
    _need(k, "k", (N, H, dk), dt, dev)
    _need(v, "v", (N, H, dv), dt, dev)
    _need(alpha, "alpha", (N, H, dk) if kda else (N, H), torch.float32, dev)
    _need(beta, "beta", (N, H), torch.float32, dev)
    _need(state, "state", (N, H, dv, dk), torch.float32, dev)
    out_dtype = out_dtype or dt
    if o is None:
        o = torch.empty((N, H, dv), dtype=out_dtype, device=dev)
    _need(o, "o", (N, H, dv), out_dtype, dev)
    fn, extra = _pick("kda_decode" if kda else "gdn_decode", prologue)
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(state), _ptr(o),
              N, H, dk, dv, _code(dt), _code(out_dtype), _stream(dev, stream), *extra))
    return o


def gdn_decode(q, k, v, alpha, beta, state, *, out_dtype=None, o=None, stream=None, prologue=0):
    """One Gated DeltaNet decode step for N sequences; ``state`` [N, H, d_v, d_k]
    float32 is updated in place.  Returns o [N, H, d_v]."""
    return _decode(False, q, k, v, alpha, beta, state, out_dtype, o, stream, prologue)


def kda_decode(q, k, v, alpha, beta, state, *, out_dtype=None, o=None, stream=None, prologue=0):
    """One Kimi Delta Attention decode step (alpha [N, H, d_k]); as ``gdn_decode``."""
    return _decode(True, q, k, v, alpha, beta, state, out_dtype, o, stream, prologue)


def _prefill_varlen(kda, q, k, v, alpha, beta, cu_seqlens, state, slots, out_dtype, o,
                    chunk, stream, workspace, prologue=0):
    if q.dim() != 3:
        raise ValueError("q must be [total, H, d_k] (sequences packed along the tokens)")
    total, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (there is no CPU path)")
    dt = q.dtype
    _need(q, "q", (total, H, dk), dt, dev)
    _need(k, "k", (total, H, dk), dt, dev)
    _need(v, "v", (total, H, dv), dt, dev)
    _need(alpha, "alpha", (total, H, dk) if kda else (total, H), torch.float32, dev)
    _need(beta, "beta", (total, H), torch.float32, dev)
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.device != dev:
        raise ValueError("cu_seqlens must be a 1-D int32 tensor on the inputs' device")
    nseq = cu_seqlens.numel() - 1
    if nseq < 0:
        raise ValueError("cu_seqlens needs nseq + 1 entries")
    if state.dim() != 4 or state.shape[1:] != (H, dv, dk) or state.dtype != torch.float32:
        raise ValueError("state must be a float32 pool [nslots, H, d_v, d_k]")
    if not state.is_contiguous() or state.device != dev:
        raise ValueError("state must be contiguous on the inputs' device")
    if slots is not None and (slots.dtype != torch.int32 or slots.numel() != nseq
                              or slots.device != dev):
        raise ValueError("slots must be an int32 tensor of nseq entries on the inputs' device")
    if slots is None and state.shape[0] < nseq:
        raise ValueError("without slots the pool needs one slot per sequence")
    out_dtype = out_dtype or dt
    if o is None:
        o = torch.empty((total, H, dv), dtype=out_dtype, device=dev)
    _need(o, "o", (total, H, dv), out_dtype, dev)
    need = lib.gdr_prefill_varlen_workspace_bytes(nseq, total, H, dk, dv, int(kda))
    if workspace is None:
        s = stream if stream is not None else torch.cuda.current_stream(dev)
        with torch.cuda.stream(s):
            workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
    fn, extra = _pick("kda_prefill_varlen" if kda else "gdn_prefill_varlen", prologue)
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(cu_seqlens), _ptr(slots),
              _ptr(state), _ptr(o), nseq, total, H, dk, dv, _code(dt), _code(out_dtype), chunk,
              _ptr(workspace), workspace.numel(), _stream(dev, stream), *extra))
    return o


def gdn_prefill_varlen(q, k, v, alpha, beta, cu_seqlens, state, *, slots=None, out_dtype=None,
                       o=None, chunk=CHUNK, stream=None, workspace=None, prologue=0):
    """Gated DeltaNet prefill of nseq sequences packed along the tokens: q, k
    [total, H, d_k], v [total, H, d_v] bf16; alpha, beta [total, H] float32; cu_seqlens
    int32 [nseq + 1] on the device; state a float32 pool [nslots, H, d_v, d_k] read
    from and written back to slot slots[i] (default i) in place.  Returns o."""
    return _prefill_varlen(False, q, k, v, alpha, beta, cu_seqlens, state, slots, out_dtype, o,
                           chunk, stream, workspace, prologue)


def kda_prefill_varlen(q, k, v, alpha, beta, cu_seqlens, state, *, slots=None, out_dtype=None,
                       o=None, chunk=CHUNK, stream=None, workspace=None, prologue=0):
    """Kimi Delta Attention (alpha [total, H, d_k]); as ``gdn_prefill_varlen``."""
    return _prefill_varlen(True, q, k, v, alpha, beta, cu_seqlens, state, slots, out_dtype, o,
                           chunk, stream, workspace, prologue)


VERIFY_MAX_TOKENS = 16


def _verify(kda, q, k, v, alpha, beta, state, snapshots, out_dtype, o, stream, prologue=0):
    if q.dim() != 4:
        raise ValueError("q must be [N, K, H, d_k]")
    N, K, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (there is no CPU path)")
    dt = q.dtype
    _need(q, "q", (N, K, H, dk), dt, dev)
    _need(k, "k", (N, K, H, dk), dt, dev)
    _need(v, "v", (N, K, H, dv), dt, dev)
    _need(alpha, "alpha", (N, K, H, dk) if kda else (N, K, H), torch.float32, dev)
    _need(beta, "beta", (N, K, H), torch.float32, dev)
    _need(state, "state", (N, H, dv, dk), torch.float32, dev)
    if snapshots is True:
        snapshots = torch.empty((K, N, H, dv, dk), dtype=torch.float32, device=dev)
    elif snapshots is False:
        snapshots = None
    if snapshots is not None:
        _need(snapshots, "snapshots", (K, N, H, dv, dk), torch.float32, dev)
    out_dtype = out_dtype or dt
    if o is None:
        o = torch.empty((N, K, H, dv), dtype=out_dtype, device=dev)
    _need(o, "o", (N, K, H, dv), out_dtype, dev)
    fn, extra = _pick("kda_verify" if kda else "gdn_verify", prologue)
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(state), _ptr(snapshots),
              _ptr(o), N, K, H, dk, dv, _code(dt), _code(out_dtype), _stream(dev, stream),
              *extra))
    return o, snapshots


def gdn_verify(q, k, v, alpha, beta, state, *, snapshots=True, out_dtype=None, o=None,
               stream=None, prologue=0):
    """Gated DeltaNet over K tokens per sequence from a carried state, keeping the
    state after every token.  q, k [N, K, H, d_k]; v [N, K, H, d_v]; alpha, beta
    [N, K, H]; state [N, H, d_v, d_k] float32.  snapshots=True allocates, or pass a
    [K, N, H, d_v, d_k] float32 tensor; snapshots[t] is the state after token t+1 and
    ``state`` is left as it was.  snapshots=False updates ``state`` in place to the
    state after the K tokens instead.  Returns (o [N, K, H, d_v], snapshots or None)."""
    return _verify(False, q, k, v, alpha, beta, state, snapshots, out_dtype, o, stream,
                   prologue)


def kda_verify(q, k, v, alpha, beta, state, *, snapshots=True, out_dtype=None, o=None,
               stream=None, prologue=0):
    """Kimi Delta Attention (alpha [N, K, H, d_k]); as ``gdn_verify``."""
    return _verify(True, q, k, v, alpha, beta, state, snapshots, out_dtype, o, stream,
                   prologue)


def _backward(kda, q, k, v, alpha, beta, s0, do, ds_final, workspace, stream):
    if q.dim() != 4:
        raise ValueError("q must be [B, T, H, d_k]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (there is no CPU path)")
    dt = q.dtype
    _need(q, "q", (B, T, H, dk), dt, dev)
    _need(k, "k", (B, T, H, dk), dt, dev)
    _need(v, "v", (B, T, H, dv), dt, dev)
    _need(alpha, "alpha", (B, T, H, dk) if kda else (B, T, H), torch.float32, dev)
    _need(beta, "beta", (B, T, H), torch.float32, dev)
    if s0 is not None:
        _need(s0, "s0", (B, H, dv, dk), torch.float32, dev)
    _need(do, "do", (B, T, H, dv), None, dev)
    if ds_final is not None:
        _need(ds_final, "ds_final", (B, H, dv, dk), torch.float32, dev)
    f32 = dict(dtype=torch.float32, device=dev)
    dq = torch.empty((B, T, H, dk), **f32)
    dk_ = torch.empty((B, T, H, dk), **f32)
    dv_ = torch.empty((B, T, H, dv), **f32)
    dalpha = torch.empty(alpha.shape, **f32)
    dbeta = torch.empty((B, T, H), **f32)
    ds0 = torch.empty((B, H, dv, dk), **f32)
    need = lib.gdr_backward_workspace_bytes(B, T, H, dk, dv, int(kda))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    nws = workspace.numel() * workspace.element_size()
    fn = lib.kda_backward if kda else lib.gdn_backward
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(s0), _ptr(do),
              _ptr(ds_final), _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(dalpha), _ptr(dbeta),
              _ptr(ds0), B, T, H, dk, dv, _code(dt), _code(do.dtype), _ptr(workspace), nws,
              _stream(dev, stream)))
    return dq, dk_, dv_, dalpha, dbeta, ds0


def gdn_backward(q, k, v, alpha, beta, s0, do, ds_final=None, *, workspace=None, stream=None):
    """Gradients (dq, dk, dv, dalpha [B,T,H], dbeta, ds0), all fp32, of
    L = sum <do, o> + <ds_final, S_T> for gdn_prefill(q, k, v, alpha, beta, s0)."""
    return _backward(False, q, k, v, alpha, beta, s0, do, ds_final, workspace, stream)


def kda_backward(q, k, v, alpha, beta, s0, do, ds_final=None, *, workspace=None, stream=None):
    """As gdn_backward with the per-channel gate: dalpha is [B, T, H, d_k]."""
    return _backward(True, q, k, v, alpha, beta, s0, do, ds_final, workspace, stream)


def backward_workspace_bytes(B, T, H, dk, dv, kda):
    return lib.gdr_backward_workspace_bytes(B, T, H, dk, dv, int(kda))


def prefill_path(dk, dv, dtype, kda):
    """"tensor-core" or "cuda-core": which prefill kernel serves these parameters."""
    p = lib.gdr_prefill_path(dk, dv, _code(dtype), int(kda))
    if p < 0:
        raise GdrError(GDR_ERR_UNSUPPORTED, f"no prefill kernel for d_k={dk} d_v={dv}")
    return "tensor-core" if p == 1 else "cuda-core"


def check_status(stream=None):
    """Synchronise and read/clear the device-side index-check word of the checks build
    (libgdr_checks.so); raises GdrError(GDR_ERR_INVALID_ARG) if a check fired, and
    GdrError(GDR_ERR_UNSUPPORTED) in the product build, which has no checks."""
    dev = torch.device("cuda", torch.cuda.current_device())
    _check(lib.gdr_check_status(_stream(dev, stream)))


def noalloc_status(stream=None):
    """Synchronise and read/clear the sticky status of gdn_prefill_noalloc on the
    current device; raises GdrError(GDR_ERR_TIMEOUT) if a bounded device wait of a
    call since the last query gave up."""
    dev = torch.device("cuda", torch.cuda.current_device())
    _check(lib.gdr_noalloc_status(_stream(dev, stream)))


def workspace_status(workspace, stream=None):
    """Synchronise and read/clear the device status word of a prefill workspace;
    raises GdrError(GDR_ERR_TIMEOUT) if a bounded device wait gave up."""
    dev = workspace.device
    _check(lib.gdr_workspace_status(_ptr(workspace), workspace.numel(), _stream(dev, stream)))


def timing_start():
    """Start recording per-kernel CUDA events for every prefill call (measurement aid)."""
    lib.gdr_timing_start()


def timing_stop(max_kernels=8):
    """Stop recording; returns (mean ms of each kernel position of a call, calls)."""
    buf = (ctypes.c_float * max_kernels)()
    n = ctypes.c_int(0)
    k = lib.gdr_timing_stop(buf, max_kernels, ctypes.byref(n))
    if k < 0:
        raise GdrError(GDR_ERR_CUDA, "gdr_timing_stop: reading a CUDA event failed")
    return [float(buf[i]) for i in range(min(k, max_kernels))], int(n.value)
