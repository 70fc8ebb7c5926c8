"""ctypes binding of libar_attn.so (argument marshalling only).

Every step of the attention core runs in the library's CUDA kernels; this
module checks tensor dtypes/devices, allocates outputs and scratch with torch's
caching allocator, and passes raw pointers plus torch's current CUDA stream.
If the library is missing or cannot be loaded, the first call raises: there is
no fallback implementation.
"""
import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libar_attn.so")

AR_OK = 0
STATUS = {
    0: "AR_OK", -1: "AR_ERR_NULL", -2: "AR_ERR_SHAPE", -3: "AR_ERR_UNSUPPORTED", -4: "AR_ERR_ALIGN",
    -5: "AR_ERR_ARG", -6: "AR_ERR_DEVICE", -7: "AR_ERR_CUDA", -8: "AR_ERR_TIMEOUT", -9: "AR_ERR_WORKSPACE",
    -10: "AR_ERR_TOO_LARGE",
    -11: "AR_ERR_LAYOUT",
}

_lib = None


class ArAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s failed: %s (%s)" % (where, STATUS.get(status, status), strerror(status)))


def lib():
    """Load libar_attn.so (raises OSError if it is absent)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError("libar_attn.so not built at %s; run sliding_window_attention_rmsnorm_b200.build"
                          % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.ar_attn_bwd_workspace_bytes.argtypes = [i, i, i, i]
        L.ar_attn_bwd_workspace_bytes.restype = sz
        L.ar_attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, f, vp]
        L.ar_attn_fwd.restype = i
        L.ar_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, f, vp, sz, vp]
        L.ar_attn_bwd.restype = i
        L.ar_attn_sync_status.argtypes = [vp]
        L.ar_attn_sync_status.restype = i
        L.ar_attn_strerror.argtypes = [i]
        L.ar_attn_strerror.restype = ctypes.c_char_p
        L.ar_attn_layer_window.argtypes = [i, i, i, ctypes.c_char_p]
        L.ar_attn_layer_window.restype = i
        L.ar_attn_unmasked_pairs.argtypes = [i, i]
        L.ar_attn_unmasked_pairs.restype = ctypes.c_longlong
        L.ar_attn_timing_enable.argtypes = [i]
        L.ar_attn_timing_enable.restype = i
        L.ar_attn_timing_read.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong)]
        L.ar_attn_timing_read.restype = i
        L.ar_attn_fwd_gqa.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, f, vp]
        L.ar_attn_fwd_gqa.restype = i
        L.ar_attn_bwd_gqa_workspace_bytes.argtypes = [i, i, i, i, i]
        L.ar_attn_bwd_gqa_workspace_bytes.restype = sz
        L.ar_attn_bwd_gqa.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, f, vp, sz, vp]
        L.ar_attn_bwd_gqa.restype = i
        L.ar_attn_fwd_rope.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, vp, vp, i, i, i, i, i, i, f, f, vp, sz, vp]
        L.ar_attn_fwd_rope_workspace_bytes.argtypes = [i, i, i, i, i]
        L.ar_attn_fwd_rope_workspace_bytes.restype = sz
        L.ar_attn_fwd_rope.restype = i
        L.ar_attn_bwd_rope_workspace_bytes.argtypes = [i, i, i, i, i, i]
        L.ar_attn_bwd_rope_workspace_bytes.restype = sz
        L.ar_attn_bwd_rope.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, vp, vp, vp, vp, vp, vp, vp,
                                       i, i, i, i, i, i, f, f, vp, sz, vp]
        L.ar_attn_bwd_rope.restype = i
        L.ar_attn_bwd_rope_saved.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, vp, vp, vp, vp, vp, vp, vp,
                                             i, i, i, i, i, i, f, f, vp, vp, sz, vp]
        L.ar_attn_bwd_rope_saved.restype = i
        L.ar_attn_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
        L.ar_attn_set_wait_limit_ns.restype = i
        L.ar_attn_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, f, vp]
        L.ar_attn_fwd_noalloc.restype = i
        _lib = L
    return _lib


def strerror(status: int) -> str:
    return lib().ar_attn_strerror(int(status)).decode()


def _check(status: int, where: str):
    if status != AR_OK:
        raise ArAttnError(status, where)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check_inputs(*ts):
    for t in ts:
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous() and t.dim() == 4):
            raise ValueError("expected contiguous bf16 CUDA tensors of shape [B, T, H, D]")
        if t.shape != ts[0].shape:
            raise ValueError("q, k, v (and o, dO) must have the same shape")


def _check_qkv(q, k, v):
    """q [B, T, H, D]; k, v [B, T, Hkv, D] with Hkv dividing H.  Returns Hkv."""
    _check_inputs(q)
    _check_inputs(k, v)
    B, T, H, D = q.shape
    Hkv = k.shape[2]
    if k.shape[0] != B or k.shape[1] != T or k.shape[3] != D or H % Hkv:
        raise ValueError("k, v must be [B, T, Hkv, D] with Hkv dividing q's head count")
    return Hkv


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)


def bwd_workspace_bytes(B, T, H, D, Hkv=None) -> int:
    if Hkv is None or Hkv == H:
        return int(lib().ar_attn_bwd_workspace_bytes(B, T, H, D))
    return int(lib().ar_attn_bwd_gqa_workspace_bytes(B, T, H, Hkv, D))


def _check_out(t, like, name):
    """A caller-supplied output must match the tensor it is shaped after."""
    if not (t.is_cuda and t.dtype == like.dtype and t.is_contiguous() and tuple(t.shape) == tuple(like.shape)
            and t.device == like.device):
        raise ValueError("%s must be a contiguous %s CUDA tensor of shape %s" % (name, like.dtype, tuple(like.shape)))


def _check_lse(t, B, H, T, device):
    if not (t.is_cuda and t.dtype == torch.float32 and t.is_contiguous() and tuple(t.shape) == (B, H, T)
            and t.device == device):
        raise ValueError("lse must be a contiguous fp32 CUDA tensor [B, H, T]")


def fwd(q, k, v, window: int, eps: float = 1e-6, scale=None, out=None, lse=None, need_lse: bool = True):
    """o, lse = attention(norm(q), norm(k), v) over the band 0 <= i - j <= window.

    q: bf16 CUDA tensor [B, T, H, 128]; k, v: [B, T, Hkv, 128] with Hkv
    dividing H (Hkv < H: grouped K/V heads, query head h reads K/V head
    h // (H // Hkv)).  Returns o (bf16, like q) and lse (fp32 [B, H, T]).
    need_lse=False is the forward-only use (no backward follows): the kernel
    does not store lse and None is returned in its place; o is unchanged.
    Enqueued on torch's current stream.
    """
    Hkv = _check_qkv(q, k, v)
    B, T, H, D = q.shape
    if scale is None:
        scale = default_scale(D)
    if out is not None:
        _check_out(out, q, "out")
    o = torch.empty_like(q) if out is None else out
    if need_lse:
        lse_t = torch.empty((B, H, T), dtype=torch.float32, device=q.device) if lse is None else lse
        _check_lse(lse_t, B, H, T, q.device)
    else:
        lse_t = None
    if Hkv != H:
        st = lib().ar_attn_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse_t), B, T, H, Hkv, D, int(window),
                                   float(eps), float(scale), _stream())
        _check(st, "ar_attn_fwd_gqa")
        return o, lse_t
    st = lib().ar_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse_t), B, T, H, D, int(window),
                           float(eps), float(scale), _stream())
    _check(st, "ar_attn_fwd")
    return o, lse_t


def bwd(q, k, v, o, dO, lse, window: int, eps: float = 1e-6, scale=None, dq=None, dk=None, dv=None,
        workspace=None):
    """dq, dk, dv of the forward above, given the upstream gradient dO.

    With grouped K/V heads, dk and dv ([B, T, Hkv, 128]) sum the gradients of
    every query head of their group.
    """
    Hkv = _check_qkv(q, k, v)
    _check_inputs(q, o, dO)
    B, T, H, D = q.shape
    _check_lse(lse, B, H, T, q.device)
    if scale is None:
        scale = default_scale(D)
    for t, like, name in ((dq, q, "dq"), (dk, k, "dk"), (dv, v, "dv")):
        if t is not None:
            _check_out(t, like, name)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(bwd_workspace_bytes(B, T, H, D, Hkv), dtype=torch.uint8, device=q.device)
    if Hkv != H:
        st = lib().ar_attn_bwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse), _ptr(dq), _ptr(dk),
                                   _ptr(dv), B, T, H, Hkv, D, int(window), float(eps), float(scale),
                                   _ptr(workspace), workspace.numel(), _stream())
        _check(st, "ar_attn_bwd_gqa")
        return dq, dk, dv
    st = lib().ar_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                           B, T, H, D, int(window), float(eps), float(scale), _ptr(workspace), workspace.numel(),
                           _stream())
    _check(st, "ar_attn_bwd")
    return dq, dk, dv


def sync_status():
    """Synchronise the current stream and raise if a kernel gave up a wait."""
    _check(lib().ar_attn_sync_status(_stream()), "ar_attn_sync_status")


def _check_rope(cos, sin, T):
    if not (cos.is_cuda and sin.is_cuda and cos.dtype == torch.bfloat16 and sin.dtype == torch.bfloat16
            and cos.is_contiguous() and sin.is_contiguous() and cos.dim() == 2 and cos.shape == sin.shape
            and cos.shape[1] == 64 and cos.shape[0] >= T):
        raise ValueError("cos, sin must be contiguous bf16 CUDA tensors [rows >= T, 64]")


def _check_ve(ve, gate, k):
    if (ve is None) != (gate is None):
        raise ValueError("ve and ve_gate go together")
    if ve is None:
        return
    _check_out(ve, k, "ve")
    B, T, Hkv, _ = k.shape
    if not (gate.is_cuda and gate.dtype == torch.bfloat16 and gate.is_contiguous()
            and tuple(gate.shape) == (B, T, Hkv)):
        raise ValueError("ve_gate must be a contiguous bf16 CUDA tensor [B, T, Hkv]")


def rope_tables(T: int, D: int = 128, base: float = 10000.0, device="cuda"):
    """cos, sin [T, D/2] bf16 as the pages' model precomputes them (angles
    t / base^(2c/D) in fp32, rounded to bf16); built once per model, outside
    the attention core."""
    c = torch.arange(0, D, 2, dtype=torch.float32)
    inv = 1.0 / (base ** (c / D))
    ang = torch.outer(torch.arange(T, dtype=torch.float32), inv)
    return ang.cos().to(torch.bfloat16).to(device), ang.sin().to(torch.bfloat16).to(device)


def fwd_rope_workspace_bytes(B, T, Hkv, D, with_ve=False) -> int:
    return int(lib().ar_attn_fwd_rope_workspace_bytes(B, T, Hkv, D, 1 if with_ve else 0))


def fwd_rope(q, k, v, cos, sin, window: int, eps: float = 1e-6, scale=None, ve=None, ve_gate=None, out=None,
             lse=None, need_lse: bool = True, workspace=None):
    """The forward with the steps before the core: q and k rotated by RoPE (cos,
    sin: bf16 [rows >= T, 64], row t = position t) and, when ve ([B, T, Hkv,
    128]) and ve_gate (the gate logits g, [B, T, Hkv]) are given, v replaced by
    v + 2 sigmoid(g) ve.  q, k, v are the unrotated, unmixed tensors; Q is
    rotated inside the kernel, k and v in one pre-pass into the workspace."""
    Hkv = _check_qkv(q, k, v)
    B, T, H, D = q.shape
    _check_rope(cos, sin, T)
    _check_ve(ve, ve_gate, k)
    if scale is None:
        scale = default_scale(D)
    if out is not None:
        _check_out(out, q, "out")
    o = torch.empty_like(q) if out is None else out
    lse_t = None
    if need_lse:
        lse_t = torch.empty((B, H, T), dtype=torch.float32, device=q.device) if lse is None else lse
        _check_lse(lse_t, B, H, T, q.device)
    if workspace is None:
        workspace = torch.empty(fwd_rope_workspace_bytes(B, T, Hkv, D, ve is not None), dtype=torch.uint8,
                                device=q.device)
    st = lib().ar_attn_fwd_rope(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse_t), _ptr(cos), _ptr(sin),
                                int(cos.shape[0]), _ptr(ve), _ptr(ve_gate), B, T, H, Hkv, D, int(window),
                                float(eps), float(scale), _ptr(workspace), workspace.numel(), _stream())
    _check(st, "ar_attn_fwd_rope")
    return o, lse_t


def bwd_rope_workspace_bytes(B, T, H, D, Hkv=None, with_ve=False) -> int:
    return int(lib().ar_attn_bwd_rope_workspace_bytes(B, T, H, Hkv or H, D, 1 if with_ve else 0))


def bwd_rope(q, k, v, o, dO, lse, cos, sin, window: int, eps: float = 1e-6, scale=None, ve=None, ve_gate=None,
             dq=None, dk=None, dv=None, dve=None, dgate=None, workspace=None, saved=None):
    """Backward of fwd_rope: (dq, dk, dv) for the unrotated, unmixed q, k, v,
    plus (dve, dgate) when the forward mixed in a value embedding (dgate: the
    gradient of the gate logits, fp32 [B, T, Hkv]).  saved: the workspace the
    forward was given for the same k, v, ve, ve_gate and tables, untouched since
    (its rotated k and mixed v are then used instead of formed again)."""
    Hkv = _check_qkv(q, k, v)
    _check_inputs(q, o, dO)
    B, T, H, D = q.shape
    _check_lse(lse, B, H, T, q.device)
    _check_rope(cos, sin, T)
    _check_ve(ve, ve_gate, k)
    if scale is None:
        scale = default_scale(D)
    for t, like, name in ((dq, q, "dq"), (dk, k, "dk"), (dv, v, "dv"), (dve, k, "dve")):
        if t is not None:
            _check_out(t, like, name)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    with_ve = ve is not None
    if with_ve:
        dve = torch.empty_like(k) if dve is None else dve
        if dgate is None:
            dgate = torch.empty((B, T, Hkv), dtype=torch.float32, device=q.device)
        elif not (dgate.is_cuda and dgate.dtype == torch.float32 and dgate.is_contiguous()
                  and tuple(dgate.shape) == (B, T, Hkv)):
            raise ValueError("dgate must be a contiguous fp32 CUDA tensor [B, T, Hkv]")
    else:
        dve = dgate = None
    if workspace is None:
        workspace = torch.empty(bwd_rope_workspace_bytes(B, T, H, D, Hkv, with_ve), dtype=torch.uint8,
                                device=q.device)
    if saved is not None:
        need = fwd_rope_workspace_bytes(B, T, Hkv, D, with_ve)
        if not (saved.is_cuda and saved.device == q.device and saved.numel() * saved.element_size() >= need):
            raise ValueError("saved must be the forward's CUDA workspace (at least %d bytes)" % need)
    st = lib().ar_attn_bwd_rope_saved(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse), _ptr(cos),
                                      _ptr(sin), int(cos.shape[0]), _ptr(ve), _ptr(ve_gate), _ptr(dq), _ptr(dk),
                                      _ptr(dv), _ptr(dve), _ptr(dgate), B, T, H, Hkv, D, int(window), float(eps),
                                      float(scale), _ptr(saved), _ptr(workspace), workspace.numel(), _stream())
    _check(st, "ar_attn_bwd_rope_saved")
    return (dq, dk, dv, dve, dgate) if with_ve else (dq, dk, dv)


def set_wait_limit_ns(ns: int = 0):
    """Limit of every device-side wait in kernels launched from now on (0: the
    default, 2 s).  A kernel whose wait runs out abandons its work and
    sync_status() raises AR_ERR_TIMEOUT; for failure-detection tests."""
    _check(lib().ar_attn_set_wait_limit_ns(int(ns)), "ar_attn_set_wait_limit_ns")


def unmasked_pairs(T: int, window: int) -> int:
    return int(lib().ar_attn_unmasked_pairs(int(T), int(window)))


KERNELS = ("fwd_prep", "fwd", "bwd_prep", "bwd", "dq", "rope_prep")


def timing_enable(on: bool = True):
    """Start (clearing earlier records) or stop per-kernel event timing."""
    _check(lib().ar_attn_timing_enable(1 if on else 0), "ar_attn_timing_enable")


def timing_read():
    """{kernel: (total_ms, launches)} recorded since timing_enable(True)."""
    ms = (ctypes.c_double * len(KERNELS))()
    n = (ctypes.c_longlong * len(KERNELS))()
    _check(lib().ar_attn_timing_read(ms, n), "ar_attn_timing_read")
    return {k: (ms[i], n[i]) for i, k in enumerate(KERNELS)}


NOALLOC_MAX_KEYS = 1 << 20


def fwd_noalloc(q, k, v, window: int, eps: float = 1e-6, scale=None, out=None, lse=None):
    """The forward through ar_attn_fwd_noalloc: no workspace is allocated.

    For callers that must not allocate device memory (a host application that
    owns the allocator).  Scratch is the library's built-in array, so
    B * H * ceil(T/128)*128 must not exceed NOALLOC_MAX_KEYS, and calls that
    can overlap on the GPU must be serialised by the caller.  The outputs o and
    lse may be passed in (out, lse) so that nothing at all is allocated here.
    """
    _check_inputs(q, k, v)
    B, T, H, D = q.shape
    if scale is None:
        scale = default_scale(D)
    if out is not None:
        _check_out(out, q, "out")
    o = torch.empty_like(q) if out is None else out
    lse_t = torch.empty((B, H, T), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_lse(lse_t, B, H, T, q.device)
    st = lib().ar_attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse_t), B, T, H, D, int(window),
                               float(eps), float(scale), _stream())
    _check(st, "ar_attn_fwd_noalloc")
    return o, lse_t
