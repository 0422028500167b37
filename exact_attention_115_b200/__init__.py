"""B200 (sm_100a) fused exact attention: thin Python binding of the C ABI.

Every computation happens in the CUDA kernels of ``libfa_b200.so`` (built by
``python -m exact_attention_115_b200.build``); this module only checks
tensors and marshals pointers, sizes and the current CUDA stream.  There is no
CPU or PyTorch fallback: if the library is missing or a tensor is not on a
CUDA device, the call raises.

Layouts follow ``include/fa.h``: Q/O/dO [B, H, Nq, d], K/V [B, H, Nk, d],
L [B, H, Nq] float32 natural-log logsumexp.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa_b200.so")

FA_FP32, FA_BF16, FA_FP16 = 0, 1, 2
FA_DECODE_NOALLOC_SCRATCH_BYTES = 8 << 20  # include/fa.h
FA_OK, FA_ERR_INVALID, FA_ERR_UNSUPPORTED, FA_ERR_WORKSPACE, FA_ERR_CUDA, FA_ERR_TIMEOUT = (
    0, -1, -2, -3, -4, -5)
FA_ERR_BOUNDS = -6  # debug builds only
STATUS_NAMES = {0: "FA_OK", -1: "FA_ERR_INVALID", -2: "FA_ERR_UNSUPPORTED",
                -3: "FA_ERR_WORKSPACE", -4: "FA_ERR_CUDA", -5: "FA_ERR_TIMEOUT",
                -6: "FA_ERR_BOUNDS"}

# Every symbol include/fa.h declares: name -> (restype, argtypes)
_VP, _I, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "fa_fwd": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _F, _I, _VP]),
    "fa_bwd_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "fa_bwd": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _F, _I,
                    _VP, _SZ, _VP]),
    "fa_fwd_ex": (_I, [_VP] * 9 + [_I, _I, _I, _I, _I, _I, _F, _I, _VP, _VP, _VP, _VP, _VP]),
    "fa_bwd_ex": (_I, [_VP] * 9 + [_VP] * 8 + [_I, _I, _I, _I, _I, _I, _F, _I, _VP, _VP, _VP, _VP,
                                               _VP, _SZ, _VP]),
    "fa_set_bwd_dq_mode": (_I, [_I]),
    "fa_set_bwd_dq_groups": (_I, [_I]),
    "fa_decode_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I]),
    "fa_decode": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _I, _I, _VP, _SZ, _VP]),
    "fa_decode_ex": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _I, _I, _VP, _VP, _SZ, _VP]),
    "fa_status": (_I, [_VP]),
    "fa_bwd_set_timing_events": (_I, [_VP, _VP]),
    "fa_last_timeout_site": (_I, []),
    "fa_last_cuda_error": (_I, []),
    "fa_decode_noalloc": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _I, _I, _VP]),
    "fa_selftest_wait_timeout": (_I, [ctypes.c_uint, _VP]),
    "fa_version": (ctypes.c_char_p, []),
}

_lib = None


class FAError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS_NAMES.get(code, code)}")
        self.code = code


def lib() -> ctypes.CDLL:
    """Load libfa_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m exact_attention_115_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _lib = h
    return _lib


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return FA_BF16
    if t.dtype == torch.float16:
        return FA_FP16
    if t.dtype == torch.float32:
        return FA_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


class Layout(ctypes.Structure):
    """fa_layout: element strides (batch, head, row) of a [B, H, N, d] tensor."""
    _fields_ = [("b", ctypes.c_longlong), ("h", ctypes.c_longlong), ("n", ctypes.c_longlong)]


class Dropout(ctypes.Structure):
    """fa_dropout: drop probability, generator seed and counter offset."""
    _fields_ = [("p", ctypes.c_float), ("seed", ctypes.c_ulonglong), ("offset", ctypes.c_uint)]


def _dropout(p, seed, offset):
    """A Dropout for the C call, or None when p == 0."""
    if p == 0:
        return None
    return Dropout(float(p), int(seed) & 0xFFFFFFFFFFFFFFFF, int(offset) & 0xFFFFFFFF)


def _kv_len_ptr(kv_len, B, device):
    """Device pointer of a key-padding length tensor (int32 [B] on the
    tensors' device), or None."""
    if kv_len is None:
        return None
    if not isinstance(kv_len, torch.Tensor) or kv_len.dtype != torch.int32:
        raise TypeError("kv_len must be an int32 torch.Tensor")
    if kv_len.device != device or tuple(kv_len.shape) != (B,) or not kv_len.is_contiguous():
        raise ValueError(f"kv_len must be a contiguous [B={B}] tensor on {device}")
    return kv_len.data_ptr()


def _bias_args(bias, q, B, H, Nq, Nk):
    """(pointer, Layout) of an additive bias broadcastable to [B, H, Nq, Nk]
    (input dtype, key columns contiguous), or (None, None)."""
    if bias is None:
        return None, None
    if not isinstance(bias, torch.Tensor) or bias.dtype != q.dtype or bias.device != q.device:
        raise TypeError("bias must be a tensor of the inputs' dtype on their device")
    if bias.dim() != 4:
        raise ValueError("bias must be 4-D, broadcastable to [B, H, Nq, Nk]")
    b = bias.expand(B, H, Nq, Nk)  # broadcast dimensions get stride 0
    if b.stride(3) != 1:
        raise ValueError("bias must have contiguous key columns")
    return b.data_ptr(), Layout(b.stride(0), b.stride(1), b.stride(2))


def _layout(t) -> Layout:
    s = t.stride()
    return Layout(s[0], s[1], s[2])


def _check(name, t, shape=None, dtype=None, strided=False):
    """Validate a tensor argument; ``strided`` allows any strides with the
    last (d) dimension contiguous, else the tensor must be contiguous."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device (no CPU path exists)")
    if strided:
        if t.dim() != 4 or t.stride(-1) != 1:
            raise ValueError(f"{name} must be [B, H, N, d] with the d dimension contiguous")
    elif not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _on(device):
    """Context that makes ``device`` current for one library call: the C side
    launches on the current device and looks up per-device state (tensor-map
    encoder, scratch addresses) there, so it must be the tensors' device."""
    return torch.cuda.device(device)


def _raise(fn, code):
    if code != FA_OK:
        err = FAError(fn, code)
        if code == FA_ERR_CUDA:  # name the CUDA error behind it
            cu = int(lib().fa_last_cuda_error())
            err.cuda_error = cu
            err.args = (f"{err.args[0]} (CUDA error {cu}"
                        + (f", tensor-map encoding CUresult {cu - 100000})" if cu >= 100000 else ")"),)
        raise err


def forward(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None,
            dropout_p: float = 0.0, seed: int = 0, offset: int = 0, kv_len=None, bias=None):
    """O, L = attention(q, k, v).  q, k, v (and out) are [B, H, N, d] with any
    strides whose d dimension is contiguous (a [B, N, H, d] tensor viewed
    with .transpose(1, 2) works as is).  ``dropout_p`` > 0 drops attention
    weights with the keep mask that ``seed`` and ``offset`` select (pass the
    same three to ``backward``).  ``kv_len`` (int32 [B] on the device) hides
    keys j >= kv_len[b] of batch element b; ``bias`` (broadcastable to
    [B, H, Nq, Nk], q's dtype) is added to the scaled scores.  Returns
    (O [B,H,Nq,d] q.dtype,
    L [B,H,Nq] fp32 contiguous)."""
    _check("q", q, strided=True)
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    _check("k", k, (B, H, Nk, d), q.dtype, strided=True)
    _check("v", v, (B, H, Nk, d), q.dtype, strided=True)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, H, Nq, d), dtype=q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _check("out", out, (B, H, Nq, d), q.dtype, strided=True)
    _check("lse", lse, (B, H, Nq), torch.float32)
    dr = _dropout(dropout_p, seed, offset)
    kvl = _kv_len_ptr(kv_len, B, q.device)
    bp, bl = _bias_args(bias, q, B, H, Nq, Nk)
    if dr is None and kvl is None and bp is None and all(t.is_contiguous() for t in (q, k, v, out)):
        with _on(q.device):
            rc = lib().fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                              lse.data_ptr(), B, H, Nq, Nk, d, int(bool(causal)), float(scale),
                              _dtype_code(q), _stream(q.device))
        _raise("fa_fwd", rc)
        return out, lse
    lq, lk, lv, lo = _layout(q), _layout(k), _layout(v), _layout(out)
    with _on(q.device):
        rc = lib().fa_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                             lse.data_ptr(), ctypes.byref(lq), ctypes.byref(lk), ctypes.byref(lv),
                             ctypes.byref(lo), B, H, Nq, Nk, d, int(bool(causal)), float(scale),
                             _dtype_code(q), None if dr is None else ctypes.byref(dr), kvl, bp,
                             None if bl is None else ctypes.byref(bl), _stream(q.device))
    _raise("fa_fwd_ex", rc)
    return out, lse


def bwd_workspace_bytes(B, H, Nq, Nk, d, dtype=torch.bfloat16) -> int:
    code = {torch.bfloat16: FA_BF16, torch.float16: FA_FP16, torch.float32: FA_FP32}[dtype]
    return int(lib().fa_bwd_workspace_bytes(B, H, Nq, Nk, d, code))


def set_bwd_dq_mode(mode: int) -> int:
    """0 auto, 1 reduce-add into one fp32 buffer, 2 per-K/V-block partials,
    3 reduce-add into G buffers (K/V block kb into buffer kb mod G; see
    set_bwd_dq_groups).  Returns the previous mode."""
    rc = lib().fa_set_bwd_dq_mode(int(mode))
    if rc < 0:
        raise FAError("fa_set_bwd_dq_mode", rc)
    return rc


def set_bwd_dq_groups(groups: int) -> int:
    """G, the buffer count of dQ mode 3 (1..16).  Returns the previous G."""
    rc = lib().fa_set_bwd_dq_groups(int(groups))
    if rc < 0:
        raise FAError("fa_set_bwd_dq_groups", rc)
    return rc


def backward(q, k, v, o, do, lse, causal: bool = False, scale: float | None = None,
             dq=None, dk=None, dv=None, workspace=None, dropout_p: float = 0.0, seed: int = 0,
             offset: int = 0, kv_len=None, bias=None):
    """dQ, dK, dV of attention given the forward's O and L and the upstream dO
    (and the forward's ``dropout_p``, ``seed``, ``offset``, ``kv_len`` and
    ``bias``; the bias gets no gradient)."""
    _check("q", q, strided=True)
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    for name, t, n in (("k", k, Nk), ("v", v, Nk), ("o", o, Nq), ("do", do, Nq)):
        _check(name, t, (B, H, n, d), q.dtype, strided=True)
    _check("lse", lse, (B, H, Nq), torch.float32)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dev = q.device
    dq = torch.empty((B, H, Nq, d), dtype=q.dtype, device=dev) if dq is None else dq
    dk = torch.empty((B, H, Nk, d), dtype=q.dtype, device=dev) if dk is None else dk
    dv = torch.empty((B, H, Nk, d), dtype=q.dtype, device=dev) if dv is None else dv
    for name, t, n in (("dq", dq, Nq), ("dk", dk, Nk), ("dv", dv, Nk)):
        _check(name, t, (B, H, n, d), q.dtype, strided=True)
    need = bwd_workspace_bytes(B, H, Nq, Nk, d, q.dtype)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _check("workspace", workspace)
    ts = (q, k, v, o, do, dq, dk, dv)
    dr = _dropout(dropout_p, seed, offset)
    kvl = _kv_len_ptr(kv_len, B, dev)
    bp, bl = _bias_args(bias, q, B, H, Nq, Nk)
    if dr is None and kvl is None and bp is None and all(t.is_contiguous() for t in ts):
        with _on(dev):
            rc = lib().fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                              dv.data_ptr(), B, H, Nq, Nk, d, int(bool(causal)), float(scale),
                              _dtype_code(q), workspace.data_ptr(),
                              workspace.numel() * workspace.element_size(), _stream(dev))
        _raise("fa_bwd", rc)
        return dq, dk, dv
    lays = [_layout(t) for t in ts]
    with _on(dev):
        rc = lib().fa_bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                             do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                             dv.data_ptr(), *[ctypes.byref(l) for l in lays], B, H, Nq, Nk, d,
                             int(bool(causal)), float(scale), _dtype_code(q),
                             None if dr is None else ctypes.byref(dr), kvl, bp,
                             None if bl is None else ctypes.byref(bl), workspace.data_ptr(),
                             workspace.numel() * workspace.element_size(), _stream(dev))
    _raise("fa_bwd_ex", rc)
    return dq, dk, dv


class _Attention(torch.autograd.Function):
    """forward() / backward() of this module as one autograd node.  Saves
    q, k, v, O and L (not P); the backward recomputes P in the kernel."""

    @staticmethod
    def forward(ctx, q, k, v, causal, scale, dropout_p, seed, offset, kv_len, bias):
        O, L = forward(q, k, v, causal=causal, scale=scale, dropout_p=dropout_p, seed=seed,
                       offset=offset, kv_len=kv_len, bias=bias)
        # bias and kv_len are saved too (None when absent), so that an
        # in-place change between the passes raises instead of silently
        # rebuilding a different P in the backward
        ctx.save_for_backward(q, k, v, O, L, kv_len, bias)
        ctx.args = (causal, scale, dropout_p, seed, offset)
        ctx.mark_non_differentiable(L)
        return O, L

    @staticmethod
    def backward(ctx, dO, dL):
        q, k, v, O, L, kv_len, bias = ctx.saved_tensors
        causal, scale, dropout_p, seed, offset = ctx.args
        if dO.stride(-1) != 1:
            dO = dO.contiguous()
        dq, dk, dv = backward(q, k, v, O, dO, L, causal=causal, scale=scale, dropout_p=dropout_p,
                              seed=seed, offset=offset, kv_len=kv_len, bias=bias)
        return dq, dk, dv, None, None, None, None, None, None, None


def attention(q, k, v, causal: bool = False, scale: float | None = None, dropout_p: float = 0.0,
              seed: int | None = None, offset: int = 0, kv_len=None, bias=None):
    """Differentiable O = attention(q, k, v) for [B, H, N, d] CUDA tensors
    (any strides with d contiguous), through forward() and backward().  With
    dropout and no ``seed``, one is drawn from torch's default CPU generator
    (so torch.manual_seed makes runs repeatable); the backward reuses it.
    Returns O only (L is kept for the backward)."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    if bias is not None and bias.requires_grad:
        raise ValueError("the bias is an input constant: its gradient is not computed "
                         "(pass bias.detach() to use it as one)")
    if dropout_p > 0 and seed is None:
        seed = int(torch.randint(0, 2**62, (1,)).item())
    O, _ = _Attention.apply(q, k, v, bool(causal), float(scale), float(dropout_p),
                            0 if seed is None else int(seed), int(offset), kv_len, bias)
    return O


def decode_workspace_bytes(B, H, Nk, d, num_splits=0) -> int:
    return int(lib().fa_decode_workspace_bytes(B, H, Nk, d, num_splits))


def decode(q, k, v, scale: float | None = None, num_splits: int = 0, out=None, lse=None,
           workspace=None, kv_len=None):
    """Split-KV decode: q [B,H,1,d], k/v [B,H,Nk,d] -> (O [B,H,1,d], L [B,H,1]).
    ``kv_len`` (int32 [B] on the device) limits batch element b to its first
    kv_len[b] keys (a padded KV cache)."""
    _check("q", q)
    B, H, one, d = q.shape
    if one != 1:
        raise ValueError("decode takes exactly one query row per (batch, head)")
    Nk = k.shape[2]
    _check("k", k, (B, H, Nk, d), q.dtype)
    _check("v", v, (B, H, Nk, d), q.dtype)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, 1), dtype=torch.float32, device=q.device) if lse is None else lse
    need = decode_workspace_bytes(B, H, Nk, d, num_splits)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    kvl = _kv_len_ptr(kv_len, B, q.device)
    if kvl is None:
        with _on(q.device):
            rc = lib().fa_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                 lse.data_ptr(), B, H, Nk, d, float(scale), _dtype_code(q),
                                 int(num_splits), workspace.data_ptr(),
                                 workspace.numel() * workspace.element_size(), _stream(q.device))
        _raise("fa_decode", rc)
        return out, lse
    with _on(q.device):
        rc = lib().fa_decode_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                lse.data_ptr(), B, H, Nk, d, float(scale), _dtype_code(q),
                                int(num_splits), kvl, workspace.data_ptr(),
                                workspace.numel() * workspace.element_size(), _stream(q.device))
    _raise("fa_decode_ex", rc)
    return out, lse


def decode_noalloc(q, k, v, scale: float | None = None, num_splits: int = 0, out=None, lse=None):
    """Split-KV decode like decode(), for callers that cannot allocate device
    memory: no workspace is created or passed; the partial results go to the
    library's own 8 MiB device scratch array (see fa_decode_noalloc in
    include/fa.h: calls share it, so overlapping calls on the GPU race)."""
    _check("q", q)
    B, H, one, d = q.shape
    if one != 1:
        raise ValueError("decode takes exactly one query row per (batch, head)")
    Nk = k.shape[2]
    _check("k", k, (B, H, Nk, d), q.dtype)
    _check("v", v, (B, H, Nk, d), q.dtype)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, 1), dtype=torch.float32, device=q.device)
    _check("out", out, q.shape, q.dtype)
    _check("lse", lse, (B, H, 1), torch.float32)
    with _on(q.device):
        rc = lib().fa_decode_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                     lse.data_ptr(), B, H, Nk, d, float(scale), _dtype_code(q),
                                     int(num_splits), _stream(q.device))
    _raise("fa_decode_noalloc", rc)
    return out, lse


def status(device=None) -> int:
    """Synchronise the current stream and return (and clear) the kernel
    error status: FA_OK, FA_ERR_TIMEOUT or FA_ERR_CUDA."""
    return int(lib().fa_status(_stream(device)))


def set_bwd_timing_events(start=None, stop=None) -> None:
    """Record torch.cuda.Event ``start``/``stop`` around the main backward
    kernel of every later backward() call (None, None switches it off).  The
    events must already exist on the device (record them once first)."""
    if start is None or stop is None:
        lib().fa_bwd_set_timing_events(None, None)
    else:
        lib().fa_bwd_set_timing_events(start.cuda_event, stop.cuda_event)


def selftest_wait_timeout(limit_us: int = 20000, device=None) -> int:
    """Enqueue the failure-detection self-test (a bounded wait that runs out
    after ``limit_us``); returns the launch status.  The next status() reads
    FA_ERR_TIMEOUT."""
    return int(lib().fa_selftest_wait_timeout(int(limit_us), _stream(device)))


def version() -> str:
    return lib().fa_version().decode()
