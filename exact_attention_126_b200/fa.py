"""Python binding of libfa.so: the C entry points of include/fa.h under the same names.

Only argument marshalling happens here: shapes, dtypes and devices are read off torch
tensors, their data pointers and the current CUDA stream are passed to the C ABI, and a
non-OK status is raised as ``FAError``. Every step of the computation runs in the
library's kernels; if the library cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(_PKG, "libfa.so")

FA_OK = 0
STATUS_NAMES = {
    0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_MISALIGNED",
    4: "FA_ERR_WORKSPACE", 5: "FA_ERR_CUDA", 6: "FA_ERR_TIMEOUT",
}

#: every symbol include/fa.h declares
EXPORTED = ("fa_fwd", "fa_fwd_ex", "fa_fwd_fp8", "fa_bwd_workspace_bytes",
            "fa_bwd_workspace_bytes_ex", "fa_bwd", "fa_bwd_ex",
            "fa_fwd_alibi", "fa_bwd_alibi", "fa_bwd_preprocess", "fa_bwd_dkdv", "fa_bwd_dq",
            "fa_bwd_fused", "fa_bwd_dq_convert", "fa_bwd_noalloc", "fa_status_string",
            "fa_debug_status", "fa_debug_set_fault", "fa_version")

#: fa_options_t.flags: the fused backward (head_dim 64; dQ by fp32 reductions)
FA_BWD_FUSED = 1


class FAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib().fa_status_string(status).decode() if _LIB is not None else STATUS_NAMES.get(status)
        super().__init__("%s returned %s" % (where, msg))


class fa_window_t(ctypes.Structure):
    _fields_ = [("left", ctypes.c_int), ("right", ctypes.c_int)]


class fa_options_t(ctypes.Structure):
    """Optional inputs and outputs of the _ex entry points (include/fa.h)."""
    _fields_ = [("alibi_slopes", ctypes.c_void_p), ("key_padding", ctypes.c_void_p),
                ("o_low", ctypes.c_void_p), ("dropout_p", ctypes.c_float),
                ("flags", ctypes.c_uint), ("dropout_seed", ctypes.c_ulonglong),
                ("dropout_offset", ctypes.c_ulonglong), ("seq_lengths", ctypes.c_void_p),
                ("cu_seqlens", ctypes.c_void_p), ("total_tokens", ctypes.c_int)]


def options(alibi_slopes=None, key_padding=None, o_low=None, dropout_p=0.0, dropout_seed=0,
            dropout_offset=0, fused=False, seq_lengths=None, cu_seqlens=None, total_tokens=0):
    """An fa_options_t holding the device pointers of the given tensors (None = absent), the
    dropout parameters (probability, 64-bit seed, 32-bit offset), the backward's flags, the
    real lengths of a variable-length batch (B int32 on the device), or the cumulative
    lengths (B + 1 int32 on the device) and token count of a packed batch."""
    return fa_options_t(_ptr(alibi_slopes), _ptr(key_padding), _ptr(o_low), float(dropout_p),
                        FA_BWD_FUSED if fused else 0,
                        int(dropout_seed) & 0xFFFFFFFFFFFFFFFF, int(dropout_offset),
                        _ptr(seq_lengths), _ptr(cu_seqlens), int(total_tokens))


_LIB = None


def _lib() -> ctypes.CDLL:
    """The loaded library (built in-tree by ``build.build()``); raises if it is absent."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIBRARY):
            raise RuntimeError("libfa.so is not built (run exact_attention_126_b200.build.build());"
                               " there is no fallback path")
        lib = ctypes.CDLL(LIBRARY)
        vp, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        W = fa_window_t
        OP = ctypes.POINTER(fa_options_t)
        lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, I, I, I, I, F, I, W, vp]
        lib.fa_fwd_ex.argtypes = [vp, vp, vp, vp, vp, I, I, I, I, F, I, W, OP, vp]
        lib.fa_fwd_fp8.argtypes = [vp, vp, vp, F, F, F, vp, vp, I, I, I, I, F, I, W, vp]
        lib.fa_bwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, I, I, I, I, F, I, W, OP,
                                  vp, ctypes.c_size_t, vp]
        lib.fa_bwd_workspace_bytes.argtypes = [I, I, I, I]
        lib.fa_bwd_workspace_bytes.restype = ctypes.c_size_t
        lib.fa_bwd_workspace_bytes_ex.argtypes = [I, I, I, I, OP]
        lib.fa_bwd_workspace_bytes_ex.restype = ctypes.c_size_t
        lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, I, I, I, I, F, I, W, vp,
                               ctypes.c_size_t, vp]
        lib.fa_fwd_alibi.argtypes = [vp, vp, vp, vp, vp, I, I, I, I, F, I, W, vp, vp]
        lib.fa_bwd_alibi.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, I, I, I, I, F, I, W, vp,
                                     vp, ctypes.c_size_t, vp]
        lib.fa_bwd_preprocess.argtypes = [vp, vp, vp, vp, I, I, I, I, OP, vp]
        lib.fa_bwd_dkdv.argtypes = [vp, vp, vp, vp, vp, vp, vp, I, I, I, I, F, I, W, OP, vp]
        lib.fa_bwd_dq.argtypes = [vp, vp, vp, vp, vp, vp, I, I, I, I, F, I, W, OP, vp]
        lib.fa_bwd_fused.argtypes = [vp, vp, vp, vp, vp, vp, vp, I, I, I, I, F, I, W, OP, vp]
        lib.fa_bwd_dq_convert.argtypes = [vp, vp, I, I, I, I, F, vp]
        lib.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, I, I, I, I, F, I, W,
                                       vp]
        lib.fa_status_string.argtypes = [I]
        lib.fa_status_string.restype = ctypes.c_char_p
        lib.fa_debug_status.argtypes = [vp]
        lib.fa_debug_set_fault.argtypes = [I]
        lib.fa_version.argtypes = []
        for name in ("fa_fwd", "fa_fwd_ex", "fa_fwd_fp8", "fa_bwd", "fa_bwd_ex", "fa_fwd_alibi",
                     "fa_bwd_alibi", "fa_bwd_preprocess", "fa_bwd_fused", "fa_bwd_dq_convert",
                     "fa_bwd_dkdv", "fa_bwd_dq", "fa_bwd_noalloc", "fa_debug_status",
                     "fa_debug_set_fault", "fa_version"):
            getattr(lib, name).restype = I
        _LIB = lib
    return _LIB


def library() -> ctypes.CDLL:
    return _lib()


def _check(status: int, where: str) -> None:
    if status != FA_OK:
        raise FAError(status, where)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _shape(q: torch.Tensor, dims=None):
    """(B, H, N, d) of a (batch, heads, seq_len, head_dim) tensor, or `dims` as given (a
    packed batch's (total, heads, head_dim) tensors do not carry B and N)."""
    if dims is not None:
        return tuple(int(x) for x in dims)
    if q.dim() != 4:
        raise ValueError("expected a (batch, heads, seq_len, head_dim) tensor")
    return tuple(int(x) for x in q.shape)


def _window(causal: bool, window) -> tuple[int, fa_window_t]:
    left, right = (-1, -1) if window is None else window
    return int(bool(causal)), fa_window_t(int(left), int(right))


def default_scale(d: int) -> float:
    """softmax_scale=None means 1/sqrt(head_dim)."""
    return 1.0 / math.sqrt(d)


# ------------------------------------------------------------------ raw entry points
def fa_fwd(q, k, v, o, lse, scale=None, causal=False, window=(-1, -1), stream=None) -> None:
    B, H, N, d = _shape(q)
    c, w = _window(causal, window)
    s = default_scale(d) if scale is None else float(scale)
    _check(_lib().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, s, c, w,
                         _stream(stream)), "fa_fwd")


def fa_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o, lse, scale=None, causal=False,
               window=(-1, -1), stream=None) -> None:
    """The forward on e4m3 tensors (torch.float8_e4m3fn or uint8 bytes) with per-tensor
    descales; o is bf16."""
    B, H, N, d = _shape(q8)
    c, w = _window(causal, window)
    s = default_scale(d) if scale is None else float(scale)
    _check(_lib().fa_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), float(q_scale), float(k_scale),
                             float(v_scale), _ptr(o), _ptr(lse), B, H, N, d, s, c, w,
                             _stream(stream)), "fa_fwd_fp8")


def attention_forward_fp8(q8, k8, v8, q_scale=1.0, k_scale=1.0, v_scale=1.0, scale=None,
                          causal=False, window=(-1, -1), stream=None):
    """Returns (O, LSE) of the attention of q8*q_scale, k8*k_scale, v8*v_scale for e4m3 CUDA
    tensors of shape (B, H, N, 128); O is bf16."""
    for t in (q8, k8, v8):
        if not t.is_cuda or t.dtype not in (torch.float8_e4m3fn, torch.uint8):
            raise ValueError("q8, k8, v8 must be float8_e4m3fn (or uint8) CUDA tensors")
        if not t.is_contiguous() or t.shape != q8.shape:
            raise ValueError("q8, k8, v8 must be contiguous and share one shape")
    B, H, N, d = _shape(q8)
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q8.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device)
    fa_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o, lse, scale, causal, window, stream)
    return o, lse


def fa_bwd_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(_lib().fa_bwd_workspace_bytes(B, H, N, d))


def fa_bwd_workspace_bytes_ex(B: int, H: int, N: int, d: int, opt=None) -> int:
    return int(_lib().fa_bwd_workspace_bytes_ex(B, H, N, d, _opt_ref(opt)))


def fa_bwd(q, k, v, o, do, lse, dq, dk, dv, workspace, scale=None, causal=False,
           window=(-1, -1), stream=None) -> None:
    B, H, N, d = _shape(q)
    c, w = _window(causal, window)
    s = default_scale(d) if scale is None else float(scale)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                         _ptr(dk), _ptr(dv), B, H, N, d, s, c, w, _ptr(workspace), nbytes,
                         _stream(stream)), "fa_bwd")


def fa_fwd_alibi(q, k, v, o, lse, alibi_slopes, scale=None, causal=False, window=(-1, -1),
                 stream=None) -> None:
    """fa_fwd with the linear bias -alibi_slopes[h] * |i - j| (alibi_slopes: H fp32 values
    on the device)."""
    B, H, N, d = _shape(q)
    c, w = _window(causal, window)
    s = default_scale(d) if scale is None else float(scale)
    _check(_lib().fa_fwd_alibi(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, s, c,
                               w, _ptr(alibi_slopes), _stream(stream)), "fa_fwd_alibi")


def fa_bwd_alibi(q, k, v, o, do, lse, dq, dk, dv, workspace, alibi_slopes, scale=None,
                 causal=False, window=(-1, -1), stream=None) -> None:
    B, H, N, d = _shape(q)
    c, w = _window(causal, window)
    s = default_scale(d) if scale is None else float(scale)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib().fa_bwd_alibi(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse),
                               _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, s, c, w,
                               _ptr(alibi_slopes), _ptr(workspace), nbytes, _stream(stream)),
           "fa_bwd_alibi")


def _opt_ref(opt):
    return None if opt is None else ctypes.byref(opt)


def fa_fwd_ex(q, k, v, o, lse, opt=None, scale=None, causal=False, window=(-1, -1),
              stream=None, dims=None) -> None:
    """fa_fwd with an fa_options_t (see options()); `dims` = (B, H, N, d) for a packed batch."""
    B, H, N, d = _shape(q, dims)
    c, w = _window(causal, window)
    s = default_scale(d) if scale is None else float(scale)
    _check(_lib().fa_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, s, c, w,
                            _opt_ref(opt), _stream(stream)), "fa_fwd_ex")


def fa_bwd_ex(q, k, v, o, do, lse, dq, dk, dv, workspace, opt=None, scale=None, causal=False,
              window=(-1, -1), stream=None, dims=None) -> None:
    """fa_bwd with an fa_options_t (see options()); `dims` = (B, H, N, d) for a packed batch."""
    B, H, N, d = _shape(q, dims)
    c, w = _window(causal, window)
    s = default_scale(d) if scale is None else float(scale)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib().fa_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                            _ptr(dk), _ptr(dv), B, H, N, d, s, c, w, _opt_ref(opt),
                            _ptr(workspace), nbytes, _stream(stream)), "fa_bwd_ex")


def fa_bwd_preprocess(o, do, lse, workspace, opt=None, stream=None, dims=None) -> None:
    B, H, N, d = _shape(o, dims)
    _check(_lib().fa_bwd_preprocess(_ptr(o), _ptr(do), _ptr(lse), _ptr(workspace), B, H, N, d,
                                    _opt_ref(opt), _stream(stream)), "fa_bwd_preprocess")


def fa_bwd_dkdv(q, k, v, do, workspace, dk, dv, scale=None, causal=False, window=(-1, -1),
                stream=None, opt=None, dims=None) -> None:
    B, H, N, d = _shape(q, dims)
    c, w = _window(causal, window)
    s = default_scale(d) if scale is None else float(scale)
    _check(_lib().fa_bwd_dkdv(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(workspace), _ptr(dk),
                              _ptr(dv), B, H, N, d, s, c, w, _opt_ref(opt), _stream(stream)),
           "fa_bwd_dkdv")


def fa_bwd_fused(q, k, v, do, workspace, dk, dv, scale=None, causal=False, window=(-1, -1),
                 stream=None, opt=None) -> None:
    B, H, N, d = _shape(q)
    c, w = _window(causal, window)
    s = default_scale(d) if scale is None else float(scale)
    _check(_lib().fa_bwd_fused(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(workspace), _ptr(dk),
                               _ptr(dv), B, H, N, d, s, c, w, _opt_ref(opt), _stream(stream)),
           "fa_bwd_fused")


def fa_bwd_dq_convert(workspace, dq, scale=None, stream=None) -> None:
    B, H, N, d = _shape(dq)
    s = default_scale(d) if scale is None else float(scale)
    _check(_lib().fa_bwd_dq_convert(_ptr(workspace), _ptr(dq), B, H, N, d, s, _stream(stream)),
           "fa_bwd_dq_convert")


def fa_bwd_dq(q, k, v, do, workspace, dq, scale=None, causal=False, window=(-1, -1),
              stream=None, opt=None, dims=None) -> None:
    B, H, N, d = _shape(q, dims)
    c, w = _window(causal, window)
    s = default_scale(d) if scale is None else float(scale)
    _check(_lib().fa_bwd_dq(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(workspace), _ptr(dq),
                            B, H, N, d, s, c, w, _opt_ref(opt), _stream(stream)), "fa_bwd_dq")


def fa_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, scale=None, causal=False, window=(-1, -1),
                   stream=None) -> None:
    """fa_bwd without a workspace argument: for callers that cannot allocate device
    memory; the library's own fixed device array holds the row statistics."""
    B, H, N, d = _shape(q)
    c, w = _window(causal, window)
    s = default_scale(d) if scale is None else float(scale)
    _check(_lib().fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse),
                                 _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, s, c, w,
                                 _stream(stream)), "fa_bwd_noalloc")



def fa_status_string(status: int) -> str:
    return _lib().fa_status_string(int(status)).decode()


def fa_debug_status(stream=None) -> int:
    return int(_lib().fa_debug_status(_stream(stream)))


def fa_debug_set_fault(fault: int) -> None:
    """Test hook: 1 makes later fa_fwd launches time out on purpose (see include/fa.h)."""
    _check(_lib().fa_debug_set_fault(int(fault)), "fa_debug_set_fault")


def fa_version() -> int:
    return int(_lib().fa_version())


# ------------------------------------------------------------------ allocating helpers
def _check_inputs(*ts):
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must be on a CUDA device")
        if t.dtype != torch.bfloat16:
            raise ValueError("tensors must be bf16")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous (B, H, N, d)")
        if t.shape != ts[0].shape:
            raise ValueError("q, k, v (and dO) must share one shape")


def _check_slopes(alibi_slopes, q):
    if not alibi_slopes.is_cuda or alibi_slopes.dtype != torch.float32:
        raise ValueError("alibi_slopes must be an fp32 CUDA tensor")
    if alibi_slopes.numel() != q.shape[1] or not alibi_slopes.is_contiguous():
        raise ValueError("alibi_slopes must hold one slope per head, contiguous")


def _check_padding(key_padding, B, N):
    if not key_padding.is_cuda or key_padding.dtype not in (torch.bool, torch.uint8):
        raise ValueError("key_padding must be a bool or uint8 CUDA tensor")
    if tuple(key_padding.shape) != (B, N) or not key_padding.is_contiguous():
        raise ValueError("key_padding must be a contiguous (batch, seq_len) tensor")


def _check_lengths(seq_lengths, q):
    if not seq_lengths.is_cuda or seq_lengths.dtype != torch.int32:
        raise ValueError("seq_lengths must be an int32 CUDA tensor")
    if seq_lengths.numel() != q.shape[0] or not seq_lengths.is_contiguous():
        raise ValueError("seq_lengths must hold one length per batch entry, contiguous")


def _packed_dims(q, cu_seqlens, max_seqlen, seq_lengths):
    """(B, H, N, d) of a packed batch: q is (total, H, d), cu_seqlens B + 1 int32 offsets."""
    if seq_lengths is not None:
        raise ValueError("seq_lengths and cu_seqlens exclude each other")
    if not cu_seqlens.is_cuda or cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1:
        raise ValueError("cu_seqlens must be a 1-D int32 CUDA tensor")
    if cu_seqlens.numel() < 2 or not cu_seqlens.is_contiguous():
        raise ValueError("cu_seqlens must hold B + 1 >= 2 offsets, contiguous")
    if q.dim() != 3:
        raise ValueError("a packed batch takes (total_tokens, heads, head_dim) tensors")
    if max_seqlen is None or int(max_seqlen) < 1:
        raise ValueError("a packed batch needs max_seqlen >= 1 (the longest sequence)")
    return cu_seqlens.numel() - 1, int(q.shape[1]), int(max_seqlen), int(q.shape[2])


def attention_forward(q, k, v, scale=None, causal=False, window=(-1, -1), stream=None,
                      alibi_slopes=None, key_padding=None, keep_residual=False, dropout=None,
                      seq_lengths=None, cu_seqlens=None, max_seqlen=None):
    """Returns (O, LSE) for bf16 CUDA tensors q, k, v of shape (B, H, N, d), or
    (O, LSE, O_low) with keep_residual: O_low = O_fp32 - bf16(O) in bf16, which
    attention_backward uses to form rowsum(dO o O) from O to about 16 bits.
    alibi_slopes (H fp32 values): the scores carry the bias -alibi_slopes[h] * |i - j|.
    key_padding ((B, N) bool or uint8, True = padded key): padded keys are masked out
    for every head and query. dropout: (p, seed, offset) drops each attention weight with
    probability p (rounded to a multiple of 1/256) after the softmax and scales the kept
    ones by 1 / (1 - p); the backward needs the same triple. seq_lengths ((B,) int32):
    entry b holds seq_lengths[b] real tokens; rows past it are zero (LSE -inf) and tiles
    wholly past it are not computed. cu_seqlens ((B + 1,) int32) with max_seqlen: a packed
    batch, q, k, v of shape (total, H, d) holding sequence b at tokens cu_seqlens[b] ..
    cu_seqlens[b+1]-1; O is (total, H, d) and LSE (H, total)."""
    _check_inputs(q, k, v)
    if cu_seqlens is not None:
        B, H, N, d = _packed_dims(q, cu_seqlens, max_seqlen, seq_lengths)
        lse = torch.empty((H, q.shape[0]), dtype=torch.float32, device=q.device)
    else:
        B, H, N, d = _shape(q)
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    o = torch.empty_like(q)
    o_low = torch.empty_like(q) if keep_residual else None
    if alibi_slopes is not None:
        _check_slopes(alibi_slopes, q)
    if key_padding is not None:
        _check_padding(key_padding, B, N)
    if seq_lengths is not None:
        _check_lengths(seq_lengths, q)
    if (alibi_slopes is None and key_padding is None and o_low is None and dropout is None
            and seq_lengths is None and cu_seqlens is None):
        fa_fwd(q, k, v, o, lse, scale, causal, window, stream)
    else:
        opt = options(alibi_slopes, key_padding, o_low, *(dropout or ()),
                      seq_lengths=seq_lengths, cu_seqlens=cu_seqlens,
                      total_tokens=q.shape[0] if cu_seqlens is not None else 0)
        fa_fwd_ex(q, k, v, o, lse, opt, scale, causal, window, stream, dims=(B, H, N, d))
    return (o, lse, o_low) if keep_residual else (o, lse)


def attention_backward(q, k, v, o, lse, do, scale=None, causal=False, window=(-1, -1),
                       stream=None, alibi_slopes=None, key_padding=None, o_low=None,
                       dropout=None, fused=False, seq_lengths=None, cu_seqlens=None,
                       max_seqlen=None):
    """Returns (dQ, dK, dV): the gradient of <O, dO>; lse (and o_low, if kept) come from
    attention_forward with the same alibi_slopes, key_padding, dropout and seq_lengths.
    fused: at head_dim 64, the backward in one pass over key tiles with dQ added up in fp32
    in no fixed order (see FA_BWD_FUSED); otherwise the deterministic dK/dV and dQ passes."""
    _check_inputs(q, k, v, o, do)
    if cu_seqlens is not None:
        B, H, N, d = _packed_dims(q, cu_seqlens, max_seqlen, seq_lengths)
    else:
        B, H, N, d = _shape(q)
    total = q.shape[0] if cu_seqlens is not None else 0
    dq = torch.empty_like(q)
    dk = torch.empty_like(q)
    dv = torch.empty_like(q)
    ws = torch.empty(max(1, fa_bwd_workspace_bytes_ex(
        B, H, N, d, options(fused=fused, seq_lengths=seq_lengths, cu_seqlens=cu_seqlens,
                            total_tokens=total))),
                     dtype=torch.uint8, device=q.device)
    if alibi_slopes is not None:
        _check_slopes(alibi_slopes, q)
    if key_padding is not None:
        _check_padding(key_padding, B, N)
    if o_low is not None:
        _check_inputs(q, o_low)
    if seq_lengths is not None:
        _check_lengths(seq_lengths, q)
    if (alibi_slopes is None and key_padding is None and o_low is None and dropout is None
            and not fused and seq_lengths is None and cu_seqlens is None):
        fa_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, scale, causal, window, stream)
    else:
        opt = options(alibi_slopes, key_padding, o_low, *(dropout or ()),
                      fused=fused, seq_lengths=seq_lengths, cu_seqlens=cu_seqlens,
                      total_tokens=total)
        fa_bwd_ex(q, k, v, o, do, lse, dq, dk, dv, ws, opt, scale, causal, window, stream,
                  dims=(B, H, N, d))
    return dq, dk, dv
