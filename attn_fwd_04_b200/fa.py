"""ctypes binding of libfa.so (include/fa.h), one Python function per C entry
point, same names.  Argument marshalling only: every step of the computation
runs in the library's CUDA kernels.  PyTorch supplies device memory and the
stream; there is no fallback -- a missing library or a non-CUDA tensor is an
error.
"""
import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfa.so")

FA_OK = 0
FA_ERR_NULL = -1
FA_ERR_SHAPE = -2
FA_ERR_UNSUPPORTED = -3
FA_ERR_ALIGN = -4
FA_ERR_CUDA = -5
FA_ERR_DEVICE_TIMEOUT = -6
FA_ERR_NOMEM = -7
FA_ERR_DEVICE_BAD_INPUT = -8

# every symbol include/fa.h declares
EXPORTS = ("fa_fwd", "fa_fwd_gqa", "fa_fwd_rope", "fa_bwd", "fa_bwd_gqa", "fa_bwd_varlen",
           "fa_fwd_varlen", "fa_fwd_varlen_gqa",
           "fa_decode_paged",
           "fa_decode_paged_gqa", "fa_decode_paged_strided",
           "fa_decode_paged_noalloc", "fa_append_paged", "fa_prefill_paged",
           "fa_gather_paged",
           "fa_get_device_error", "fa_selftest_bounded_wait", "fa_selftest_fwd_stall",
           "fa_selftest_decode_stall",
           "fa_release_workspace", "fa_status_str", "fa_version", "fa_fwd_set_cta_pairs")

_lib = None


class FaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {fa_status_str(status)} ({status})")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libfa.so (built in-tree by attn_fwd_04_b200.build); raise if absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libfa.so not found at {LIB_PATH}; build it with "
                              "`python -m attn_fwd_04_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.fa_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, F, P]
        L.fa_fwd_gqa.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, P]
        L.fa_fwd_varlen.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, F, P]
        L.fa_fwd_varlen_gqa.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, F, P]
        L.fa_fwd_rope.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, P]
        L.fa_bwd.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, F, P]
        L.fa_bwd_gqa.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, P]
        L.fa_bwd_varlen.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, P]
        L.fa_decode_paged.argtypes = [P, P, P, P, P, P, I, I, I, I, P]
        L.fa_decode_paged_gqa.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, P]
        L.fa_decode_paged_noalloc.argtypes = [P, P, P, P, P, P, I, I, I, I, P]
        L.fa_decode_paged_strided.argtypes = [P, P, P, P, I, P, P, I, I, I, I, I, I, P]
        L.fa_gather_paged.argtypes = [P, P, P, P, I, I, I, I, P]
        L.fa_append_paged.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, P]
        L.fa_prefill_paged.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, F, P]
        L.fa_get_device_error.argtypes = [ctypes.POINTER(ctypes.c_int), P]
        L.fa_selftest_bounded_wait.argtypes = [P]
        L.fa_selftest_fwd_stall.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P]
        L.fa_selftest_decode_stall.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, P]
        L.fa_release_workspace.argtypes = []
        L.fa_status_str.argtypes = [I]
        L.fa_status_str.restype = ctypes.c_char_p
        L.fa_version.argtypes = []
        L.fa_fwd_set_cta_pairs.argtypes = [I]
        for name in ("fa_fwd", "fa_fwd_gqa", "fa_fwd_rope", "fa_bwd", "fa_bwd_gqa", "fa_bwd_varlen",
                     "fa_fwd_varlen", "fa_fwd_varlen_gqa",
                     "fa_decode_paged",
                     "fa_decode_paged_gqa", "fa_decode_paged_strided", "fa_decode_paged_noalloc",
                     "fa_append_paged",
                     "fa_prefill_paged", "fa_gather_paged",
                     "fa_get_device_error", "fa_selftest_bounded_wait", "fa_selftest_fwd_stall",
                     "fa_selftest_decode_stall",
                     "fa_release_workspace", "fa_version", "fa_fwd_set_cta_pairs"):
            getattr(L, name).restype = I
        _lib = L
    return _lib


def fa_status_str(status: int) -> str:
    return lib().fa_status_str(int(status)).decode()


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# device types the wrappers accept (the library reads device memory only)
_DEVICE_TYPES = ("cuda",)


def _check(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int):
    if not isinstance(t, torch.Tensor) or t.device.type not in _DEVICE_TYPES:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _expect(t, name: str, dtype: torch.dtype, shape, device):
    """t must be a contiguous CUDA tensor of this dtype and exact shape on
    `device` (the device of the call's first input)."""
    _check(t, name, dtype, len(shape))
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, the call's inputs on {device}")


def _same_device(device, **tensors):
    for name, t in tensors.items():
        if t.device != device:
            raise ValueError(f"{name} is on {t.device}, the call's inputs on {device}")


def _pages(k_pages, v_pages, page_size: int, d: int, heads=None):
    """k_pages, v_pages: the same [P, heads, page_size, d] shape."""
    if v_pages.shape != k_pages.shape:
        raise ValueError("k_pages and v_pages must have the same shape")
    want = (heads if heads is not None else k_pages.shape[1], int(page_size), d)
    if tuple(k_pages.shape[1:]) != want:
        raise ValueError(f"pages must be [P, {want[0]}, {want[1]}, {want[2]}], got "
                         f"{tuple(k_pages.shape)}")


def _raise_if(status: int, what: str):
    if status != FA_OK:
        raise FaError(status, what)


def fa_fwd(q, k, v, causal: bool, scale: Optional[float] = None, o=None, lse=None, stream=None):
    """Fused attention forward over [B,H,N,d] bf16 tensors -> (o, lse [B,H,N] fp32)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, torch.bfloat16, 4)
    B, H, N, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same [B,H,N,d] shape")
    _same_device(q.device, k=k, v=v)
    if scale is None:
        scale = d ** -0.5
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _expect(o, "o", torch.bfloat16, q.shape, q.device)
    _expect(lse, "lse", torch.float32, (B, H, N), q.device)
    rc = lib().fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                      B, H, N, d, int(bool(causal)), float(scale), _stream(stream))
    _raise_if(rc, "fa_fwd")
    return o, lse


def fa_fwd_gqa(q, k, v, causal: bool, scale: Optional[float] = None, o=None, lse=None,
               stream=None):
    """Grouped-query forward: q [B,H,N,d], k/v [B,H_kv,N,d] bf16 with H a
    multiple of H_kv -> (o [B,H,N,d], lse [B,H,N] fp32)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, torch.bfloat16, 4)
    B, H, N, d = q.shape
    H_kv = k.shape[1]
    if k.shape != (B, H_kv, N, d) or v.shape != k.shape:
        raise ValueError("k, v must be [B,H_kv,N,d] with q's B, N, d")
    _same_device(q.device, k=k, v=v)
    if scale is None:
        scale = d ** -0.5
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _expect(o, "o", torch.bfloat16, q.shape, q.device)
    _expect(lse, "lse", torch.float32, (B, H, N), q.device)
    rc = lib().fa_fwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                          B, H, H_kv, N, d, int(bool(causal)), float(scale), _stream(stream))
    _raise_if(rc, "fa_fwd_gqa")
    return o, lse


def fa_fwd_rope(q, k, v, rope_cos, rope_sin, causal: bool, scale: Optional[float] = None,
                o=None, lse=None, stream=None):
    """Forward with rotary embedding applied in the kernel: q [B,H,N,d],
    k/v [B,H_kv,N,d] bf16 (unrotated), tables [max_pos,d/2] fp32 ->
    (o [B,H,N,d], lse [B,H,N])."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, torch.bfloat16, 4)
    _check(rope_cos, "rope_cos", torch.float32, 2)
    _check(rope_sin, "rope_sin", torch.float32, 2)
    B, H, N, d = q.shape
    H_kv = k.shape[1]
    if k.shape != (B, H_kv, N, d) or v.shape != k.shape:
        raise ValueError("k, v must be [B,H_kv,N,d] with q's B, N, d")
    if rope_cos.shape[1] != d // 2 or rope_sin.shape != rope_cos.shape:
        raise ValueError("rope tables must be [max_pos, d/2]")
    _same_device(q.device, k=k, v=v, rope_cos=rope_cos, rope_sin=rope_sin)
    if scale is None:
        scale = d ** -0.5
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _expect(o, "o", torch.bfloat16, q.shape, q.device)
    _expect(lse, "lse", torch.float32, (B, H, N), q.device)
    rc = lib().fa_fwd_rope(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                           rope_cos.data_ptr(), rope_sin.data_ptr(), rope_cos.shape[0], B, H,
                           H_kv, N, d, int(bool(causal)), float(scale), _stream(stream))
    _raise_if(rc, "fa_fwd_rope")
    return o, lse


def fa_bwd(q, k, v, o, lse, dout, causal: bool, scale: Optional[float] = None, dq=None,
           dk=None, dv=None, stream=None):
    """Gradients of fa_fwd: (dq, dk, dv), each [B,H,N,d] bf16, from q, k, v, o,
    dout [B,H,N,d] bf16 and lse [B,H,N] fp32 (as fa_fwd returned them)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _check(t, n, torch.bfloat16, 4)
        if t.shape != q.shape:
            raise ValueError(f"{n} must have q's shape")
    B, H, N, d = q.shape
    _expect(lse, "lse", torch.float32, (B, H, N), q.device)
    _same_device(q.device, k=k, v=v, o=o, dout=dout)
    if scale is None:
        scale = d ** -0.5
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _expect(t, n, torch.bfloat16, q.shape, q.device)
    rc = lib().fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                      dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d,
                      int(bool(causal)), float(scale), _stream(stream))
    _raise_if(rc, "fa_bwd")
    return dq, dk, dv


def fa_bwd_gqa(q, k, v, o, lse, dout, causal: bool, scale: Optional[float] = None, dq=None,
               dk=None, dv=None, stream=None):
    """Gradients of fa_fwd_gqa: dq [B,H,N,d] and dk, dv [B,H_kv,N,d] bf16, from
    q, o, dout [B,H,N,d], k, v [B,H_kv,N,d] bf16 and lse [B,H,N] fp32."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _check(t, n, torch.bfloat16, 4)
    B, H, N, d = q.shape
    H_kv = k.shape[1]
    if o.shape != q.shape or dout.shape != q.shape or k.shape != (B, H_kv, N, d) or \
            v.shape != k.shape:
        raise ValueError("q, o, dout must be [B,H,N,d] and k, v [B,H_kv,N,d]")
    _expect(lse, "lse", torch.float32, (B, H, N), q.device)
    _same_device(q.device, k=k, v=v, o=o, dout=dout)
    if scale is None:
        scale = d ** -0.5
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _expect(dq, "dq", torch.bfloat16, q.shape, q.device)
    _expect(dk, "dk", torch.bfloat16, k.shape, q.device)
    _expect(dv, "dv", torch.bfloat16, k.shape, q.device)
    rc = lib().fa_bwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                          dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H,
                          H_kv, N, d, int(bool(causal)), float(scale), _stream(stream))
    _raise_if(rc, "fa_bwd_gqa")
    return dq, dk, dv


def fa_bwd_varlen(q, k, v, o, lse, dout, cu_seqlens, max_seqlen: int, causal: bool,
                  scale: Optional[float] = None, dq=None, dk=None, dv=None, stream=None):
    """Gradients of fa_fwd_varlen over packed sequences: dq [total,H,d] and dk, dv
    [total,H_kv,d] bf16, from q, o, dout [total,H,d], k, v [total,H_kv,d] bf16 and
    lse [H,total] fp32 (as fa_fwd_varlen returned it)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _check(t, n, torch.bfloat16, 3)
    _check(cu_seqlens, "cu_seqlens", torch.int32, 1)
    total, H, d = q.shape
    H_kv = k.shape[1]
    if o.shape != q.shape or dout.shape != q.shape or k.shape != (total, H_kv, d) or \
            v.shape != k.shape:
        raise ValueError("q, o, dout must be [total,H,d] and k, v [total,H_kv,d]")
    _expect(lse, "lse", torch.float32, (H, total), q.device)
    _same_device(q.device, k=k, v=v, o=o, dout=dout, cu_seqlens=cu_seqlens)
    B = cu_seqlens.numel() - 1
    if scale is None:
        scale = d ** -0.5
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _expect(dq, "dq", torch.bfloat16, q.shape, q.device)
    _expect(dk, "dk", torch.bfloat16, k.shape, q.device)
    _expect(dv, "dv", torch.bfloat16, k.shape, q.device)
    rc = lib().fa_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                             lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                             dv.data_ptr(), cu_seqlens.data_ptr(), B, H, H_kv, total,
                             int(max_seqlen), d, int(bool(causal)), float(scale), _stream(stream))
    _raise_if(rc, "fa_bwd_varlen")
    return dq, dk, dv


def fa_fwd_varlen(q, k, v, cu_seqlens, max_seqlen: int, causal: bool,
                  scale: Optional[float] = None, o=None, lse=None, stream=None):
    """Forward over packed [total,H,d] sequences -> (o, lse [H,total] fp32)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, torch.bfloat16, 3)
    _check(cu_seqlens, "cu_seqlens", torch.int32, 1)
    total, H, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same [total,H,d] shape")
    _same_device(q.device, k=k, v=v, cu_seqlens=cu_seqlens)
    B = cu_seqlens.numel() - 1
    if scale is None:
        scale = d ** -0.5
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((H, total), dtype=torch.float32, device=q.device)
    _expect(o, "o", torch.bfloat16, q.shape, q.device)
    _expect(lse, "lse", torch.float32, (H, total), q.device)
    rc = lib().fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                             lse.data_ptr(), cu_seqlens.data_ptr(), B, H, total,
                             int(max_seqlen), d, int(bool(causal)), float(scale),
                             _stream(stream))
    _raise_if(rc, "fa_fwd_varlen")
    return o, lse


def fa_fwd_varlen_gqa(q, k, v, cu_seqlens, max_seqlen: int, causal: bool,
                      scale: Optional[float] = None, o=None, lse=None, stream=None):
    """Forward over packed sequences with grouped K/V heads: q [total,H,d], k, v
    [total,H_kv,d] -> (o [total,H,d], lse [H,total] fp32)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, torch.bfloat16, 3)
    _check(cu_seqlens, "cu_seqlens", torch.int32, 1)
    total, H, d = q.shape
    H_kv = k.shape[1]
    if k.shape != (total, H_kv, d) or v.shape != k.shape:
        raise ValueError("k, v must be [total,H_kv,d]")
    _same_device(q.device, k=k, v=v, cu_seqlens=cu_seqlens)
    B = cu_seqlens.numel() - 1
    if scale is None:
        scale = d ** -0.5
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((H, total), dtype=torch.float32, device=q.device)
    _expect(o, "o", torch.bfloat16, q.shape, q.device)
    _expect(lse, "lse", torch.float32, (H, total), q.device)
    rc = lib().fa_fwd_varlen_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                 lse.data_ptr(), cu_seqlens.data_ptr(), B, H, H_kv, total,
                                 int(max_seqlen), d, int(bool(causal)), float(scale),
                                 _stream(stream))
    _raise_if(rc, "fa_fwd_varlen_gqa")
    return o, lse


def fa_decode_paged(q, k_pages, v_pages, page_table, seq_lens, page_size: int = 256, o=None,
                    stream=None):
    """Single-token decode over a paged cache -> o [B,H,d] bf16."""
    _check(q, "q", torch.bfloat16, 3)
    _check(k_pages, "k_pages", torch.bfloat16, 4)
    _check(v_pages, "v_pages", torch.bfloat16, 4)
    _check(page_table, "page_table", torch.int32, 1)
    _check(seq_lens, "seq_lens", torch.int32, 1)
    B, H, d = q.shape
    # the multi-head call takes no pool size, so the pool's layout is checked
    # here: a cache of another head count or page size would be misread
    _pages(k_pages, v_pages, page_size, d, heads=H)
    if seq_lens.numel() != B:
        raise ValueError(f"seq_lens must hold one length per sequence ({B})")
    _same_device(q.device, k_pages=k_pages, v_pages=v_pages, page_table=page_table,
                 seq_lens=seq_lens)
    if o is None:
        o = torch.empty_like(q)
    _expect(o, "o", torch.bfloat16, q.shape, q.device)
    rc = lib().fa_decode_paged(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(),
                               page_table.data_ptr(), seq_lens.data_ptr(), o.data_ptr(),
                               B, H, d, int(page_size), _stream(stream))
    _raise_if(rc, "fa_decode_paged")
    return o


def fa_decode_paged_gqa(q, k_pages, v_pages, page_table, seq_lens, page_size: int = 256, o=None,
                        stream=None):
    """Decode with grouped K/V heads: q [B,H,d], pages [P,H_kv,page_size,d]
    -> o [B,H,d] bf16.  The pool size P bounds the page indices read."""
    _check(q, "q", torch.bfloat16, 3)
    _check(k_pages, "k_pages", torch.bfloat16, 4)
    _check(v_pages, "v_pages", torch.bfloat16, 4)
    _check(page_table, "page_table", torch.int32, 1)
    _check(seq_lens, "seq_lens", torch.int32, 1)
    B, H, d = q.shape
    H_kv = k_pages.shape[1]
    _pages(k_pages, v_pages, page_size, d)
    if H_kv == 0 or H % H_kv != 0:
        raise ValueError(f"H ({H}) must be a multiple of the cache's K/V heads ({H_kv})")
    if seq_lens.numel() != B:
        raise ValueError(f"seq_lens must hold one length per sequence ({B})")
    _same_device(q.device, k_pages=k_pages, v_pages=v_pages, page_table=page_table,
                 seq_lens=seq_lens)
    if o is None:
        o = torch.empty_like(q)
    _expect(o, "o", torch.bfloat16, q.shape, q.device)
    rc = lib().fa_decode_paged_gqa(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(),
                                   page_table.data_ptr(), seq_lens.data_ptr(), o.data_ptr(),
                                   B, H, H_kv, k_pages.shape[0], d, int(page_size),
                                   _stream(stream))
    _raise_if(rc, "fa_decode_paged_gqa")
    return o


def fa_decode_paged_strided(q, k_pages, v_pages, block_table, seq_lens, page_size: int = 256,
                            o=None, stream=None):
    """Decode through a block table [B, max_pages] int32 (row b lists sequence
    b's pages): q [B,H,d], pages [P,H_kv,page_size,d] -> o [B,H,d] bf16."""
    _check(q, "q", torch.bfloat16, 3)
    _check(k_pages, "k_pages", torch.bfloat16, 4)
    _check(v_pages, "v_pages", torch.bfloat16, 4)
    _check(block_table, "block_table", torch.int32, 2)
    _check(seq_lens, "seq_lens", torch.int32, 1)
    B, H, d = q.shape
    H_kv = k_pages.shape[1]
    if block_table.shape[0] != B:
        raise ValueError("block_table must have one row per sequence")
    _pages(k_pages, v_pages, page_size, d)
    if H_kv == 0 or H % H_kv != 0:
        raise ValueError(f"H ({H}) must be a multiple of the cache's K/V heads ({H_kv})")
    if seq_lens.numel() != B:
        raise ValueError(f"seq_lens must hold one length per sequence ({B})")
    _same_device(q.device, k_pages=k_pages, v_pages=v_pages, block_table=block_table,
                 seq_lens=seq_lens)
    if o is None:
        o = torch.empty_like(q)
    _expect(o, "o", torch.bfloat16, q.shape, q.device)
    rc = lib().fa_decode_paged_strided(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(),
                                       block_table.data_ptr(), block_table.shape[1],
                                       seq_lens.data_ptr(), o.data_ptr(), B, H, H_kv,
                                       k_pages.shape[0], d, int(page_size), _stream(stream))
    _raise_if(rc, "fa_decode_paged_strided")
    return o


def fa_decode_paged_noalloc(q, k_pages, v_pages, page_table, seq_lens, page_size: int = 256,
                            o=None, stream=None):
    """fa_decode_paged without any device allocation by the library (its scratch
    is a fixed 16 MiB device array).  `o` should be preallocated by callers that
    cannot allocate; it is created here only as a convenience."""
    _check(q, "q", torch.bfloat16, 3)
    _check(k_pages, "k_pages", torch.bfloat16, 4)
    _check(v_pages, "v_pages", torch.bfloat16, 4)
    _check(page_table, "page_table", torch.int32, 1)
    _check(seq_lens, "seq_lens", torch.int32, 1)
    B, H, d = q.shape
    # the multi-head call takes no pool size, so the pool's layout is checked
    # here: a cache of another head count or page size would be misread
    _pages(k_pages, v_pages, page_size, d, heads=H)
    if seq_lens.numel() != B:
        raise ValueError(f"seq_lens must hold one length per sequence ({B})")
    _same_device(q.device, k_pages=k_pages, v_pages=v_pages, page_table=page_table,
                 seq_lens=seq_lens)
    if o is None:
        o = torch.empty_like(q)
    _expect(o, "o", torch.bfloat16, q.shape, q.device)
    rc = lib().fa_decode_paged_noalloc(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(),
                                       page_table.data_ptr(), seq_lens.data_ptr(), o.data_ptr(),
                                       B, H, d, int(page_size), _stream(stream))
    _raise_if(rc, "fa_decode_paged_noalloc")
    return o


def fa_append_paged(k_new, v_new, cu_new, k_pages, v_pages, page_table, seq_lens,
                    page_size: int = 256, stream=None):
    """Write new rows [total_new,H_kv,d] into the [P,H_kv,page_size,d] pages
    (in place) as the last tokens of their sequences; seq_lens are the
    lengths after the append."""
    for t, n in ((k_new, "k_new"), (v_new, "v_new")):
        _check(t, n, torch.bfloat16, 3)
    _check(k_pages, "k_pages", torch.bfloat16, 4)
    _check(v_pages, "v_pages", torch.bfloat16, 4)
    _check(cu_new, "cu_new", torch.int32, 1)
    _check(page_table, "page_table", torch.int32, 1)
    _check(seq_lens, "seq_lens", torch.int32, 1)
    total_new, H_kv, d = k_new.shape
    if v_new.shape != k_new.shape:
        raise ValueError("k_new and v_new must have the same shape")
    _pages(k_pages, v_pages, page_size, d, heads=H_kv)
    if seq_lens.numel() != cu_new.numel() - 1:
        raise ValueError("seq_lens must hold one length per sequence of cu_new")
    _same_device(k_new.device, v_new=v_new, cu_new=cu_new, k_pages=k_pages, v_pages=v_pages,
                 page_table=page_table, seq_lens=seq_lens)
    rc = lib().fa_append_paged(k_new.data_ptr(), v_new.data_ptr(), cu_new.data_ptr(),
                               k_pages.data_ptr(), v_pages.data_ptr(), page_table.data_ptr(),
                               seq_lens.data_ptr(), cu_new.numel() - 1, H_kv, total_new,
                               k_pages.shape[0], d, int(page_size), _stream(stream))
    _raise_if(rc, "fa_append_paged")


def fa_prefill_paged(q, k_pages, v_pages, page_table, seq_lens, cu_q, max_q: int, causal: bool,
                     scale: Optional[float] = None, page_size: int = 256, o=None, lse=None,
                     stream=None):
    """Queries [total_q,H,d] that end their cached sequences, attending
    through the page table -> (o [total_q,H,d], lse [H,total_q] fp32)."""
    _check(q, "q", torch.bfloat16, 3)
    _check(k_pages, "k_pages", torch.bfloat16, 4)
    _check(v_pages, "v_pages", torch.bfloat16, 4)
    _check(page_table, "page_table", torch.int32, 1)
    _check(seq_lens, "seq_lens", torch.int32, 1)
    _check(cu_q, "cu_q", torch.int32, 1)
    total_q, H, d = q.shape
    _pages(k_pages, v_pages, page_size, d)
    if k_pages.shape[1] == 0 or H % k_pages.shape[1] != 0:
        raise ValueError(f"H ({H}) must be a multiple of the cache's K/V heads "
                         f"({k_pages.shape[1]})")
    if seq_lens.numel() != cu_q.numel() - 1:
        raise ValueError("seq_lens must hold one length per sequence of cu_q")
    _same_device(q.device, k_pages=k_pages, v_pages=v_pages, page_table=page_table,
                 seq_lens=seq_lens, cu_q=cu_q)
    if scale is None:
        scale = d ** -0.5
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((H, total_q), dtype=torch.float32, device=q.device)
    _expect(o, "o", torch.bfloat16, q.shape, q.device)
    _expect(lse, "lse", torch.float32, (H, total_q), q.device)
    rc = lib().fa_prefill_paged(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(),
                                page_table.data_ptr(), seq_lens.data_ptr(), cu_q.data_ptr(),
                                o.data_ptr(), lse.data_ptr(), cu_q.numel() - 1, H,
                                k_pages.shape[1], total_q, int(max_q), k_pages.shape[0], d,
                                int(page_size), int(bool(causal)), float(scale), _stream(stream))
    _raise_if(rc, "fa_prefill_paged")
    return o, lse


def fa_gather_paged(pages, page_table, seq_lens, total_tokens: int, page_size: int = 256,
                    out=None, stream=None):
    """Copy cached tokens out of [P,H,page_size,d] pages -> [total_tokens,H,d]."""
    _check(pages, "pages", torch.bfloat16, 4)
    _check(page_table, "page_table", torch.int32, 1)
    _check(seq_lens, "seq_lens", torch.int32, 1)
    _, H, _, d = pages.shape
    if pages.shape[2] != int(page_size):
        raise ValueError(f"pages must hold {page_size} tokens each, got {pages.shape[2]}")
    B = seq_lens.numel()
    _same_device(pages.device, page_table=page_table, seq_lens=seq_lens)
    if out is None:
        out = torch.empty((total_tokens, H, d), dtype=torch.bfloat16, device=pages.device)
    _expect(out, "out", torch.bfloat16, (total_tokens, H, d), pages.device)
    rc = lib().fa_gather_paged(pages.data_ptr(), page_table.data_ptr(), seq_lens.data_ptr(),
                               out.data_ptr(), B, H, d, int(page_size), _stream(stream))
    _raise_if(rc, "fa_gather_paged")
    return out


def fa_get_device_error(stream=None) -> int:
    """Synchronise the stream, read and clear the device error word (FA_* code)."""
    code = ctypes.c_int(0)
    rc = lib().fa_get_device_error(ctypes.byref(code), _stream(stream))
    _raise_if(rc, "fa_get_device_error")
    return code.value


def fa_selftest_bounded_wait(stream=None) -> None:
    """Launch the bounded-wait self test; read the result with fa_get_device_error."""
    _raise_if(lib().fa_selftest_bounded_wait(_stream(stream)), "fa_selftest_bounded_wait")


def fa_selftest_fwd_stall(q, k, v, withheld: int, wait_us: int, o=None, lse=None,
                          stream=None):
    """Launch the causal forward pass with K/V copy `withheld` never issued and
    every wait bounded by wait_us; read the outcome with fa_get_device_error."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, torch.bfloat16, 4)
    B, H, N, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same [B,H,N,d] shape")
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _expect(o, "o", torch.bfloat16, q.shape, q.device)
    _expect(lse, "lse", torch.float32, (B, H, N), q.device)
    rc = lib().fa_selftest_fwd_stall(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                     lse.data_ptr(), B, H, N, d, int(withheld), int(wait_us),
                                     _stream(stream))
    _raise_if(rc, "fa_selftest_fwd_stall")
    return o, lse


def fa_selftest_decode_stall(q, k_pages, v_pages, page_table, seq_lens, withheld: int,
                             wait_us: int, page_size: int = 256, o=None, stream=None):
    """Launch the paged decode with no copy issued from ring use `withheld` on
    and every wait bounded by wait_us; read the outcome with
    fa_get_device_error."""
    _check(q, "q", torch.bfloat16, 3)
    _check(k_pages, "k_pages", torch.bfloat16, 4)
    _check(v_pages, "v_pages", torch.bfloat16, 4)
    _check(page_table, "page_table", torch.int32, 1)
    _check(seq_lens, "seq_lens", torch.int32, 1)
    B, H, d = q.shape
    _pages(k_pages, v_pages, page_size, d, heads=H)
    if seq_lens.numel() != B:
        raise ValueError(f"seq_lens must hold one length per sequence ({B})")
    _same_device(q.device, k_pages=k_pages, v_pages=v_pages, page_table=page_table,
                 seq_lens=seq_lens)
    o = torch.empty_like(q) if o is None else o
    _expect(o, "o", torch.bfloat16, q.shape, q.device)
    rc = lib().fa_selftest_decode_stall(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(),
                                        page_table.data_ptr(), seq_lens.data_ptr(), o.data_ptr(),
                                        B, H, d, int(page_size), int(withheld), int(wait_us),
                                        _stream(stream))
    _raise_if(rc, "fa_selftest_decode_stall")
    return o


def fa_release_workspace() -> None:
    _raise_if(lib().fa_release_workspace(), "fa_release_workspace")


def fa_version() -> int:
    return lib().fa_version()


def fa_fwd_set_cta_pairs(enable: bool) -> bool:
    """Select the CTA-pair (True) or single-CTA (False, default) forward kernel
    for d = 128; returns the previous setting."""
    return bool(lib().fa_fwd_set_cta_pairs(int(bool(enable))))
