"""fp64 CPU oracle for exact attention, paged gather and paged decode.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
benchmark's CPU-baseline / reference leg may import this package.  It shares
no code with the CUDA library (attn_fwd_04_b200), and the CUDA library never
imports it.

The arithmetic lives in attn_oracle.c (plain loops, fp64); this module only
marshals numpy arrays into it.  `method.py` beside it holds the CPU
restatements of the method's own steps (online softmax, split merge) that
the pin tests compare with the plain definition.

Inputs are whatever values the GPU receives (bf16 upcast exactly to fp64);
outputs are fp64.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        L.oracle_attention.argtypes = [P, P, P, P, P, I64, I64, I64, I64, I64,
                                       ctypes.c_int, ctypes.c_double, P, I64]
        L.oracle_attention.restype = ctypes.c_int
        L.oracle_attention_probs.argtypes = [P, P, P, I64, I64, ctypes.c_int,
                                             ctypes.c_double]
        L.oracle_attention_probs.restype = ctypes.c_int
        L.oracle_attention_varlen.argtypes = [P, P, P, P, P, P, I64, I64, I64,
                                              ctypes.c_int, ctypes.c_double, P, I64]
        L.oracle_attention_varlen.restype = ctypes.c_int
        L.oracle_gather_paged.argtypes = [P, P, P, P, I64, I64, I64, I64]
        L.oracle_gather_paged.restype = ctypes.c_int
        L.oracle_decode_paged.argtypes = [P, P, P, P, P, P, P, I64, I64, I64, I64]
        L.oracle_decode_paged.restype = ctypes.c_int
        L.oracle_attention_gqa.argtypes = [P, P, P, P, P, I64, I64, I64, I64, I64, I64,
                                           ctypes.c_int, ctypes.c_double, P, I64]
        L.oracle_attention_gqa.restype = ctypes.c_int
        L.oracle_decode_paged_gqa.argtypes = [P, P, P, P, P, P, P, I64, I64, I64, I64, I64]
        L.oracle_decode_paged_gqa.restype = ctypes.c_int
        L.oracle_decode_paged_strided.argtypes = [P, P, P, P, I64, P, P, P, I64, I64, I64,
                                                  I64, I64]
        L.oracle_decode_paged_strided.restype = ctypes.c_int
        L.oracle_append_paged.argtypes = [P, P, P, P, P, I64, I64, I64, I64]
        L.oracle_append_paged.restype = ctypes.c_int
        L.oracle_prefill_paged.argtypes = [P, P, P, P, P, P, P, P, I64, I64, I64, I64, I64,
                                           ctypes.c_int, ctypes.c_double]
        L.oracle_prefill_paged.restype = ctypes.c_int
        L.oracle_rope_exact.argtypes = [P, P, P, I64, I64, I64]
        L.oracle_rope_exact.restype = None
        L.oracle_rope_bf16.argtypes = [P, P, P, I64, I64, I64]
        L.oracle_rope_bf16.restype = None
        L.oracle_attention_bwd.argtypes = [P, P, P, P, P, P, P, I64, I64, I64, I64, I64,
                                           ctypes.c_int, ctypes.c_double]
        L.oracle_attention_bwd.restype = ctypes.c_int
        L.oracle_num_threads.argtypes = []
        L.oracle_num_threads.restype = ctypes.c_int
        _LIB = L
    return _LIB


def _f64(a):
    """Any array-like (numpy or torch, any float dtype) -> C-contiguous fp64."""
    if hasattr(a, "detach"):  # torch tensor: upcast on the CPU, exactly
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i64(a):
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.int64))


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def num_threads() -> int:
    return lib().oracle_num_threads()


def attention(q, k, v, causal: bool, scale: float, rows=None):
    """Plain fp64 attention over q,k [B,H,N,d] and v [B,H,N,dv].

    Returns (o [B,H,N,dv], lse [B,H,N]).  With `rows` (flat ids
    (b*H + h)*N + i) only those rows are computed; the other entries of the
    returned arrays are NaN.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, H, N, d) and v.shape == (B, H, N, dv)
    o = np.full((B, H, N, dv), np.nan)
    lse = np.full((B, H, N), np.nan)
    r = _i64(rows) if rows is not None else None
    rc = lib().oracle_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                B, H, N, d, dv, int(bool(causal)), float(scale),
                                _ptr(r), 0 if r is None else r.size)
    if rc != 0:
        raise RuntimeError(f"oracle_attention failed ({rc})")
    return o, lse


def attention_gqa(q, k, v, causal: bool, scale: float, rows=None):
    """Grouped-query attention: q [B,H,N,d], k [B,Hkv,N,d], v [B,Hkv,N,dv];
    query head h reads K/V head h // (H // Hkv).  Returns (o [B,H,N,dv],
    lse [B,H,N]); `rows` as in attention()."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    dv = v.shape[-1]
    assert k.shape == (B, Hkv, N, d) and v.shape == (B, Hkv, N, dv) and H % Hkv == 0
    o = np.full((B, H, N, dv), np.nan)
    lse = np.full((B, H, N), np.nan)
    r = _i64(rows) if rows is not None else None
    rc = lib().oracle_attention_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                    B, H, Hkv, N, d, dv, int(bool(causal)), float(scale),
                                    _ptr(r), 0 if r is None else r.size)
    if rc != 0:
        raise RuntimeError(f"oracle_attention_gqa failed ({rc})")
    return o, lse


def probs(q, k, causal: bool, scale: float):
    """The full N x N probability matrix of one head; q, k are [N, d]."""
    q, k = _f64(q), _f64(k)
    N, d = q.shape
    p = np.zeros((N, N))
    lib().oracle_attention_probs(_ptr(q), _ptr(k), _ptr(p), N, d,
                                 int(bool(causal)), float(scale))
    return p


def attention_varlen(q, k, v, cu_seqlens, causal: bool, scale: float, rows=None):
    """Plain fp64 attention over packed [total,H,d] sequences.

    Returns (o [total,H,d], lse [H,total]); `rows` are flat ids h*total + g.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    cu = _i64(cu_seqlens)
    total, H, d = q.shape
    B = cu.size - 1
    assert cu[-1] == total
    o = np.full((total, H, d), np.nan)
    lse = np.full((H, total), np.nan)
    r = _i64(rows) if rows is not None else None
    rc = lib().oracle_attention_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                       _ptr(cu), B, H, d, int(bool(causal)),
                                       float(scale), _ptr(r), 0 if r is None else r.size)
    if rc != 0:
        raise RuntimeError(f"oracle_attention_varlen failed ({rc})")
    return o, lse


def gather_paged(pages, page_table, seq_lens, page_size: int):
    """Contiguous [sum(seq_lens), H, d] rows gathered from [P,H,page_size,d] pages."""
    pages = _f64(pages)
    pt = _i64(page_table)
    sl = _i64(seq_lens)
    _, H, ps, d = pages.shape
    assert ps == page_size
    out = np.zeros((int(sl.sum()), H, d))
    rc = lib().oracle_gather_paged(_ptr(pages), _ptr(pt), _ptr(sl), _ptr(out),
                                   sl.size, H, d, page_size)
    if rc != 0:
        raise RuntimeError(f"oracle_gather_paged failed ({rc})")
    return out


def decode_paged(q, k_pages, v_pages, page_table, seq_lens, page_size: int):
    """Single-token decode; returns (o [B,H,d], lse [B,H]).  Scale is 1/sqrt(d)."""
    q = _f64(q)
    kp, vp = _f64(k_pages), _f64(v_pages)
    pt, sl = _i64(page_table), _i64(seq_lens)
    B, H, d = q.shape
    o = np.zeros((B, H, d))
    lse = np.zeros((B, H))
    rc = lib().oracle_decode_paged(_ptr(q), _ptr(kp), _ptr(vp), _ptr(pt), _ptr(sl),
                                   _ptr(o), _ptr(lse), B, H, d, page_size)
    if rc != 0:
        raise RuntimeError(f"oracle_decode_paged failed ({rc})")
    return o, lse


def decode_paged_gqa(q, k_pages, v_pages, page_table, seq_lens, page_size: int):
    """Single-token decode with grouped K/V heads: q [B,H,d], pages
    [P,Hkv,page_size,d]; returns (o [B,H,d], lse [B,H]).  Scale 1/sqrt(d)."""
    q = _f64(q)
    kp, vp = _f64(k_pages), _f64(v_pages)
    pt, sl = _i64(page_table), _i64(seq_lens)
    B, H, d = q.shape
    Hkv = kp.shape[1]
    assert H % Hkv == 0
    o = np.zeros((B, H, d))
    lse = np.zeros((B, H))
    rc = lib().oracle_decode_paged_gqa(_ptr(q), _ptr(kp), _ptr(vp), _ptr(pt), _ptr(sl),
                                       _ptr(o), _ptr(lse), B, H, Hkv, d, page_size)
    if rc != 0:
        raise RuntimeError(f"oracle_decode_paged_gqa failed ({rc})")
    return o, lse


def decode_paged_strided(q, k_pages, v_pages, block_table, seq_lens, page_size: int):
    """Single-token decode through a block table [B, max_pages] (sequence b's
    k-th page at block_table[b, k]; entries past its pages unused): q [B,H,d],
    pages [P,Hkv,page_size,d]; returns (o [B,H,d], lse [B,H]).  Scale 1/sqrt(d)."""
    q = _f64(q)
    kp, vp = _f64(k_pages), _f64(v_pages)
    bt, sl = _i64(block_table), _i64(seq_lens)
    B, H, d = q.shape
    Hkv = kp.shape[1]
    assert bt.ndim == 2 and bt.shape[0] == B and H % Hkv == 0
    o = np.zeros((B, H, d))
    lse = np.zeros((B, H))
    rc = lib().oracle_decode_paged_strided(_ptr(q), _ptr(kp), _ptr(vp), _ptr(bt), bt.shape[1],
                                           _ptr(sl), _ptr(o), _ptr(lse), B, H, Hkv, d,
                                           page_size)
    if rc != 0:
        raise RuntimeError(f"oracle_decode_paged_strided failed ({rc})")
    return o, lse


def append_paged(pages, page_table, seq_lens, new_rows, cu_new, page_size: int):
    """Pages after writing each sequence's new rows [cu_new[B],Hkv,d] at its
    last positions (seq_lens are the lengths after the append).  Returns a new
    fp64 array; the input is not modified."""
    out = _f64(pages).copy()
    pt, sl, cu = _i64(page_table), _i64(seq_lens), _i64(cu_new)
    rows = _f64(new_rows)
    _, Hkv, ps, d = out.shape
    assert ps == page_size and rows.shape[1:] == (Hkv, d)
    rc = lib().oracle_append_paged(_ptr(out), _ptr(pt), _ptr(sl), _ptr(rows), _ptr(cu),
                                   sl.size, Hkv, d, page_size)
    if rc != 0:
        raise RuntimeError(f"oracle_append_paged failed ({rc})")
    return out


def prefill_paged(q, k_pages, v_pages, page_table, seq_lens, cu_q, page_size: int,
                  causal: bool, scale: float):
    """Queries [cu_q[B],H,d] that are the last positions of their cached
    sequences, attending through the page table; returns (o [cu_q[B],H,d],
    lse [H,cu_q[B]])."""
    q = _f64(q)
    kp, vp = _f64(k_pages), _f64(v_pages)
    pt, sl, cu = _i64(page_table), _i64(seq_lens), _i64(cu_q)
    total, H, d = q.shape
    Hkv = kp.shape[1]
    o = np.full((total, H, d), np.nan)
    lse = np.full((H, total), np.nan)
    rc = lib().oracle_prefill_paged(_ptr(q), _ptr(kp), _ptr(vp), _ptr(pt), _ptr(sl), _ptr(cu),
                                    _ptr(o), _ptr(lse), sl.size, H, Hkv, d, page_size,
                                    int(bool(causal)), float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle_prefill_paged failed ({rc})")
    return o, lse


def attention_bwd_varlen(q, k, v, dout, cu_seqlens, causal: bool, scale: float):
    """Gradients over packed sequences: q, dout [total,H,d], k, v [total,Hkv,d]
    (query head h uses K/V head h // (H/Hkv)); sequence b owns rows
    cu_seqlens[b] .. cu_seqlens[b+1]-1 and attends within itself only (the
    variable-length batches of the page "Flash Attention 是什么", section
    典型应用场景).  Each sequence's gradients are those of attention_bwd on
    its own rows.  Returns (dq [total,H,d], dk, dv [total,Hkv,d])."""
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(dout)
    cu = _i64(cu_seqlens)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(cu.size - 1):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        if s1 <= s0:
            continue
        per = [x[s0:s1].transpose(1, 0, 2)[None] for x in (q, k, v, g)]  # [1, heads, len, d]
        gq, gk, gv = attention_bwd(*per, causal, scale)
        dq[s0:s1], dk[s0:s1], dv[s0:s1] = (x[0].transpose(1, 0, 2) for x in (gq, gk, gv))
    return dq, dk, dv


def rope(x, cos_t, sin_t, bf16_round: bool = True):
    """Rotary embedding of x [..., N, d] (positions 0..N-1) with the fp32 tables
    cos_t, sin_t [>=N, d/2]; returns a new fp64 array.  Without bf16_round the
    rotation is computed in fp64; with it, each rotated value is that fp64
    rotation rounded once to the nearest bf16 (ties to even), the values the
    bf16 tensor-core products consume."""
    xs = _f64(x).copy()
    N, d = xs.shape[-2], xs.shape[-1]
    c = np.ascontiguousarray(np.asarray(cos_t.cpu() if hasattr(cos_t, "cpu") else cos_t,
                                        dtype=np.float32)[:N])
    s_ = np.ascontiguousarray(np.asarray(sin_t.cpu() if hasattr(sin_t, "cpu") else sin_t,
                                         dtype=np.float32)[:N])
    assert c.shape == (N, d // 2) and s_.shape == (N, d // 2)
    rows = int(np.prod(xs.shape[:-2])) if xs.ndim > 2 else 1
    fn = lib().oracle_rope_bf16 if bf16_round else lib().oracle_rope_exact
    fn(_ptr(xs), c.ctypes.data_as(ctypes.c_void_p), s_.ctypes.data_as(ctypes.c_void_p), rows, N, d)
    return xs


def attention_bwd(q, k, v, dout, causal: bool, scale: float):
    """Gradients (dq, dk, dv) of attention over q [B,H,N,d] and k, v
    [B,Hkv,N,d] (query head h uses K/V head h // (H/Hkv); Hkv = H is plain
    multi-head) for the output gradient dout [B,H,N,d], in fp64."""
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    assert k.shape == v.shape == (B, Hkv, N, d) and g.shape == q.shape and H % Hkv == 0
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    rc = lib().oracle_attention_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(dq), _ptr(dk),
                                    _ptr(dv), B, H, Hkv, N, d, int(bool(causal)), float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle_attention_bwd failed ({rc})")
    return dq, dk, dv
