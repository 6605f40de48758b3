"""Seeded synthetic inputs shaped like the attention workloads.

This module holds input generation only -- no attention arithmetic -- so that
the CUDA path and the CPU oracle can be fed the very same values.  Every draw
goes through a torch.Generator seeded explicitly; draw order within a
workload is fixed: q, k, v, then lengths, then the page permutation.

Small workloads are drawn on the CPU (so the CPU-only tests can build them);
large ones on the CUDA device with torch's own Philox generator (their
host-side fp32 temporaries would not fit the host), in the chunk order the
code below fixes.  Either way the values are a pure function of the seed,
shape and device kind.

Shapes follow the workloads the pages describe: the [1, 32, 16384, 128]
query/key/value layout of the page "为什么“Flash”突然成了AI圈的高频词"
(lqnn.cn), section 2.1; variable-length batches of the page "Flash Attention
是什么" (ai.lansai.wang), section on typical applications; 256-token KV
pages of the page "“Flash”不是那个被时代淘汰的插件" (0539edu.com), section 2.
"""
from dataclasses import dataclass, field
from typing import List, Optional

import torch

PAGE_SIZE = 256


@dataclass(frozen=True)
class FwdWorkload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    seed: int
    std: float = 1.0
    fp32_source: bool = False  # drawn as fp32 and rounded once to bf16


@dataclass(frozen=True)
class VarlenWorkload:
    name: str
    B: int
    H: int
    d: int
    len_lo: int
    len_hi: int  # inclusive
    causal: bool
    seed: int
    std: float = 1.0


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int
    H: int
    d: int
    len_lo: int
    len_hi: int  # inclusive
    seed: int
    page_size: int = PAGE_SIZE


# The five workloads: tiny, long prefill, batched prefill (+ varlen),
# 128K context, paged decode.
TINY = FwdWorkload("tiny_fwd_b1_h2_n256_d64", 1, 2, 256, 64, False, 1, fp32_source=True)
TINY_CAUSAL = FwdWorkload("tiny_fwd_causal_b1_h2_n256_d64", 1, 2, 256, 64, True, 1, fp32_source=True)
LONG_PREFILL = FwdWorkload("long_prefill_fwd_b1_h32_n16384_d128_causal", 1, 32, 16384, 128, True, 2)
BATCHED = FwdWorkload("batched_prefill_fwd_b8_h32_n8192_d128_causal", 8, 32, 8192, 128, True, 3)
BATCHED_VARLEN = VarlenWorkload("varlen_prefill_fwd_b8_h32_len1024to8192_d128_causal",
                                8, 32, 128, 1024, 8192, True, 31)
CTX128K = FwdWorkload("ctx128k_fwd_b1_h32_n131072_d128_causal", 1, 32, 131072, 128, True, 4, std=0.5)
PAGED_DECODE = DecodeWorkload("paged_decode_b64_h32_d128_len1024to32768_page256",
                              64, 32, 128, 1024, 32768, 5)

# Above this many elements per tensor the draw happens on the device.
_HOST_LIMIT = 1 << 26


def _gen(seed: int, device: str) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _device_for(numel: int, device: Optional[str]) -> str:
    if device is not None:
        return device
    return "cpu" if numel <= _HOST_LIMIT else "cuda"


def _randn_bf16(shape, g: torch.Generator, std: float, device: str) -> torch.Tensor:
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def fwd_inputs(w: FwdWorkload, device: Optional[str] = None):
    """q, k, v as bf16 [B,H,N,d] tensors (on the generation device).

    For fp32-sourced workloads the fp32 draws are returned too, as
    (q, k, v, (q32, k32, v32)); the bf16 tensors are their one-time RNE
    rounding.
    """
    shape = (w.B, w.H, w.N, w.d)
    n = w.B * w.H * w.N * w.d
    dev = _device_for(n, device)
    g = _gen(w.seed, dev)
    if w.fp32_source:
        f = [torch.randn(shape, generator=g, device=dev, dtype=torch.float32) * w.std
             for _ in range(3)]
        return tuple(x.to(torch.bfloat16) for x in f) + (tuple(f),)
    q = _randn_bf16(shape, g, w.std, dev)
    k = _randn_bf16(shape, g, w.std, dev)
    v = _randn_bf16(shape, g, w.std, dev)
    return q, k, v


def custom_fwd_inputs(B, H, N, d, seed, std=1.0, device="cpu"):
    """Same recipe for arbitrary (test) shapes."""
    return fwd_inputs(FwdWorkload("custom", B, H, N, d, False, seed, std), device)


def gqa_fwd_inputs(B, H, H_kv, N, d, seed, std=1.0, device=None):
    """q [B,H,N,d] and k, v [B,H_kv,N,d] (grouped-query attention), same
    recipe: q, then k, then v from one seeded generator."""
    n = B * H * N * d
    dev = _device_for(n, device)
    g = _gen(seed, dev)
    q = _randn_bf16((B, H, N, d), g, std, dev)
    k = _randn_bf16((B, H_kv, N, d), g, std, dev)
    v = _randn_bf16((B, H_kv, N, d), g, std, dev)
    return q, k, v


def rope_tables(max_pos: int, d: int, base: float = 10000.0, device: Optional[str] = None):
    """The rotary-embedding lookup tables: cos and sin of p * base^(-2i/d) for
    positions p < max_pos and i < d/2, evaluated in fp64 and stored as fp32
    [max_pos, d/2] (the caller-side precomputation the attention calls take as
    input)."""
    i = torch.arange(d // 2, dtype=torch.float64)
    inv = base ** (-2.0 * i / d)
    ang = torch.arange(max_pos, dtype=torch.float64)[:, None] * inv[None, :]
    dev = device or "cpu"
    return ang.cos().float().to(dev).contiguous(), ang.sin().float().to(dev).contiguous()


def varlen_lengths(B: int, lo: int, hi: int, seed: int) -> List[int]:
    g = _gen(seed, "cpu")
    return [int(x) for x in torch.randint(lo, hi + 1, (B,), generator=g)]


def cu_seqlens_of(lengths: List[int]) -> torch.Tensor:
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + int(L))
    return torch.tensor(cu, dtype=torch.int32)


def varlen_inputs(H: int, d: int, lengths: List[int], seed: int, std: float = 1.0,
                  device: Optional[str] = None):
    """Packed q, k, v [total,H,d] bf16 plus cu_seqlens (int32, CPU)."""
    total = sum(lengths)
    dev = _device_for(total * H * d, device)
    g = _gen(seed + 1, dev)  # the lengths were drawn from `seed`
    q = _randn_bf16((total, H, d), g, std, dev)
    k = _randn_bf16((total, H, d), g, std, dev)
    v = _randn_bf16((total, H, d), g, std, dev)
    return q, k, v, cu_seqlens_of(lengths)


def varlen_workload_inputs(w: VarlenWorkload, device: Optional[str] = None):
    lengths = varlen_lengths(w.B, w.len_lo, w.len_hi, w.seed)
    return varlen_inputs(w.H, w.d, lengths, w.seed, w.std, device)


@dataclass
class PagedCache:
    q: torch.Tensor            # [B,H,d] bf16
    k_pages: torch.Tensor      # [P,H,page_size,d] bf16
    v_pages: torch.Tensor      # [P,H,page_size,d] bf16
    page_table: torch.Tensor   # [P] int32, packed per sequence
    seq_lens: torch.Tensor     # [B] int32
    page_size: int
    pages_per_seq: List[int] = field(default_factory=list)


def paged_inputs(B: int, H: int, d: int, lengths: List[int], seed: int,
                 page_size: int = PAGE_SIZE, device: Optional[str] = None,
                 poison_unused: bool = True, H_kv: Optional[int] = None) -> PagedCache:
    """A paged KV cache holding `lengths[b]` tokens for sequence b.

    The pool holds exactly the pages the sequences need; the pages are
    handed out through a seeded random permutation, so consecutive pages of
    a sequence sit at unrelated pool slots.  The page table lists every
    sequence's pages in order, sequences back to back.  With poison_unused,
    the slots past a sequence's last token in its last page hold NaN, so any
    read of them shows up in the output.  H_kv (default H) is the number of
    K/V heads the pages hold (grouped-query caches); q keeps H heads.
    """
    Hk = H if H_kv is None else H_kv
    pages_per_seq = [(int(L) + page_size - 1) // page_size for L in lengths]
    P = sum(pages_per_seq)
    n = max(P, 1) * Hk * page_size * d
    dev = _device_for(n, device)
    g = _gen(seed, dev)
    q = _randn_bf16((B, H, d), g, 1.0, dev)
    k_pages = torch.empty((P, Hk, page_size, d), dtype=torch.bfloat16, device=dev)
    v_pages = torch.empty((P, Hk, page_size, d), dtype=torch.bfloat16, device=dev)
    chunk = max(1, (1 << 26) // (Hk * page_size * d))
    for dst in (k_pages, v_pages):
        for p0 in range(0, P, chunk):
            p1 = min(P, p0 + chunk)
            dst[p0:p1] = _randn_bf16((p1 - p0, Hk, page_size, d), g, 1.0, dev)
    gperm = _gen(seed + 1, "cpu")
    perm = torch.randperm(P, generator=gperm).to(torch.int32)
    if poison_unused:
        pos = 0
        for L, npg in zip(lengths, pages_per_seq):
            if npg:
                used = int(L) - (npg - 1) * page_size
                last = int(perm[pos + npg - 1])
                if used < page_size:
                    k_pages[last, :, used:, :] = float("nan")
                    v_pages[last, :, used:, :] = float("nan")
            pos += npg
    seq_lens = torch.tensor([int(L) for L in lengths], dtype=torch.int32)
    return PagedCache(q, k_pages, v_pages, perm, seq_lens, page_size, pages_per_seq)


@dataclass
class PrefillWorkload:
    """Chunked prefill over a paged cache: sequence b has ctx_lens[b] cached
    tokens followed by q_len new ones (the queries)."""
    name: str
    B: int
    H: int
    H_kv: int
    d: int
    q_len: int
    ctx_lo: int
    ctx_hi: int
    causal: bool
    seed: int
    page_size: int = PAGE_SIZE


PAGED_PREFILL = PrefillWorkload("paged_prefill_b8_h32_d128_ctx1024to8192_q1024_page256",
                                8, 32, 32, 128, 1024, 1024, 8192, True, 61)


def prefill_inputs(B: int, H: int, H_kv: int, d: int, lens_after: List[int], q_lens: List[int],
                   seed: int, page_size: int = PAGE_SIZE, device: Optional[str] = None):
    """A paged cache holding lens_after[b] tokens per sequence (pages from a
    shuffled pool, NaN past each sequence's end) and packed queries for the
    last q_lens[b] positions: returns (cache, q [sum q_lens, H, d], cu_q)."""
    cache = paged_inputs(B, H, d, lens_after, seed, page_size, device, H_kv=H_kv)
    total_q = int(sum(q_lens))
    dev = cache.k_pages.device.type
    g = _gen(seed + 2, dev)
    q = _randn_bf16((max(total_q, 1), H, d), g, 1.0, dev)[:total_q]
    return cache, q, cu_seqlens_of(q_lens)


def prefill_workload_inputs(w: PrefillWorkload, device: Optional[str] = None):
    ctx = varlen_lengths(w.B, w.ctx_lo, w.ctx_hi, w.seed)
    lens_after = [c + w.q_len for c in ctx]
    return prefill_inputs(w.B, w.H, w.H_kv, w.d, lens_after, [w.q_len] * w.B, w.seed,
                          w.page_size, device)


def decode_workload_inputs(w: DecodeWorkload, device: Optional[str] = None) -> PagedCache:
    lengths = varlen_lengths(w.B, w.len_lo, w.len_hi, w.seed)
    return paged_inputs(w.B, w.H, w.d, lengths, w.seed, w.page_size, device)
