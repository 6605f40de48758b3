"""fa_decode_paged_noalloc: paged decode for callers that cannot allocate
device memory (serving loops with all memory reserved up front, host programs
whose own allocator forbids other allocations).  Called straight through the C ABI and checked against the
allocating fa_decode_paged on the same inputs, twice in a row, within the
tolerances the parity tests use.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it also passes alone in a fresh
process (it builds its own inputs and needs no earlier state).
"""
import ctypes

import pytest
import torch

import attn_fwd_04_b200 as fa
import oracle
from attn_fwd_04_b200 import workloads as W
from helpers import assert_o_close, to64

pytestmark = pytest.mark.gpu

PS = 256


def _noalloc_raw(c: W.PagedCache, o: torch.Tensor) -> int:
    B, H, d = c.q.shape
    return fa.lib().fa_decode_paged_noalloc(
        ctypes.c_void_p(c.q.data_ptr()), ctypes.c_void_p(c.k_pages.data_ptr()),
        ctypes.c_void_p(c.v_pages.data_ptr()), ctypes.c_void_p(c.page_table.data_ptr()),
        ctypes.c_void_p(c.seq_lens.data_ptr()), ctypes.c_void_p(o.data_ptr()),
        B, H, d, PS, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _cuda(c: W.PagedCache) -> W.PagedCache:
    return W.PagedCache(c.q.cuda(), c.k_pages.cuda(), c.v_pages.cuda(), c.page_table.cuda(),
                        c.seq_lens.cuda(), c.page_size, c.pages_per_seq)


def _case_small():
    lens = [1, 255, 256, 257, 3000, 0, 700]
    return W.paged_inputs(len(lens), 4, 128, lens, seed=41, device="cpu")


def _case_many_heads():
    # 64 sequences x 32 heads: the fixed scratch holds fewer splits per
    # sequence than the allocating path uses, so the two differ by rounding
    lens = W.varlen_lengths(64, 256, 3000, seed=42)
    return W.paged_inputs(64, 32, 128, lens, seed=42, device="cuda")


def test_noalloc_matches_allocating_decode_twice_in_a_row():
    small = _case_small()
    cases = [_cuda(small), _cuda(_case_many_heads())]
    results = []
    for c in cases:                      # two calls in a row, different shapes
        o_ref = fa.fa_decode_paged(c.q, c.k_pages, c.v_pages, c.page_table, c.seq_lens, PS)
        o = torch.full_like(c.q, float("nan"))
        assert _noalloc_raw(c, o) == fa.FA_OK
        assert fa.fa_get_device_error() == fa.FA_OK
        assert_o_close(to64(o), to64(o_ref), "noalloc vs fa_decode_paged")
        results.append(o)
    # the first case again: the scratch still holds the second call's data
    c = cases[0]
    o_again = torch.full_like(c.q, float("nan"))
    assert _noalloc_raw(c, o_again) == fa.FA_OK
    assert fa.fa_get_device_error() == fa.FA_OK
    assert torch.equal(o_again, results[0])
    # through the Python wrapper, into a preallocated output, on a side stream
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    o_side = torch.full_like(c.q, float("nan"))
    got = fa.fa_decode_paged_noalloc(c.q, c.k_pages, c.v_pages, c.page_table, c.seq_lens, PS,
                                     o=o_side, stream=side)
    assert got is o_side
    assert fa.fa_get_device_error(stream=side) == fa.FA_OK
    torch.cuda.current_stream().wait_stream(side)
    assert torch.equal(o_side, results[0])
    # and against the fp64 oracle directly
    o64, _ = oracle.decode_paged(small.q, small.k_pages, small.v_pages, small.page_table,
                                 small.seq_lens, PS)
    assert_o_close(to64(results[0]), o64, "noalloc vs oracle")
    assert torch.all(results[0][5] == 0)  # the empty sequence


def test_noalloc_rejects_sizes_beyond_its_scratch():
    c = _cuda(_case_small())
    o = torch.empty_like(c.q)
    B_too_many = 40000  # 40000 x 1 head x (128+1) floats of partials > 16 MiB
    rc = fa.lib().fa_decode_paged_noalloc(
        ctypes.c_void_p(c.q.data_ptr()), ctypes.c_void_p(c.k_pages.data_ptr()),
        ctypes.c_void_p(c.v_pages.data_ptr()), ctypes.c_void_p(c.page_table.data_ptr()),
        ctypes.c_void_p(c.seq_lens.data_ptr()), ctypes.c_void_p(o.data_ptr()),
        B_too_many, 1, 128, PS, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == fa.FA_ERR_SHAPE
    assert fa.fa_get_device_error() == fa.FA_OK
