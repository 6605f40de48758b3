"""Calls on different streams of one GPU may overlap: each stream has its own
library workspace (decode split partials, page offsets), so a paged decode on
one stream and a paged prefill on another, enqueued back to back many times,
give exactly what each gives alone (neither has a run-to-run rounding
difference: no atomics in either)."""
import math

import pytest
import torch

import attn_fwd_04_b200 as fa
from attn_fwd_04_b200 import workloads as W

pytestmark = pytest.mark.gpu

PS = 256


def test_decode_and_prefill_on_two_streams_overlap():
    H, d = 32, 128
    # decode: 16 sequences of 1K..16K cached tokens, 32 heads
    dlens = W.varlen_lengths(16, 1024, 16384, 41)
    dc = W.paged_inputs(16, H, d, dlens, seed=41, device="cuda")
    dpt, dsl = dc.page_table.cuda(), dc.seq_lens.cuda()
    # prefill: 8 sequences, 256 new queries after 1K..8K cached tokens, 8 K/V heads
    ctx = W.varlen_lengths(8, 1024, 8192, 42)
    pc, pq, pcu = W.prefill_inputs(8, H, 8, d, [n + 256 for n in ctx], [256] * 8, seed=42,
                                   device="cuda")
    ppt, psl, pcud = pc.page_table.cuda(), pc.seq_lens.cuda(), pcu.cuda()
    scale = 1 / math.sqrt(d)

    def decode(o, stream=None):
        fa.fa_decode_paged(dc.q, dc.k_pages, dc.v_pages, dpt, dsl, PS, o=o, stream=stream)

    def prefill(o, lse, stream=None):
        fa.fa_prefill_paged(pq, pc.k_pages, pc.v_pages, ppt, psl, pcud, 256, True, scale,
                            page_size=PS, o=o, lse=lse, stream=stream)

    # each alone, on the default stream
    od_ref = torch.empty_like(dc.q)
    decode(od_ref)
    op_ref = torch.empty_like(pq)
    lp_ref = torch.empty((H, pq.shape[0]), dtype=torch.float32, device="cuda")
    prefill(op_ref, lp_ref)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == fa.FA_OK
    assert bool(torch.isfinite(od_ref.float()).all()) and bool(torch.isfinite(op_ref.float()).all())

    # both, interleaved on two streams
    n = 12
    od = [torch.full_like(od_ref, float("nan")) for _ in range(n)]
    op = [torch.full_like(op_ref, float("nan")) for _ in range(n)]
    lp = [torch.full_like(lp_ref, float("nan")) for _ in range(n)]
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    for i in range(n):
        decode(od[i], stream=s1)
        prefill(op[i], lp[i], stream=s2)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == fa.FA_OK
    for i in range(n):
        assert torch.equal(od[i], od_ref), f"decode {i}"
        assert torch.equal(op[i], op_ref) and torch.equal(lp[i], lp_ref), f"prefill {i}"
    fa.fa_release_workspace()  # frees every stream's workspace on this GPU (raises on failure)
    decode(od_ref, stream=s1)      # a released workspace is allocated again on demand
    torch.cuda.synchronize()
    assert torch.equal(od_ref, od[0])
