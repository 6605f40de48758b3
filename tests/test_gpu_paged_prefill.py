"""GPU parity of the paged-cache write (fa_append_paged, byte-exact against
the oracle) and of attention for several new queries per sequence through
the page table (fa_prefill_paged, within the tolerances), through the C ABI.

The pages past each sequence's last token hold NaN, so a read of them, or a
product of zero probabilities with them, shows up in the output."""
import math

import numpy as np
import pytest
import torch

import attn_fwd_04_b200 as fa
import oracle
from attn_fwd_04_b200 import workloads as W
from helpers import assert_lse_close, assert_o_close, to64

pytestmark = pytest.mark.gpu

PS = 256


def _prefill(cache, q, cu, max_q, causal, scale):
    qc = q.cuda()
    o = torch.full_like(qc, float("nan"))
    lse = torch.full((q.shape[1], q.shape[0]), float("nan"), device="cuda")
    fa.fa_prefill_paged(qc, cache.k_pages.cuda(), cache.v_pages.cuda(), cache.page_table.cuda(),
                        cache.seq_lens.cuda(), cu.cuda(), max_q, causal, scale, o=o, lse=lse)
    assert fa.fa_get_device_error() == fa.FA_OK
    return o, lse


CASES = [  # (lens_after, q_lens)
    ([1, 300, 1000, 4103, 256, 513], [1, 127, 1000, 129, 200, 513]),
    ([2049, 130, 77], [128, 130, 3]),
]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("H,H_kv", [(4, 4), (8, 2)])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("case", [0, 1])
def test_prefill_small_full_compare(d, H, H_kv, causal, case):
    lens, nq = CASES[case]
    cache, q, cu = W.prefill_inputs(len(lens), H, H_kv, d, lens, nq, seed=300 + d + H + case,
                                    device="cpu")
    scale = 1 / math.sqrt(d)
    o, lse = _prefill(cache, q, cu, max(nq), causal, scale)
    o_ref, lse_ref = oracle.prefill_paged(q, cache.k_pages, cache.v_pages, cache.page_table,
                                          cache.seq_lens, cu, PS, causal, scale)
    assert_o_close(to64(o), o_ref, f"prefill d={d} H={H}/{H_kv} causal={causal}")
    assert_lse_close(to64(lse), lse_ref, "prefill lse")


def test_prefill_one_query_matches_decode():
    lens = [1, 255, 257, 3000]
    cache, q, cu = W.prefill_inputs(4, 4, 4, 128, lens, [1] * 4, seed=310, device="cpu")
    o, _ = _prefill(cache, q, cu, 1, True, 1 / math.sqrt(128))
    g = W.PagedCache(q.cuda(), cache.k_pages.cuda(), cache.v_pages.cuda(),
                     cache.page_table.cuda(), cache.seq_lens.cuda(), PS, cache.pages_per_seq)
    od = fa.fa_decode_paged(g.q, g.k_pages, g.v_pages, g.page_table, g.seq_lens, PS)
    assert fa.fa_get_device_error() == fa.FA_OK
    # both within tolerance of the oracle, so within twice of each other
    assert (o.float() - od.float()).abs().max().item() <= 4e-2


def test_prefill_whole_sequences_equal_varlen_bitwise():
    """Every cached token a query: the same key tiles, masks and arithmetic
    as the variable-length forward pass on the gathered sequences."""
    lens = [300, 129, 1024]
    H, d = 2, 128
    cache, q, cu = W.prefill_inputs(3, H, H, d, lens, lens, seed=311, device="cpu")
    o, lse = _prefill(cache, q, cu, max(lens), True, 0.1)
    total = sum(lens)
    kc = fa.fa_gather_paged(cache.k_pages.cuda(), cache.page_table.cuda(),
                            cache.seq_lens.cuda(), total, PS)
    vc = fa.fa_gather_paged(cache.v_pages.cuda(), cache.page_table.cuda(),
                            cache.seq_lens.cuda(), total, PS)
    ov, lv = fa.fa_fwd_varlen(q.cuda(), kc, vc, cu.cuda(), max(lens), True, 0.1)
    assert fa.fa_get_device_error() == fa.FA_OK
    assert torch.equal(o, ov) and torch.equal(lse, lv)


def test_prefill_heaviest_first_keeps_each_sequence():
    """Paged prefill runs its sequences heaviest first (a device-side ranking
    by attended pairs): a batch whose cached lengths are not in that order,
    with a tie, gives each sequence bit for bit what a call on that sequence
    alone gives."""
    ctx = [700, 3000, 257, 3000, 1200]
    ql = [128, 64, 257, 64, 300]
    H, d = 4, 128
    cache, q, cu = W.prefill_inputs(len(ctx), H, H, d, ctx, ql, seed=313, device="cpu")
    o, lse = _prefill(cache, q, cu, max(ql), True, 0.1)
    for b in range(len(ctx)):
        pages = cache.pages_per_seq
        p0 = sum(pages[:b])
        one = W.PagedCache(cache.q, cache.k_pages, cache.v_pages,
                           cache.page_table[p0:p0 + pages[b]].contiguous(),
                           cache.seq_lens[b:b + 1].contiguous(), cache.page_size, [pages[b]])
        s0, s1 = int(cu[b]), int(cu[b + 1])
        cu1 = torch.tensor([0, s1 - s0], dtype=torch.int32)
        o1, l1 = _prefill(one, q[s0:s1].contiguous(), cu1, s1 - s0, True, 0.1)
        assert torch.equal(o1, o[s0:s1]), f"sequence {b}"
        assert torch.equal(l1, lse[:, s0:s1]), f"sequence {b}"


def test_prefill_more_queries_than_tokens_reported():
    lens, nq = [100, 50], [10, 60]
    cache, q, cu = W.prefill_inputs(2, 2, 2, 64, lens, [10, 50], seed=312, device="cpu")
    q2 = torch.cat([q, q[:10]], dim=0)  # 70 rows: sequence 1 claims 60 queries
    cu2 = torch.tensor([0, 10, 70], dtype=torch.int32)
    qc = q2.cuda()
    o = torch.zeros_like(qc)
    lse = torch.zeros((2, 70), device="cuda")
    fa.fa_prefill_paged(qc, cache.k_pages.cuda(), cache.v_pages.cuda(), cache.page_table.cuda(),
                        cache.seq_lens.cuda(), cu2.cuda(), 60, True, 0.125, o=o, lse=lse)
    assert fa.fa_get_device_error() == fa.FA_ERR_DEVICE_BAD_INPUT
    o_ref, lse_ref = oracle.prefill_paged(q[:10], cache.k_pages, cache.v_pages, cache.page_table,
                                          cache.seq_lens[:1], cu[:2], PS, True, 0.125)
    assert_o_close(to64(o[:10]), o_ref, "valid sequence")


def test_paged_prefill_workload_sampled():
    w = W.PAGED_PREFILL
    cache, q, cu = W.prefill_workload_inputs(w, device="cuda")
    scale = 1 / math.sqrt(w.d)
    o, lse = fa.fa_prefill_paged(q, cache.k_pages, cache.v_pages, cache.page_table.cuda(),
                                 cache.seq_lens.cuda(), cu.cuda(), w.q_len, w.causal, scale)
    assert fa.fa_get_device_error() == fa.FA_OK
    assert bool(torch.isfinite(o).all()) and bool(torch.isfinite(lse).all())
    # sequences 0 and B-1, each on its own small pool (pages in table order)
    got_o, ref_o, got_l, ref_l = [], [], [], []
    for b in (0, w.B - 1):
        off = sum(cache.pages_per_seq[:b])
        n = cache.pages_per_seq[b]
        idx = cache.page_table[off:off + n].long().to(cache.k_pages.device)
        kp, vp = cache.k_pages.index_select(0, idx).cpu(), cache.v_pages.index_select(0, idx).cpu()
        rows = slice(int(cu[b]), int(cu[b + 1]))
        o_ref, lse_ref = oracle.prefill_paged(q[rows].cpu(), kp, vp, torch.arange(n),
                                              cache.seq_lens[b:b + 1], torch.tensor([0, w.q_len]),
                                              PS, True, scale)
        got_o.append(to64(o[rows]))
        ref_o.append(o_ref)
        got_l.append(to64(lse[:, rows]))
        ref_l.append(lse_ref)
    assert_o_close(np.concatenate(got_o), np.concatenate(ref_o), w.name)
    assert_lse_close(np.concatenate(got_l, axis=1), np.concatenate(ref_l, axis=1), w.name)


# -- appending new rows ---------------------------------------------------------------

@pytest.mark.parametrize("d", [64, 128])
def test_append_bit_exact(d):
    """Rows appended into their slots: the pool afterwards equals the
    oracle's append byte for byte (slots nobody writes keep their content)."""
    H_kv = 2
    lens_before, n_new = [0, 255, 256, 700, 9], [300, 1, 257, 0, 3]
    lens_after = [a + n for a, n in zip(lens_before, n_new)]
    cache = W.paged_inputs(len(lens_after), H_kv, d, lens_after, seed=320 + d, device="cpu",
                           H_kv=H_kv)
    g = torch.Generator().manual_seed(321)
    total = sum(n_new)
    k_new = torch.randn((total, H_kv, d), generator=g).to(torch.bfloat16)
    v_new = torch.randn((total, H_kv, d), generator=g).to(torch.bfloat16)
    cu = W.cu_seqlens_of(n_new)
    kp, vp = cache.k_pages.cuda(), cache.v_pages.cuda()
    fa.fa_append_paged(k_new.cuda(), v_new.cuda(), cu.cuda(), kp, vp, cache.page_table.cuda(),
                       cache.seq_lens.cuda(), PS)
    assert fa.fa_get_device_error() == fa.FA_OK
    for got, pages, new in ((kp, cache.k_pages, k_new), (vp, cache.v_pages, v_new)):
        ref = oracle.append_paged(pages, cache.page_table, cache.seq_lens, new, cu, PS)
        ref_bf16 = torch.from_numpy(ref).to(torch.bfloat16)  # exact: values are bf16 or NaN
        same = got.cpu().view(torch.int16) == ref_bf16.view(torch.int16)
        both_nan = torch.isnan(got.cpu()) & torch.isnan(ref_bf16)
        assert bool((same | both_nan).all())


def test_append_then_decode_equals_decode_of_full_cache():
    """Serving-loop order: append the new token, then decode -- the same as
    decoding a cache that held the token from the start."""
    H, d = 4, 128
    lens = [1, 256, 1000]
    full = W.paged_inputs(3, H, d, lens, seed=330, device="cpu")
    # the last token of every sequence, taken out and written back
    starts = np.concatenate([[0], np.cumsum(lens)])
    kc = oracle.gather_paged(full.k_pages, full.page_table, full.seq_lens, PS)
    vc = oracle.gather_paged(full.v_pages, full.page_table, full.seq_lens, PS)
    last = [int(s) - 1 for s in starts[1:]]
    k_new = torch.from_numpy(kc[last]).to(torch.bfloat16)
    v_new = torch.from_numpy(vc[last]).to(torch.bfloat16)
    kp, vp = full.k_pages.clone(), full.v_pages.clone()
    off = 0
    for b, L in enumerate(lens):  # wipe the last token's slot
        page = int(full.page_table[off + (L - 1) // PS])
        kp[page, :, (L - 1) % PS] = float("nan")
        vp[page, :, (L - 1) % PS] = float("nan")
        off += (L + PS - 1) // PS
    kp, vp = kp.cuda(), vp.cuda()
    pt, sl = full.page_table.cuda(), full.seq_lens.cuda()
    fa.fa_append_paged(k_new.cuda(), v_new.cuda(), W.cu_seqlens_of([1, 1, 1]).cuda(), kp, vp, pt,
                       sl, PS)
    o = fa.fa_decode_paged(full.q.cuda(), kp, vp, pt, sl, PS)
    o_full = fa.fa_decode_paged(full.q.cuda(), full.k_pages.cuda(), full.v_pages.cuda(), pt, sl, PS)
    assert fa.fa_get_device_error() == fa.FA_OK
    assert torch.equal(o, o_full)


def test_append_bad_page_reported_and_skipped():
    lens = [10, 20]
    cache = W.paged_inputs(2, 2, 64, lens, seed=340, device="cpu", poison_unused=False)
    bad_table = cache.page_table.clone()
    bad_table[0] = 10_000  # outside the pool
    k_new = torch.ones((3, 2, 64), dtype=torch.bfloat16)
    kp, vp = cache.k_pages.cuda(), cache.v_pages.cuda()
    fa.fa_append_paged(k_new.cuda(), k_new.cuda(), torch.tensor([0, 1, 3], dtype=torch.int32).cuda(),
                       kp, vp, bad_table.cuda(), cache.seq_lens.cuda(), PS)
    assert fa.fa_get_device_error() == fa.FA_ERR_DEVICE_BAD_INPUT
    # sequence 1 (valid pages) was written
    page = int(cache.page_table[1])
    assert torch.all(kp[page, :, 18:20].cpu() == 1)
