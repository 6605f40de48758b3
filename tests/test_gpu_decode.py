"""GPU parity of paged decode (fa_decode_paged) and of the paged gather
(fa_gather_paged) against the fp64 CPU oracle, through the C ABI.

The gather is integer/byte work and must match the oracle's gather bit for
bit.  Decode is compared within the floating-point tolerances, element by
element on small caches and on sampled sequences of the full-size workload.
"""
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


def _on_gpu(c: W.PagedCache) -> W.PagedCache:
    return W.PagedCache(c.q.cuda(), c.k_pages.cuda(), c.v_pages.cuda(), c.page_table.cuda(),
                        c.seq_lens.cuda(), c.page_size, c.pages_per_seq)


def _decode(c: W.PagedCache):
    o = torch.full_like(c.q, float("nan"))
    fa.fa_decode_paged(c.q, c.k_pages, c.v_pages, c.page_table, c.seq_lens, c.page_size, o=o)
    assert fa.fa_get_device_error() == fa.FA_OK
    return o


def _mini(c: W.PagedCache, b: int):
    """Sequence b alone: its pages (in table order) as a small pool, with the
    identity page table -- so the oracle can gather and decode it on the host."""
    off = sum(c.pages_per_seq[:b])
    n = c.pages_per_seq[b]
    idx = c.page_table[off:off + n].long()
    kp = c.k_pages.index_select(0, idx.to(c.k_pages.device)).cpu()
    vp = c.v_pages.index_select(0, idx.to(c.v_pages.device)).cpu()
    return kp, vp, torch.arange(n, dtype=torch.int32), c.seq_lens[b:b + 1].cpu()


LENS_SMALL = [1, 2, 255, 256, 257, 511, 512, 513, 1000, 4103]


@pytest.mark.parametrize("d", [64, 128])
def test_gather_bit_exact_small(d):
    c = W.paged_inputs(len(LENS_SMALL) + 1, 3, d, LENS_SMALL + [0], seed=21, device="cpu")
    g = _on_gpu(c)
    total = int(c.seq_lens.sum())
    out = torch.full((total, 3, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    fa.fa_gather_paged(g.k_pages, g.page_table, g.seq_lens, total, PS, out=out)
    assert fa.fa_get_device_error() == fa.FA_OK
    ref = oracle.gather_paged(c.k_pages, c.page_table, c.seq_lens, PS)
    ref_bf16 = torch.from_numpy(ref).to(torch.bfloat16)  # exact: values are bf16
    assert torch.equal(out.cpu().view(torch.int16), ref_bf16.view(torch.int16))


@pytest.mark.parametrize("d", [64, 128])
def test_decode_small_full_compare(d):
    c = W.paged_inputs(len(LENS_SMALL), 4, d, LENS_SMALL, seed=22, device="cpu")
    o = _decode(_on_gpu(c))
    o_ref, _ = oracle.decode_paged(c.q, c.k_pages, c.v_pages, c.page_table, c.seq_lens, PS)
    assert_o_close(to64(o), o_ref, f"decode d={d}")


def test_decode_long_sequence_bigger_splits():
    # more pages than splits x chunk (64 x 4): each split covers more than the minimum
    lens = [256 * 260 + 17, 300]
    c = W.paged_inputs(2, 2, 128, lens, seed=23, device="cpu")
    o = _decode(_on_gpu(c))
    o_ref, _ = oracle.decode_paged(c.q, c.k_pages, c.v_pages, c.page_table, c.seq_lens, PS)
    assert_o_close(to64(o), o_ref, "long decode")


def test_decode_empty_sequence_is_zero():
    c = W.paged_inputs(3, 2, 128, [0, 700, 0], seed=24, device="cpu")
    o = _decode(_on_gpu(c))
    assert torch.all(o[0] == 0) and torch.all(o[2] == 0)
    o_ref, _ = oracle.decode_paged(c.q, c.k_pages, c.v_pages, c.page_table, c.seq_lens, PS)
    assert_o_close(to64(o[1]), o_ref[1], "middle sequence")


def test_decode_negative_length_reported():
    c = W.paged_inputs(2, 2, 64, [300, 5], seed=25, device="cpu")
    g = _on_gpu(c)
    bad = torch.tensor([300, -5], dtype=torch.int32, device="cuda")
    o = torch.full_like(g.q, float("nan"))
    fa.fa_decode_paged(g.q, g.k_pages, g.v_pages, g.page_table, bad, PS, o=o)
    assert fa.fa_get_device_error() == fa.FA_ERR_DEVICE_BAD_INPUT
    assert torch.all(o[1] == 0)
    o_ref, _ = oracle.decode_paged(c.q[:1], c.k_pages, c.v_pages, c.page_table, c.seq_lens[:1], PS)
    assert_o_close(to64(o[0:1]), o_ref, "valid sequence")


def test_decode_deterministic_and_pool_order_invariant():
    lens = [3000, 77, 1025]
    H, d = 4, 128
    c = W.paged_inputs(3, H, d, lens, seed=26, device="cpu", poison_unused=False)
    g = _on_gpu(c)
    o1 = _decode(g)
    o2 = _decode(g)
    assert torch.equal(o1, o2)
    # move every page to another pool slot; same content through the table
    P = c.k_pages.shape[0]
    perm = torch.randperm(P, generator=torch.Generator().manual_seed(27))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(P)
    k2 = c.k_pages[perm].contiguous()   # new slot s holds old page perm[s]
    v2 = c.v_pages[perm].contiguous()
    pt2 = inv[c.page_table.long()].to(torch.int32)
    g2 = W.PagedCache(g.q, k2.cuda(), v2.cuda(), pt2.cuda(), g.seq_lens, PS, c.pages_per_seq)
    o3 = _decode(g2)
    assert torch.equal(o1, o3)


def test_decode_equals_last_causal_row_of_fwd():
    """Decode of a sequence's last token equals the last row of the causal
    forward pass over the same keys, gathered into contiguous memory."""
    H, d, L = 4, 128, 1500
    c = W.paged_inputs(1, H, d, [L], seed=28, device="cpu")
    g = _on_gpu(c)
    kc = fa.fa_gather_paged(g.k_pages, g.page_table, g.seq_lens, L, PS)  # [L,H,d]
    vc = fa.fa_gather_paged(g.v_pages, g.page_table, g.seq_lens, L, PS)
    qf = torch.randn((1, H, L, d), generator=torch.Generator().manual_seed(29)).to(torch.bfloat16).cuda()
    qf[0, :, L - 1] = g.q[0]
    kf = kc.permute(1, 0, 2).contiguous()[None]
    vf = vc.permute(1, 0, 2).contiguous()[None]
    of, _ = fa.fa_fwd(qf, kf, vf, True, 1 / math.sqrt(d))
    od = _decode(g)
    # both are within tolerance of the oracle, so within 2x of each other
    diff = (of[0, :, L - 1].float() - od[0].float()).abs().max().item()
    assert diff <= 4e-2


def test_paged_decode_workload_sampled():
    w = W.PAGED_DECODE
    c = W.decode_workload_inputs(w, device="cuda")
    c = W.PagedCache(c.q, c.k_pages, c.v_pages, c.page_table.cuda(), c.seq_lens.cuda(),
                     c.page_size, c.pages_per_seq)
    o = _decode(c)
    assert bool(torch.isfinite(o).all())
    lens = c.seq_lens.cpu().tolist()
    order = sorted(range(w.B), key=lambda b: lens[b])
    picks = sorted({order[0], order[-1], order[w.B // 2], 0, w.B - 1, 17})
    got, ref = [], []
    for b in picks:
        kp, vp, pt, sl = _mini(c, b)
        o_ref, _ = oracle.decode_paged(c.q[b:b + 1].cpu(), kp, vp, pt, sl, PS)
        got.append(to64(o[b:b + 1]))
        ref.append(o_ref)
    assert_o_close(np.concatenate(got), np.concatenate(ref), w.name)


def test_paged_gather_workload_sampled_bit_exact():
    w = W.PAGED_DECODE
    c = W.decode_workload_inputs(w, device="cuda")
    pt, sl = c.page_table.cuda(), c.seq_lens.cuda()
    total = int(c.seq_lens.sum())
    out = fa.fa_gather_paged(c.k_pages, pt, sl, total, PS)
    assert fa.fa_get_device_error() == fa.FA_OK
    starts = np.concatenate([[0], np.cumsum(c.seq_lens.numpy())])
    for b in (0, 31, w.B - 1):
        kp, _, ptb, slb = _mini(c, b)
        ref = oracle.gather_paged(kp, ptb, slb, PS)
        got = out[int(starts[b]):int(starts[b + 1])].cpu()
        assert torch.equal(got.view(torch.int16),
                           torch.from_numpy(ref).to(torch.bfloat16).view(torch.int16))


@pytest.mark.parametrize("withheld", [0, 5, 20])
def test_decode_kernel_stall_is_reported_and_recovered(withheld):
    """Failure detection inside the production decode kernel: from one ring
    use on (the first chunk, the sixth, the 21st: the longest units here hold
    24 chunks of 64 tokens) the producer issues no copy
    and every wait is bounded by 50 ms.  The stall comes back as
    FA_ERR_DEVICE_TIMEOUT (no trap, no fault), and a normal decode on the same
    stream right after it computes correctly."""
    lens = [1000, 4103, 9000, 257]
    c = _on_gpu(W.paged_inputs(len(lens), 4, 128, lens, seed=23, device="cpu"))
    assert fa.fa_get_device_error() == fa.FA_OK
    fa.fa_selftest_decode_stall(c.q, c.k_pages, c.v_pages, c.page_table, c.seq_lens, withheld,
                                50_000)
    assert fa.fa_get_device_error() == fa.FA_ERR_DEVICE_TIMEOUT
    assert fa.fa_get_device_error() == fa.FA_OK
    o = _decode(c)
    o_ref, _ = oracle.decode_paged(c.q.cpu(), c.k_pages.cpu(), c.v_pages.cpu(),
                                   c.page_table.cpu(), c.seq_lens.cpu(), PS)
    assert_o_close(to64(o), o_ref, "decode after a stalled decode")


# -- grouped K/V heads (fa_decode_paged_gqa) ---------------------------------------

def _decode_gqa(c: W.PagedCache):
    o = torch.full_like(c.q, float("nan"))
    fa.fa_decode_paged_gqa(c.q, c.k_pages, c.v_pages, c.page_table, c.seq_lens, c.page_size,
                           o=o)
    assert fa.fa_get_device_error() == fa.FA_OK
    return o


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("H,H_kv", [(4, 2), (8, 2), (8, 1), (16, 2), (3, 3), (16, 1), (32, 2),
                                    (32, 1), (64, 2), (48, 1), (6, 2), (12, 1), (40, 2), (17, 1)])
def test_decode_gqa_small_full_compare(d, H, H_kv):
    lens = [1, 255, 257, 1000, 4103, 0]
    c = W.paged_inputs(len(lens), H, d, lens, seed=40 + H + H_kv, device="cpu", H_kv=H_kv)
    o = _decode_gqa(_on_gpu(c))
    o_ref, _ = oracle.decode_paged_gqa(c.q, c.k_pages, c.v_pages, c.page_table, c.seq_lens, PS)
    assert torch.all(o[-1] == 0)  # the empty sequence
    assert_o_close(to64(o), o_ref, f"decode gqa d={d} H={H} H_kv={H_kv}")


def test_decode_gqa_group1_equals_decode():
    """With one query head per K/V head the grouped entry point is decode."""
    lens = [700, 3, 2049]
    c = W.paged_inputs(3, 4, 128, lens, seed=48, device="cpu")
    g = _on_gpu(c)
    assert torch.equal(_decode_gqa(g), _decode(g))


@pytest.mark.parametrize("H_kv", [16, 8, 4, 2, 1])
def test_decode_gqa_workload_sampled(H_kv):
    """The paged-decode workload's lengths with 16, 8, 4, 2 or 1 K/V heads for
    32 query heads (every CTA of the persistent grid runs many units)."""
    w = W.PAGED_DECODE
    lengths = W.varlen_lengths(w.B, w.len_lo, w.len_hi, w.seed)
    c = W.paged_inputs(w.B, w.H, w.d, lengths, w.seed, w.page_size, device="cuda", H_kv=H_kv)
    c = W.PagedCache(c.q, c.k_pages, c.v_pages, c.page_table.cuda(), c.seq_lens.cuda(),
                     c.page_size, c.pages_per_seq)
    o = _decode_gqa(c)
    assert bool(torch.isfinite(o).all())
    got, ref = [], []
    for b in (0, 17, w.B - 1):
        kp, vp, pt, sl = _mini(c, b)
        o_ref, _ = oracle.decode_paged_gqa(c.q[b:b + 1].cpu(), kp, vp, pt, sl, PS)
        got.append(to64(o[b:b + 1]))
        ref.append(o_ref)
    assert_o_close(np.concatenate(got), np.concatenate(ref), f"gqa decode workload H_kv={H_kv}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("H,H_kv", [(8, 4), (8, 2), (16, 2), (16, 1), (32, 1), (40, 2)])
def test_decode_gqa_chunk_and_warp_edges(d, H, H_kv):
    """Lengths that end inside, and right at, the 16- or 32-token slices the
    warps own (32 when two sub-groups share a unit: 32 and 40 query heads per
    K/V head) and the 64-token chunks the crews take in turn; the poisoned
    (NaN) slots past each length must not reach the output."""
    lens = [15, 16, 17, 31, 32, 33, 48, 49, 64, 65, 97, 127, 128, 129, 191, 320, 513, 767]
    c = W.paged_inputs(len(lens), H, d, lens, seed=90 + H + H_kv + d, device="cpu", H_kv=H_kv)
    o = _decode_gqa(_on_gpu(c))
    o_ref, _ = oracle.decode_paged_gqa(c.q, c.k_pages, c.v_pages, c.page_table, c.seq_lens, PS)
    assert_o_close(to64(o), o_ref, f"decode gqa edges d={d} H={H} H_kv={H_kv}")


@pytest.mark.parametrize("H,H_kv", [(32, 1), (16, 2)])
@pytest.mark.parametrize("lens", [[0, 0, 0], [5, 0, 64, 65], [131072], [0, 40000, 1]],
                         ids=["all-empty", "fewer-chunks-than-ctas", "one-128k-sequence",
                              "long-between-empty-and-short"])
def test_decode_gqa_even_split_edges(H, H_kv, lens):
    """Few unit heads per sequence (one or two) split the chunk stream evenly
    over the CTAs: no work at all; fewer 64-token chunks than CTAs (only
    some CTAs take part); one sequence whose chunks span every CTA (its
    merge combines more than 32 pieces); a long sequence beside an empty and
    a one-token one."""
    # the pool must hold a page: with no tokens at all, one sequence's page is
    # allocated and its length then set to 0
    alloc = lens if sum(lens) else [1] + lens[1:]
    c = W.paged_inputs(len(lens), H, 128, alloc, seed=7 + len(lens) + H_kv, device="cpu",
                       H_kv=H_kv)
    c = W.PagedCache(c.q, c.k_pages, c.v_pages, c.page_table,
                     torch.tensor(lens, dtype=torch.int32), c.page_size, c.pages_per_seq)
    o = _decode_gqa(_on_gpu(c))
    assert bool(torch.isfinite(o).all())
    for b, n in enumerate(lens):
        if n == 0:
            assert torch.all(o[b] == 0)
    if sum(lens) == 0:
        return
    o_ref, _ = oracle.decode_paged_gqa(c.q, c.k_pages, c.v_pages, c.page_table, c.seq_lens, PS)
    assert_o_close(to64(o), o_ref, f"decode gqa even split H={H} H_kv={H_kv} lens={lens}")


@pytest.mark.parametrize("H,H_kv", [(8, 2), (4, 4)])
def test_decode_gqa_page_outside_pool_reported(H, H_kv):
    """A page index past the pool is reported through the device error word and
    nothing outside the pool is read; the other sequences are unaffected."""
    lens = [300, 700, 40]
    c = _on_gpu(W.paged_inputs(len(lens), H, 128, lens, seed=77, device="cpu", H_kv=H_kv))
    P = c.k_pages.shape[0]
    good = _decode_gqa(c)
    pt = c.page_table.clone()
    pt[c.pages_per_seq[0]] = P + 5  # the first page of sequence 1
    o = torch.zeros_like(c.q)
    fa.fa_decode_paged_gqa(c.q, c.k_pages, c.v_pages, pt, c.seq_lens, c.page_size, o=o)
    assert fa.fa_get_device_error() == fa.FA_ERR_DEVICE_BAD_INPUT
    assert torch.equal(o[0], good[0]) and torch.equal(o[2], good[2])


# -- decode through a block table (fa_decode_paged_strided) -----------------------

def _block_table(c: W.PagedCache, max_pages: int, pad: int = -1) -> torch.Tensor:
    """The packed table's pages, one row of max_pages per sequence; unused
    entries hold `pad` (an index outside the pool: reading one is reported)."""
    bt = torch.full((len(c.pages_per_seq), max_pages), pad, dtype=torch.int32)
    pt = c.page_table.cpu()
    off = 0
    for b, n in enumerate(c.pages_per_seq):
        bt[b, :n] = pt[off:off + n]
        off += n
    return bt


def _decode_strided(c: W.PagedCache, bt: torch.Tensor, lens=None):
    o = torch.full_like(c.q, float("nan"))
    fa.fa_decode_paged_strided(c.q, c.k_pages, c.v_pages, bt.cuda(),
                               c.seq_lens if lens is None else lens, c.page_size, o=o)
    return o


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("H,H_kv", [(4, 4), (8, 2)])
def test_decode_strided_small_full_compare(d, H, H_kv):
    lens = [1, 255, 257, 1000, 0, 4103]
    c = W.paged_inputs(len(lens), H, d, lens, seed=120 + H + d, device="cpu", H_kv=H_kv)
    bt = _block_table(c, 20)
    o = _decode_strided(_on_gpu(c), bt)
    assert fa.fa_get_device_error() == fa.FA_OK  # no padding entry was read
    o_ref, _ = oracle.decode_paged_strided(c.q, c.k_pages, c.v_pages, bt, c.seq_lens, PS)
    assert torch.all(o[4] == 0)
    assert_o_close(to64(o), o_ref, f"decode strided d={d} H={H} H_kv={H_kv}")


@pytest.mark.parametrize("H,H_kv", [(4, 4), (8, 2)])
def test_decode_strided_equals_packed_bitwise(H, H_kv):
    """The block table is packed on the device, then the same decode runs."""
    lens = [700, 3, 2049, 256]
    c = _on_gpu(W.paged_inputs(len(lens), H, 128, lens, seed=130 + H, device="cpu", H_kv=H_kv))
    o1 = _decode_strided(c, _block_table(c, 9))
    assert fa.fa_get_device_error() == fa.FA_OK
    assert torch.equal(o1, _decode_gqa(c))


def test_decode_strided_row_overflow_reported_and_cut():
    """A length past its row is reported; the sequence is decoded over the
    row's pages only (entries of the next row are not read)."""
    lens = [600, 1024]  # 3 pages, 4 full pages
    c = _on_gpu(W.paged_inputs(len(lens), 4, 128, lens, seed=140, device="cpu"))
    bt = _block_table(c, 4)
    too_long = torch.tensor([600, 1500], dtype=torch.int32, device="cuda")
    o = _decode_strided(c, bt, too_long)
    assert fa.fa_get_device_error() == fa.FA_ERR_DEVICE_BAD_INPUT
    assert torch.equal(o, _decode_gqa(c))  # row 1 cut to its 4 pages = 1024 tokens
    neg = torch.tensor([600, -5], dtype=torch.int32, device="cuda")
    o = _decode_strided(c, bt, neg)
    assert fa.fa_get_device_error() == fa.FA_ERR_DEVICE_BAD_INPUT
    assert torch.all(o[1] == 0)


def test_decode_strided_workload_bitwise():
    """The paged-decode workload (64 sequences of 1K-32K tokens) through a
    block table of 128 pages per row equals the packed-table decode."""
    c = W.decode_workload_inputs(W.PAGED_DECODE, device="cuda")
    c = W.PagedCache(c.q, c.k_pages, c.v_pages, c.page_table.cuda(), c.seq_lens.cuda(),
                     c.page_size, c.pages_per_seq)
    o1 = _decode_strided(c, _block_table(c, 128))
    assert fa.fa_get_device_error() == fa.FA_OK
    assert torch.equal(o1, _decode(c))
