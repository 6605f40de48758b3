"""GPU parity of the fused forward pass (fa_fwd, fa_fwd_varlen) against the
fp64 CPU oracle, through the C ABI.

Small shapes are compared element by element over every output; the
full-size workloads (long prefill, batched prefill, varlen, 128K context) run
the same launch the benchmark times and are compared on sampled query rows
the oracle computes one by one.
"""
import math

import numpy as np
import pytest
import torch

import attn_fwd_04_b200 as fa
import oracle
from attn_fwd_04_b200 import workloads as W
from helpers import assert_lse_close, assert_o_close, assert_o_close_scaled, sample_rows, to64

pytestmark = pytest.mark.gpu


def _fwd_gpu(q, k, v, causal, scale):
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    B, H, N, d = q.shape
    o = torch.full_like(qc, float("nan"))
    lse = torch.full((B, H, N), float("nan"), device="cuda")
    fa.fa_fwd(qc, kc, vc, causal, scale, o=o, lse=lse)
    assert fa.fa_get_device_error() == fa.FA_OK
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
def test_tiny_workload(causal):
    w = W.TINY_CAUSAL if causal else W.TINY
    q, k, v, _fp32 = W.fwd_inputs(w, device="cpu")
    scale = 1 / math.sqrt(w.d)
    o, lse = _fwd_gpu(q, k, v, causal, scale)
    o_ref, lse_ref = oracle.attention(q, k, v, causal, scale)
    assert_o_close(to64(o), o_ref, w.name)
    assert_lse_close(to64(lse), lse_ref, w.name)


SHAPES = [(1, 1, 1, 64), (1, 1, 1, 128), (1, 2, 127, 128), (2, 3, 129, 64), (1, 2, 255, 128),
          (1, 1, 1000, 128), (2, 2, 384, 64), (1, 4, 1024, 128), (1, 2, 2049, 64)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("causal", [False, True])
def test_shapes_full_compare(shape, causal):
    B, H, N, d = shape
    q, k, v = W.custom_fwd_inputs(B, H, N, d, seed=100 + N + d)
    scale = 1 / math.sqrt(d)
    o, lse = _fwd_gpu(q, k, v, causal, scale)
    o_ref, lse_ref = oracle.attention(q, k, v, causal, scale)
    assert_o_close(to64(o), o_ref, str(shape))
    assert_lse_close(to64(lse), lse_ref, str(shape))


@pytest.fixture(params=[True, False], ids=["pairs", "single"])
def cta_pairs(request):
    """Run a d = 128 test on the CTA-pair kernel and on the single-CTA kernel."""
    prev = fa.fa_fwd_set_cta_pairs(request.param)
    yield request.param
    fa.fa_fwd_set_cta_pairs(prev)


# d = 128 lengths around the pair kernel's 512-row blocks: a pair whose odd
# CTA's tile starts past the end (1, 127, 257), whose second tile pair is
# empty (255, 256), partial blocks (384, 511, 513, 1000) and several heads,
# batches and grouped K/V heads
PAIR_SHAPES = [(1, 1, 1, 1), (1, 2, 2, 127), (1, 2, 2, 256), (2, 2, 1, 257), (1, 3, 3, 384),
               (1, 2, 2, 511), (1, 1, 1, 513), (1, 4, 2, 1000), (2, 2, 2, 1536)]


@pytest.mark.parametrize("shape", PAIR_SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("causal", [False, True])
def test_d128_both_kernels_full_compare(shape, causal, cta_pairs):
    B, H, Hkv, N = shape
    q, k, v = W.gqa_fwd_inputs(B, H, Hkv, N, 128, seed=900 + N + H, device="cpu")
    scale = 1 / math.sqrt(128)
    o, lse = _gqa_gpu(q, k, v, causal, scale)
    o_ref, lse_ref = oracle.attention_gqa(q, k, v, causal, scale)
    assert_o_close(to64(o), o_ref, f"{shape} pairs={cta_pairs}")
    assert_lse_close(to64(lse), lse_ref, f"{shape} pairs={cta_pairs}")


def test_pair_kernel_matches_single_kernel():
    """Both kernels take the same steps per query row (the pair kernel's extra
    fully masked step adds exact zeros), so they agree to the tolerance; the
    comparison also reports whether they agree bit for bit."""
    q, k, v = W.custom_fwd_inputs(1, 4, 1500, 128, seed=910)
    got = {}
    for pairs in (True, False):
        prev = fa.fa_fwd_set_cta_pairs(pairs)
        try:
            got[pairs] = _fwd_gpu(q, k, v, True, 0.09)
        finally:
            fa.fa_fwd_set_cta_pairs(prev)
    (o1, l1), (o2, l2) = got[True], got[False]
    assert_o_close(to64(o1), to64(o2), "pairs vs single")
    assert_lse_close(to64(l1), to64(l2), "pairs vs single")


@pytest.mark.parametrize("scale", [0.0, 0.02, 0.3, -0.1])
def test_other_scales(scale):
    q, k, v = W.custom_fwd_inputs(1, 2, 300, 128, seed=7)
    for causal in (False, True):
        o, lse = _fwd_gpu(q, k, v, causal, scale)
        o_ref, lse_ref = oracle.attention(q, k, v, causal, scale)
        assert_o_close(to64(o), o_ref, f"scale {scale}")
        assert_lse_close(to64(lse), lse_ref, f"scale {scale}")


def test_large_magnitude_scores_stay_finite():
    # scores up to ~+-200: the running max must be subtracted before exp.
    # V stays unit-scale so the absolute O tolerance keeps its meaning.
    q, k, _ = W.custom_fwd_inputs(1, 1, 512, 64, seed=8, std=4.0)
    _, _, v = W.custom_fwd_inputs(1, 1, 512, 64, seed=18)
    o, lse = _fwd_gpu(q, k, v, True, 1.0)
    o_ref, lse_ref = oracle.attention(q, k, v, True, 1.0)
    assert_o_close(to64(o), o_ref, "large scores")
    # lse magnitudes are in the hundreds here; compare relative to them
    np.testing.assert_allclose(to64(lse), lse_ref, rtol=2e-6, atol=1e-3)


@pytest.mark.parametrize("causal", [False, True])
def test_large_magnitude_values(causal):
    """Large scores (q, k with std 4) and large values (V with std 4, |V| up
    to ~18): O is compared with a max-abs gate relative to max |V|, the
    log-sum-exp at the usual absolute tolerance scaled by its magnitude."""
    q, k, v = W.custom_fwd_inputs(1, 2, 640, 128, seed=8, std=4.0)
    o, lse = _fwd_gpu(q, k, v, causal, 1 / math.sqrt(128))
    o_ref, lse_ref = oracle.attention(q, k, v, causal, 1 / math.sqrt(128))
    vmax = float(v.float().abs().max())
    assert vmax > 12
    assert_o_close_scaled(to64(o), o_ref, vmax, f"large |V| causal={causal}")
    np.testing.assert_allclose(to64(lse), lse_ref, rtol=2e-6, atol=1e-3)


def test_deterministic():
    q, k, v = W.custom_fwd_inputs(1, 3, 700, 128, seed=9)
    o1, l1 = _fwd_gpu(q, k, v, True, 0.1)
    o2, l2 = _fwd_gpu(q, k, v, True, 0.1)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def _sampled_parity(q, k, v, causal, scale, o, lse, rows_per_head, seed):
    """Oracle on sampled rows, one head at a time (keeps host memory small)."""
    B, H, N, d = q.shape
    g = torch.Generator().manual_seed(seed)
    pairs = [(int(b), int(h)) for b, h in zip(torch.randint(0, B, (8,), generator=g),
                                             torch.randint(0, H, (8,), generator=g))]
    pairs = sorted(set(pairs) | {(0, 0), (B - 1, H - 1)})
    got_o, ref_o, got_l, ref_l = [], [], [], []
    for (b, h) in pairs:
        rows = sample_rows(N, rows_per_head, seed + 31 * b + h)
        qh, kh, vh = q[b, h][None, None], k[b, h][None, None], v[b, h][None, None]
        o_ref, lse_ref = oracle.attention(qh, kh, vh, causal, scale, rows=rows)
        got_o.append(to64(o[b, h, rows]))
        ref_o.append(o_ref[0, 0, rows])
        got_l.append(to64(lse[b, h, rows]))
        ref_l.append(lse_ref[0, 0, rows])
    assert_o_close(np.concatenate(got_o), np.concatenate(ref_o), "sampled")
    assert_lse_close(np.concatenate(got_l), np.concatenate(ref_l), "sampled")


@pytest.mark.parametrize("w", [W.LONG_PREFILL, W.BATCHED], ids=lambda w: w.name)
def test_full_size_sampled(w):
    q, k, v = W.fwd_inputs(w, device="cuda")
    scale = 1 / math.sqrt(w.d)
    o, lse = fa.fa_fwd(q, k, v, w.causal, scale)
    assert fa.fa_get_device_error() == fa.FA_OK
    assert bool(torch.isfinite(o).all()) and bool(torch.isfinite(lse).all())
    _sampled_parity(q.cpu(), k.cpu(), v.cpu(), w.causal, scale, o.cpu(), lse.cpu(), 24, w.seed)


def test_ctx128k_sampled():
    """128K context: 256 query rows in total, seeded, across heads (the first
    and last row of head 0 always included); K/V of each head copied to the
    host one at a time."""
    w = W.CTX128K
    q, k, v = W.fwd_inputs(w, device="cuda")
    scale = 1 / math.sqrt(w.d)
    o, lse = fa.fa_fwd(q, k, v, w.causal, scale)
    assert fa.fa_get_device_error() == fa.FA_OK
    g = torch.Generator().manual_seed(4)
    hs = torch.randint(0, w.H, (254,), generator=g).tolist()
    rs = torch.randint(0, w.N, (254,), generator=g).tolist()
    picks = {}
    for h, r in [(0, 0), (0, w.N - 1)] + list(zip(hs, rs)):
        picks.setdefault(h, set()).add(r)
    got_o, ref_o, got_l, ref_l = [], [], [], []
    for h, rows in sorted(picks.items()):
        rows = sorted(rows)
        qh, kh, vh = q[0, h].cpu(), k[0, h].cpu(), v[0, h].cpu()
        o_ref, lse_ref = oracle.attention(qh[None, None], kh[None, None], vh[None, None],
                                          True, scale, rows=rows)
        got_o.append(to64(o[0, h, rows]))
        ref_o.append(o_ref[0, 0, rows])
        got_l.append(to64(lse[0, h, rows]))
        ref_l.append(lse_ref[0, 0, rows])
    assert_o_close(np.concatenate(got_o), np.concatenate(ref_o), w.name)
    assert_lse_close(np.concatenate(got_l), np.concatenate(ref_l), w.name)


# -- variable length -----------------------------------------------------------

def _varlen_gpu(q, k, v, cu, maxlen, causal, scale):
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    total, H, d = q.shape
    o = torch.full_like(qc, float("nan"))
    lse = torch.full((H, total), float("nan"), device="cuda")
    fa.fa_fwd_varlen(qc, kc, vc, cu.cuda(), maxlen, causal, scale, o=o, lse=lse)
    assert fa.fa_get_device_error() == fa.FA_OK
    return o, lse


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_varlen_small_full_compare(d, causal):
    lens = [1, 127, 128, 129, 300, 5, 256]
    q, k, v, cu = W.varlen_inputs(3, d, lens, seed=11)
    scale = 1 / math.sqrt(d)
    o, lse = _varlen_gpu(q, k, v, cu, max(lens), causal, scale)
    o_ref, lse_ref = oracle.attention_varlen(q, k, v, cu, causal, scale)
    assert_o_close(to64(o), o_ref, f"varlen d={d}")
    assert_lse_close(to64(lse), lse_ref, f"varlen d={d}")


def test_varlen_equals_fixed_per_sequence():
    """Each packed sequence gives bit-identical results to a fixed-length call
    on that sequence alone (same tiles, same arithmetic)."""
    lens = [200, 64, 513]
    H, d = 2, 128
    q, k, v, cu = W.varlen_inputs(H, d, lens, seed=12)
    o, lse = _varlen_gpu(q, k, v, cu, max(lens), True, 0.125)
    for b, L in enumerate(lens):
        s0 = int(cu[b])
        sl = slice(s0, s0 + L)
        qf = q[sl].permute(1, 0, 2).contiguous()[None]
        kf = k[sl].permute(1, 0, 2).contiguous()[None]
        vf = v[sl].permute(1, 0, 2).contiguous()[None]
        of, lf = _fwd_gpu(qf, kf, vf, True, 0.125)
        assert torch.equal(of[0].permute(1, 0, 2), o[sl])
        assert torch.equal(lf[0], lse[:, sl])


def test_varlen_workload_sampled():
    w = W.BATCHED_VARLEN
    q, k, v, cu = W.varlen_workload_inputs(w, device="cuda")
    lens = (cu[1:] - cu[:-1]).tolist()
    scale = 1 / math.sqrt(w.d)
    o, lse = fa.fa_fwd_varlen(q, k, v, cu.cuda(), max(lens), w.causal, scale)
    assert fa.fa_get_device_error() == fa.FA_OK
    total = q.shape[0]
    g = torch.Generator().manual_seed(w.seed)
    rows = []
    for b, L in enumerate(lens):
        s0 = int(cu[b])
        for r in {0, L - 1, min(127, L - 1), min(128, L - 1)} | set(torch.randint(0, L, (6,), generator=g).tolist()):
            h = int(torch.randint(0, w.H, (1,), generator=g))
            rows.append(h * total + s0 + r)
    rows = sorted(set(rows))
    o_ref, lse_ref = oracle.attention_varlen(q.cpu(), k.cpu(), v.cpu(), cu, True, scale, rows=rows)
    hs = [r // total for r in rows]
    gs = [r % total for r in rows]
    oc, lc = o.cpu(), lse.cpu()
    assert_o_close(np.stack([to64(oc[g_, h_]) for h_, g_ in zip(hs, gs)]),
                   np.stack([o_ref[g_, h_] for h_, g_ in zip(hs, gs)]), w.name)
    assert_lse_close(np.array([float(lc[h_, g_]) for h_, g_ in zip(hs, gs)]),
                     np.array([lse_ref[h_, g_] for h_, g_ in zip(hs, gs)]), w.name)


def test_bounded_wait_reports_timeout():
    assert fa.fa_get_device_error() == fa.FA_OK
    fa.fa_selftest_bounded_wait()
    assert fa.fa_get_device_error() == fa.FA_ERR_DEVICE_TIMEOUT
    assert fa.fa_get_device_error() == fa.FA_OK  # read clears it
    # the context is still usable afterwards
    q, k, v = W.custom_fwd_inputs(1, 1, 130, 64, seed=13)
    o, lse = _fwd_gpu(q, k, v, True, 0.125)
    o_ref, lse_ref = oracle.attention(q, k, v, True, 0.125)
    assert_o_close(to64(o), o_ref, "after timeout")


@pytest.mark.parametrize("withheld", [0, 3, 6])
def test_forward_kernel_stall_is_reported_and_recovered(withheld):
    """Failure detection inside the production forward kernel: one K/V copy
    (K of tile 0, V of tile 1, or K of tile 3) is never issued and every wait
    is bounded by 50 ms.  The stall comes back as FA_ERR_DEVICE_TIMEOUT (no
    trap, no fault), and a normal call on the same stream right after it
    computes correctly -- its CTAs allocate TMEM and use every barrier again,
    which they could not if the stalled CTAs had leaked them."""
    q, k, v = W.custom_fwd_inputs(1, 2, 1000, 128, seed=14)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    assert fa.fa_get_device_error() == fa.FA_OK
    fa.fa_selftest_fwd_stall(qc, kc, vc, withheld, 50_000)
    assert fa.fa_get_device_error() == fa.FA_ERR_DEVICE_TIMEOUT
    assert fa.fa_get_device_error() == fa.FA_OK
    o, lse = _fwd_gpu(q, k, v, True, 1 / math.sqrt(128))
    o_ref, lse_ref = oracle.attention(q, k, v, True, 1 / math.sqrt(128))
    assert_o_close(to64(o), o_ref, "after a stalled forward")
    assert_lse_close(to64(lse), lse_ref, "after a stalled forward")


# -- grouped-query attention (fa_fwd_gqa) ----------------------------------------

def _gqa_gpu(q, k, v, causal, scale):
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    B, H, N, d = q.shape
    o = torch.full_like(qc, float("nan"))
    lse = torch.full((B, H, N), float("nan"), device="cuda")
    fa.fa_fwd_gqa(qc, kc, vc, causal, scale, o=o, lse=lse)
    assert fa.fa_get_device_error() == fa.FA_OK
    return o, lse


# (B, H, H_kv, N, d): groups of 2, 3, 8, 1 (plain multi-head) and 4
GQA_SHAPES = [(1, 4, 2, 129, 128), (2, 6, 3, 300, 64), (1, 3, 1, 255, 128), (1, 8, 1, 1000, 64),
              (1, 2, 2, 127, 128), (2, 8, 4, 1, 64), (1, 16, 2, 2049, 128)]


@pytest.mark.parametrize("shape", GQA_SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_full_compare(shape, causal):
    B, H, Hkv, N, d = shape
    q, k, v = W.gqa_fwd_inputs(B, H, Hkv, N, d, seed=200 + N + H, device="cpu")
    scale = 1 / math.sqrt(d)
    o, lse = _gqa_gpu(q, k, v, causal, scale)
    o_ref, lse_ref = oracle.attention_gqa(q, k, v, causal, scale)
    assert_o_close(to64(o), o_ref, f"gqa {shape}")
    assert_lse_close(to64(lse), lse_ref, f"gqa {shape}")


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_equals_fwd_on_repeated_heads(causal):
    """A query head's rows are computed with the same tiles in the same order
    whether its K/V head is shared or repeated (fa_fwd): the results are
    bit-identical."""
    B, H, Hkv, N, d = 2, 8, 2, 700, 128
    q, k, v = W.gqa_fwd_inputs(B, H, Hkv, N, d, seed=17, device="cpu")
    o, lse = _gqa_gpu(q, k, v, causal, 0.1)
    g = H // Hkv
    o2, l2 = _fwd_gpu(q, k.repeat_interleave(g, dim=1), v.repeat_interleave(g, dim=1), causal, 0.1)
    assert torch.equal(o, o2) and torch.equal(lse, l2)


def test_gqa_long_prefill_sampled():
    """The long-prefill shape with 8 K/V heads for 32 query heads (groups of
    4), sampled rows against the oracle."""
    B, H, Hkv, N, d = 1, 32, 8, 16384, 128
    q, k, v = W.gqa_fwd_inputs(B, H, Hkv, N, d, seed=21, device="cuda")
    scale = 1 / math.sqrt(d)
    o, lse = fa.fa_fwd_gqa(q, k, v, True, scale)
    assert fa.fa_get_device_error() == fa.FA_OK
    qc, kc, vc, oc, lc = q.cpu(), k.cpu(), v.cpu(), o.cpu(), lse.cpu()
    got_o, ref_o, got_l, ref_l = [], [], [], []
    for h in (0, 1, 5, 30, 31):
        rows = sample_rows(N, 24, 500 + h)
        o_ref, lse_ref = oracle.attention_gqa(qc[:, h:h + 1], kc[:, h // 4:h // 4 + 1],
                                              vc[:, h // 4:h // 4 + 1], True, scale, rows=rows)
        got_o.append(to64(oc[0, h, rows]))
        ref_o.append(o_ref[0, 0, rows])
        got_l.append(to64(lc[0, h, rows]))
        ref_l.append(lse_ref[0, 0, rows])
    assert_o_close(np.concatenate(got_o), np.concatenate(ref_o), "gqa long prefill")
    assert_lse_close(np.concatenate(got_l), np.concatenate(ref_l), "gqa long prefill")


# -- rotary embedding fused into the forward pass (fa_fwd_rope) -------------------

def _rope_ref(q, k, v, c, s, causal, scale):
    """Oracle: rotate q and k (the exact rotation rounded once to bf16, the
    precision of the tensor-core inputs), then grouped-query attention in fp64."""
    qr = oracle.rope(q, c, s, bf16_round=True)
    kr = oracle.rope(k, c, s, bf16_round=True)
    return oracle.attention_gqa(qr, kr, v, causal, scale), qr, kr


ROPE_SHAPES = [(1, 2, 2, 300, 128), (2, 4, 2, 129, 64), (1, 2, 1, 1, 128), (1, 4, 4, 1000, 128),
               (1, 2, 2, 2049, 64)]


@pytest.mark.parametrize("shape", ROPE_SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("causal", [False, True])
def test_rope_full_compare(shape, causal):
    B, H, Hkv, N, d = shape
    q, k, v = W.gqa_fwd_inputs(B, H, Hkv, N, d, seed=400 + N + d, device="cpu")
    c, s = W.rope_tables(N + 17, d)
    scale = 1 / math.sqrt(d)
    o = torch.full_like(q.cuda(), float("nan"))
    lse = torch.full((B, H, N), float("nan"), device="cuda")
    fa.fa_fwd_rope(q.cuda(), k.cuda(), v.cuda(), c.cuda(), s.cuda(), causal, scale, o=o, lse=lse)
    assert fa.fa_get_device_error() == fa.FA_OK
    (o_ref, lse_ref), _, _ = _rope_ref(q, k, v, c, s, causal, scale)
    assert_o_close(to64(o), o_ref, f"rope {shape}")
    assert_lse_close(to64(lse), lse_ref, f"rope {shape}")


def _rope_torch_fp32(x, c, s):
    """The rotation in the library's own fp32 operation order (each product
    rounded to fp32, then the difference or sum, then bf16), written with
    plain PyTorch ops on the GPU.  A self-consistency aid, not the oracle."""
    h = x.shape[-1] // 2
    N = x.shape[-2]
    a, b = x[..., :h].float(), x[..., h:].float()
    cc, ss = c[:N].float(), s[:N].float()
    ra = a * cc - b * ss
    rb = b * cc + a * ss
    return torch.cat([ra, rb], dim=-1).to(torch.bfloat16).contiguous()


def test_rope_self_consistent_with_fp32_rotation():
    """GPU self-consistency, not an oracle check: the in-kernel rotation (Q in
    shared memory, K by the row kernel) gives exactly the bf16 values of the
    same fp32 formula evaluated by PyTorch on the GPU, so fa_fwd_rope equals
    fa_fwd_gqa on inputs pre-rotated that way, bit for bit."""
    B, H, Hkv, N, d = 1, 4, 2, 777, 128
    q, k, v = W.gqa_fwd_inputs(B, H, Hkv, N, d, seed=410, device="cpu")
    c, s = W.rope_tables(N, d)
    q, k, v, c, s = q.cuda(), k.cuda(), v.cuda(), c.cuda(), s.cuda()
    o, lse = fa.fa_fwd_rope(q, k, v, c, s, True, 0.1)
    qr, kr = _rope_torch_fp32(q, c, s), _rope_torch_fp32(k, c, s)
    prev = fa.fa_fwd_set_cta_pairs(False)  # the kernel fa_fwd_rope runs on (the default)
    try:
        o2, l2 = fa.fa_fwd_gqa(qr, kr, v, True, 0.1)
    finally:
        fa.fa_fwd_set_cta_pairs(prev)
    assert fa.fa_get_device_error() == fa.FA_OK
    assert torch.equal(o, o2) and torch.equal(lse, l2)


def test_rope_rotation_matches_oracle_rounding_almost_everywhere():
    """The fp32 rotation (library order) against the oracle's exactly rounded
    rotation: equal except where the fp32 rounding error crosses a bf16
    rounding boundary, where they differ by one bf16 step."""
    B, H, N, d = 1, 4, 2048, 128
    q = W.gqa_fwd_inputs(B, H, H, N, d, seed=411, device="cpu")[0]
    c, s = W.rope_tables(N, d)
    got = _rope_torch_fp32(q.cuda(), c.cuda(), s.cuda()).cpu().double().numpy()
    want = oracle.rope(q, c, s, True)
    diff = got != want
    assert diff.mean() < 1e-3, diff.mean()
    step = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(want[diff]), 1e-30))) - 7)
    assert np.all(np.abs(got[diff] - want[diff]) <= step * 1.0000001)


def test_rope_long_prefill_sampled():
    w = W.LONG_PREFILL
    q, k, v = W.fwd_inputs(w, device="cuda")
    c, s = W.rope_tables(w.N, w.d, device="cuda")
    scale = 1 / math.sqrt(w.d)
    o, lse = fa.fa_fwd_rope(q, k, v, c, s, True, scale)
    assert fa.fa_get_device_error() == fa.FA_OK
    cc, sc = c.cpu(), s.cpu()
    got_o, ref_o, got_l, ref_l = [], [], [], []
    for h in (0, 13, 31):
        rows = sample_rows(w.N, 24, 600 + h)
        qh, kh, vh = q[0, h].cpu()[None, None], k[0, h].cpu()[None, None], v[0, h].cpu()[None, None]
        qr, kr = oracle.rope(qh, cc, sc, True), oracle.rope(kh, cc, sc, True)
        o_ref, lse_ref = oracle.attention(qr, kr, vh, True, scale, rows=rows)
        got_o.append(to64(o[0, h, rows]))
        ref_o.append(o_ref[0, 0, rows])
        got_l.append(to64(lse[0, h, rows]))
        ref_l.append(lse_ref[0, 0, rows])
    assert_o_close(np.concatenate(got_o), np.concatenate(ref_o), "rope long prefill")
    assert_lse_close(np.concatenate(got_l), np.concatenate(ref_l), "rope long prefill")
