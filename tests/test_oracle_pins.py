"""Pins for the fp64 CPU oracle: it is checked against things other than
itself -- a hand-worked example, high-precision brute force, closed forms,
invariants and special cases -- chosen so that a plausible slip (a dropped
max subtraction, a transposed operand, a wrong index, a mask off by one,
a natural-log / log2 mix-up) fails at least one of them.

The definition pinned here is standard attention, page "Flash Attention
是什么：2026 最新原理、架构演进与实战详解" (ai.lansai.wang), section
核心工作机制; the causal switch is flash_attn_causal on the page
"为什么“Flash”突然成了AI圈的高频词" (lqnn.cn), section 3.3.
"""
import json
import math
import os

import mpmath
import numpy as np
import pytest

import oracle
from oracle import method

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TOL = 1e-12


def _num(x):
    if isinstance(x, str):
        return math.log(float(x[2:]))  # "lnK"
    return float(x)


def _rand(shape, seed, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


def _mp_attention(q, k, v, causal, scale):
    """Brute force at 50 significant digits, straight from the definition."""
    mpmath.mp.dps = 50
    N, d = q.shape
    o = np.zeros((N, v.shape[1]))
    lse = np.zeros(N)
    for i in range(N):
        js = range(i + 1) if causal else range(k.shape[0])
        s = [mpmath.mpf(scale) * mpmath.fsum(mpmath.mpf(float(q[i, c])) * mpmath.mpf(float(k[j, c]))
                                             for c in range(d)) for j in js]
        e = [mpmath.exp(x) for x in s]
        tot = mpmath.fsum(e)
        for c in range(v.shape[1]):
            o[i, c] = float(mpmath.fsum(e[t] * mpmath.mpf(float(v[j, c]))
                                        for t, j in enumerate(js)) / tot)
        lse[i] = float(mpmath.log(tot))
    return o, lse


def _att(q, k, v, causal, scale):
    o, lse = oracle.attention(q[None, None], k[None, None], v[None, None], causal, scale)
    return o[0, 0], lse[0, 0]


# -- hand-worked example -----------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_hand_worked_2x2(causal):
    g = json.load(open(os.path.join(GOLDEN, "hand_worked_2x2.json")))
    q = np.array([[_num(x) for x in r] for r in g["q"]])
    k = np.array(g["k"], float)
    v = np.array(g["v"], float)
    exp = g["causal" if causal else "noncausal"]
    o, lse = _att(q, k, v, causal, g["scale"])
    np.testing.assert_allclose(o, np.array(exp["o"], float), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, [_num(x) for x in exp["lse"]], rtol=0, atol=1e-14)


# -- brute force at high precision -------------------------------------------

@pytest.mark.parametrize("N,d,causal", [(1, 1, False), (3, 2, True), (5, 4, False),
                                        (7, 8, True), (16, 8, False), (16, 5, True)])
def test_brute_force_mpmath(N, d, causal):
    q = _rand((N, d), 10 + N)
    k = _rand((N, d), 20 + N)
    v = _rand((N, d + 1), 30 + N)  # dv != d catches a q/v shape mix-up
    v2 = v[:, :d]
    scale = 0.37 + 0.1 * d
    o, lse = _att(q, k, v2, causal, scale)
    ob, lseb = _mp_attention(q, k, v2, causal, scale)
    np.testing.assert_allclose(o, ob, rtol=0, atol=TOL)
    np.testing.assert_allclose(lse, lseb, rtol=0, atol=TOL)


def test_brute_force_nonsquare_values_catch_transpose():
    # Q K^T differs from K Q^T here; a transposed operand changes the output
    N, d = 6, 3
    q = _rand((N, d), 1)
    k = _rand((N, d), 2) * 3.0
    v = _rand((N, d), 3)
    o, _ = _att(q, k, v, False, 1.0)
    ob, _ = _mp_attention(q, k, v, False, 1.0)
    ot, _ = _mp_attention(k, q, v, False, 1.0)
    np.testing.assert_allclose(o, ob, atol=TOL)
    assert np.abs(o - ot).max() > 1e-3


# -- invariants ---------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows_sum_to_one(causal):
    N, d = 33, 8
    q, k = _rand((N, d), 4), _rand((N, d), 5)
    p = oracle.probs(q, k, causal, 1 / math.sqrt(d))
    np.testing.assert_allclose(p.sum(axis=1), np.ones(N), atol=TOL)
    assert (p >= 0).all()
    if causal:
        assert np.all(np.triu(p, 1) == 0.0)
        assert np.all(np.diag(p) > 0)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_returns_v(causal):
    N, d = 40, 16
    q, k = _rand((N, d), 6, 2.0), _rand((N, d), 7, 2.0)
    c = _rand((d,), 8)
    v = np.tile(c, (N, 1))
    o, _ = _att(q, k, v, causal, 0.5)
    np.testing.assert_allclose(o, np.tile(c, (N, 1)), atol=TOL)


def test_causal_row0_is_v0():
    N, d = 21, 8
    q, k, v = _rand((N, d), 9), _rand((N, d), 10), _rand((N, d), 11)
    scale = 0.3
    o, lse = _att(q, k, v, True, scale)
    np.testing.assert_allclose(o[0], v[0], atol=TOL)
    assert abs(lse[0] - scale * float(q[0] @ k[0])) < TOL


def test_causal_last_row_equals_noncausal_last_row():
    N, d = 19, 4
    q, k, v = _rand((N, d), 12), _rand((N, d), 13), _rand((N, d), 14)
    oc, lc = _att(q, k, v, True, 0.7)
    on, ln = _att(q, k, v, False, 0.7)
    np.testing.assert_allclose(oc[-1], on[-1], atol=TOL)
    assert abs(lc[-1] - ln[-1]) < TOL
    # and the rows before it differ (the mask does something)
    assert np.abs(oc[:-1] - on[:-1]).max() > 1e-3


def test_v_linearity():
    N, d = 25, 8
    q, k = _rand((N, d), 15), _rand((N, d), 16)
    v1, v2 = _rand((N, d), 17), _rand((N, d), 18)
    a, b = 1.7, -0.4
    o1, _ = _att(q, k, v1, True, 0.5)
    o2, _ = _att(q, k, v2, True, 0.5)
    o12, _ = _att(q, k, a * v1 + b * v2, True, 0.5)
    np.testing.assert_allclose(o12, a * o1 + b * o2, atol=1e-11)


def test_noncausal_key_permutation_invariance():
    N, d = 30, 8
    q, k, v = _rand((N, d), 19), _rand((N, d), 20), _rand((N, d), 21)
    perm = np.random.default_rng(22).permutation(N)
    o, lse = _att(q, k, v, False, 0.4)
    # permute keys and values jointly: unchanged
    op, lsep = _att(q, k[perm], v[perm], False, 0.4)
    np.testing.assert_allclose(op, o, atol=TOL)
    np.testing.assert_allclose(lsep, lse, atol=TOL)
    # permute values only: changed (catches using the wrong index for V)
    ow, _ = _att(q, k, v[perm], False, 0.4)
    assert np.abs(ow - o).max() > 1e-3


@pytest.mark.parametrize("shift", [3.0, 800.0])
def test_score_shift_moves_lse_only(shift):
    """Adding a constant c to every score of a row leaves o unchanged and adds
    c to the log-sum-exp.  The constant enters through an extra feature:
    q' = [q, 1], k' = [k, c/scale].  c = 800 overflows exp() unless the row
    max is subtracted first."""
    N, d = 17, 8
    scale = 0.25
    q, k, v = _rand((N, d), 23), _rand((N, d), 24), _rand((N, d), 25)
    q2 = np.concatenate([q, np.ones((N, 1))], axis=1)
    k2 = np.concatenate([k, np.full((N, 1), shift / scale)], axis=1)
    for causal in (False, True):
        o, lse = _att(q, k, v, causal, scale)
        o2, lse2 = _att(q2, k2, v, causal, scale)
        assert np.all(np.isfinite(o2))
        np.testing.assert_allclose(o2, o, atol=1e-10)
        np.testing.assert_allclose(lse2, lse + shift, rtol=0, atol=1e-9)


# -- closed forms -------------------------------------------------------------

def test_zero_query_closed_form():
    N, d = 37, 8
    q = np.zeros((N, d))
    k, v = _rand((N, d), 26), _rand((N, d), 27)
    o, lse = _att(q, k, v, False, 1.0)
    np.testing.assert_allclose(o, np.tile(v.mean(axis=0), (N, 1)), atol=TOL)
    np.testing.assert_allclose(lse, np.full(N, math.log(N)), atol=TOL)
    oc, lsec = _att(q, k, v, True, 1.0)
    prefix_mean = np.cumsum(v, axis=0) / np.arange(1, N + 1)[:, None]
    np.testing.assert_allclose(oc, prefix_mean, atol=TOL)
    np.testing.assert_allclose(lsec, np.log(np.arange(1, N + 1)), atol=TOL)


def test_large_scale_is_hard_argmax():
    N, d = 12, 6
    q, k, v = _rand((N, d), 28), _rand((N, d), 29), _rand((N, d), 30)
    scale = 1e4
    o, lse = _att(q, k, v, False, scale)
    s = q @ k.T
    j = s.argmax(axis=1)
    np.testing.assert_allclose(o, v[j], atol=1e-9)
    np.testing.assert_allclose(lse, scale * s.max(axis=1), rtol=1e-12)


def test_lse_is_natural_log():
    # two equal scores: lse = s + ln 2 (a log2 slip would give s + 1)
    q = np.array([[1.0, 0.0], [1.0, 0.0]])
    k = np.array([[2.0, 0.0], [2.0, 0.0]])
    v = np.eye(2)
    _, lse = _att(q, k, v, False, 1.0)
    assert abs(lse[0] - (2.0 + math.log(2.0))) < 1e-15
    assert abs(lse[1] - (2.0 + math.log(2.0))) < 1e-15


def test_row_subset_matches_full():
    B, H, N, d = 2, 3, 50, 8
    q, k, v = _rand((B, H, N, d), 31), _rand((B, H, N, d), 32), _rand((B, H, N, d), 33)
    o, lse = oracle.attention(q, k, v, True, 0.3)
    rows = np.array([0, 7, 49, 50, 149, 299])
    os_, ls = oracle.attention(q, k, v, True, 0.3, rows=rows)
    fo, fl = o.reshape(-1, d), lse.reshape(-1)
    np.testing.assert_array_equal(os_.reshape(-1, d)[rows], fo[rows])
    np.testing.assert_array_equal(ls.reshape(-1)[rows], fl[rows])
    assert np.isnan(ls.reshape(-1)[1])


def test_batch_heads_are_independent():
    B, H, N, d = 2, 2, 9, 4
    q, k, v = _rand((B, H, N, d), 34), _rand((B, H, N, d), 35), _rand((B, H, N, d), 36)
    o, lse = oracle.attention(q, k, v, True, 0.5)
    for b in range(B):
        for h in range(H):
            ob, lb = _mp_attention(q[b, h], k[b, h], v[b, h], True, 0.5)
            np.testing.assert_allclose(o[b, h], ob, atol=TOL)
            np.testing.assert_allclose(lse[b, h], lb, atol=TOL)


# -- the method's steps reach the definition ---------------------------------

@pytest.mark.parametrize("block", [1, 7, 64, 128, 200])
@pytest.mark.parametrize("causal", [False, True])
def test_online_softmax_equals_two_pass(block, causal):
    N, d = 200, 16
    q, k, v = _rand((N, d), 40, 2.0), _rand((N, d), 41, 2.0), _rand((N, d), 42)
    o, lse = _att(q, k, v, causal, 1 / math.sqrt(d))
    oo, lo = method.online_attention(q, k, v, causal, 1 / math.sqrt(d), block)
    np.testing.assert_allclose(oo, o, rtol=0, atol=TOL)
    np.testing.assert_allclose(lo, lse, rtol=0, atol=TOL)


def test_online_softmax_without_correction_is_wrong():
    """Planted slip on the CPU: dropping the correction of earlier partial
    results (alpha = 1) changes the answer, so the test above is sensitive."""
    N, d = 64, 8
    q, k, v = _rand((N, d), 43, 3.0), _rand((N, d), 44, 3.0), _rand((N, d), 45)
    o, _ = _att(q, k, v, False, 1.0)
    m = np.full(N, -np.inf)
    acc = np.zeros((N, d))
    l = np.zeros(N)
    for j0 in range(0, N, 8):
        x = q @ k[j0:j0 + 8].T
        m = np.maximum(m, x.max(axis=1))
        p = np.exp(x - m[:, None])
        l = l + p.sum(axis=1)
        acc = acc + p @ v[j0:j0 + 8]
    assert np.abs(acc / l[:, None] - o).max() > 1e-3


@pytest.mark.parametrize("nsplit", [1, 2, 3, 8, 40])
def test_split_merge_equals_unsplit(nsplit):
    N, d = 300, 16
    rng = np.random.default_rng(50 + nsplit)
    q, k, v = rng.standard_normal(d) * 2, rng.standard_normal((N, d)) * 2, rng.standard_normal((N, d))
    cuts = sorted(rng.integers(0, N + 1, size=nsplit - 1).tolist())
    edges = [0] + cuts + [N]
    bounds = list(zip(edges[:-1], edges[1:]))
    if nsplit >= 3:
        bounds.append((N, N))  # an empty split must carry no weight
    o, lse = method.split_merge_attention(q, k, v, 1 / math.sqrt(d), bounds)
    # the plain definition for this one query: every row of the tiled query
    # block is the same row
    ref_o, ref_l = _att(np.tile(q, (N, 1)), k, v, False, 1 / math.sqrt(d))
    np.testing.assert_allclose(o, ref_o[0], atol=TOL)
    assert abs(lse - ref_l[0]) < TOL


# -- variable length ----------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equals_per_sequence(causal):
    lens = [5, 1, 17, 9]
    H, d = 3, 8
    total = sum(lens)
    q, k, v = _rand((total, H, d), 60), _rand((total, H, d), 61), _rand((total, H, d), 62)
    cu = np.concatenate([[0], np.cumsum(lens)])
    o, lse = oracle.attention_varlen(q, k, v, cu, causal, 0.35)
    for b, L in enumerate(lens):
        s0 = cu[b]
        for h in range(H):
            ob, lb = _mp_attention(q[s0:s0 + L, h], k[s0:s0 + L, h], v[s0:s0 + L, h], causal, 0.35)
            np.testing.assert_allclose(o[s0:s0 + L, h], ob, atol=TOL)
            np.testing.assert_allclose(lse[h, s0:s0 + L], lb, atol=TOL)


def test_varlen_row_subset_matches_full():
    lens = [4, 11, 6]
    H, d = 2, 4
    total = sum(lens)
    q, k, v = _rand((total, H, d), 63), _rand((total, H, d), 64), _rand((total, H, d), 65)
    cu = np.concatenate([[0], np.cumsum(lens)])
    o, lse = oracle.attention_varlen(q, k, v, cu, True, 0.5)
    rows = np.array([0, 3, 4, 14, 15, 20, 21 + 14])
    o2, l2 = oracle.attention_varlen(q, k, v, cu, True, 0.5, rows=rows)
    for r in rows:
        h, g = divmod(int(r), total)
        np.testing.assert_array_equal(o2[g, h], o[g, h])
        assert l2[h, g] == lse[h, g]


# -- paged gather and decode --------------------------------------------------

def _append_simulation(seqs, H, d, page_size, n_pool, seed):
    """Build a paged cache the way a serving loop fills it: tokens arrive one
    at a time per sequence (round robin); a sequence whose current page is
    full takes a fresh page from a shuffled free list (page "“Flash”不是那个
    被时代淘汰的插件", 0539edu.com, section 2: pages come from a fixed pool,
    a new token goes to a page allocated from the pool).  Returns the pool,
    the packed page table and the lengths."""
    rng = np.random.default_rng(seed)
    free = list(rng.permutation(n_pool))
    pool = np.full((n_pool, H, page_size, d), np.nan)
    owned = [[] for _ in seqs]
    fill = [page_size for _ in seqs]  # current page full -> allocate on first token
    pos = [0 for _ in seqs]
    active = True
    while active:
        active = False
        for b, x in enumerate(seqs):
            if pos[b] >= x.shape[0]:
                continue
            active = True
            if fill[b] == page_size:
                owned[b].append(free.pop())
                fill[b] = 0
            pool[owned[b][-1], :, fill[b], :] = x[pos[b]]
            fill[b] += 1
            pos[b] += 1
    table = np.array([p for o in owned for p in o], dtype=np.int64)
    return pool, table, np.array([x.shape[0] for x in seqs], dtype=np.int64)


@pytest.mark.parametrize("page_size", [4, 256])
def test_gather_inverts_append(page_size):
    H, d = 2, 3
    lens = [1, page_size, page_size + 1, 3 * page_size - 1, 0, 2]
    seqs = [_rand((L, H, d), 70 + i) for i, L in enumerate(lens)]
    n_pool = sum((L + page_size - 1) // page_size for L in lens) + 3  # spare pages
    pool, table, sl = _append_simulation(seqs, H, d, page_size, n_pool, 71)
    out = oracle.gather_paged(pool, table, sl, page_size)
    np.testing.assert_array_equal(out, np.concatenate(seqs, axis=0))


def test_decode_equals_attention_over_gathered_cache():
    H, d, page_size = 3, 8, 4
    lens = [1, 4, 5, 13]
    kseqs = [_rand((L, H, d), 80 + i) for i, L in enumerate(lens)]
    vseqs = [_rand((L, H, d), 90 + i) for i, L in enumerate(lens)]
    n_pool = sum((L + page_size - 1) // page_size for L in lens)
    kpool, table, sl = _append_simulation(kseqs, H, d, page_size, n_pool, 81)
    vpool, table2, _ = _append_simulation(vseqs, H, d, page_size, n_pool, 81)
    assert np.array_equal(table, table2)
    q = _rand((len(lens), H, d), 82)
    o, lse = oracle.decode_paged(q, kpool, vpool, table, sl, page_size)
    assert np.all(np.isfinite(o))  # the NaN-filled spare slots were never read
    for b, L in enumerate(lens):
        for h in range(H):
            ob, lb = _mp_attention(q[b, h][None], kseqs[b][:, h], vseqs[b][:, h], False,
                                   1 / math.sqrt(d))
            np.testing.assert_allclose(o[b, h], ob[0], atol=TOL)
            assert abs(lse[b, h] - lb[0]) < TOL


def test_decode_empty_sequence_gives_zero():
    H, d, page_size = 2, 4, 4
    kpool = _rand((2, H, page_size, d), 83)
    vpool = _rand((2, H, page_size, d), 84)
    q = _rand((2, H, d), 85)
    o, lse = oracle.decode_paged(q, kpool, vpool, np.array([1, 0]), np.array([0, 5]), page_size)
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(np.isfinite(o[1]))


def test_decode_is_last_causal_row():
    """Decode of the last token equals the last row of causal attention over
    the same (gathered) keys -- the tie between the two entry points."""
    H, d, page_size = 2, 8, 4
    L = 11
    qs, ks, vs = _rand((L, H, d), 86), _rand((L, H, d), 87), _rand((L, H, d), 88)
    n_pool = (L + page_size - 1) // page_size
    kpool, table, sl = _append_simulation([ks], H, d, page_size, n_pool, 89)
    vpool, _, _ = _append_simulation([vs], H, d, page_size, n_pool, 89)
    o, lse = oracle.decode_paged(qs[-1][None], kpool, vpool, table, sl, page_size)
    oc, lc = oracle.attention(qs.transpose(1, 0, 2)[None], ks.transpose(1, 0, 2)[None],
                              vs.transpose(1, 0, 2)[None], True, 1 / math.sqrt(d))
    np.testing.assert_allclose(o[0], oc[0, :, -1], atol=TOL)
    np.testing.assert_allclose(lse[0], lc[0, :, -1], atol=TOL)


def test_bf16_inputs_are_upcast_exactly():
    torch = pytest.importorskip("torch")
    x = torch.randn(4, 8, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    q = x[None, None]
    o, _ = oracle.attention(q, q, q, False, 0.5)
    o2, _ = oracle.attention(x.float().double().numpy()[None, None],
                             x.float().double().numpy()[None, None],
                             x.float().double().numpy()[None, None], False, 0.5)
    np.testing.assert_array_equal(o, o2)


# -- grouped-query attention (MQA/GQA: page "Flash Attention 是什么",
#    section 进阶学习路径, item 4) --------------------------------------------

@pytest.mark.parametrize("H,Hkv,causal", [(4, 2, True), (6, 3, False), (4, 1, True)])
def test_gqa_brute_force_mpmath(H, Hkv, causal):
    """Query head h against K/V head h // (H // Hkv), brute force per head;
    a mapping by h % Hkv (the plausible slip) fails the (4, 2) and (6, 3)
    cases, where the two mappings differ."""
    N, d = 6, 4
    q, k, v = _rand((1, H, N, d), 130), _rand((1, Hkv, N, d), 131), _rand((1, Hkv, N, d), 132)
    o, lse = oracle.attention_gqa(q, k, v, causal, 0.6)
    g = H // Hkv
    for h in range(H):
        ob, lb = _mp_attention(q[0, h], k[0, h // g], v[0, h // g], causal, 0.6)
        np.testing.assert_allclose(o[0, h], ob, atol=TOL)
        np.testing.assert_allclose(lse[0, h], lb, atol=TOL)


def test_gqa_equals_attention_with_repeated_heads():
    """GQA is ordinary attention after repeating each K/V head H // Hkv times
    (np.repeat puts copies of head g at h = g*G .. g*G + G - 1)."""
    B, H, Hkv, N, d = 2, 8, 2, 37, 8
    q, k, v = _rand((B, H, N, d), 133), _rand((B, Hkv, N, d), 134), _rand((B, Hkv, N, d), 135)
    for causal in (False, True):
        o, lse = oracle.attention_gqa(q, k, v, causal, 0.4)
        o2, l2 = oracle.attention(q, np.repeat(k, H // Hkv, axis=1),
                                  np.repeat(v, H // Hkv, axis=1), causal, 0.4)
        np.testing.assert_allclose(o, o2, atol=1e-15)
        np.testing.assert_allclose(lse, l2, atol=1e-15)


def test_mqa_zero_query_closed_form():
    """Hkv = 1, q = 0: every head of every row averages the shared V (prefix
    means when causal) and lse = ln(#keys)."""
    B, H, N, d = 1, 3, 9, 4
    k, v = _rand((B, 1, N, d), 136), _rand((B, 1, N, d), 137)
    q = np.zeros((B, H, N, d))
    o, lse = oracle.attention_gqa(q, k, v, True, 1.0)
    for h in range(H):
        for i in range(N):
            np.testing.assert_allclose(o[0, h, i], v[0, 0, :i + 1].mean(axis=0), atol=1e-14)
            assert abs(lse[0, h, i] - math.log(i + 1)) < 1e-14


def test_decode_gqa_equals_brute_force():
    H, Hkv, d, page_size = 6, 2, 8, 4
    lens = [1, 5, 12]
    kseqs = [_rand((L, Hkv, d), 140 + i) for i, L in enumerate(lens)]
    vseqs = [_rand((L, Hkv, d), 150 + i) for i, L in enumerate(lens)]
    n_pool = sum((L + page_size - 1) // page_size for L in lens) + 1
    kpool, table, sl = _append_simulation(kseqs, Hkv, d, page_size, n_pool, 141)
    vpool, _, _ = _append_simulation(vseqs, Hkv, d, page_size, n_pool, 141)
    q = _rand((len(lens), H, d), 142)
    o, lse = oracle.decode_paged_gqa(q, kpool, vpool, table, sl, page_size)
    assert np.all(np.isfinite(o))
    g = H // Hkv
    for b in range(len(lens)):
        for h in range(H):
            ob, lb = _mp_attention(q[b, h][None], kseqs[b][:, h // g], vseqs[b][:, h // g],
                                   False, 1 / math.sqrt(d))
            np.testing.assert_allclose(o[b, h], ob[0], atol=TOL)
            assert abs(lse[b, h] - lb[0]) < TOL


def _block_table(table, lens, page_size, max_pages, pad):
    """The packed table's pages laid out one row of max_pages per sequence,
    unused entries set to `pad`."""
    bt = np.full((len(lens), max_pages), pad, dtype=np.int64)
    off = 0
    for b, L in enumerate(lens):
        n = (L + page_size - 1) // page_size
        bt[b, :n] = table[off:off + n]
        off += n
    return bt


def test_decode_strided_equals_brute_force():
    """Decode through a block table: each sequence reads its own row; the
    padding entries point at a NaN-filled page and are never read."""
    H, Hkv, d, page_size = 4, 2, 8, 4
    lens = [1, 7, 12, 0, 4]
    kseqs = [_rand((L, Hkv, d), 160 + i) for i, L in enumerate(lens)]
    vseqs = [_rand((L, Hkv, d), 170 + i) for i, L in enumerate(lens)]
    n_pool = sum((L + page_size - 1) // page_size for L in lens) + 1  # last page: spare
    kpool, table, sl = _append_simulation(kseqs, Hkv, d, page_size, n_pool, 161)
    vpool, _, _ = _append_simulation(vseqs, Hkv, d, page_size, n_pool, 161)
    spare = sorted(set(range(n_pool)) - set(table.tolist()))[0]
    assert np.all(np.isnan(kpool[spare]))
    bt = _block_table(table, lens, page_size, 5, spare)
    q = _rand((len(lens), H, d), 162)
    o, lse = oracle.decode_paged_strided(q, kpool, vpool, bt, sl, page_size)
    g = H // Hkv
    for b, L in enumerate(lens):
        for h in range(H):
            if L == 0:
                assert np.all(o[b, h] == 0) and np.isneginf(lse[b, h])
                continue
            ob, lb = _mp_attention(q[b, h][None], kseqs[b][:, h // g], vseqs[b][:, h // g],
                                   False, 1 / math.sqrt(d))
            np.testing.assert_allclose(o[b, h], ob[0], atol=TOL)
            assert abs(lse[b, h] - lb[0]) < TOL


def test_decode_strided_equals_packed_decode():
    """The same pages listed one row per sequence or back to back give the same
    decode; a row index slip (reading row b+1) would not."""
    H, d, page_size = 3, 8, 4
    lens = [9, 3, 16]
    kseqs = [_rand((L, H, d), 180 + i) for i, L in enumerate(lens)]
    vseqs = [_rand((L, H, d), 190 + i) for i, L in enumerate(lens)]
    n_pool = sum((L + page_size - 1) // page_size for L in lens)
    kpool, table, sl = _append_simulation(kseqs, H, d, page_size, n_pool, 181)
    vpool, _, _ = _append_simulation(vseqs, H, d, page_size, n_pool, 181)
    bt = _block_table(table, lens, page_size, 6, 0)
    q = _rand((len(lens), H, d), 182)
    o1, l1 = oracle.decode_paged_strided(q, kpool, vpool, bt, sl, page_size)
    o2, l2 = oracle.decode_paged(q, kpool, vpool, table, sl, page_size)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)
    shifted = np.roll(bt, 1, axis=0)  # each sequence reading its neighbour's row
    o3, _ = oracle.decode_paged_strided(q, kpool, vpool, shifted, [3, 9, 3], page_size)
    assert np.abs(o3 - o1).max() > 1e-3


def test_decode_strided_rejects_a_row_overflow():
    H, d, page_size = 1, 4, 4
    pool = _rand((2, H, page_size, d), 195)
    with pytest.raises(RuntimeError):
        oracle.decode_paged_strided(_rand((1, H, d), 196), pool, pool, np.array([[0, 1]]),
                                    [9], page_size)


# -- appending to the paged cache and prefill through it (page
#    "“Flash”不是那个被时代淘汰的插件", 0539edu.com, section 2) ------------------

def _split_append(lens_before, n_new, Hkv, d, page_size, seed, table_seed=7):
    """A cache built by the append simulation for the first lens_before[b]
    tokens, with the pages for the n_new[b] further tokens already owned;
    returns (pool, table, lens_after, full token arrays per sequence).  Pools
    built with the same table_seed share their page table (K and V)."""
    lens_after = [a + n for a, n in zip(lens_before, n_new)]
    full = [_rand((L, Hkv, d), seed + i) for i, L in enumerate(lens_after)]
    n_pool = sum((L + page_size - 1) // page_size for L in lens_after) + 2
    pool, table, sl = _append_simulation(full, Hkv, d, page_size, n_pool, table_seed)
    return pool, table, sl, full


def test_append_then_gather_is_concatenation():
    """Writing the new rows over their slots restores exactly the tokens a
    one-at-a-time append produced: gather(append(...)) == concatenation."""
    Hkv, d, ps = 2, 3, 4
    lens_before, n_new = [0, 3, 4, 9, 5], [5, 1, 4, 0, 7]
    pool, table, sl, full = _split_append(lens_before, n_new, Hkv, d, ps, 160)
    # wipe the new tokens' slots, then append them back
    wiped = pool.copy()
    for b, (a, n) in enumerate(zip(lens_before, n_new)):
        off = sum((L + ps - 1) // ps for L in sl[:b])
        for pos in range(a, a + n):
            wiped[table[off + pos // ps], :, pos % ps, :] = np.nan
    new_rows = np.concatenate([full[b][a:] for b, a in enumerate(lens_before)], axis=0)
    cu = np.concatenate([[0], np.cumsum(n_new)])
    out = oracle.append_paged(wiped, table, sl, new_rows, cu, ps)
    np.testing.assert_array_equal(oracle.gather_paged(out, table, sl, ps),
                                  np.concatenate(full, axis=0))
    # slots nobody owns (NaN before) stay NaN: nothing else was written
    assert np.array_equal(np.isnan(out), np.isnan(pool))


def test_prefill_paged_brute_force_bottom_right_mask():
    """Queries are the LAST q_b positions: query i sees keys 0..L-q_b+i.  A
    top-left mask (keys 0..i) is the plausible slip and fails here."""
    H, Hkv, d, ps = 4, 2, 4, 4
    lens, nq = [7, 10, 3], [3, 10, 1]
    pool_k, table, sl, ks = _split_append([0, 0, 0], lens, Hkv, d, ps, 170)
    pool_v, table_v, _, vs = _split_append([0, 0, 0], lens, Hkv, d, ps, 170 + 50)
    assert np.array_equal(table, table_v)
    cu = np.concatenate([[0], np.cumsum(nq)])
    q = _rand((int(cu[-1]), H, d), 171)
    for causal in (True, False):
        o, lse = oracle.prefill_paged(q, pool_k, pool_v, table, sl, cu, ps, causal, 0.7)
        g = H // Hkv
        for b, (L, n) in enumerate(zip(lens, nq)):
            for i in range(n):
                keys = (L - n + i + 1) if causal else L
                for h in range(H):
                    ob, lb = _mp_attention(q[cu[b] + i, h][None], ks[b][:keys, h // g],
                                           vs[b][:keys, h // g], False, 0.7)
                    np.testing.assert_allclose(o[cu[b] + i, h], ob[0], atol=TOL)
                    assert abs(lse[h, cu[b] + i] - lb[0]) < TOL


def test_prefill_paged_one_query_is_decode():
    H, d, ps = 3, 8, 4
    lens = [1, 6, 13]
    pool_k, table, sl, _ = _split_append([0, 0, 0], lens, H, d, ps, 180)
    pool_v, table_v, _, _ = _split_append([0, 0, 0], lens, H, d, ps, 185)
    assert np.array_equal(table, table_v)
    q = _rand((3, H, d), 182)
    o, lse = oracle.prefill_paged(q, pool_k, pool_v, table, sl, np.arange(4), ps, True,
                                  1 / math.sqrt(d))
    od, ld = oracle.decode_paged(q, pool_k, pool_v, table, sl, ps)
    np.testing.assert_allclose(o, od, atol=1e-15)
    np.testing.assert_allclose(lse.T, ld, atol=1e-15)


def test_prefill_paged_whole_sequence_is_causal_varlen():
    """When every cached token is a query, prefill is causal attention over
    the (gathered) sequence."""
    H, d, ps = 2, 8, 4
    lens = [5, 12, 1]
    pool_k, table, sl, ks = _split_append([0, 0, 0], lens, H, d, ps, 190)
    pool_v, table_v, _, vs = _split_append([0, 0, 0], lens, H, d, ps, 195)
    assert np.array_equal(table, table_v)
    cu = np.concatenate([[0], np.cumsum(lens)])
    q = _rand((int(cu[-1]), H, d), 192)
    o, lse = oracle.prefill_paged(q, pool_k, pool_v, table, sl, cu, ps, True, 0.3)
    o2, l2 = oracle.attention_varlen(q, np.concatenate(ks), np.concatenate(vs), cu, True, 0.3)
    np.testing.assert_allclose(o, o2, atol=1e-15)
    np.testing.assert_allclose(lse, l2, atol=1e-15)


# -- rotary position embedding (page "“Flash”不是那个被时代淘汰的插件",
#    sections 2 and 3: RoPE fused into the kernel, sin/cos from a table) -----------

def test_rope_table_closed_form():
    from attn_fwd_04_b200 import workloads as W
    c, s = W.rope_tables(300, 8, base=10000.0)
    for p in (0, 1, 7, 299):
        for i in range(4):
            ang = p * 10000.0 ** (-2.0 * i / 8)
            assert abs(float(c[p, i]) - math.cos(ang)) < 1e-7
            assert abs(float(s[p, i]) - math.sin(ang)) < 1e-7
    assert bool((c[0] == 1).all()) and bool((s[0] == 0).all())


def test_rope_hand_worked_d2():
    """d = 2: the single pair rotates by angle p (theta_0 = base^0 = 1):
    (1, 0) -> (cos p, sin p) and (0, 1) -> (-sin p, cos p)."""
    from attn_fwd_04_b200 import workloads as W
    c, s = W.rope_tables(4, 2)
    x = np.array([[[1.0, 0.0], [1.0, 0.0], [0.0, 1.0], [0.0, 1.0]]])
    y = oracle.rope(x, c, s, bf16_round=False)
    for p in range(4):
        cp, sp = float(c[p, 0]), float(s[p, 0])
        exp = (cp, sp) if p < 2 else (-sp, cp)
        np.testing.assert_allclose(y[0, p], exp, atol=1e-15)
    assert abs(float(c[3, 0]) - math.cos(3.0)) < 1e-7


def test_rope_preserves_pair_norms_and_is_relative():
    from attn_fwd_04_b200 import workloads as W
    d, N = 16, 40
    c, s = W.rope_tables(N, d)
    q, k = _rand((1, N, d), 200), _rand((1, N, d), 201)
    qr, kr = oracle.rope(q, c, s, False), oracle.rope(k, c, s, False)
    h = d // 2
    # norms are kept up to cos^2 + sin^2 = 1 of the fp32 table entries (~1e-7)
    np.testing.assert_allclose(qr[..., :h] ** 2 + qr[..., h:] ** 2,
                               q[..., :h] ** 2 + q[..., h:] ** 2, rtol=1e-6)
    # the score of rotated q at p and k at p' depends on p - p' only (to the
    # fp32 precision of the tables): shift both positions by 5
    qs, ks = np.zeros_like(q), np.zeros_like(k)
    qs[0, 5:], ks[0, 5:] = q[0, :-5], k[0, :-5]
    qsr, ksr = oracle.rope(qs, c, s, False), oracle.rope(ks, c, s, False)
    for p, pp in ((3, 1), (10, 0), (20, 20)):
        a = qr[0, p] @ kr[0, pp]
        b = qsr[0, p + 5] @ ksr[0, pp + 5]
        assert abs(a - b) < 1e-5 * (1 + abs(a))


def _rne_bf16_py(x: float) -> float:
    """Nearest bf16 value (8 significant bits), ties to even: an independent
    restatement with Python's own rounding (round() on a float rounds half to
    even, and the power-of-two scalings are exact)."""
    if x == 0.0 or not math.isfinite(x):
        return x
    _, e = math.frexp(x)
    qe = max(e - 8, -133)
    return math.ldexp(round(math.ldexp(x, -qe)), qe)


def test_rope_bf16_is_the_rounded_rotation():
    """The bf16 variant is the exact fp64 rotation rounded once to the nearest
    bf16, element by element (checked against a Python rounding of the exact
    rotation), and every value it returns is a bf16 number."""
    from attn_fwd_04_b200 import workloads as W
    torch = pytest.importorskip("torch")
    d, N = 64, 50
    c, s = W.rope_tables(N, d)
    x = torch.randn((2, N, d), generator=torch.Generator().manual_seed(202)).to(torch.bfloat16)
    ex = oracle.rope(x, c, s, False)
    rb = oracle.rope(x, c, s, True)
    want = np.vectorize(_rne_bf16_py)(ex)
    np.testing.assert_array_equal(rb, want)
    assert np.all(np.abs(rb - ex) <= np.abs(ex) * 2.0 ** -8 + 1e-30)
    rt = torch.from_numpy(rb).float().to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(rt, rb)


def test_rope_bf16_hand_worked_d2():
    """d = 2, the table of base 10000 (theta_0 = 1): (1, 0) at position 1 turns
    to (cos 1, sin 1) = (0.540302..., 0.841470...).  In [1/2, 1) a bf16 step is
    2^-8: 0.540302 * 256 = 138.32 -> 138/256 = 0.5390625 and 0.841471 * 256 =
    215.42 -> 215/256 = 0.83984375.  (0, 1) at position 2 turns to
    (-sin 2, cos 2) = (-0.909297..., -0.416147...): -232.78 -> -233/256 =
    -0.91015625, and in [1/4, 1/2) the step is 2^-9: -213.07 -> -213/512 =
    -0.416015625."""
    from attn_fwd_04_b200 import workloads as W
    c, s = W.rope_tables(3, 2)
    x = np.array([[[0.0, 0.0], [1.0, 0.0], [0.0, 1.0]]])
    y = oracle.rope(x, c, s, bf16_round=True)
    np.testing.assert_array_equal(y[0, 1], [0.5390625, 0.83984375])
    np.testing.assert_array_equal(y[0, 2], [-0.91015625, -0.416015625])
    np.testing.assert_array_equal(y[0, 0], [0.0, 0.0])


def test_rope_bf16_ties_to_even():
    """A hand-made table (cos 1, sin 2^-8, exact in fp32) puts the rotation on
    bf16 midpoints: with (a, b) = (1, -1), a cos - b sin = 1 + 2^-8, halfway
    between 1 and 1 + 2^-7, goes to the even 1; with a = 1 + 2^-7 the value
    1 + 2^-7 + 2^-8 goes up to the even 1 + 2^-6.  The second component
    b cos + a sin = -1 + 2^-8 (resp. -1 + 2^-8 + 2^-15) is exact, resp. rounds
    to -1 + 2^-8."""
    cos_t = np.ones((2, 1), np.float32)
    sin_t = np.full((2, 1), 2.0 ** -8, np.float32)
    x = np.array([[[1.0, -1.0], [1.0 + 2.0 ** -7, -1.0]]])
    y = oracle.rope(x, cos_t, sin_t, bf16_round=True)
    np.testing.assert_array_equal(y[0, 0], [1.0, -1.0 + 2.0 ** -8])
    np.testing.assert_array_equal(y[0, 1], [1.0 + 2.0 ** -6, -1.0 + 2.0 ** -8])
    ex = oracle.rope(x, cos_t, sin_t, bf16_round=False)
    np.testing.assert_array_equal(ex[0, 0], [1.0 + 2.0 ** -8, -1.0 + 2.0 ** -8])


def test_rope_second_frequency_d4():
    """d = 4: component 1 pairs with component 3 and turns at
    theta_1 = base^(-1/2) = 0.01: e_1 at position p -> (0, cos, 0, sin)."""
    from attn_fwd_04_b200 import workloads as W
    c, s = W.rope_tables(60, 4)
    x = np.zeros((1, 60, 4))
    x[0, :, 1] = 1.0
    y = oracle.rope(x, c, s, bf16_round=False)
    for p in (0, 17, 59):
        np.testing.assert_allclose(y[0, p], [0.0, math.cos(0.01 * p), 0.0, math.sin(0.01 * p)],
                                   atol=1e-7)


# -- backward pass (the saved statistics serve it: page "Flash Attention 是什么",
#    section 核心工作机制, recomputation paragraph) -----------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_bwd_equals_finite_differences(causal):
    """dq, dk, dv are the gradients of L = sum(O * G) for the forward
    definition: central differences of L in every input entry."""
    B, H, N, d = 1, 2, 5, 3
    q, k, v = _rand((B, H, N, d), 210), _rand((B, H, N, d), 211), _rand((B, H, N, d), 212)
    g = _rand((B, H, N, d), 213)
    scale = 0.7
    dq, dk, dv = oracle.attention_bwd(q, k, v, g, causal, scale)

    def loss(q_, k_, v_):
        o, _ = oracle.attention(q_, k_, v_, causal, scale)
        return float(np.sum(o * g))

    h = 1e-5
    for x, grad, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[which], args_m[which] = xp, xm
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(grad, num, atol=1e-8)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_gqa_equals_finite_differences(causal):
    """Grouped K/V heads: a K/V entry feeds every query head of its group, so
    its gradient is the central difference of the loss summed over them (a
    gradient written to only the first query head's share would fail)."""
    B, H, Hkv, N, d = 1, 4, 2, 4, 3
    q, g = _rand((B, H, N, d), 230), _rand((B, H, N, d), 231)
    k, v = _rand((B, Hkv, N, d), 232), _rand((B, Hkv, N, d), 233)
    scale = 0.6
    dq, dk, dv = oracle.attention_bwd(q, k, v, g, causal, scale)

    def loss(q_, k_, v_):
        o, _ = oracle.attention_gqa(q_, k_, v_, causal, scale)
        return float(np.sum(o * g))

    h = 1e-5
    for x, grad, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[which], args_m[which] = xp, xm
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(grad, num, atol=1e-8)


def test_bwd_gqa_equals_repeated_heads_summed():
    """Attention with grouped heads is attention with each K/V head repeated
    for its query heads; dK, dV of a K/V head are then the sums of the
    repeated copies' gradients."""
    B, H, Hkv, N, d = 2, 6, 2, 9, 4
    q, g = _rand((B, H, N, d), 234), _rand((B, H, N, d), 235)
    k, v = _rand((B, Hkv, N, d), 236), _rand((B, Hkv, N, d), 237)
    dq, dk, dv = oracle.attention_bwd(q, k, v, g, True, 0.5)
    r = H // Hkv
    dq2, dk2, dv2 = oracle.attention_bwd(q, np.repeat(k, r, axis=1), np.repeat(v, r, axis=1), g,
                                         True, 0.5)
    np.testing.assert_allclose(dq, dq2, atol=1e-13)
    np.testing.assert_allclose(dk, dk2.reshape(B, Hkv, r, N, d).sum(axis=2), atol=1e-13)
    np.testing.assert_allclose(dv, dv2.reshape(B, Hkv, r, N, d).sum(axis=2), atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_varlen_equals_finite_differences(causal):
    """Packed sequences: central differences of L = sum(O * G) with O from the
    varlen forward definition; a gradient leaking across a sequence boundary
    (or a boundary read off by one row) would fail."""
    lens = [3, 1, 4]
    H, Hkv, d = 2, 1, 3
    total = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)])
    q, g = _rand((total, H, d), 240), _rand((total, H, d), 241)
    k, v = _rand((total, Hkv, d), 242), _rand((total, Hkv, d), 243)
    scale = 0.8
    dq, dk, dv = oracle.attention_bwd_varlen(q, k, v, g, cu, causal, scale)

    def loss(q_, k_, v_):
        o = np.zeros_like(q_)
        for b in range(len(lens)):
            s0, s1 = cu[b], cu[b + 1]
            ob, _ = oracle.attention_gqa(q_[s0:s1].transpose(1, 0, 2)[None],
                                         k_[s0:s1].transpose(1, 0, 2)[None],
                                         v_[s0:s1].transpose(1, 0, 2)[None], causal, scale)
            o[s0:s1] = ob[0].transpose(1, 0, 2)
        return float(np.sum(o * g))

    h = 1e-5
    for x, grad, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[which], args_m[which] = xp, xm
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(grad, num, atol=1e-8)


def test_bwd_varlen_single_sequence_is_fixed_length():
    N, H, d = 11, 2, 4
    q, k, v, g = (_rand((N, H, d), s) for s in (244, 245, 246, 247))
    dq, dk, dv = oracle.attention_bwd_varlen(q, k, v, g, [0, N], True, 0.5)
    t = lambda x: x.transpose(1, 0, 2)[None]
    rq, rk, rv = oracle.attention_bwd(t(q), t(k), t(v), t(g), True, 0.5)
    for a, b in ((dq, rq), (dk, rk), (dv, rv)):
        np.testing.assert_allclose(t(a), b, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_key_gradients_sum_to_zero(causal):
    """Each row of dS sums to zero (the softmax Jacobian annihilates
    constants), so sum_j dK_j = scale sum_i q_i sum_j dS_ij = 0; dropping the
    row term D_i breaks it."""
    q, k, v, g = (_rand((1, 1, 40, 8), s) for s in (214, 215, 216, 217))
    _, dk, _ = oracle.attention_bwd(q, k, v, g, causal, 0.4)
    assert np.all(np.abs(dk.sum(axis=2)) < 1e-12)


def test_bwd_zero_query_closed_form():
    """q = 0, non-causal: P is uniform, so dV_j = mean_i dO_i for every key j,
    and dQ_i = scale sum_j (1/N)(dO_i.v_j - dO_i.mean(v)) k_j."""
    N, d = 7, 4
    k, v, g = _rand((1, 1, N, d), 218), _rand((1, 1, N, d), 219), _rand((1, 1, N, d), 220)
    q = np.zeros((1, 1, N, d))
    dq, dk, dv = oracle.attention_bwd(q, k, v, g, False, 0.5)
    for j in range(N):
        np.testing.assert_allclose(dv[0, 0, j], g[0, 0].mean(axis=0), atol=1e-14)
    vbar = v[0, 0].mean(axis=0)
    for i in range(N):
        exp = 0.5 * sum((g[0, 0, i] @ (v[0, 0, j] - vbar)) / N * k[0, 0, j] for j in range(N))
        np.testing.assert_allclose(dq[0, 0, i], exp, atol=1e-14)
    np.testing.assert_allclose(dk, 0.0, atol=1e-15)  # q = 0 -> dK = scale dS^T q = 0
