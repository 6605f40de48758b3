"""CPU restatements of the fused method's own steps, in fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring).  These are not the
oracle's definition of the result -- that is the plain two-pass attention in
attn_oracle.c -- but the steps the fused method takes, written out so that the
pin tests can show that the steps reach the definition exactly (up to
rounding), independently of any GPU code:

online_attention
    The single-pass online softmax of the page "Flash Attention 是什么：2026
    最新原理、架构演进与实战详解" (ai.lansai.wang), section "关键术语解析",
    item 4 (在线 Softmax): walking the keys block by block, keep the running
    max m and normaliser l,
        m_new = max(m_old, max(x_block))
        l_new = exp(m_old - m_new) * l_old + sum(exp(x_block - m_new)),
    and correct the partial output by the same factor exp(m_old - m_new)
    (section "核心工作机制": the earlier partial results are corrected).
    The division by the final normaliser happens once, after the last block,
    as the page "zwxr.cn/news/208202", section 3.1 (从“读内存”到“原地算”),
    describes: every block is folded in, then the result is scaled once by the
    final values.

split_merge_attention
    Split-K over the keys followed by a log-sum-exp merge (the paged-decode
    entry point splits a sequence's pages over several workers).  The pages do
    not describe the merge; it is the plain identity for combining softmax
    partial results:  with (o_s, lse_s) the normalised output and log-sum-exp
    of split s,  lse = M + ln sum_s exp(lse_s - M)  (M = max_s lse_s) and
    o = sum_s exp(lse_s - lse) o_s.  An empty split has lse_s = -inf and
    weight 0.
"""
import math

import numpy as np


def _scores(q, k, scale):
    return scale * (q @ k.T)


def online_attention(q, k, v, causal: bool, scale: float, block: int):
    """Single-query-block online softmax over key blocks of size `block`.

    q [Nq,d], k [Nk,d], v [Nk,d] fp64; causal means key j is admissible for
    query i when j <= i.  Returns (o [Nq,dv], lse [Nq]).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    nq, nk = q.shape[0], k.shape[0]
    m = np.full(nq, -np.inf)
    l = np.zeros(nq)
    acc = np.zeros((nq, v.shape[1]))
    rows = np.arange(nq)[:, None]
    for j0 in range(0, nk, block):
        j1 = min(nk, j0 + block)
        x = _scores(q, k[j0:j1], scale)
        if causal:
            cols = np.arange(j0, j1)[None, :]
            x = np.where(cols <= rows, x, -np.inf)
        m_blk = x.max(axis=1)
        m_new = np.maximum(m, m_blk)
        # rows that have seen no admissible key yet keep m = -inf; their
        # correction factor and block terms are zero
        seen = np.isfinite(m_new)
        alpha = np.where(seen, np.exp(np.where(seen, m - m_new, 0.0)), 0.0)
        alpha = np.where(np.isfinite(m), alpha, 0.0)
        p = np.where(seen[:, None], np.exp(x - np.where(seen, m_new, 0.0)[:, None]), 0.0)
        l = alpha * l + p.sum(axis=1)
        acc = alpha[:, None] * acc + p @ v[j0:j1]
        m = m_new
    with np.errstate(divide="ignore", invalid="ignore"):
        o = np.where((l > 0)[:, None], acc / np.where(l > 0, l, 1.0)[:, None], 0.0)
        lse = np.where(l > 0, m + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    return o, lse


def split_partials(q, k, v, scale: float, bounds):
    """Normalised partial results of one query row over key splits.

    q [d], k/v [Nk,d]; bounds is a list of (j0, j1) key ranges.  Returns a
    list of (o_s [d], lse_s) with lse_s = -inf for an empty range.
    """
    out = []
    for j0, j1 in bounds:
        if j1 <= j0:
            out.append((np.zeros(v.shape[1]), -math.inf))
            continue
        s = scale * (k[j0:j1] @ q)
        m = s.max()
        e = np.exp(s - m)
        l = e.sum()
        out.append(((e / l) @ v[j0:j1], m + math.log(l)))
    return out


def merge(partials):
    """Log-sum-exp merge of normalised partial results (see module doc)."""
    lses = np.array([p[1] for p in partials])
    if not np.any(np.isfinite(lses)):
        return np.zeros_like(partials[0][0]), -math.inf
    M = lses[np.isfinite(lses)].max()
    w = np.where(np.isfinite(lses), np.exp(lses - M), 0.0)
    lse = M + math.log(w.sum())
    o = np.zeros_like(partials[0][0])
    for (o_s, lse_s) in partials:
        if np.isfinite(lse_s):
            o = o + math.exp(lse_s - lse) * o_s
    return o, lse


def split_merge_attention(q, k, v, scale: float, bounds):
    """One query row attended over all keys via split + merge."""
    return merge(split_partials(q, k, v, scale, bounds))
