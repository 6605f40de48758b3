"""GPU parity of the backward pass (fa_bwd) against the fp64 oracle's
gradients, through the C ABI.  The oracle's gradients are pinned by finite
differences of the forward definition (test_oracle_pins.py)."""
import math

import numpy as np
import pytest
import torch

import attn_fwd_04_b200 as fa
import oracle
from attn_fwd_04_b200 import workloads as W
from helpers import assert_grad_close, assert_lse_close, assert_o_close, to64

pytestmark = pytest.mark.gpu


def _bwd_gpu(q, k, v, g, causal, scale):
    qc, kc, vc, gc = q.cuda(), k.cuda(), v.cuda(), g.cuda()
    o, lse = fa.fa_fwd(qc, kc, vc, causal, scale)
    dq = torch.full_like(qc, float("nan"))
    dk = torch.full_like(qc, float("nan"))
    dv = torch.full_like(qc, float("nan"))
    fa.fa_bwd(qc, kc, vc, o, lse, gc, causal, scale, dq=dq, dk=dk, dv=dv)
    assert fa.fa_get_device_error() == fa.FA_OK
    return dq, dk, dv


def _grad_out(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


SHAPES = [(1, 1, 128, 64), (1, 2, 127, 128), (2, 2, 300, 64), (1, 1, 1, 128), (1, 2, 1000, 128),
          (1, 1, 129, 64)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_full_compare(shape, causal):
    B, H, N, d = shape
    q, k, v = W.custom_fwd_inputs(B, H, N, d, seed=700 + N + d)
    g = _grad_out((B, H, N, d), 701 + N)
    scale = 1 / math.sqrt(d)
    dq, dk, dv = _bwd_gpu(q, k, v, g, causal, scale)
    rq, rk, rv = oracle.attention_bwd(q, k, v, g, causal, scale)
    assert_grad_close(to64(dv), rv, f"dv {shape}")
    assert_grad_close(to64(dk), rk, f"dk {shape}")
    assert_grad_close(to64(dq), rq, f"dq {shape}")


def test_bwd_4k_two_heads():
    """Several 128-key blocks per head and many query tiles per block."""
    B, H, N, d = 1, 2, 4096, 128
    q, k, v = W.custom_fwd_inputs(B, H, N, d, seed=710)
    g = _grad_out((B, H, N, d), 711)
    scale = 1 / math.sqrt(d)
    dq, dk, dv = _bwd_gpu(q, k, v, g, True, scale)
    rq, rk, rv = oracle.attention_bwd(q, k, v, g, True, scale)
    assert_grad_close(to64(dv), rv, "dv 4k")
    assert_grad_close(to64(dk), rk, "dk 4k")
    assert_grad_close(to64(dq), rq, "dq 4k")


def test_bwd_linear_in_dout():
    """dk and dv are linear in the output gradient and scaling by 2 is exact
    in every step, so bwd(2 g) = 2 bwd(g) bit for bit (dq is summed with
    atomics in a varying order and is compared within the tolerance)."""
    q, k, v = W.custom_fwd_inputs(1, 2, 513, 64, seed=712)
    g = _grad_out((1, 2, 513, 64), 713)
    a = _bwd_gpu(q, k, v, g, True, 0.2)
    b = _bwd_gpu(q, k, v, (g.float() * 2).to(torch.bfloat16), True, 0.2)
    for x, y in zip(a[1:], b[1:]):
        assert torch.equal((x.float() * 2).to(torch.bfloat16), y)
    assert_grad_close(to64(b[0]), 2 * to64(a[0]), "dq linearity")


def _cpu_head(x, h):
    """Head h of a [B, heads, N, d] CUDA tensor as a [1, 1, N, d] CPU tensor."""
    return x[:, h:h + 1].cpu()


def test_bwd_long_prefill_one_head_full():
    """The long-prefill workload's backward pass (B=1 H=32 N=16384 d=128,
    causal) in the launch configuration the benchmark times: every gradient
    finite, and query head 13 (dq) with its K/V head (dk, dv) compared whole
    against the oracle (a head's gradients depend on that head alone)."""
    w = W.LONG_PREFILL
    q, k, v = W.fwd_inputs(w, device="cuda")
    scale = 1 / math.sqrt(w.d)
    o, lse = fa.fa_fwd(q, k, v, True, scale)
    g = torch.randn(q.shape, generator=torch.Generator(device="cuda").manual_seed(7),
                    device="cuda").to(torch.bfloat16)
    dq, dk, dv = fa.fa_bwd(q, k, v, o, lse, g, True, scale)
    assert fa.fa_get_device_error() == fa.FA_OK
    for t in (dq, dk, dv):
        assert bool(torch.isfinite(t).all())
    h = 13
    rq, rk, rv = oracle.attention_bwd(*(_cpu_head(t, h) for t in (q, k, v, g)), True, scale)
    assert_grad_close(to64(_cpu_head(dv, h)), rv, "dv head 13")
    assert_grad_close(to64(_cpu_head(dk, h)), rk, "dk head 13")
    assert_grad_close(to64(_cpu_head(dq, h)), rq, "dq head 13")


def test_bwd_gqa_long_prefill_one_group_full():
    """The grouped backward on the long-prefill shape with 8 K/V heads, as the
    benchmark runs it: K/V head 5 and its four query heads 20..23 compared
    whole against the oracle (dk, dv sum the group's four query heads)."""
    w = W.LONG_PREFILL
    H_kv, kv = 8, 5
    q, k, v = W.gqa_fwd_inputs(w.B, w.H, H_kv, w.N, w.d, seed=21, device="cuda")
    scale = 1 / math.sqrt(w.d)
    o, lse = fa.fa_fwd_gqa(q, k, v, True, scale)
    g = torch.randn(q.shape, generator=torch.Generator(device="cuda").manual_seed(7),
                    device="cuda").to(torch.bfloat16)
    dq, dk, dv = fa.fa_bwd_gqa(q, k, v, o, lse, g, True, scale)
    assert fa.fa_get_device_error() == fa.FA_OK
    G = w.H // H_kv
    hs = slice(kv * G, (kv + 1) * G)
    rq, rk, rv = oracle.attention_bwd(q[:, hs].cpu(), _cpu_head(k, kv), _cpu_head(v, kv),
                                      g[:, hs].cpu(), True, scale)
    assert_grad_close(to64(_cpu_head(dv, kv)), rv, "dv K/V head 5")
    assert_grad_close(to64(_cpu_head(dk, kv)), rk, "dk K/V head 5")
    assert_grad_close(to64(dq[:, hs].cpu()), rq, "dq query heads 20..23")


def test_bwd_varlen_workload_one_head_full():
    """The packed backward on the variable-length prefill workload (8
    sequences of 1024..8192 tokens, H=32, d=128, causal), as the benchmark
    runs it: head 30 of every sequence compared whole against the oracle."""
    wv = W.BATCHED_VARLEN
    q, k, v, cu = W.varlen_workload_inputs(wv, device="cuda")
    lens = (cu[1:] - cu[:-1]).tolist()
    scale = 1 / math.sqrt(wv.d)
    cud = cu.cuda()
    o, lse = fa.fa_fwd_varlen(q, k, v, cud, max(lens), wv.causal, scale)
    g = torch.randn(q.shape, generator=torch.Generator(device="cuda").manual_seed(8),
                    device="cuda").to(torch.bfloat16)
    dq, dk, dv = fa.fa_bwd_varlen(q, k, v, o, lse, g, cud, max(lens), wv.causal, scale)
    assert fa.fa_get_device_error() == fa.FA_OK
    for t in (dq, dk, dv):
        assert bool(torch.isfinite(t).all())
    h = 30
    sl = lambda x: x[:, h:h + 1].cpu()  # packed [total, heads, d] -> [total, 1, d]
    rq, rk, rv = oracle.attention_bwd_varlen(sl(q), sl(k), sl(v), sl(g), cu.cpu(), wv.causal,
                                             scale)
    assert_grad_close(to64(sl(dv)), rv, "dv head 30")
    assert_grad_close(to64(sl(dk)), rk, "dk head 30")
    assert_grad_close(to64(sl(dq)), rq, "dq head 30")


# -- grouped K/V heads (fa_bwd_gqa) -----------------------------------------------

def _bwd_gqa_gpu(q, k, v, g, causal, scale):
    qc, kc, vc, gc = q.cuda(), k.cuda(), v.cuda(), g.cuda()
    o, lse = fa.fa_fwd_gqa(qc, kc, vc, causal, scale)
    dq = torch.full_like(qc, float("nan"))
    dk = torch.full_like(kc, float("nan"))
    dv = torch.full_like(vc, float("nan"))
    fa.fa_bwd_gqa(qc, kc, vc, o, lse, gc, causal, scale, dq=dq, dk=dk, dv=dv)
    assert fa.fa_get_device_error() == fa.FA_OK
    return dq, dk, dv


# (B, H, H_kv, N, d): groups of 2, 4, 3 and multi-query
GQA_SHAPES = [(1, 4, 2, 300, 128), (2, 8, 2, 129, 64), (1, 6, 2, 1000, 128), (1, 4, 1, 257, 128)]


@pytest.mark.parametrize("shape", GQA_SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_gqa_full_compare(shape, causal):
    B, H, Hkv, N, d = shape
    q, k, v = W.gqa_fwd_inputs(B, H, Hkv, N, d, seed=800 + N + H, device="cpu")
    g = _grad_out((B, H, N, d), 801 + N)
    scale = 1 / math.sqrt(d)
    dq, dk, dv = _bwd_gqa_gpu(q, k, v, g, causal, scale)
    rq, rk, rv = oracle.attention_bwd(q, k, v, g, causal, scale)
    assert_grad_close(to64(dv), rv, f"dv {shape}")
    assert_grad_close(to64(dk), rk, f"dk {shape}")
    assert_grad_close(to64(dq), rq, f"dq {shape}")


def test_bwd_gqa_group1_equals_bwd():
    """With one query head per K/V head the grouped entry point is fa_bwd: dk
    and dv bit for bit (dq sums key blocks with atomics, so only closely)."""
    q, k, v = W.custom_fwd_inputs(1, 3, 700, 128, seed=810)
    g = _grad_out((1, 3, 700, 128), 811)
    a = _bwd_gpu(q, k, v, g, True, 0.1)
    b = _bwd_gqa_gpu(q, k, v, g, True, 0.1)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert_grad_close(to64(b[0]), to64(a[0]), "dq group 1")



# -- packed variable-length sequences (fa_bwd_varlen) --------------------------------

def _varlen(lengths, H, Hkv, d, seed):
    total = sum(lengths)
    cu = torch.tensor([0] + list(np.cumsum(lengths)), dtype=torch.int32)
    q, k, v = W.gqa_fwd_inputs(1, H, Hkv, total, d, seed=seed, device="cpu")
    # [1, heads, total, d] -> packed [total, heads, d]
    q, k, v = (x[0].transpose(0, 1).contiguous() for x in (q, k, v))
    g = _grad_out((total, H, d), seed + 1)
    return q, k, v, g, cu


def _bwd_varlen_gpu(q, k, v, g, cu, o, lse, causal, scale):
    dq = torch.full_like(q.cuda(), float("nan"))
    dk = torch.full_like(k.cuda(), float("nan"))
    dv = torch.full_like(v.cuda(), float("nan"))
    maxlen = int((cu[1:] - cu[:-1]).max())
    fa.fa_bwd_varlen(q.cuda(), k.cuda(), v.cuda(), o, lse, g.cuda(), cu.cuda(), maxlen, causal,
                     scale, dq=dq, dk=dk, dv=dv)
    assert fa.fa_get_device_error() == fa.FA_OK
    return dq, dk, dv


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_varlen_full_compare(d, causal):
    lengths = [300, 1, 129, 0, 513, 128]
    q, k, v, g, cu = _varlen(lengths, 2, 2, d, 820 + d)
    scale = 1 / math.sqrt(d)
    o, lse = fa.fa_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), max(lengths), causal,
                              scale)
    dq, dk, dv = _bwd_varlen_gpu(q, k, v, g, cu, o, lse, causal, scale)
    rq, rk, rv = oracle.attention_bwd_varlen(q, k, v, g, cu, causal, scale)
    assert_grad_close(to64(dv), rv, "dv varlen")
    assert_grad_close(to64(dk), rk, "dk varlen")
    assert_grad_close(to64(dq), rq, "dq varlen")


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_gqa_forward_and_backward(causal):
    """Grouped K/V heads over packed sequences: the forward pass against the
    oracle, then the backward pass from its o and lse."""
    lengths = [257, 40, 700]
    H, Hkv, d = 4, 2, 128
    q, k, v, g, cu = _varlen(lengths, H, Hkv, d, 830)
    scale = 1 / math.sqrt(d)
    o, lse = fa.fa_fwd_varlen_gqa(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), max(lengths), causal,
                                  scale)
    assert fa.fa_get_device_error() == fa.FA_OK
    for b in range(len(lengths)):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        ob, lb = oracle.attention_gqa(q[s0:s1].transpose(0, 1)[None], k[s0:s1].transpose(0, 1)[None],
                                      v[s0:s1].transpose(0, 1)[None], causal, scale)
        assert_o_close(to64(o[s0:s1].transpose(0, 1)), ob[0], f"fwd varlen gqa seq {b}")
        assert_lse_close(to64(lse[:, s0:s1]), lb[0], f"fwd varlen gqa seq {b}")
    dq, dk, dv = _bwd_varlen_gpu(q, k, v, g, cu, o, lse, causal, scale)
    rq, rk, rv = oracle.attention_bwd_varlen(q, k, v, g, cu, causal, scale)
    assert_grad_close(to64(dv), rv, "dv varlen gqa")
    assert_grad_close(to64(dk), rk, "dk varlen gqa")
    assert_grad_close(to64(dq), rq, "dq varlen gqa")


def test_bwd_varlen_one_sequence_equals_fixed():
    """A single packed sequence gives fa_bwd's dk, dv bit for bit."""
    N, H, d = 700, 2, 128
    q, k, v, g, cu = _varlen([N], H, H, d, 840)
    o, lse = fa.fa_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), N, True, 0.1)
    a = _bwd_varlen_gpu(q, k, v, g, cu, o, lse, True, 0.1)
    t = lambda x: x.transpose(0, 1)[None].contiguous()
    b = _bwd_gpu(t(q), t(k), t(v), t(g), True, 0.1)
    assert torch.equal(t(a[1]), b[1]) and torch.equal(t(a[2]), b[2])
    assert_grad_close(to64(t(a[0])), to64(b[0]), "dq one sequence")
