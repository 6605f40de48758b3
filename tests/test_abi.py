"""The C-ABI library without a GPU: it loads, exports every entry point the
header declares, names its status codes, and rejects bad arguments before
touching CUDA.  No compute call runs here."""
import ctypes
import os
import re

import pytest
import torch

import attn_fwd_04_b200 as fa
from attn_fwd_04_b200 import build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


@pytest.fixture(scope="module")
def L():
    fa_build.build()
    return fa.lib()


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"FA_API\s+[\w\s\*]*?\b(fa_\w+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert _declared() == sorted(fa.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in _declared():
        assert hasattr(L, name), name


def _prototypes():
    """name -> parameter kinds ('p' pointer or stream, 'i' integer, 'f' float)
    and the return kind, parsed from the header's FA_API declarations."""
    text = re.sub(r"/\*.*?\*/", " ", open(HEADER).read(), flags=re.S)
    out = {}
    for ret, name, params in re.findall(r"FA_API\s+([\w\s\*]*?)\s*\b(fa_\w+)\s*\(([^)]*)\)\s*;",
                                        text, flags=re.S):
        kinds = []
        for prm in (x.strip() for x in params.split(",")):
            if not prm or prm == "void":
                continue
            if "*" in prm or prm.startswith("fa_stream_t"):
                kinds.append("p")
            elif prm.split()[0] in ("float", "double"):
                kinds.append("f" if prm.split()[0] == "float" else "d")
            else:
                kinds.append("i")
        out[name] = (kinds, "p" if "*" in ret else "i")
    return out


def _kind(t):
    if t in (ctypes.c_void_p, ctypes.c_char_p) or issubclass(t, ctypes._Pointer):
        return "p"
    return {ctypes.c_int: "i", ctypes.c_float: "f", ctypes.c_double: "d"}[t]


def test_binding_argtypes_match_the_header(L):
    """Each binding's ctypes signature has the header prototype's parameter
    count and kinds, so a pointer never lands in an int slot (or a float in
    an int) when the header changes and the binding does not."""
    protos = _prototypes()
    assert sorted(protos) == _declared()
    for name, (kinds, ret) in protos.items():
        fn = getattr(L, name)
        assert [_kind(t) for t in fn.argtypes] == kinds, name
        assert _kind(fn.restype) == ret, name


def test_status_strings(L):
    codes = [fa.FA_OK, fa.FA_ERR_NULL, fa.FA_ERR_SHAPE, fa.FA_ERR_UNSUPPORTED, fa.FA_ERR_ALIGN,
             fa.FA_ERR_CUDA, fa.FA_ERR_DEVICE_TIMEOUT, fa.FA_ERR_NOMEM, fa.FA_ERR_DEVICE_BAD_INPUT]
    names = [fa.fa_status_str(c) for c in codes]
    assert names[0] == "FA_OK"
    assert len(set(names)) == len(names)
    assert fa.fa_status_str(12345) == "unknown fa status"
    assert fa.fa_version() == 100


def test_cta_pair_setting_round_trips(L):
    prev = fa.fa_fwd_set_cta_pairs(True)
    try:
        assert fa.fa_fwd_set_cta_pairs(False) is True
        assert fa.fa_fwd_set_cta_pairs(False) is False
    finally:
        fa.fa_fwd_set_cta_pairs(prev)
    assert prev is False  # the default


# Fake, never-dereferenced device addresses: validation rejects the calls
# before any CUDA call is made.
A = 1 << 20          # 16-byte aligned
MIS = A + 8          # not 16-byte aligned
S = None             # default stream


def fwd(L, q=A, k=A, v=A, o=A, lse=A, B=1, H=2, N=256, d=64, causal=0, scale=0.125):
    return L.fa_fwd(q, k, v, o, lse, B, H, N, d, causal, scale, S)


def fwd_gqa(L, q=A, k=A, v=A, o=A, lse=A, B=1, H=8, H_kv=2, N=256, d=128, causal=1,
            scale=0.1):
    return L.fa_fwd_gqa(q, k, v, o, lse, B, H, H_kv, N, d, causal, scale, S)


def varlen(L, q=A, k=A, v=A, o=A, lse=A, cu=A, B=2, H=2, total=100, maxlen=60, d=128,
           causal=1, scale=0.1):
    return L.fa_fwd_varlen(q, k, v, o, lse, cu, B, H, total, maxlen, d, causal, scale, S)


def decode(L, q=A, kp=A, vp=A, pt=A, sl=A, o=A, B=4, H=2, d=128, ps=256):
    return L.fa_decode_paged(q, kp, vp, pt, sl, o, B, H, d, ps, S)


def decode_gqa(L, q=A, kp=A, vp=A, pt=A, sl=A, o=A, B=4, H=8, H_kv=2, P=64, d=128, ps=256):
    return L.fa_decode_paged_gqa(q, kp, vp, pt, sl, o, B, H, H_kv, P, d, ps, S)


def decode_strided(L, q=A, kp=A, vp=A, bt=A, mp=70, sl=A, o=A, B=4, H=8, H_kv=2, P=64, d=128,
                   ps=256):
    return L.fa_decode_paged_strided(q, kp, vp, bt, mp, sl, o, B, H, H_kv, P, d, ps, S)


def append(L, kn=A, vn=A, cu=A, kp=A, vp=A, pt=A, sl=A, B=2, H_kv=2, total=10, P=8, d=128,
           ps=256):
    return L.fa_append_paged(kn, vn, cu, kp, vp, pt, sl, B, H_kv, total, P, d, ps, S)


def prefill(L, q=A, kp=A, vp=A, pt=A, sl=A, cu=A, o=A, lse=A, B=2, H=8, H_kv=2, total=100,
            maxq=60, P=8, d=128, ps=256, causal=1, scale=0.1):
    return L.fa_prefill_paged(q, kp, vp, pt, sl, cu, o, lse, B, H, H_kv, total, maxq, P, d, ps,
                              causal, scale, S)


def bwd_gqa(L, q=A, k=A, v=A, o=A, lse=A, do=A, dq=A, dk=A, dv=A, B=1, H=8, H_kv=2, N=256,
            d=128, causal=1, scale=0.1):
    return L.fa_bwd_gqa(q, k, v, o, lse, do, dq, dk, dv, B, H, H_kv, N, d, causal, scale, S)


def bwd_varlen(L, q=A, k=A, v=A, o=A, lse=A, do=A, dq=A, dk=A, dv=A, cu=A, B=2, H=8, H_kv=2,
               total=100, maxlen=60, d=128, causal=1, scale=0.1):
    return L.fa_bwd_varlen(q, k, v, o, lse, do, dq, dk, dv, cu, B, H, H_kv, total, maxlen, d,
                           causal, scale, S)


def varlen_gqa(L, q=A, k=A, v=A, o=A, lse=A, cu=A, B=2, H=8, H_kv=2, total=100, maxlen=60,
               d=128, causal=1, scale=0.1):
    return L.fa_fwd_varlen_gqa(q, k, v, o, lse, cu, B, H, H_kv, total, maxlen, d, causal, scale,
                               S)


def test_bwd_argument_errors(L):
    assert L.fa_bwd(A, A, A, A, A, None, A, A, A, 1, 2, 256, 64, 1, 0.125, S) == fa.FA_ERR_NULL
    assert bwd_gqa(L, dk=None) == fa.FA_ERR_NULL
    assert bwd_gqa(L, N=0) == fa.FA_ERR_SHAPE
    assert bwd_gqa(L, H=6, H_kv=4) == fa.FA_ERR_SHAPE       # H not a multiple of H_kv
    assert bwd_gqa(L, d=96) == fa.FA_ERR_UNSUPPORTED
    assert bwd_gqa(L, scale=float("inf")) == fa.FA_ERR_SHAPE
    assert bwd_gqa(L, dq=MIS) == fa.FA_ERR_ALIGN
    assert bwd_gqa(L, lse=MIS) == fa.FA_ERR_ALIGN


def test_bwd_varlen_argument_errors(L):
    assert bwd_varlen(L, cu=None) == fa.FA_ERR_NULL
    assert bwd_varlen(L, dv=None) == fa.FA_ERR_NULL
    assert bwd_varlen(L, total=0) == fa.FA_ERR_SHAPE
    assert bwd_varlen(L, maxlen=0) == fa.FA_ERR_SHAPE
    assert bwd_varlen(L, H=8, H_kv=3) == fa.FA_ERR_SHAPE
    assert bwd_varlen(L, d=32) == fa.FA_ERR_UNSUPPORTED
    assert bwd_varlen(L, scale=float("nan")) == fa.FA_ERR_SHAPE
    assert bwd_varlen(L, do=MIS) == fa.FA_ERR_ALIGN


def test_varlen_gqa_argument_errors(L):
    assert varlen_gqa(L, cu=None) == fa.FA_ERR_NULL
    assert varlen_gqa(L, H_kv=0) == fa.FA_ERR_SHAPE
    assert varlen_gqa(L, H=8, H_kv=3) == fa.FA_ERR_SHAPE
    assert varlen_gqa(L, total=0) == fa.FA_ERR_SHAPE
    assert varlen_gqa(L, d=256) == fa.FA_ERR_UNSUPPORTED
    assert varlen_gqa(L, k=MIS) == fa.FA_ERR_ALIGN


def test_append_and_prefill_argument_errors(L):
    assert append(L, cu=None) == fa.FA_ERR_NULL
    assert append(L, P=0) == fa.FA_ERR_SHAPE
    assert append(L, total=-1) == fa.FA_ERR_SHAPE
    assert append(L, ps=128) == fa.FA_ERR_UNSUPPORTED
    assert append(L, d=96) == fa.FA_ERR_UNSUPPORTED
    assert append(L, kp=MIS) == fa.FA_ERR_ALIGN
    assert prefill(L, cu=None) == fa.FA_ERR_NULL
    assert prefill(L, H_kv=3) == fa.FA_ERR_SHAPE
    assert prefill(L, maxq=0) == fa.FA_ERR_SHAPE
    assert prefill(L, P=0) == fa.FA_ERR_SHAPE
    assert prefill(L, ps=64) == fa.FA_ERR_UNSUPPORTED
    assert prefill(L, scale=float("nan")) == fa.FA_ERR_SHAPE
    assert prefill(L, lse=MIS) == fa.FA_ERR_ALIGN


def gather(L, pages=A, pt=A, sl=A, out=A, B=4, H=2, d=128, ps=256):
    return L.fa_gather_paged(pages, pt, sl, out, B, H, d, ps, S)


def test_fwd_argument_errors(L):
    assert fwd(L, q=None) == fa.FA_ERR_NULL
    assert fwd(L, lse=None) == fa.FA_ERR_NULL
    assert fwd(L, N=0) == fa.FA_ERR_SHAPE
    assert fwd(L, B=0) == fa.FA_ERR_SHAPE
    assert fwd(L, H=-1) == fa.FA_ERR_SHAPE
    assert fwd(L, B=256, H=256) == fa.FA_ERR_SHAPE       # B*H > 65535
    assert fwd(L, d=96) == fa.FA_ERR_UNSUPPORTED
    assert fwd(L, d=256) == fa.FA_ERR_UNSUPPORTED
    assert fwd(L, scale=float("nan")) == fa.FA_ERR_SHAPE
    assert fwd(L, scale=float("inf")) == fa.FA_ERR_SHAPE
    assert fwd(L, k=MIS) == fa.FA_ERR_ALIGN
    assert fwd(L, o=MIS) == fa.FA_ERR_ALIGN


def test_fwd_gqa_argument_errors(L):
    assert fwd_gqa(L, k=None) == fa.FA_ERR_NULL
    assert fwd_gqa(L, H_kv=0) == fa.FA_ERR_SHAPE
    assert fwd_gqa(L, H_kv=3) == fa.FA_ERR_SHAPE        # H not a multiple of H_kv
    assert fwd_gqa(L, H=4, H_kv=8) == fa.FA_ERR_SHAPE
    assert fwd_gqa(L, d=80) == fa.FA_ERR_UNSUPPORTED
    assert fwd_gqa(L, v=MIS) == fa.FA_ERR_ALIGN


def rope_fwd(L, q=A, k=A, v=A, o=A, lse=A, c=A, sn=A, maxpos=256, B=1, H=4, H_kv=2, N=256,
             d=128, causal=1, scale=0.1):
    return L.fa_fwd_rope(q, k, v, o, lse, c, sn, maxpos, B, H, H_kv, N, d, causal, scale, S)


def test_fwd_rope_argument_errors(L):
    assert rope_fwd(L, c=None) == fa.FA_ERR_NULL
    assert rope_fwd(L, sn=None) == fa.FA_ERR_NULL
    assert rope_fwd(L, maxpos=100) == fa.FA_ERR_SHAPE      # table shorter than N
    assert rope_fwd(L, c=MIS) == fa.FA_ERR_ALIGN
    assert rope_fwd(L, H_kv=3) == fa.FA_ERR_SHAPE
    assert rope_fwd(L, d=32) == fa.FA_ERR_UNSUPPORTED


def test_varlen_argument_errors(L):
    assert varlen(L, cu=None) == fa.FA_ERR_NULL
    assert varlen(L, total=0) == fa.FA_ERR_SHAPE
    assert varlen(L, maxlen=0) == fa.FA_ERR_SHAPE
    assert varlen(L, d=32) == fa.FA_ERR_UNSUPPORTED
    assert varlen(L, v=MIS) == fa.FA_ERR_ALIGN


def test_decode_argument_errors(L):
    assert decode(L, pt=None) == fa.FA_ERR_NULL
    assert decode(L, sl=None) == fa.FA_ERR_NULL
    assert decode(L, B=0) == fa.FA_ERR_SHAPE
    assert decode(L, ps=128) == fa.FA_ERR_UNSUPPORTED
    assert decode(L, ps=16) == fa.FA_ERR_UNSUPPORTED
    assert decode(L, d=80) == fa.FA_ERR_UNSUPPORTED
    assert decode(L, kp=MIS) == fa.FA_ERR_ALIGN
    assert decode_gqa(L, vp=None) == fa.FA_ERR_NULL
    assert decode_gqa(L, H_kv=0) == fa.FA_ERR_SHAPE
    assert decode_gqa(L, H_kv=3) == fa.FA_ERR_SHAPE       # 8 is not a multiple of 3
    assert decode_gqa(L, P=0) == fa.FA_ERR_SHAPE          # empty pool
    assert decode_gqa(L, H=24, H_kv=5) == fa.FA_ERR_SHAPE  # 24 is not a multiple of 5
    assert decode_gqa(L, ps=128) == fa.FA_ERR_UNSUPPORTED
    assert decode_gqa(L, o=MIS) == fa.FA_ERR_ALIGN
    assert decode_strided(L, bt=None) == fa.FA_ERR_NULL
    assert decode_strided(L, mp=0) == fa.FA_ERR_SHAPE
    assert decode_strided(L, mp=1 << 24) == fa.FA_ERR_SHAPE  # row of 2^32 tokens
    assert decode_strided(L, B=1 << 10, mp=1 << 22) == fa.FA_ERR_SHAPE  # 2^32 entries
    assert decode_strided(L, H=24, H_kv=7) == fa.FA_ERR_SHAPE
    assert decode_strided(L, ps=128) == fa.FA_ERR_UNSUPPORTED
    assert decode_strided(L, q=MIS) == fa.FA_ERR_ALIGN
    assert gather(L, out=None) == fa.FA_ERR_NULL
    assert gather(L, ps=255) == fa.FA_ERR_UNSUPPORTED
    assert gather(L, pages=MIS) == fa.FA_ERR_ALIGN


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")
def test_valid_call_without_gpu_reports_cuda_error(L):
    # arguments pass validation; the device lookup then fails cleanly
    assert fwd(L) == fa.FA_ERR_CUDA
    assert fwd_gqa(L) == fa.FA_ERR_CUDA
    assert rope_fwd(L) == fa.FA_ERR_CUDA
    assert decode(L) == fa.FA_ERR_CUDA
    assert decode_gqa(L) == fa.FA_ERR_CUDA
    assert decode_strided(L) == fa.FA_ERR_CUDA
    assert append(L) == fa.FA_ERR_CUDA
    assert prefill(L) == fa.FA_ERR_CUDA
    code = ctypes.c_int(7)
    assert L.fa_get_device_error(ctypes.byref(code), S) == fa.FA_ERR_CUDA


def test_binding_refuses_cpu_tensors():
    x = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        fa.fa_fwd(x, x, x, causal=False)


def test_binding_fails_loudly_without_library(monkeypatch):
    from attn_fwd_04_b200 import fa as binding
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "LIB_PATH", "/nonexistent/libfa.so")
    with pytest.raises(ImportError):
        binding.lib()


# -- the Python wrappers reject inconsistent tensors before calling the library --
# (meta tensors carry shapes, dtypes and devices without memory; the library
# handle is replaced by one that fails the test if any call reaches it)

@pytest.fixture
def meta_binding(monkeypatch):
    from attn_fwd_04_b200 import fa as binding

    def no_library():
        raise AssertionError("the library was called")

    monkeypatch.setattr(binding, "_DEVICE_TYPES", ("cuda", "meta"))
    monkeypatch.setattr(binding, "lib", no_library)
    return binding


def _m(*shape, dtype=torch.bfloat16):
    return torch.empty(shape, dtype=dtype, device="meta")


def _decode_args(B=3, H=4, P=5, Hc=None, PS=256, d=128, nlen=None):
    Hc = H if Hc is None else Hc
    return (_m(B, H, d), _m(P, Hc, PS, d), _m(P, Hc, PS, d), _m(7, dtype=torch.int32),
            _m(B if nlen is None else nlen, dtype=torch.int32))


@pytest.mark.parametrize("name", ["fa_decode_paged", "fa_decode_paged_noalloc"])
def test_multihead_decode_wrappers_check_the_pool(meta_binding, name):
    f = getattr(meta_binding, name)
    with pytest.raises(AssertionError, match="library was called"):
        f(*_decode_args())                      # consistent: reaches the library
    with pytest.raises(ValueError, match="pages"):
        f(*_decode_args(Hc=2))                  # a grouped pool: other head count
    q, kp, vp, pt, sl = _decode_args()
    with pytest.raises(ValueError, match="pages"):
        f(q, _m(5, 4, 128, 128), _m(5, 4, 128, 128), pt, sl)   # page size 128, not 256
    with pytest.raises(ValueError, match="same shape"):
        f(q, kp, _m(6, 4, 256, 128), pt, sl)    # k and v pools differ
    with pytest.raises(ValueError, match="one length per sequence"):
        f(*_decode_args(nlen=2))
    with pytest.raises(ValueError, match="shape"):
        f(q, kp, vp, pt, sl, o=_m(3, 4, 64))    # output of another shape
    with pytest.raises(TypeError):
        f(q, kp, vp, pt, sl, o=_m(3, 4, 128, dtype=torch.float32))


def test_grouped_decode_wrappers_check_the_pool(meta_binding):
    q, kp, vp, pt, sl = _decode_args(H=8, Hc=2)
    with pytest.raises(AssertionError, match="library was called"):
        meta_binding.fa_decode_paged_gqa(q, kp, vp, pt, sl)
    q3, kp3, vp3, _, _ = _decode_args(H=8, Hc=3)
    with pytest.raises(ValueError, match="multiple"):
        meta_binding.fa_decode_paged_gqa(q3, kp3, vp3, pt, sl)
    with pytest.raises(ValueError, match="one length per sequence"):
        meta_binding.fa_decode_paged_gqa(q, kp, vp, pt, _m(4, dtype=torch.int32))
    bt = _m(3, 6, dtype=torch.int32)
    with pytest.raises(AssertionError, match="library was called"):
        meta_binding.fa_decode_paged_strided(q, kp, vp, bt, sl)
    with pytest.raises(ValueError, match="pages"):
        meta_binding.fa_decode_paged_strided(q, kp, vp, bt, sl, page_size=128)


def test_forward_and_backward_wrappers_check_outputs(meta_binding):
    q = _m(1, 2, 64, 128)
    with pytest.raises(AssertionError, match="library was called"):
        meta_binding.fa_fwd(q, q, q, True)
    with pytest.raises(ValueError, match="shape"):
        meta_binding.fa_fwd(q, q, q, True, lse=_m(1, 2, 63, dtype=torch.float32))
    with pytest.raises(ValueError, match="shape"):
        meta_binding.fa_fwd(q, q, q, True, o=_m(1, 2, 64, 64))
    lse = _m(1, 2, 64, dtype=torch.float32)
    with pytest.raises(AssertionError, match="library was called"):
        meta_binding.fa_bwd(q, q, q, q, lse, q, True)
    with pytest.raises(ValueError, match="shape"):
        meta_binding.fa_bwd(q, q, q, q, _m(1, 2, 32, dtype=torch.float32), q, True)
    with pytest.raises(ValueError, match="shape"):
        meta_binding.fa_bwd(q, q, q, q, lse, q, True, dk=_m(1, 1, 64, 128))
    qp = _m(100, 4, 128)
    cu = _m(3, dtype=torch.int32)
    with pytest.raises(ValueError, match="shape"):
        meta_binding.fa_fwd_varlen(qp, _m(100, 2, 128), _m(100, 2, 128), cu, 64, True)
    with pytest.raises(ValueError, match="shape"):
        meta_binding.fa_fwd_varlen(qp, qp, qp, cu, 64, True, lse=_m(100, 4, dtype=torch.float32))
