"""Exact scaled-dot-product attention on B200 (sm_100a).

The computation lives in libfa.so (CUDA, C ABI in include/fa.h); this package
is its Python binding plus seeded synthetic workloads.
"""
from .fa import (EXPORTS, FA_ERR_ALIGN, FA_ERR_CUDA, FA_ERR_DEVICE_BAD_INPUT,  # noqa: F401
                 FA_ERR_DEVICE_TIMEOUT, FA_ERR_NOMEM, FA_ERR_NULL, FA_ERR_SHAPE,
                 FA_ERR_UNSUPPORTED, FA_OK, FaError, fa_decode_paged, fa_decode_paged_gqa,
                 fa_decode_paged_strided,
                 fa_decode_paged_noalloc, fa_append_paged, fa_prefill_paged,
                 fa_bwd, fa_bwd_gqa, fa_bwd_varlen, fa_fwd, fa_fwd_gqa, fa_fwd_rope,
                 fa_fwd_set_cta_pairs, fa_fwd_varlen_gqa,
                 fa_fwd_varlen,
                 fa_gather_paged, fa_get_device_error, fa_release_workspace, fa_selftest_bounded_wait,
                 fa_selftest_decode_stall, fa_selftest_fwd_stall,
                 fa_status_str,
                 fa_version, lib)
