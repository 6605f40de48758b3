"""Shared comparison helpers for the GPU parity tests.

Tolerances (fixed by the accuracy target for bf16 inputs with fp32
accumulation): O within max-abs 2e-2 and relative RMS 5e-3 of the fp64
oracle, the log-sum-exp within 1e-3 absolute.
"""
import numpy as np
import torch

O_MAX_ABS = 2e-2
O_REL_RMS = 5e-3
LSE_MAX_ABS = 1e-3
# Gradients (backward pass; not fixed by the accuracy target, derived here):
# P and dS enter their products rounded to bf16 (2^-9 relative each) and the
# outputs are bf16, so over the compared tensor the relative RMS error is
# about 4e-3 and single elements reach a few 2^-8 of the tensor's largest
# magnitude; the gates leave a factor of 2-3 above that.
GRAD_REL_RMS = 1e-2
GRAD_MAX_ABS_REL = 3e-2


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def o_errors(o_gpu: np.ndarray, o_ref: np.ndarray):
    diff = o_gpu - o_ref
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    denom = float(np.sqrt(np.sum(o_ref * o_ref)))
    rel_rms = float(np.sqrt(np.sum(diff * diff)) / denom) if denom > 0 else float(np.sqrt(np.sum(diff * diff)))
    return max_abs, rel_rms


def assert_o_close(o_gpu, o_ref, what=""):
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite output"
    max_abs, rel_rms = o_errors(o_gpu, o_ref)
    assert max_abs <= O_MAX_ABS, f"{what}: O max-abs {max_abs:.3e} > {O_MAX_ABS}"
    assert rel_rms <= O_REL_RMS, f"{what}: O rel-RMS {rel_rms:.3e} > {O_REL_RMS}"
    return max_abs, rel_rms


def assert_o_close_scaled(o_gpu, o_ref, v_max_abs: float, what=""):
    """O for values of any magnitude: the max-abs gate is taken relative to the
    largest |V| (O is a convex combination of V's rows, and its error -- bf16
    rounding of P and of O itself -- grows with |V|); relative RMS as usual."""
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite output"
    max_abs, rel_rms = o_errors(o_gpu, o_ref)
    gate = O_MAX_ABS * max(1.0, v_max_abs)
    assert max_abs <= gate, f"{what}: O max-abs {max_abs:.3e} > {gate:.3e}"
    assert rel_rms <= O_REL_RMS, f"{what}: O rel-RMS {rel_rms:.3e} > {O_REL_RMS}"
    return max_abs, rel_rms


def assert_lse_close(lse_gpu, lse_ref, what=""):
    assert np.all(np.isfinite(lse_gpu)), f"{what}: non-finite lse"
    err = float(np.max(np.abs(lse_gpu - lse_ref))) if np.size(lse_ref) else 0.0
    assert err <= LSE_MAX_ABS, f"{what}: LSE max-abs {err:.3e} > {LSE_MAX_ABS}"
    return err


def sample_rows(N: int, count: int, seed: int, tile: int = 128):
    """Query rows to check at full size: the first and last rows, both sides
    of every few tile boundaries, and seeded random rows."""
    g = torch.Generator().manual_seed(seed)
    fixed = {0, 1, N - 1, N - 2}
    for t in range(tile, N, max(tile, (N // 8) // tile * tile)):
        fixed.update({t - 1, t})
    rand = torch.randint(0, N, (max(0, count - len(fixed)),), generator=g).tolist()
    return sorted({r for r in fixed | set(rand) if 0 <= r < N})


def assert_grad_close(g_gpu, g_ref, what=""):
    """Gradient tensors: relative RMS over the tensor and max-abs relative to
    the reference's largest magnitude."""
    assert np.all(np.isfinite(g_gpu)), f"{what}: non-finite gradient"
    diff = g_gpu - g_ref
    scale = float(np.max(np.abs(g_ref))) or 1.0
    max_rel = float(np.max(np.abs(diff))) / scale if diff.size else 0.0
    denom = float(np.sqrt(np.sum(g_ref * g_ref)))
    rel_rms = float(np.sqrt(np.sum(diff * diff)) / denom) if denom > 0 else 0.0
    assert rel_rms <= GRAD_REL_RMS, f"{what}: rel-RMS {rel_rms:.3e} > {GRAD_REL_RMS}"
    assert max_rel <= GRAD_MAX_ABS_REL, f"{what}: max-abs/max {max_rel:.3e} > {GRAD_MAX_ABS_REL}"
    return rel_rms, max_rel
