"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
import numpy as np
import torch

import svg_workloads as W


def dev(a: np.ndarray, device="cuda"):
    t = torch.from_numpy(np.ascontiguousarray(a)).to(device)
    return t.view(torch.bfloat16) if a.dtype == np.uint16 else t


def host_bits(t) -> np.ndarray:
    """bf16 device tensor -> uint16 numpy bit patterns."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f64(bits: np.ndarray) -> np.ndarray:
    return W.bf16_bits_to_f32(bits).astype(np.float64)


def bf16_ulp_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in representable bf16 steps between two bit-pattern arrays."""
    def ordered(x):
        x = x.astype(np.int32)
        return np.where(x & 0x8000, 0x8000 - (x & 0x7FFF), 0x8000 + (x & 0x7FFF))
    return np.abs(ordered(a) - ordered(b))


def assert_norm_rope_close(got_bits: np.ndarray, ref_bits: np.ndarray, what=""):
    """QK-Norm + RoPE bar.  The kernel computes in fp32 and rounds once to
    bf16; the oracle computes in fp64 and rounds once.  A RoPE output is
    u*cos - v*sin: where it cancels, fp32 leaves an absolute error of a few
    fp32 ulps of the pair's norm (rotation preserves |(u, v)|), far below one
    bf16 ulp of the pair but possibly many ulps of the tiny result.  So the
    bar is: |got - ref| <= 1 bf16 ulp(ref) + 2^-20 * |pair|, and at least 99%
    of the elements bit-equal."""
    g = f64(got_bits).reshape(-1, 2)
    r = f64(ref_bits).reshape(-1, 2)
    pair = np.sqrt((r ** 2).sum(1, keepdims=True))
    big = np.maximum(np.maximum(np.abs(r), np.abs(g)), 2.0 ** -126)   # ulp of the larger binade
    ulp = np.exp2(np.floor(np.log2(big)) - 7)
    bound = ulp + 2.0 ** -20 * pair
    err = np.abs(g - r)
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} elements over the bound, worst excess {(err - bound).max():.3e}"
    eq = (got_bits.reshape(-1) == ref_bits.reshape(-1)).mean()
    assert eq > 0.99, f"{what}: only {eq:.4f} bit-equal"


def assert_attention_close(got_bits_rows: np.ndarray, ref: np.ndarray, max_abs=2e-2, mean_abs=2e-3, what=""):
    g = f64(got_bits_rows)
    err = np.abs(g - ref)
    assert np.isfinite(g).all(), f"{what}: non-finite outputs"
    assert err.max() <= max_abs and err.mean() <= mean_abs, \
        f"{what}: max_abs={err.max():.3e} mean_abs={err.mean():.3e} (rows {np.argmax(err.max(1))})"
    return err.max(), err.mean()
