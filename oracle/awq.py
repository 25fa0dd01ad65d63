"""CPU oracle for the AWQ scale search -- TEST INFRASTRUCTURE ONLY.

Page 2 (learn.longtimenohack.com/chasing/pages/quantization.html, AWQ section,
the ``awq_search_scale`` listing) picks the per-input-channel smoothing vector
by a grid search: act = the mean magnitude of each input channel over the
calibration rows; for alpha on an even grid over [0, 1], s = act^alpha
normalised to mean 1; the weight W * s is quantized and dequantized; the loss
is the mean squared difference between W X^T and (W^ / s) X^T; the alpha with
the smallest loss wins.  This module restates those steps with the oracle's
quantizer, dequantizer and fp64 product (``oracle/__init__.py``); it shares no
code with the CUDA library.

Readings (where the page leaves a step open):
  * alpha_i = i / (n - 1) in fp64, i = 0 .. n-1 (an even grid including both
    ends, like the listing's linspace);
  * act and s are computed in fp64; s is rounded once to fp32, the precision
    in which the quantizer folds it (w' = fl32(w * s));
  * (W^ / s) X^T is evaluated as W^ . (X / s)^T, the product the W4A16 path
    computes: x / s in fp32 (IEEE division), rounded to bf16, then the fp64
    product with the dequantized weight, rounded to bf16 like the path's
    output; the page's listing divides the weight instead, which is the same
    product in exact arithmetic (page 5 section 2.4, the smoothing identity);
  * W X^T is the fp64 product of the bf16 inputs;
  * the loss is the mean over all M x N outputs, in fp64;
  * the first index reaching the minimum wins (a strict "<" in the listing).
"""
from __future__ import annotations

import numpy as np

from . import ASYM, SYM, gemm_f64, quant_pack, w4a16_reference  # noqa: F401


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite fp32 values to bf16, ties to even, as bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def f64_to_bf16_f64(y: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 (via the fp32 the path accumulates in) -> fp64."""
    return bf16_bits_to_f64(f32_to_bf16_bits(np.asarray(y, dtype=np.float64).astype(np.float32)))


def alphas(n_alpha: int) -> np.ndarray:
    return np.array([i / (n_alpha - 1) for i in range(n_alpha)], dtype=np.float64)


def act_magnitude(X_bits: np.ndarray) -> np.ndarray:
    """act[k] = mean over calibration rows of |x[m][k]|, fp64."""
    return np.mean(np.abs(bf16_bits_to_f64(X_bits)), axis=0)


def smoothing(act: np.ndarray, alpha: float) -> np.ndarray:
    """s = act^alpha / mean(act^alpha) in fp64, rounded once to fp32."""
    p = np.power(act, alpha)
    return (p / np.mean(p)).astype(np.float32)


def awq_losses(W_bits: np.ndarray, X_bits: np.ndarray, g: int, mode: int, n_alpha: int = 20, threads: int = 1):
    """Returns (losses fp64 [n_alpha], best index, s of the best alpha fp32 [K])."""
    W_bits = np.ascontiguousarray(W_bits, dtype=np.uint16)
    X_bits = np.ascontiguousarray(X_bits, dtype=np.uint16)
    K = W_bits.shape[1]
    Y_ref = gemm_f64(X_bits, W_bits, threads=threads)
    act = act_magnitude(X_bits)
    X32 = bf16_bits_to_f64(X_bits).astype(np.float32)
    losses = np.zeros(n_alpha, dtype=np.float64)
    scales = []
    for i, a in enumerate(alphas(n_alpha)):
        s = smoothing(act, a)
        scales.append(s)
        q, sc, z = quant_pack(W_bits, g, mode, s=s, threads=threads)
        Xs_bits = f32_to_bf16_bits(X32 / s[None, :])
        Y_q = f64_to_bf16_f64(w4a16_reference(Xs_bits, q, sc, z, K, g, mode, threads=threads))
        losses[i] = np.mean((Y_ref - Y_q) ** 2)
    best = int(np.argmin(losses))
    return losses, best, scales[best]
