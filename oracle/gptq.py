"""CPU oracle for GPTQ (Hessian-aware INT4 rounding with error feedback) --
TEST INFRASTRUCTURE ONLY.

What it computes (fp64 unless stated):

  objective   choose W^ minimising || W X^T - W^ X^T ||_F^2 over the
              calibration rows X (page 2, GPTQ section; page 3 section 3.1)
  Hessian     H = 2 X^T X + lambda I, lambda = 0.01 trace(X^T X) / K
              (page 3 section 3.1, implementation detail 1)
  factor      U = the upper Cholesky factor of H^-1 (H^-1 = U^T U)
              (page 5 section 2.5)
  columns     in their natural order j = 0 .. K-1:
                at the first column of each group of g columns, the group's
                per-row scale (and zero-point) are taken from the group's
                CURRENT, already updated weights, with the quantizer's own
                rules (fp32 statistics, fp16 scale, page 5 section 2.2);
                u_j  = the INT4 code of fl32(w_j) on that grid (IEEE fp32
                       division, round half to even, clip to the code range);
                w^_j = (u_j - zp) * s16, the grid point;
                e    = (w_j - w^_j) / U[j, j];
                w_k -= e * U[j, k] for every k > j
              (page 5 section 2.5; page 2's update w_k -= (w_j - w^_j)
              [H^-1]_jk / [H^-1]_jj is the same step written with the inverse
              of the remaining columns' Hessian)

Readings where the pages leave a step open or disagree:
  * lambda: page 3's relative rule above; page 2's teaching listing adds a
    fixed 1e-3 instead, and is not followed.
  * Groups: page 3 says groups of columns share a scale in practice; its
    listing takes a per-column scale over the output channels and propagates
    only inside the group, page 2 and page 5 propagate to every later column.
    The oracle propagates to every later column and takes each row's group
    scale from the group's weights when its first column is reached.
  * Page 1's outline updates with H itself (not its inverse) and with the
    opposite sign; pages 2, 3 and 5 agree on the inverse, which is followed.
  * The error fed back is the distance to the grid point (u - zp) * s16, which
    is exact in fp32; the W4A16 product later uses the same value rounded to
    bf16.
  * If trace(X^T X) is 0 (no calibration signal), H would be singular; the
    oracle then takes U = I, which feeds nothing back (plain round-to-nearest).
  * No act-order (column permutation) and no lazy block updates: both only
    reorder the same arithmetic or change the column order, which the pages
    do not specify.

Weights enter as bf16 bit patterns [N, K] (the library's input format),
calibration rows as bf16 bits [M, K]. The output is the packed format that
``oracle.quant_pack`` and the library use. This module restates the method
with numpy (Cholesky, inverse) and the oracle's group quantizer; it shares no
code with the CUDA library.
"""
from __future__ import annotations

import numpy as np

from . import ASYM, SYM, packed_shapes, quant_group  # noqa: F401


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f16_bits_to_f64(bits) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def hessian(X_bits: np.ndarray) -> np.ndarray:
    """H = 2 X^T X + lambda I with lambda = 0.01 trace(X^T X) / K, fp64 [K, K]."""
    X = bf16_bits_to_f64(X_bits)
    XtX = X.T @ X
    K = XtX.shape[0]
    lam = 0.01 * np.trace(XtX) / K
    return 2.0 * XtX + lam * np.eye(K)


def inverse_cholesky_upper(H: np.ndarray) -> np.ndarray:
    """U upper triangular with H^-1 = U^T U (U = I when H is all zero)."""
    if not np.any(H):
        return np.eye(H.shape[0])
    Hinv = np.linalg.inv(H)
    Hinv = 0.5 * (Hinv + Hinv.T)              # symmetric to the last bit before factoring
    return np.linalg.cholesky(Hinv).T         # numpy gives lower L, Hinv = L L^T


def _codes(w32: np.ndarray, d: np.ndarray, zp: np.ndarray, mode: int) -> np.ndarray:
    """INT4 codes of the fp32 values w32 on the grids (d = float(s16), zp) per row."""
    u = np.zeros(w32.shape, dtype=np.int64)
    live = d != 0
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.rint(np.divide(w32, d.astype(np.float32), dtype=np.float32)).astype(np.float64)
    if mode == SYM:
        u = np.where(live, np.clip(q, -8, 7) + 8, 8)
    else:
        u = np.where(live, np.clip(q + zp, 0, 15), 0)
    return u.astype(np.int64)


def gptq_quantize(W_bits: np.ndarray, X_bits: np.ndarray, g: int, mode: int, return_trace: bool = False):
    """GPTQ over bf16 W [N, K] with calibration rows X [M, K].

    Returns (u int codes [N, K] in 0..15, s16 fp16 bits [N, K/g], zp [N, K/g]);
    with ``return_trace`` also W_pre fp64 [N, K], each column's value at the
    moment it was quantized. Any g dividing K is accepted here; the packed
    format needs K % 8 == 0 (``gptq_pack``)."""
    W = bf16_bits_to_f64(W_bits).copy()
    N, K = W.shape
    if K % g != 0:
        raise ValueError("K must be a multiple of g")
    U = inverse_cholesky_upper(hessian(X_bits))
    G = K // g
    u = np.zeros((N, K), dtype=np.int64)
    s16 = np.zeros((N, G), dtype=np.uint16)
    zp = np.zeros((N, G), dtype=np.int64)
    W_pre = np.zeros((N, K)) if return_trace else None
    d = None
    for j in range(K):
        gi = j // g
        if j % g == 0:                          # this group's grid, from its current weights
            blk = W[:, j:j + g].astype(np.float32)
            for n in range(N):
                s, z, _ = quant_group(blk[n], mode)
                s16[n, gi], zp[n, gi] = s, z
            d = f16_bits_to_f64(s16[:, gi])
        if return_trace:
            W_pre[:, j] = W[:, j]
        w32 = W[:, j].astype(np.float32)
        u[:, j] = _codes(w32, d, zp[:, gi], mode)
        what = (u[:, j] - zp[:, gi]) * d       # the grid point, exact
        e = (W[:, j] - what) / U[j, j]
        W[:, j + 1:] -= np.outer(e, U[j, j + 1:])
    if return_trace:
        return u, s16, zp, W_pre
    return u, s16, zp


def pack(u: np.ndarray, s16: np.ndarray, zp: np.ndarray, mode: int):
    """The library's packed format: qweight uint32 [N, K/8], element k in word
    k / 8 with e = k % 8 at bit 4 (e / 2) when e is even and at bit
    16 + 4 (e / 2) when e is odd (even elements in the low half-word, odd in
    the high); scales fp16 bits [N, G]; qzeros uint32 [N, ceil(G/8)], zero-point
    j at bit 4 (j % 8) of word j / 8 (asymmetric only)."""
    N, K = u.shape
    G = s16.shape[1]
    qweight = np.zeros((N, K // 8), dtype=np.uint32)
    for e in range(8):
        shift = 4 * (e // 2) + (16 if e % 2 else 0)
        qweight |= (u[:, e::8].astype(np.uint32) << np.uint32(shift))
    qzeros = None
    if mode == ASYM:
        qzeros = np.zeros((N, (G + 7) // 8), dtype=np.uint32)
        for gi in range(G):
            qzeros[:, gi // 8] |= (zp[:, gi].astype(np.uint32) << np.uint32(4 * (gi % 8)))
    return qweight, s16.copy(), qzeros


def gptq_pack(W_bits: np.ndarray, X_bits: np.ndarray, g: int, mode: int):
    """GPTQ in the library's packed format: (qweight, scales, qzeros or None)."""
    if W_bits.shape[1] % 8 != 0:
        raise ValueError("K must be a multiple of 8")
    u, s16, zp = gptq_quantize(W_bits, X_bits, g, mode)
    return pack(u, s16, zp, mode)


def dequantize(u: np.ndarray, s16: np.ndarray, zp: np.ndarray, g: int) -> np.ndarray:
    """Grid points (u - zp) * s16, fp64 [N, K] (exact)."""
    d = np.repeat(f16_bits_to_f64(s16), g, axis=1)
    z = np.repeat(zp, g, axis=1)
    return (u - z) * d


def output_error(W_bits: np.ndarray, What: np.ndarray, X_bits: np.ndarray) -> float:
    """|| W X^T - W^ X^T ||_F / || W X^T ||_F in fp64."""
    W = bf16_bits_to_f64(W_bits)
    X = bf16_bits_to_f64(X_bits)
    ref = W @ X.T
    return float(np.linalg.norm(ref - What @ X.T) / np.linalg.norm(ref))
