"""The MX path on the GPU against the CPU oracle.

w4_mxfp8_quant: every code and scale byte equals oracle.mxfp8_quant, in both
scale layouts.  w4_mx_scale_layout: a byte permutation, checked against the
layout's definition written out in numpy.  w4_mx_gemm: the whole GPU chain
(w4_fp4_quant MXFP4 -> w4_mx_scale_layout, w4_mxfp8_quant -> w4_mx_gemm)
against oracle.mx_reference, the fp64 product of the two dequantized operands.
"""
import numpy as np
import pytest

import oracle
from bit_gemm_quant_b200 import synth
from parity import THREADS, assert_codes_equal, assert_y_close, assert_y_elementwise, dev_bf16

MXFP4 = 1


@pytest.fixture(scope="module")
def w4():
    from bit_gemm_quant_b200 import build
    build.build()
    import bit_gemm_quant_b200 as w4
    oracle.build()
    return w4


def mma_layout(scales_rows: np.ndarray, K: int) -> np.ndarray:
    """The tensor-core scale layout of include/w4.h, written out: the scale of
    (r, kb) at ((r/128) * (K/128) + kb/4) * 512 + (r%32) * 16 + ((r%128)/32) * 4
    + kb%4, the rows that pad the last 128-row band zero."""
    R = scales_rows.shape[0]
    bands = (R + 127) // 128
    out = np.zeros(bands * 128 * (K // 32), dtype=np.uint8)
    r = np.arange(R)[:, None]
    kb = np.arange(K // 32)[None, :]
    off = ((r // 128) * (K // 128) + kb // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + kb % 4
    out[off] = scales_rows
    return out


# ------------------------------------------------------ MXFP8 quantizer --

def quant_both(w4, X_bits, layout):
    import torch
    M, K = X_bits.shape
    codes, scales = w4.mxfp8_quant(dev_bf16(X_bits), layout)
    torch.cuda.synchronize()
    oc, osc = oracle.mxfp8_quant(X_bits)
    assert_codes_equal(codes.cpu().numpy(), oc, "codes")
    if layout == w4.MX_SCALES_ROWS:
        assert_codes_equal(scales.cpu().numpy(), osc, "scales")
    else:
        assert_codes_equal(scales.cpu().numpy(), mma_layout(osc, K), "scales (tensor-core layout)")


@pytest.mark.gpu
@pytest.mark.parametrize("M,K", [(1, 4096), (4, 512), (7, 8224), (33, 1056), (1, 32), (129, 384)])
def test_mxfp8_quant_rows_layout(w4, M, K):
    X = synth.activations(5, M, K, outlier_frac=0.01, outlier_mult=40.0)
    quant_both(w4, X, w4.MX_SCALES_ROWS)


@pytest.mark.gpu
@pytest.mark.parametrize("M,K", [(1, 4096), (16, 8192), (130, 640), (300, 128)])
def test_mxfp8_quant_tensor_core_layout(w4, M, K):
    X = synth.activations(6, M, K, outlier_frac=0.005, outlier_mult=30.0)
    quant_both(w4, X, w4.MX_SCALES_MMA)


def edge_rows() -> np.ndarray:
    """Blocks of 32 that reach every branch of the rule: an all-zero block,
    bf16 subnormals (scale clamped to 2^-127), a maximum at an exact power of
    two, maxima with mantissa in [1.75, 2) (saturation at 448), every E4M3
    rounding tie at one scale, signed zeros, elements that underflow E4M3's
    subnormals, the largest finite bf16 values, and a block whose elements
    span the whole E4M3 range."""
    f = lambda a: synth.to_bf16_bits(np.asarray(a, dtype=np.float32))
    blocks = [np.zeros(32, np.uint16)]
    sub = np.arange(1, 33, dtype=np.uint16)                       # bf16 subnormal bit patterns
    blocks.append(sub)
    blocks.append(sub | np.uint16(0x8000))
    blocks.append(f(np.linspace(-1.0, 1.0, 32)))                  # amax = 1 exactly: scale 2^-8
    blocks.append(f(np.concatenate([[1.99, -1.875, 1.75], np.linspace(-1, 1, 29)])))   # saturating maxima
    # amax = 256 -> scale 1: midpoints between neighbouring E4M3 values in
    # [8, 16) and [256, 448) are exact ties in fp32
    ties = [8.5 + i for i in range(7)] + [-(9.5 + i) for i in range(6)] + [272.0, 304.0, -336.0, 400.0, 432.0]
    ties += [2.5 * 2.0 ** -9, -3.5 * 2.0 ** -9, 0.5 * 2.0 ** -9, 256.0]   # subnormal ties (2^-9 spacing)
    blocks.append(f(ties + [0.0] * (32 - len(ties))))
    blocks.append(np.array([0x8000] * 16 + [0] * 15 + [0x3F80], np.uint16))    # -0, +0 and a 1.0
    blocks.append(f([3.0e-6] * 16 + [-1.0e-7] * 15 + [100.0]))    # underflow to zero / subnormal codes
    blocks.append(f([3.0e38, -3.3e38] + [1.0e38] * 30))            # near the bf16 maximum
    blocks.append(f(2.0 ** np.arange(-16, 16, dtype=np.float64)))  # one element per binade
    row = np.concatenate(blocks)
    K = 128 * ((row.size + 127) // 128)
    row = np.concatenate([row, np.zeros(K - row.size, np.uint16)])
    return np.stack([row, row[::-1].copy(), np.roll(row, 32)])


@pytest.mark.gpu
@pytest.mark.parametrize("layout", [0, 1])
def test_mxfp8_quant_edge_blocks(w4, layout):
    quant_both(w4, edge_rows(), layout)


@pytest.mark.gpu
@pytest.mark.parametrize("R,K", [(1, 128), (100, 640), (128, 256), (129, 128), (300, 1024)])
def test_mx_scale_layout_is_the_defined_permutation(w4, R, K):
    import torch
    src = np.random.default_rng(R * 7 + K).integers(0, 256, size=(R, K // 32), dtype=np.uint8)
    dst = w4.mx_scale_layout(torch.from_numpy(src).cuda(), K)
    torch.cuda.synchronize()
    assert_codes_equal(dst.cpu().numpy(), mma_layout(src, K), "tensor-core layout")


# -------------------------------------------------------- the MX product --

def gpu_chain(w4, X_bits, W_bits):
    """The product path as a user runs it, every step in the library's kernels."""
    import torch
    K = X_bits.shape[1]
    wc, ws_rows = w4.fp4_quant(dev_bf16(W_bits), w4.MXFP4)
    ws = w4.mx_scale_layout(ws_rows, K)
    xc, xs = w4.mxfp8_quant(dev_bf16(X_bits), w4.MX_SCALES_MMA)
    Y = w4.mx_gemm(xc, xs, wc, ws)
    torch.cuda.synchronize()
    return Y, wc, ws_rows, xc


def oracle_chain(X_bits, W_bits):
    wc, ws = oracle.fp4_quant(W_bits, MXFP4)
    xc, xs = oracle.mxfp8_quant(X_bits)
    Y = oracle.mx_reference(xc, xs, wc, ws)
    Xd = np.abs(oracle.mxfp8_dequant(xc, xs).astype(np.float64))
    Wd = np.abs(oracle.fp4_dequant(wc, ws, MXFP4).astype(np.float64))
    return Y, Xd @ Wd.T, wc, ws, xc


def check_product(w4, X_bits, W_bits, what):
    Y, wc, ws, xc = gpu_chain(w4, X_bits, W_bits)
    Y_ref, Y_abs, owc, ows, oxc = oracle_chain(X_bits, W_bits)
    assert_codes_equal(wc.cpu().numpy(), owc, "weight codes")
    assert_codes_equal(ws.cpu().numpy(), ows, "weight scales")
    assert_codes_equal(xc.cpu().numpy(), oxc, "activation codes")
    Yh = Y.float().cpu().numpy().astype(np.float64)
    assert_y_elementwise(Yh, Y_ref, Y_abs, X_bits.shape[1], what)
    if Yh.size >= 1024:
        assert_y_close(Yh, Y_ref, what)
    return Y


# (M, N, K): one stage; several tiles with ragged edges in N and M; every
# activation tile width (16, 32, 64, 128, 256 tokens); two 256-token tiles
# whose second reaches into a partial 128-row scale band; split k
SHAPES = [(3, 128, 128), (4, 256, 512), (1, 300, 384), (20, 700, 1024), (64, 256, 2048), (100, 384, 512),
          (200, 256, 1024), (300, 130, 640), (1, 4096, 4096), (16, 1000, 2048),
          # single tiles and few k-stages, many tiles with long k, the decode widths
          (1, 128, 256), (2, 1024, 1024), (9, 8192, 512), (16, 11008, 4096)]


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_mx_gemm_matches_the_oracle(w4, M, N, K):
    W = synth.weights(21, N, K, std=0.02, outlier_frac=0.01, outlier_mult=5.0)
    X = synth.activations(22, M, K, outlier_frac=0.01, outlier_mult=40.0)
    check_product(w4, X, W, "Y[%d,%d,%d]" % (M, N, K))


@pytest.mark.gpu
def test_mx_gemm_repeats_bit_for_bit(w4):
    """Split-K partials are summed in split order: the result does not depend
    on which CTA finishes first; W4_WEIGHTS_STATIC gives the same bits."""
    import torch
    W = synth.weights(23, 4096, 4096, std=0.02)
    X = synth.activations(24, 1, 4096)
    Y0, wc, _, _ = gpu_chain(w4, X, W)
    ws = w4.mx_scale_layout(w4.fp4_quant(dev_bf16(W), w4.MXFP4)[1], 4096)
    xc, xs = w4.mxfp8_quant(dev_bf16(X), w4.MX_SCALES_MMA)
    for static in (False, True, False, True):
        assert torch.equal(w4.mx_gemm(xc, xs, wc, ws, weights_static=static), Y0)


@pytest.mark.gpu
@pytest.mark.parametrize("prob", synth.workload("mxdecode"), ids=lambda p: p.name)
def test_mx_decode_workload(w4, prob):
    """The decode layers (M = 1, K = 4096, N = 4096 / 11008 / 12288), every output."""
    check_product(w4, prob.X(), prob.W(), prob.name)


def sampled_rows(N: int, count: int, seed: int) -> np.ndarray:
    rows = np.random.default_rng(seed).choice(N, size=count, replace=False)
    return np.sort(np.concatenate([rows, [0, N - 1]]))


@pytest.mark.gpu
@pytest.mark.parametrize("wl,M", [("smallbatch", 16), ("smallbatch", 32), ("prefill", 512)])
def test_mx_large_shapes_on_sampled_rows(w4, wl, M):
    """Full-size products (N = 28672, K = 8192; N = 14336, K = 4096): every
    output of 384 sampled weight rows against the oracle (each output row of
    the oracle depends on its weight row only)."""
    prob = [p for p in synth.workload(wl) if p.M == M][0]
    W = prob.W()
    X = prob.X()
    Y = gpu_chain(w4, X, W)[0].float().cpu().numpy().astype(np.float64)
    rows = sampled_rows(prob.N, 384, M)
    Y_ref, Y_abs, _, _, _ = oracle_chain(X, np.ascontiguousarray(W[rows]))
    assert_y_elementwise(Y[:, rows], Y_ref, Y_abs, prob.K, prob.name)
    assert_y_close(Y[:, rows], Y_ref, prob.name)
