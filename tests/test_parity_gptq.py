"""w4_gptq on the GPU against the GPTQ oracle (oracle/gptq.py).

The GPU computes the same fp64 procedure in another summation order (a
reversed-index Cholesky and a triangular inverse instead of an explicit
inverse and a second Cholesky; the later columns updated 32 at a time), so a
code may differ where a value lies within rounding of a decision boundary,
and the differences can cascade along a row.  The criteria:
  * codes: at least 99.9% equal to the oracle's, scales at least 99.9%;
  * the output error ||W X^T - W^ X^T|| / ||W X^T|| within 1% of the oracle's;
  * on correlated calibration features GPTQ's output error is well below
    round-to-nearest's (page 5 section 2.5, Scene 4, qualitatively);
  * with no calibration signal (X = 0) GPTQ is plain rounding: every byte
    equals w4_quant_pack's (the already pinned quantizer).
"""
import numpy as np
import pytest

import oracle
from oracle import gptq as ogptq
from bit_gemm_quant_b200 import synth
from parity import THREADS, assert_codes_equal, dev_bf16, host_u16, host_u32

SYM, ASYM = 0, 1


@pytest.fixture(scope="module")
def w4():
    from bit_gemm_quant_b200 import build
    build.build()
    import bit_gemm_quant_b200 as w4
    oracle.build()
    return w4


def unpack_codes(qweight: np.ndarray) -> np.ndarray:
    N, W = qweight.shape
    u = np.zeros((N, W * 8), dtype=np.int64)
    for e in range(8):
        shift = 4 * (e // 2) + (16 if e % 2 else 0)
        u[:, e::8] = (qweight >> np.uint32(shift)) & np.uint32(15)
    return u


def unpack_zeros(qzeros: np.ndarray, G: int) -> np.ndarray:
    j = np.arange(G)
    return ((qzeros[:, j // 8] >> (4 * (j % 8)).astype(np.uint32)) & np.uint32(15)).astype(np.int64)


def correlated_calibration(seed: int, M: int, K: int, rank: int = 8) -> np.ndarray:
    """Calibration rows whose features share a few directions (plus a little
    noise), so that the Hessian couples columns strongly."""
    rng = np.random.default_rng(seed)
    B = rng.standard_normal((rank, K)).astype(np.float32)
    A = rng.standard_normal((M, rank)).astype(np.float32)
    X = A @ B + 0.1 * rng.standard_normal((M, K)).astype(np.float32)
    return synth.to_bf16_bits(X)


def gpu_gptq(w4, W, X, g, mode):
    import torch
    q, sc, z = w4.gptq(dev_bf16(W), dev_bf16(X), g, mode)
    torch.cuda.synchronize()
    return host_u32(q), host_u16(sc), (host_u32(z) if z is not None else None)


def output_error(W, u, s16, zp, g, X):
    return ogptq.output_error(W, ogptq.dequantize(u, s16, zp, g), X)


CASES = [
    # N, K, M, g, mode, calibration
    (64, 256, 64, 32, SYM, "normal"),
    (96, 512, 128, 64, ASYM, "correlated"),
    (200, 1024, 256, 128, ASYM, "correlated"),
    (128, 512, 48, 128, SYM, "correlated"),      # M < K: X^T X is rank deficient, the damping carries it
    (33, 384, 100, 128, ASYM, "outliers"),       # ragged row count
]


@pytest.mark.gpu
@pytest.mark.parametrize("N,K,M,g,mode,calib", CASES)
def test_gptq_matches_the_oracle(w4, N, K, M, g, mode, calib):
    W = synth.weights(61, N, K, 0.02, 0.01, 5.0)
    if calib == "normal":
        X = synth.activations(62, M, K)
    elif calib == "outliers":
        X = synth.activations(62, M, K, 0.01, 40.0)
    else:
        X = correlated_calibration(62, M, K)
    q, sc, z = gpu_gptq(w4, W, X, g, mode)
    u_ref, s_ref, zp_ref = ogptq.gptq_quantize(W, X, g, mode)
    u = unpack_codes(q)
    zp = unpack_zeros(z, K // g) if mode == ASYM else np.full(sc.shape, 8, dtype=np.int64)
    code_agree = float(np.mean(u == u_ref))
    scale_agree = float(np.mean(sc == s_ref))
    assert code_agree >= 0.999, "codes agree on %.5f" % code_agree
    assert scale_agree >= 0.999, "scales agree on %.5f" % scale_agree
    if mode == ASYM:
        assert float(np.mean(zp == zp_ref)) >= 0.999
    err = output_error(W, u, sc, zp, g, X)
    err_ref = output_error(W, u_ref, s_ref, zp_ref, g, X)
    assert abs(err - err_ref) <= 0.01 * err_ref, (err, err_ref)
    if calib == "correlated":
        # plain rounding of the same weights (the pinned quantizer)
        qr, sr, zr = oracle.quant_pack(W, g, mode, threads=THREADS)
        zr_u = unpack_zeros(zr, K // g) if mode == ASYM else np.full(sr.shape, 8, dtype=np.int64)
        err_rtn = output_error(W, unpack_codes(qr), sr, zr_u, g, X)
        assert err < 0.8 * err_rtn, (err, err_rtn)


@pytest.mark.gpu
@pytest.mark.parametrize("mode", [SYM, ASYM])
def test_gptq_without_calibration_signal_is_plain_rounding(w4, mode):
    N, K, g = 80, 512, 64
    W = synth.weights(63, N, K, 0.02, 0.01, 5.0)
    X = np.zeros((16, K), dtype=np.uint16)
    q, sc, z = gpu_gptq(w4, W, X, g, mode)
    oq, osc, oz = oracle.quant_pack(W, g, mode, threads=THREADS)
    assert_codes_equal(q, oq, "qweight")
    assert_codes_equal(sc, osc, "scales")
    if mode == ASYM:
        assert_codes_equal(z, oz, "qzeros")


@pytest.mark.gpu
def test_gptq_repeats_bit_for_bit(w4):
    W = synth.weights(64, 128, 512, 0.02)
    X = correlated_calibration(65, 64, 512)
    a = gpu_gptq(w4, W, X, 128, ASYM)
    b = gpu_gptq(w4, W, X, 128, ASYM)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
