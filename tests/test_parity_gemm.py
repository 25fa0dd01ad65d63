"""w4a16_gemm on the GPU against the CPU oracle's fp64 product with the
dequantized weights: relative Frobenius error <= 2e-3 and max error <=
1e-2 * max|Y_ref| (the output is rounded to bf16, which alone accounts for
about 1.6e-3 of relative Frobenius error)."""
import numpy as np
import pytest

import oracle
from bit_gemm_quant_b200 import synth
from parity import THREADS, assert_y_close, dev_bf16, host_bf16_as_f64

SYM, ASYM = 0, 1


@pytest.fixture(scope="module")
def w4():
    from bit_gemm_quant_b200 import build
    build.build()
    import bit_gemm_quant_b200 as w4
    oracle.build()
    return w4


def gpu_path(w4, W_bits, X_bits, g, mode):
    """Quantize on the GPU, then multiply on the GPU (the product path)."""
    import torch
    q, sc, z = w4.quant_pack(dev_bf16(W_bits), g, mode)
    Y = w4.gemm(dev_bf16(X_bits), q, sc, z, g, mode)
    torch.cuda.synchronize()
    return host_bf16_as_f64(Y)


def oracle_ref(W_bits, X_bits, g, mode, channels=None):
    K = W_bits.shape[1]
    oq, osc, oz = oracle.quant_pack(W_bits, g, mode, threads=THREADS)
    return oracle.w4a16_reference(X_bits, oq, osc, oz, K, g, mode, channels=channels, threads=THREADS)


@pytest.mark.gpu
@pytest.mark.parametrize("M", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("g", [32, 64, 128])
@pytest.mark.parametrize("mode", [SYM, ASYM])
def test_gemv_small_ragged_shapes(w4, M, g, mode):
    # N not a multiple of the 16-channel tile, K not a multiple of the 512-wide super-chunk
    N, K = 200, 640 if g != 128 else 1152
    W = synth.weights(M + g, N, K, 0.02, 0.01, 5.0)
    X = synth.activations(M + g, M, K, 0.01, 40.0)
    Y = gpu_path(w4, W, X, g, mode)
    assert_y_close(Y, oracle_ref(W, X, g, mode))


@pytest.mark.gpu
@pytest.mark.parametrize("N,K", [(1, 128), (15, 256), (17, 512), (16, 8192)])
def test_gemv_edge_sizes(w4, N, K):
    W = synth.weights(N + K, N, K, 0.02)
    X = synth.activations(N + K, 3, K)
    assert_y_close(gpu_path(w4, W, X, 128, ASYM), oracle_ref(W, X, 128, ASYM))


@pytest.mark.gpu
def test_tiny_workload(w4):
    (p,) = synth.workload("tiny")
    W, X = p.W(), p.X()
    assert_y_close(gpu_path(w4, W, X, p.group, p.mode), oracle_ref(W, X, p.group, p.mode))


@pytest.mark.gpu
@pytest.mark.parametrize("prob", synth.workload("decode"), ids=lambda p: p.name)
def test_decode_workload_full(w4, prob):
    """M = 1, K = 4096, N in {4096, 11008, 12288}: every output."""
    W, X = prob.W(), prob.X()
    assert_y_close(gpu_path(w4, W, X, prob.group, prob.mode), oracle_ref(W, X, prob.group, prob.mode))


@pytest.mark.gpu
@pytest.mark.parametrize("prob", [p for p in synth.workload("smallbatch") if p.M <= 8], ids=lambda p: p.name)
def test_smallbatch_workload_sampled(w4, prob):
    """K = 8192, N = 28672 at full size; the oracle checks a seeded sample of 1024 channels."""
    W, X = prob.W(), prob.X()
    Y = gpu_path(w4, W, X, prob.group, prob.mode)
    ch = np.sort(np.random.default_rng(77).choice(prob.N, 1024, replace=False))
    assert_y_close(Y[:, ch], oracle_ref(W, X, prob.group, prob.mode, channels=ch))
