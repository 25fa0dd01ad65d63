"""w4a16_gemm on the GPU against the CPU oracle's fp64 product with the
dequantized weights: relative Frobenius error <= 2e-3 and max error <=
1e-2 * max|Y_ref| (the output is rounded to bf16, which alone accounts for
about 1.6e-3 of relative Frobenius error)."""
import numpy as np
import pytest

import oracle
from bit_gemm_quant_b200 import synth
from parity import THREADS, assert_y_close, assert_y_elementwise, dev_bf16, host_bf16_as_f64

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


def oracle_abs(W_bits, X_bits, g, mode):
    K = W_bits.shape[1]
    oq, osc, oz = oracle.quant_pack(W_bits, g, mode, threads=THREADS)
    return oracle.w4a16_abs_reference(X_bits, oq, osc, oz, K, g, mode, threads=THREADS)


def check(Y, W, X, g, mode):
    """Every output within the rigorous rounding bound; outputs of >= 1024
    elements also within the relative Frobenius / max criteria."""
    Y_ref = oracle_ref(W, X, g, mode)
    assert_y_elementwise(Y, Y_ref, oracle_abs(W, X, g, mode), W.shape[1])
    if Y.size >= 1024:
        assert_y_close(Y, Y_ref)


@pytest.mark.gpu
@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 9, 13, 16])
@pytest.mark.parametrize("g", [32, 64, 128])
@pytest.mark.parametrize("mode", [SYM, ASYM])
def test_gemv_small_ragged_shapes(w4, M, g, mode):
    # N not a multiple of the 16-channel tile, K not a multiple of the 256-wide k-box
    N, K = 200, 640 if g != 128 else 1152
    W = synth.weights(M + g, N, K, 0.02, 0.01, 5.0)
    X = synth.activations(M + g, M, K, 0.01, 40.0)
    check(gpu_path(w4, W, X, g, mode), W, X, g, mode)


@pytest.mark.gpu
@pytest.mark.parametrize("N,K", [(1, 128), (15, 256), (17, 512), (16, 8192)])
def test_gemv_edge_sizes(w4, N, K):
    W = synth.weights(N + K, N, K, 0.02)
    X = synth.activations(N + K, 3, K)
    check(gpu_path(w4, W, X, 128, ASYM), W, X, 128, ASYM)


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K", [(1, 4800, 8192), (7, 1000, 2304), (12, 37904, 256)])
def test_gemv_more_shapes(w4, M, N, K):
    """Long rows (K = 8192), a ragged K (2304 = 9 k-boxes) and many one-box rows
    (K = 256, N = 37904 channels: 2369 tiles, more than one resident wave)."""
    W = synth.weights(N + K + M, N, K, 0.02, 0.01, 5.0)
    X = synth.activations(N + K + M, M, K, 0.01, 40.0)
    check(gpu_path(w4, W, X, 128, ASYM), W, X, 128, ASYM)


@pytest.mark.gpu
@pytest.mark.parametrize("M", [1, 12])
def test_gemv_is_deterministic(w4, M):
    """Repeated calls give the same bits."""
    import torch
    N, K = 4096, 4096
    W = synth.weights(93 + M, N, K, 0.02)
    X = synth.activations(93 + M, M, K, 0.01, 40.0)
    q, sc, z = w4.quant_pack(dev_bf16(W), 128, ASYM)
    Xd = dev_bf16(X)
    Ys = [host_bf16_as_f64(w4.gemm(Xd, q, sc, z, 128, ASYM)) for _ in range(5)]
    torch.cuda.synchronize()
    assert all(np.array_equal(Ys[0], Y) for Y in Ys[1:])
    check(Ys[0], W, X, 128, ASYM)
    assert w4.w4_device_error() == 0


@pytest.mark.gpu
def test_tiny_workload(w4):
    (p,) = synth.workload("tiny")
    W, X = p.W(), p.X()
    check(gpu_path(w4, W, X, p.group, p.mode), W, X, p.group, p.mode)


@pytest.mark.gpu
@pytest.mark.parametrize("prob", synth.workload("decode"), ids=lambda p: p.name)
def test_decode_workload_full(w4, prob):
    """M = 1, K = 4096, N in {4096, 11008, 12288}: every output."""
    W, X = prob.W(), prob.X()
    check(gpu_path(w4, W, X, prob.group, prob.mode), W, X, prob.group, prob.mode)


TC_SHAPES = [  # (M, N, K): every token-tile width, channels not a multiple of 128, split-K for few tiles
    # (M <= 16 runs the GEMV's two-token-group kernel, M >= 17 the tensor-core kernel)
    (9, 300, 1024), (16, 256, 4096), (17, 130, 2048), (20, 300, 1024), (24, 256, 4096), (32, 512, 1024), (33, 384, 640), (64, 200, 4096),
    (100, 256, 512), (128, 128, 8192), (129, 640, 1024), (256, 384, 1024), (300, 256, 640), (512, 1024, 1024),
]


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K", TC_SHAPES)
@pytest.mark.parametrize("g,mode", [(128, ASYM), (64, SYM), (32, ASYM)])
def test_tc_shapes(w4, M, N, K, g, mode):
    W = synth.weights(M * 3 + N, N, K, 0.02, 0.01, 5.0)
    X = synth.activations(M * 3 + N, M, K, 0.01, 40.0)
    check(gpu_path(w4, W, X, g, mode), W, X, g, mode)


@pytest.mark.gpu
@pytest.mark.parametrize("M", [12, 40, 200])
def test_tc_k_tail(w4, M):
    """K = 2080 ends with half a 64-wide k-block (g = 32)."""
    N, K = 160, 2080
    W = synth.weights(M + 5, N, K, 0.02)
    X = synth.activations(M + 5, M, K, 0.01, 40.0)
    check(gpu_path(w4, W, X, 32, SYM), W, X, 32, SYM)


@pytest.mark.gpu
def test_tc_workspace_is_left_zeroed_and_reusable(w4):
    """Split-K calls leave their counters zeroed: the same workspace serves repeated calls."""
    import torch
    M, N, K = 24, 256, 4096                      # M > 16: the tensor-core path, split over k
    need = w4.w4a16_workspace_bytes(M, N, K, 128)
    assert need > 0
    W = synth.weights(91, N, K, 0.02)
    X = synth.activations(91, M, K)
    q, sc, z = w4.quant_pack(dev_bf16(W), 128, ASYM)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    Xd = dev_bf16(X)
    Ys = [host_bf16_as_f64(w4.gemm(Xd, q, sc, z, 128, ASYM, workspace=ws)) for _ in range(3)]
    torch.cuda.synchronize()
    counters_tail = ws[-((N + 127) // 128) * 4:].cpu()
    assert int(counters_tail.sum()) == 0
    assert np.array_equal(Ys[0], Ys[1]) and np.array_equal(Ys[1], Ys[2])
    check(Ys[0], W, X, 128, ASYM)
    assert w4.w4_device_error() == 0


_ORACLE_PACKED = {}


def oracle_packed(prob):
    """The oracle's quantization of a workload weight, computed once per weight
    (the small-batch problems share one W[28672, 8192])."""
    key = (prob.seed, prob.N, prob.K, prob.group, prob.mode, prob.w_std, prob.w_outlier)
    if key not in _ORACLE_PACKED:
        _ORACLE_PACKED.clear()
        W = prob.W()
        _ORACLE_PACKED[key] = (W, oracle.quant_pack(W, prob.group, prob.mode, threads=THREADS))
    return _ORACLE_PACKED[key]


def check_full_or_rows(w4, prob, rows=None):
    """Every output channel of the given rows (all rows when None) against the
    oracle: the per-element rounding bound, and the relative Frobenius and max
    criteria."""
    W, (oq, osc, oz) = oracle_packed(prob)
    X = prob.X()
    Y = gpu_path(w4, W, X, prob.group, prob.mode)
    Xr = X if rows is None else X[rows]
    Yg = Y if rows is None else Y[rows]
    Y_ref = oracle.w4a16_reference(Xr, oq, osc, oz, prob.K, prob.group, prob.mode, threads=THREADS)
    Y_abs = oracle.w4a16_abs_reference(Xr, oq, osc, oz, prob.K, prob.group, prob.mode, threads=THREADS)
    assert_y_elementwise(Yg, Y_ref, Y_abs, prob.K)
    assert_y_close(Yg, Y_ref)
    assert w4.w4_device_error() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("prob", synth.workload("prefill"), ids=lambda p: p.name)
def test_prefill_workload(w4, prob):
    """K = 4096, N = 14336 at full size: every output of M = 512; every channel
    of 256 seeded rows at M = 2048 and 8192."""
    rows = None if prob.M <= 512 else np.sort(np.random.default_rng(78).choice(prob.M, 256, replace=False))
    check_full_or_rows(w4, prob, rows)


@pytest.mark.gpu
@pytest.mark.parametrize("prob", synth.workload("smallbatch"), ids=lambda p: p.name)
def test_smallbatch_workload_full(w4, prob):
    """K = 8192, N = 28672 at full size, M = 2..32: every output."""
    check_full_or_rows(w4, prob)


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K,g,mode", [(1, 4096, 4096, 128, ASYM), (1, 12288, 4096, 128, ASYM),
                                           (1, 11008, 4096, 128, ASYM), (4, 200, 1152, 128, SYM),
                                           (8, 28672, 8192, 128, SYM), (13, 1000, 2304, 64, ASYM),
                                           (2, 37904, 256, 32, SYM)])
def test_weights_static_flag_gives_the_same_bits(w4, M, N, K, g, mode):
    """W4_WEIGHTS_STATIC only lets the weight stream start before the previous
    kernel on the stream finishes: with the weight quantized (and synchronized)
    beforehand, the flagged product gives exactly the unflagged bits, on every
    launch shape of the GEMV (few tiles, five and six tiles per SM, two token
    groups, one-box rows), in a chain of back-to-back products."""
    import torch
    W = synth.weights(M + N + K, N, K, 0.02, 0.01, 5.0)
    X = synth.activations(M + N + K, M, K, 0.01, 40.0)
    q, sc, z = w4.quant_pack(dev_bf16(W), g, mode)
    Xd = dev_bf16(X)
    torch.cuda.synchronize()
    ref = host_bf16_as_f64(w4.gemm(Xd, q, sc, z, g, mode))
    outs = [w4.gemm(Xd, q, sc, z, g, mode, weights_static=True) for _ in range(4)]
    torch.cuda.synchronize()
    for Y in outs:
        assert np.array_equal(host_bf16_as_f64(Y), ref)
    assert w4.w4_device_error() == 0
    if M * N <= 300000:
        check(ref, W, X, g, mode)
