"""w4_awq_search on the GPU against the oracle's search (page 2, AWQ section):
every alpha's loss within 1e-3 (relative), the chosen alpha optimal for the
oracle too (a near-tie may pick the other index), and s for it as the oracle
computes it."""
import numpy as np
import pytest

from oracle import awq
from bit_gemm_quant_b200 import synth
from parity import THREADS, dev_bf16

SYM, ASYM = 0, 1
CASES = [  # (M, N, K, g, mode): the GEMV path, the tensor-core path with split K, ragged N
    (8, 128, 1024, 32, ASYM),
    (24, 200, 640, 64, ASYM),
    (64, 256, 512, 128, SYM),
]


@pytest.fixture(scope="module")
def w4():
    from bit_gemm_quant_b200 import build
    build.build()
    import bit_gemm_quant_b200 as w4
    w4.lib()
    return w4


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K,g,mode", CASES)
def test_awq_search_matches_oracle(w4, M, N, K, g, mode):
    import torch
    W = synth.weights(M + N + K, N, K, 0.02, 0.01, 5.0)
    X = synth.activations(M + N, M, K, 0.02, 40.0)
    n_alpha = 12
    losses, best, s_best = w4.awq_search(dev_bf16(W), dev_bf16(X), g, mode, n_alpha=n_alpha)
    torch.cuda.synchronize()
    losses = losses.cpu().numpy()
    best = int(best.cpu().numpy()[0])
    s_best = s_best.cpu().numpy()
    ref, ref_best, _ = awq.awq_losses(W, X, g, mode, n_alpha=n_alpha, threads=THREADS)
    assert np.all(np.isfinite(losses))
    np.testing.assert_allclose(losses, ref, rtol=1e-3, atol=0)
    assert ref[best] <= ref[ref_best] * (1 + 2e-3), (best, ref_best)
    s_ref = awq.smoothing(awq.act_magnitude(X), awq.alphas(n_alpha)[best])
    np.testing.assert_allclose(s_best, s_ref, rtol=2e-7, atol=0)
    assert w4.w4_device_error() == 0
