"""w4_repack and the GEMV on repacked codes (W4_REPACKED).

The repack is a permutation of words, checked against its definition written
out in numpy; the GEMV on the repacked codes must give every bit of Y that it
gives on the canonical layout (the same boxes land in shared memory), and Y is
checked against the oracle once more on its own.
"""
import numpy as np
import pytest

import oracle
from bit_gemm_quant_b200 import synth
from parity import THREADS, assert_codes_equal, assert_y_elementwise, dev_bf16, host_bf16_as_f64

SYM, ASYM = 0, 1


@pytest.fixture(scope="module")
def w4():
    from bit_gemm_quant_b200 import build
    build.build()
    import bit_gemm_quant_b200 as w4
    oracle.build()
    return w4


def repack_reference(q: np.ndarray, N: int, K: int) -> np.ndarray:
    """Word kw of channel n at (((n/16) * (K/256) + kw/32) * 16 + n%16) * 32 + kw%32."""
    KW, KC = K // 8, K // 256
    Np = (N + 15) // 16 * 16
    out = np.zeros(Np * KW, dtype=np.uint32)
    n = np.arange(N)[:, None]
    kw = np.arange(KW)[None, :]
    idx = (((n // 16) * KC + kw // 32) * 16 + n % 16) * 32 + kw % 32
    out[idx] = q
    return out


@pytest.mark.gpu
@pytest.mark.parametrize("N,K", [(16, 256), (1000, 512), (37, 4096), (4096, 4352)])
def test_repack_is_the_defined_permutation(w4, N, K):
    import torch
    q = np.random.default_rng(N + K).integers(0, 2 ** 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    qd = torch.from_numpy(q.view(np.int32)).cuda()
    out = w4.repack(qd, N, K)
    torch.cuda.synchronize()
    assert_codes_equal(out.cpu().numpy().view(np.uint32), repack_reference(q, N, K), "repacked words")


CASES = [
    # M, N, K, g, mode
    (1, 4096, 4096, 128, ASYM),
    (1, 11008, 4096, 128, ASYM),
    (1, 12288, 4096, 128, ASYM),
    (4, 1000, 4352, 64, SYM),       # ragged N, and K/256 odd: the last 512-k stage's second box is out of range
    (16, 28672, 8192, 128, SYM),
    (8, 300, 2048, 32, ASYM),
]


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K,g,mode", CASES)
def test_gemv_on_repacked_codes_gives_the_same_bits(w4, M, N, K, g, mode):
    import torch
    W = synth.weights(71 + M, N, K, 0.02, 0.01, 5.0)
    X = synth.activations(72 + M, M, K, 0.01, 40.0)
    q, sc, z = w4.quant_pack(dev_bf16(W), g, mode)
    rq = w4.repack(q, N, K)
    Xd = dev_bf16(X)
    for static in (False, True):
        Y0 = w4.gemm(Xd, q, sc, z, g, mode, weights_static=static)
        Y1 = w4.gemm(Xd, rq, sc, z, g, mode, N=N, weights_static=static, repacked=True)
        assert torch.equal(Y0, Y1)
    F0 = w4.gemm(Xd, q, sc, z, g, mode, out_f32=True)
    F1 = w4.gemm(Xd, rq, sc, z, g, mode, N=N, out_f32=True, repacked=True)
    assert torch.equal(F0, F1)
    if N <= 4096:
        torch.cuda.synchronize()
        oq, osc, oz = oracle.quant_pack(W, g, mode, threads=THREADS)
        Y_ref = oracle.w4a16_reference(X, oq, osc, oz, K, g, mode, threads=THREADS)
        Y_abs = oracle.w4a16_abs_reference(X, oq, osc, oz, K, g, mode, threads=THREADS)
        assert_y_elementwise(host_bf16_as_f64(Y1), Y_ref, Y_abs, K, "Y from repacked codes")
