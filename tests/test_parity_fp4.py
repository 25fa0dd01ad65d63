"""w4_fp4_quant on the GPU against the CPU oracle: every code byte and every
scale byte must match, for NVFP4 (blocks of 16, E4M3 scales) and MXFP4
(blocks of 32, E8M0 scales)."""
import numpy as np
import pytest

import oracle
from bit_gemm_quant_b200 import synth
from parity import assert_codes_equal, dev_bf16

NVFP4, MXFP4 = 0, 1
KINDS = [NVFP4, MXFP4]


@pytest.fixture(scope="module")
def w4():
    from bit_gemm_quant_b200 import build
    build.build()
    import bit_gemm_quant_b200 as w4
    oracle.build()
    return w4


def run_both(w4, W_bits, kind):
    import torch
    codes, scales = w4.fp4_quant(dev_bf16(W_bits), kind)
    torch.cuda.synchronize()
    oc, osc = oracle.fp4_quant(W_bits, kind)
    assert_codes_equal(codes.cpu().numpy(), oc, "codes")
    assert_codes_equal(scales.cpu().numpy(), osc, "scales")


@pytest.mark.gpu
@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("N,K", [(1, 32), (3, 96), (37, 160), (64, 4096), (5, 8224), (129, 1056)])
def test_random_weights(w4, kind, N, K):
    W = synth.weights(11, N, K, std=0.02, outlier_frac=0.01)
    run_both(w4, W, kind)


@pytest.mark.gpu
@pytest.mark.parametrize("kind", KINDS)
def test_every_tie_and_the_saturation_edge(w4, kind):
    # amax = 6 gives the scale 1 in both formats (6/6 = 1 in E4M3; 2^(2-2) in
    # E8M0), so w / s = w exactly: the row holds every midpoint between
    # neighbouring E2M1 values, points just beside them, and both signs.
    mids = synth.to_bf16_bits(np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32))
    vals = []
    for m in mids.astype(np.int64):          # the tie, its bf16 neighbours, both signs
        for b in (m, m - 1, m + 1):
            vals += [b, b | 0x8000]
    six = int(synth.to_bf16_bits(np.array([6.0], dtype=np.float32))[0])
    B = 16 if kind == NVFP4 else 32
    row = []
    for start in range(0, len(vals), B - 1):
        chunk = vals[start:start + B - 1] + [six]
        row += chunk + [0] * (B - len(chunk))
    W = np.array(row, dtype=np.uint16).reshape(1, -1)
    run_both(w4, W, kind)


@pytest.mark.gpu
@pytest.mark.parametrize("kind", KINDS)
def test_zero_blocks_signed_zeros_and_tiny_values(w4, kind):
    rng = np.random.default_rng(5)
    K = 256
    W = np.zeros((6, K), dtype=np.float32)
    W[1] = -0.0
    W[2] = rng.standard_normal(K) * 1e-38          # bf16 subnormals and near-subnormals
    W[3] = rng.standard_normal(K) * 1e-3
    W[3, ::32] = 0.0
    W[4, :K // 2] = -0.0
    W[4, K // 2:] = rng.standard_normal(K // 2) * 3e-6   # E4M3 scale rounds to 0 or a subnormal
    W[5] = rng.standard_normal(K) * 1e-8
    run_both(w4, synth.to_bf16_bits(W), kind)


@pytest.mark.gpu
@pytest.mark.parametrize("kind", KINDS)
def test_large_magnitudes_saturate(w4, kind):
    rng = np.random.default_rng(6)
    K = 128
    W = np.zeros((4, K), dtype=np.float32)
    W[0] = rng.standard_normal(K) * 1e3             # NVFP4 scale above 448 saturates
    W[1] = rng.standard_normal(K) * 1e30
    W[2] = rng.standard_normal(K) * 1e38            # MXFP4 exponent near the top of E8M0
    W[3] = np.where(rng.random(K) < 0.5, 3e38, -3e38)
    run_both(w4, synth.to_bf16_bits(W), kind)


@pytest.mark.gpu
@pytest.mark.parametrize("kind", KINDS)
def test_decode_size_matrix(w4, kind):
    # one projection of the decode workload's size class, every byte compared
    W = synth.weights(12, 4096, 12288, std=0.02, outlier_frac=0.01)
    run_both(w4, W, kind)


@pytest.mark.gpu
def test_rejects_bad_arguments(w4):
    import torch
    W = torch.zeros((4, 48), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(w4.W4Error):
        w4.fp4_quant(W, MXFP4)                      # K not a multiple of 32
    with pytest.raises(w4.W4Error):
        w4.fp4_quant(W, 7)                          # unknown kind
