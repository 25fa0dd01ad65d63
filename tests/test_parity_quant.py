"""w4_quant_pack on the GPU against the CPU oracle: every byte of codes,
scales and zero-points must match."""
import numpy as np
import pytest

import oracle
from bit_gemm_quant_b200 import synth
from parity import THREADS, assert_codes_equal, dev_bf16, dev_f32, host_u16, host_u32

SYM, ASYM = 0, 1


@pytest.fixture(scope="module")
def w4():
    from bit_gemm_quant_b200 import build
    build.build()
    import bit_gemm_quant_b200 as w4
    oracle.build()
    return w4


def run_both(w4, W_bits, g, mode, s=None):
    import torch
    Wd = dev_bf16(W_bits)
    sd = dev_f32(s) if s is not None else None
    q, sc, z = w4.quant_pack(Wd, g, mode, s=sd)
    torch.cuda.synchronize()
    oq, osc, oz = oracle.quant_pack(W_bits, g, mode, s=s, threads=THREADS)
    assert_codes_equal(host_u32(q), oq, "qweight")
    assert_codes_equal(host_u16(sc), osc, "scales")
    if mode == ASYM:
        assert_codes_equal(host_u32(z), oz, "qzeros")
    else:
        assert z is None


SMALL = [  # (N, K, g) including ragged row lengths (K not a multiple of 256 or 1024)
    (1, 32, 32), (3, 96, 32), (7, 192, 64), (16, 128, 128), (33, 1088, 64),
    (5, 1280, 128), (64, 4096, 128), (17, 8448, 32),
]


@pytest.mark.gpu
@pytest.mark.parametrize("N,K,g", SMALL)
@pytest.mark.parametrize("mode", [SYM, ASYM])
@pytest.mark.parametrize("fold", [False, True])
def test_quant_pack_small_and_ragged(w4, N, K, g, mode, fold):
    W = synth.weights(N * 7 + K, N, K, 0.02, 0.05, 8.0)
    s = synth.smoothing_vector(K, K) if fold else None
    run_both(w4, W, g, mode, s)


def tie_rows(g, mode):
    """Rows whose groups hold exact ties x = (n + 1/2) d and their bf16 neighbours."""
    import torch
    if mode == SYM:
        d, top = 0.75, 5.25           # amax = 7 d -> s16 = d exactly
        ends = [top, -top]
    else:
        d, top = 0.25, 1.875          # range 15 d, zp = rint(7.5) = 8
        ends = [top, -top]
    vals = []
    for n in range(-7, 7):
        x = np.float32((n + 0.5) * d)
        xb = torch.tensor([x]).to(torch.bfloat16)
        up = torch.nextafter(xb.float(), torch.tensor([np.inf])).to(torch.bfloat16)
        vals += [float(xb), float(xb.view(torch.int16).add(1).view(torch.bfloat16)),
                 float(xb.view(torch.int16).sub(1).view(torch.bfloat16)), float(up)]
    rows = []
    per = g - 2
    for a in range(0, len(vals), per):
        grp = np.zeros(g, np.float32)
        chunk = vals[a:a + per]
        grp[:len(chunk)] = chunk
        grp[g - 2], grp[g - 1] = ends
        rows.append(grp)
    W = np.concatenate(rows).reshape(1, -1)
    K = W.shape[1]
    K8 = ((K + 255) // 256) * 256
    W = np.pad(W, ((0, 0), (0, K8 - K)))
    W = np.repeat(W, 4, axis=0)
    return synth.to_bf16_bits(W)


@pytest.mark.gpu
@pytest.mark.parametrize("g", [32, 64, 128])
@pytest.mark.parametrize("mode", [SYM, ASYM])
def test_quant_pack_exact_ties(w4, g, mode):
    W = tie_rows(g, mode)
    run_both(w4, W, g, mode)
    # the same rows with a smoothing fold whose products land near ties in fp32
    K = W.shape[1]
    s = (1.0 + (np.arange(K) % 7 - 3) * 2.0 ** -20).astype(np.float32)
    run_both(w4, W, g, mode, s)


@pytest.mark.gpu
@pytest.mark.parametrize("mode", [SYM, ASYM])
def test_quant_pack_degenerate_groups(w4, mode):
    K, g = 256, 32
    W = np.zeros((6, K), np.float32)
    W[1, :] = 1e-8                       # fp16 underflow of the scale
    W[2, :32] = 3.0e5                    # scale saturates at 65504
    W[2, 32:64] = -2.0e6
    W[3, :] = np.linspace(-1, 1, K)
    W[4, ::2] = 0.5                      # single-signed groups
    W[5, :] = -np.abs(np.linspace(-3, 3, K))
    run_both(w4, synth.to_bf16_bits(W), g, mode)


@pytest.mark.gpu
@pytest.mark.parametrize("prob", synth.workload("quantizer"), ids=lambda p: p.name)
def test_quant_pack_quantizer_workload_full_size(w4, prob):
    """The quantizer sweep at full size, W[28672, 8192]: every byte."""
    run_both(w4, prob.W(), prob.group, prob.mode, prob.s())


@pytest.mark.gpu
@pytest.mark.parametrize("prob", synth.workload("decode") + synth.workload("tiny"), ids=lambda p: p.name)
def test_quant_pack_decode_and_tiny_weights(w4, prob):
    run_both(w4, prob.W(), prob.group, prob.mode, prob.s())
