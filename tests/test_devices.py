"""Every kernel that opts into more than 48 KB of dynamic shared memory does
so per device (the attribute is a property of the current device).  The paths
run on device 0 and, when the machine has one, device 1, and must give the
same bits on both."""
import numpy as np
import pytest

from bit_gemm_quant_b200 import synth
from parity import dev_bf16


@pytest.fixture(scope="module")
def w4():
    from bit_gemm_quant_b200 import build
    build.build()
    import bit_gemm_quant_b200 as w4
    return w4


def run_all_paths(w4, device):
    import torch
    with torch.cuda.device(device):
        to = lambda bits: dev_bf16(bits).to(device)
        W = to(synth.weights(91, 512, 1024, 0.02, 0.01, 5.0))
        out = {}
        q, sc, z = w4.quant_pack(W, 128, 1)                                   # TMA quantizer
        out["qweight"] = q
        for M in (1, 64):                                                      # GEMV and tcgen05 paths
            X = to(synth.activations(92, M, 1024, 0.01, 40.0))
            out["Y%d" % M] = w4.gemm(X, q, sc, z, 128, 1)
        wc, ws_rows = w4.fp4_quant(W, w4.MXFP4)
        ws = w4.mx_scale_layout(ws_rows, 1024)
        for M in (1, 40):                                                      # MX decode form and cluster form
            X = to(synth.activations(93, M, 1024))
            xc, xs = w4.mxfp8_quant(X, w4.MX_SCALES_MMA)
            out["MX%d" % M] = w4.mx_gemm(xc, xs, wc, ws)
        torch.cuda.synchronize(device)
        return {k: v.cpu() for k, v in out.items()}


@pytest.mark.gpu
def test_every_large_shared_memory_path_on_each_device(w4):
    import torch
    n = min(2, torch.cuda.device_count())
    results = [run_all_paths(w4, d) for d in range(n)]
    # a repeated run on the first device after the others: its attribute is still set
    results.append(run_all_paths(w4, 0))
    for r in results[1:]:
        for k in results[0]:
            assert torch.equal(results[0][k], r[k]), k
