"""The failure path of the bounded waits, exercised without a fault.

Every wait of a kernel on a copy, an MMA or another warp gives up after a time
limit, records a code in the library's error word and ends the kernel early
(after letting its own copies and MMAs finish, so that shared and tensor
memory are released).  These tests lower the limit to 1 us
(w4_set_wait_limit_ns) and point each warp's first wait at a barrier that
nothing completes (w4_test_stall_first_wait), so that it runs out
deterministically; they check the recorded code, restore the limit, and
check that the next call on the same data is correct (for the tensor-core
kernel this also shows that tensor memory was freed: a leaked allocation would
stall the next launch's allocation)."""
import numpy as np
import pytest

import oracle
from bit_gemm_quant_b200 import synth
from parity import THREADS, assert_codes_equal, assert_y_close, dev_bf16, host_bf16_as_f64, host_u16, host_u32

SYM, ASYM = 0, 1


@pytest.fixture(scope="module")
def w4():
    from bit_gemm_quant_b200 import build
    build.build()
    import bit_gemm_quant_b200 as w4
    oracle.build()
    return w4


def run_with_short_limit(w4, fn):
    import torch
    torch.cuda.synchronize()
    assert w4.w4_device_error() == 0
    w4.w4_set_wait_limit_ns(1000)             # 1 us
    w4.w4_test_stall_first_wait(1)
    try:
        fn()
        torch.cuda.synchronize()
        code = w4.w4_device_error()
    finally:
        w4.w4_test_stall_first_wait(0)
        w4.w4_set_wait_limit_ns(0)
    return code


def product_ref(W, X, g, mode):
    K = W.shape[1]
    q, sc, z = oracle.quant_pack(W, g, mode, threads=THREADS)
    return oracle.w4a16_reference(X, q, sc, z, K, g, mode, threads=THREADS)


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K,lo,hi", [(1, 4096, 4096, 0x201, 0x202), (64, 1024, 2048, 0x101, 0x106)],
                         ids=["gemv", "tensor_core"])
def test_product_wait_runs_out_then_next_call_is_correct(w4, M, N, K, lo, hi):
    import torch
    W = synth.weights(7 + M, N, K, 0.02, 0.01, 5.0)
    X = synth.activations(7 + M, M, K, 0.01, 40.0)
    q, sc, z = w4.quant_pack(dev_bf16(W), 128, ASYM)
    Xd = dev_bf16(X)
    ws = torch.zeros(max(w4.w4a16_workspace_bytes(M, N, K, 128), 256), dtype=torch.uint8, device="cuda")
    code = run_with_short_limit(w4, lambda: w4.gemm(Xd, q, sc, z, 128, ASYM, workspace=ws))
    assert lo <= code <= hi, hex(code)
    Y = host_bf16_as_f64(w4.gemm(Xd, q, sc, z, 128, ASYM, workspace=ws))
    torch.cuda.synchronize()
    assert w4.w4_device_error() == 0
    assert_y_close(Y, product_ref(W, X, 128, ASYM))


@pytest.mark.gpu
def test_quantizer_wait_runs_out_then_next_call_is_correct(w4):
    import torch
    N, K = 2048, 4096
    W = synth.weights(71, N, K, 0.02)
    Wd = dev_bf16(W)
    code = run_with_short_limit(w4, lambda: w4.quant_pack(Wd, 128, SYM))
    assert code in (0x401, 0x402), hex(code)
    q, sc, _ = w4.quant_pack(Wd, 128, SYM)
    torch.cuda.synchronize()
    assert w4.w4_device_error() == 0
    oq, osc, _ = oracle.quant_pack(W, 128, SYM, threads=THREADS)
    assert_codes_equal(host_u32(q), oq, "qweight")
    assert_codes_equal(host_u16(sc), osc, "scales")


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (200, 512, 1024)], ids=["split_cluster", "single"])
def test_mx_product_wait_runs_out_then_next_call_is_correct(w4, M, N, K):
    """The block-scaled product: the MMA issuer's first wait runs out; the CTA
    drains its copies, still takes part in the cluster barriers of a split-k
    grid, frees its tensor memory and the next call is correct."""
    import torch
    from test_parity_mx import oracle_chain
    from parity import assert_y_elementwise
    W = synth.weights(81, N, K, 0.02, 0.01, 5.0)
    X = synth.activations(82, M, K, 0.01, 40.0)
    wc, ws_rows = w4.fp4_quant(dev_bf16(W), w4.MXFP4)
    ws = w4.mx_scale_layout(ws_rows, K)
    xc, xs = w4.mxfp8_quant(dev_bf16(X), w4.MX_SCALES_MMA)
    code = run_with_short_limit(w4, lambda: w4.mx_gemm(xc, xs, wc, ws))
    assert 0x301 <= code <= 0x304, hex(code)
    Y = host_bf16_as_f64(w4.mx_gemm(xc, xs, wc, ws))
    torch.cuda.synchronize()
    assert w4.w4_device_error() == 0
    Y_ref, Y_abs = oracle_chain(X, W)[:2]
    assert_y_elementwise(Y, Y_ref, Y_abs, K, "Y after a failed call")
