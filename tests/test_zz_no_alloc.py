"""w4a16_gemm_noalloc: the entry point for callers that cannot allocate
device memory.  It must give the product the CPU oracle defines (and the same
product as w4a16_gemm, which takes a caller-allocated workspace) on a split-K
shape, on consecutive calls that share the library's fixed scratch array, and
must reject shapes whose scratch need exceeds that array before launching
anything.

This file is collected last so that it runs both after every other test and,
alone, in a fresh process."""
import ctypes
import re

import numpy as np
import pytest

import oracle
from bit_gemm_quant_b200 import synth
from conftest import ROOT
from parity import THREADS, assert_y_close, dev_bf16, host_bf16_as_f64

SYM, ASYM = 0, 1


@pytest.fixture(scope="module")
def w4():
    from bit_gemm_quant_b200 import build
    build.build()
    import bit_gemm_quant_b200 as w4
    w4.lib()
    return w4


def scratch_limit():
    text = open(ROOT + "/include/w4.h").read()
    m = re.search(r"#define\s+W4_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", text)
    return int(m.group(1)) << int(m.group(2))


def test_oversized_scratch_need_is_rejected_on_the_host(w4):
    # fake, aligned device addresses: the call must return before touching them
    P, FAKE = ctypes.c_void_p, 1 << 20
    limit = scratch_limit()
    M, N, K = 16, 28672, 8192
    need = w4.w4a16_workspace_bytes(M, N, K, 128)
    if need <= limit:
        M, N = 64, 1 << 17
        need = w4.w4a16_workspace_bytes(M, N, K, 128)
    assert need > limit
    st = w4.w4a16_gemm_noalloc(P(FAKE), M, N, K, P(FAKE), P(FAKE), None, 128, SYM, P(FAKE), None)
    assert st == w4.W4_ERR_UNSUPPORTED
    st = w4.w4a16_gemm_noalloc(None, M, N, K, P(FAKE), P(FAKE), None, 128, SYM, P(FAKE), None)
    assert st == w4.W4_ERR_INVALID_ARG


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K,g,mode", [(32, 4096, 4096, 128, ASYM), (24, 2000, 2048, 64, SYM)])
def test_noalloc_matches_workspace_entry_point_twice(w4, M, N, K, g, mode):
    import torch
    need = w4.w4a16_workspace_bytes(M, N, K, g)
    assert 0 < need <= scratch_limit(), need          # a split-K shape that the scratch holds
    W = synth.weights(M + N + K, N, K, 0.02, 0.01, 5.0)
    X = synth.activations(M + N + K, M, K, 0.01, 40.0)
    q, sc, z = w4.quant_pack(dev_bf16(W), g, mode)
    Xd = dev_bf16(X)
    Y_ws = host_bf16_as_f64(w4.gemm(Xd, q, sc, z, g, mode))   # caller-allocated, zeroed workspace
    oracle.build()
    oq, osc, oz = oracle.quant_pack(W, g, mode, threads=THREADS)
    Y_ref = oracle.w4a16_reference(X, oq, osc, oz, K, g, mode, threads=THREADS)
    stream = torch.cuda.current_stream()
    for call in range(2):                                       # the second call reuses the scratch
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = w4.w4a16_gemm_noalloc(ctypes.c_void_p(Xd.data_ptr()), M, N, K, ctypes.c_void_p(q.data_ptr()),
                                   ctypes.c_void_p(sc.data_ptr()),
                                   None if z is None else ctypes.c_void_p(z.data_ptr()), g, mode,
                                   ctypes.c_void_p(Y.data_ptr()), ctypes.c_void_p(stream.cuda_stream))
        assert st == w4.W4_OK, w4.w4_status_string(st)
        torch.cuda.synchronize()
        Yn = host_bf16_as_f64(Y)
        assert np.isfinite(Yn).all(), "call %d left outputs unwritten" % call
        assert_y_close(Yn, Y_ref, what="noalloc call %d against the oracle" % call)
        assert_y_close(Yn, Y_ws, what="noalloc call %d against w4a16_gemm" % call)
    assert w4.w4_device_error() == 0
