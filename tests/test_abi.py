"""The C ABI: the library loads without a GPU, exports every function that
include/w4.h declares, and rejects malformed calls on the host before anything
is launched (so these run on a CPU-only machine)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "w4.h")


@pytest.fixture(scope="module")
def w4():
    from bit_gemm_quant_b200 import build
    build.build()
    import bit_gemm_quant_b200 as w4
    w4.lib()
    return w4


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z0-9_]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("w4_quant_pack", "w4a16_gemm", "w4a16_workspace_bytes", "w4_status_string",
              "w4_layout_version", "w4_device_error", "w4_fp4_quant"):
        assert n in names


def test_library_exports_every_declared_symbol(w4):
    L = ctypes.CDLL(w4._LIB_PATH)
    for name in declared_functions():
        assert hasattr(L, name), name


def test_layout_version_matches_header(w4):
    m = re.search(r"#define\s+W4_LAYOUT_VERSION\s+(\d+)", open(HEADER).read())
    assert w4.w4_layout_version() == int(m.group(1))


def test_status_strings(w4):
    for st in range(4):
        assert w4.w4_status_string(st).startswith("W4_")
    assert w4.w4_status_string(99) == "unknown w4 status"


FAKE = 1 << 20          # 16-byte aligned fake device addresses: never dereferenced,
P = ctypes.c_void_p     # every call below is rejected during host-side validation


def qp(w4, W=FAKE, N=16, K=256, g=128, mode=0, s=None, q=FAKE, sc=FAKE, z=None):
    return w4.w4_quant_pack(P(W) if W else None, N, K, g, mode, P(s) if s else None, P(q) if q else None,
                            P(sc) if sc else None, P(z) if z else None, None)


def test_quant_pack_rejects_bad_arguments(w4):
    E = w4.W4_ERR_INVALID_ARG
    assert qp(w4, W=0) == E
    assert qp(w4, q=0) == E
    assert qp(w4, sc=0) == E
    assert qp(w4, N=0) == E                      # empty input
    assert qp(w4, N=-3) == E
    assert qp(w4, K=0) == E
    assert qp(w4, K=200) == E                    # K % g != 0
    assert qp(w4, g=16) == E and qp(w4, g=256) == E and qp(w4, g=96) == E
    assert qp(w4, mode=2) == E
    assert qp(w4, mode=1, z=None) == E           # asymmetric needs qzeros
    assert qp(w4, mode=0, z=FAKE) == E           # symmetric must not get qzeros
    assert qp(w4, W=FAKE + 2) == E               # misaligned bf16 input
    assert qp(w4, W=FAKE + 16) == E              # W needs 32-byte alignment (256-bit loads)
    assert qp(w4, q=FAKE + 4) == E
    assert qp(w4, s=FAKE + 4) == E
    assert qp(w4, sc=FAKE + 1) == E
    assert qp(w4, mode=1, z=FAKE + 2) == E
    assert qp(w4, N=1 << 40, K=1 << 30) == E     # N*K overflows int64


def mm(w4, X=FAKE, M=1, N=16, K=256, q=FAKE, sc=FAKE, z=None, g=128, mode=0, Y=FAKE, ws=None, wsb=0):
    return w4.w4a16_gemm(P(X) if X else None, M, N, K, P(q) if q else None, P(sc) if sc else None,
                         P(z) if z else None, g, mode, P(Y) if Y else None, P(ws) if ws else None, wsb, None)


def test_gemm_rejects_bad_arguments(w4):
    E = w4.W4_ERR_INVALID_ARG
    assert mm(w4, X=0) == E
    assert mm(w4, Y=0) == E
    assert mm(w4, q=0) == E
    assert mm(w4, sc=0) == E
    assert mm(w4, M=0) == E                      # empty batch
    assert mm(w4, N=0) == E
    assert mm(w4, K=64) == E                     # K < g
    assert mm(w4, K=300) == E
    assert mm(w4, g=8) == E
    assert mm(w4, mode=1) == E                   # asymmetric without qzeros
    assert mm(w4, mode=0, z=FAKE) == E
    assert mm(w4, X=FAKE + 8) == E
    assert mm(w4, q=FAKE + 4) == E
    assert mm(w4, Y=FAKE + 1) == E


def test_gemm_rejects_a_missing_or_short_split_k_workspace(w4):
    """Skinny tensor-core shapes split K and need the caller's workspace: a
    missing, short or misaligned one is rejected before anything launches."""
    E = w4.W4_ERR_INVALID_ARG
    for M, N, K in ((32, 512, 4096), (24, 256, 4096), (17, 130, 2048)):
        need = w4.w4a16_workspace_bytes(M, N, K, 128)
        assert need > 0
        assert mm(w4, M=M, N=N, K=K) == E                                  # no workspace
        assert mm(w4, M=M, N=N, K=K, ws=FAKE, wsb=need - 1) == E           # one byte short
        assert mm(w4, M=M, N=N, K=K, ws=FAKE + 64, wsb=need) == E          # not 256-byte aligned


def fq(w4, W=FAKE, N=4, K=64, kind=0, c=FAKE, sc=FAKE):
    return w4.w4_fp4_quant(P(W) if W else None, N, K, kind, P(c) if c else None, P(sc) if sc else None, None)


def test_fp4_quant_rejects_bad_arguments(w4):
    E = w4.W4_ERR_INVALID_ARG
    assert fq(w4, W=0) == E
    assert fq(w4, c=0) == E
    assert fq(w4, sc=0) == E
    assert fq(w4, kind=2) == E and fq(w4, kind=-1) == E
    assert fq(w4, N=0) == E                      # empty input
    assert fq(w4, K=0) == E
    assert fq(w4, K=8) == E                      # shorter than an NVFP4 block
    assert fq(w4, K=48, kind=1) == E             # not a whole number of MXFP4 blocks
    assert fq(w4, K=16, kind=1) == E
    assert fq(w4, K=40, kind=0) == E
    assert fq(w4, W=FAKE + 2) == E               # uint4 loads need 16-byte alignment
    assert fq(w4, c=FAKE + 8) == E
    assert fq(w4, N=1 << 40, K=1 << 30) == E     # N*K overflows int64


def test_workspace_query_is_host_only(w4):
    for M in (1, 4, 8, 16, 32, 512, 8192):
        assert w4.w4a16_workspace_bytes(M, 4096, 4096, 128) >= 0
    assert w4.w4a16_workspace_bytes(1, 4096, 4096, 128) == 0


def test_awq_workspace_query_is_host_only(w4):
    a = w4.w4_awq_workspace_bytes(128, 4096, 4096, 128, 1, 20)
    b = w4.w4_awq_workspace_bytes(128, 4096, 4096, 128, 1, 40)
    assert a > 0 and b > a                       # scale vectors and divided activations per alpha
    assert b - a >= 20 * (4096 * 4 + 128 * 4096 * 2)
    assert w4.w4_awq_workspace_bytes(128, 4096, 4096, 128, 1, 1) == 0    # a grid needs two points
    assert w4.w4_awq_workspace_bytes(128, 4096, 4000, 128, 1, 20) == 0   # K not a multiple of g
    assert w4.w4_awq_workspace_bytes(0, 4096, 4096, 128, 1, 20) == 0


def test_awq_search_rejects_malformed_arguments_before_any_launch(w4):
    P = 1 << 12                                  # never dereferenced: rejected first
    ok = dict(W=P, X=P, N=256, K=512, M=8, g=128, mode=0, na=8, losses=P, best=P, s=P, ws=P, wsb=1 << 30)

    def call(**kw):
        a = dict(ok, **kw)
        return w4.w4_awq_search(a["W"], a["X"], a["N"], a["K"], a["M"], a["g"], a["mode"], a["na"], a["losses"],
                                a["best"], a["s"], a["ws"], a["wsb"], None)
    E = w4.W4_ERR_INVALID_ARG
    assert call(na=1) == E
    assert call(na=5000) == E
    assert call(W=0) == E
    assert call(ws=P + 128) == E                 # workspace not 256-byte aligned
    assert call(wsb=1024) == E                   # workspace too small
    assert call(K=500) == E
    assert call(s=P + 4) == E


def test_weights_static_flag_is_accepted_only_in_the_product_mode(w4):
    """W4_WEIGHTS_STATIC is stripped from the product's mode before the mode is
    checked (a well-formed flagged call fails only for its other defects); any
    other bit, or the flag on the quantizer, is an invalid mode."""
    E = w4.W4_ERR_INVALID_ARG
    flag = w4.WEIGHTS_STATIC
    m = re.search(r"#define\s+W4_WEIGHTS_STATIC\s+(0x[0-9a-fA-F]+)", open(HEADER).read())
    assert int(m.group(1), 16) == flag
    assert mm(w4, mode=w4.ASYM | flag) == E                  # asymmetric without qzeros: the mode was read as ASYM
    assert mm(w4, mode=w4.SYM | flag, z=FAKE) == E           # symmetric with qzeros: read as SYM
    assert mm(w4, mode=0x800) == E                           # an unknown bit
    assert mm(w4, mode=flag | 0x800) == E
    assert qp(w4, mode=flag) == E                            # the quantizer has no such flag


def test_fp32_output_flag(w4):
    """W4_OUT_F32 is a product-mode flag like W4_WEIGHTS_STATIC; an fp32 Y must
    be 4-byte aligned; the quantizer rejects it."""
    E = w4.W4_ERR_INVALID_ARG
    f32 = w4.OUT_F32
    m = re.search(r"#define\s+W4_OUT_F32\s+(0x[0-9a-fA-F]+)", open(HEADER).read())
    assert int(m.group(1), 16) == f32
    assert mm(w4, mode=w4.ASYM | f32) == E                   # read as ASYM (no qzeros given)
    assert mm(w4, mode=w4.SYM | f32 | w4.WEIGHTS_STATIC, z=FAKE) == E
    assert mm(w4, mode=w4.SYM | f32, Y=FAKE + 2) == E        # bf16 alignment is not enough for fp32
    assert qp(w4, mode=f32) == E
    assert w4.w4_f32_to_bf16(None, 4, P(FAKE), None) == E
    assert w4.w4_f32_to_bf16(P(FAKE), 0, P(FAKE), None) == E
    assert w4.w4_f32_to_bf16(P(FAKE + 2), 4, P(FAKE), None) == E
    assert w4.w4_f32_to_bf16(P(FAKE), 4, P(FAKE + 1), None) == E


def test_noalloc_rejects_an_unsupported_shape_before_enqueuing_anything(w4):
    """A shape outside the kernels' index range is rejected on the host, before
    the entry point enqueues its counter clear (fake pointers: nothing may touch
    them, and no CUDA call may be made on a machine without a GPU)."""
    U = w4.W4_ERR_UNSUPPORTED
    st = w4.w4a16_gemm_noalloc(P(FAKE), 64, 128, 1 << 26, P(FAKE), P(FAKE), None, 128, 0, P(FAKE), None)
    assert st == U
    need = w4.w4a16_workspace_bytes(64, 128, 1 << 26, 128)
    assert mm(w4, M=64, N=128, K=1 << 26, ws=FAKE, wsb=need) == U   # w4a16_gemm agrees


def mq(w4, X=FAKE, M=4, K=256, c=FAKE, sc=FAKE, layout=1):
    return w4.w4_mxfp8_quant(P(X) if X else None, M, K, P(c) if c else None, P(sc) if sc else None, layout, None)


def test_mxfp8_quant_rejects_bad_arguments(w4):
    E = w4.W4_ERR_INVALID_ARG
    assert mq(w4, X=0) == E and mq(w4, c=0) == E and mq(w4, sc=0) == E
    assert mq(w4, layout=2) == E and mq(w4, layout=-1) == E
    assert mq(w4, M=0) == E                      # empty input
    assert mq(w4, K=0) == E and mq(w4, K=16) == E and mq(w4, K=48) == E
    assert mq(w4, K=96, layout=1) == E           # the tensor-core layout needs K % 128 == 0
    assert mq(w4, X=FAKE + 2) == E               # 16-byte loads
    assert mq(w4, c=FAKE + 8) == E
    assert mq(w4, sc=FAKE + 4, layout=1) == E    # bulk-copied atoms need 16-byte alignment
    assert mq(w4, M=1 << 40, K=1 << 30) == E     # M*K overflows int64


def test_mx_scale_layout_rejects_bad_arguments(w4):
    E = w4.W4_ERR_INVALID_ARG
    f = lambda src=FAKE, R=256, K=512, dst=FAKE: w4.w4_mx_scale_layout(P(src) if src else None, R, K,
                                                                      P(dst) if dst else None, None)
    assert f(src=0) == E and f(dst=0) == E
    assert f(R=0) == E and f(K=64) == E and f(K=160) == E
    assert f(src=FAKE + 2) == E and f(dst=FAKE + 8) == E


def mxg(w4, xc=FAKE, xs=FAKE, M=1, N=256, K=512, wc=FAKE, wsf=FAKE, Y=FAKE, flags=0):
    return w4.w4_mx_gemm(P(xc) if xc else None, P(xs) if xs else None, M, N, K, P(wc) if wc else None,
                         P(wsf) if wsf else None, P(Y) if Y else None, flags, None)


def test_mx_gemm_rejects_bad_arguments(w4):
    E = w4.W4_ERR_INVALID_ARG
    for kw in ("xc", "xs", "wc", "wsf", "Y"):
        assert mxg(w4, **{kw: 0}) == E
    assert mxg(w4, M=0) == E and mxg(w4, N=0) == E
    assert mxg(w4, K=64) == E and mxg(w4, K=192) == E        # whole 128-wide k-stages only
    assert mxg(w4, wc=FAKE + 16) == E                         # the FP4 tensor map wants 32-byte alignment
    assert mxg(w4, xc=FAKE + 8) == E and mxg(w4, xs=FAKE + 8) == E and mxg(w4, wsf=FAKE + 4) == E
    assert mxg(w4, Y=FAKE + 1) == E
    assert mxg(w4, flags=1) == E and mxg(w4, flags=0x300) == E   # W4_WEIGHTS_STATIC is the only flag
    assert mxg(w4, M=1 << 40, K=1 << 30) == E                 # M*K overflows int64


def test_gptq_rejects_bad_arguments(w4):
    E = w4.W4_ERR_INVALID_ARG
    need = w4.w4_gptq_workspace_bytes(64, 256, 128)
    assert need >= 16 * 256 * 256 + 8 * 64 * 256
    assert w4.w4_gptq_workspace_bytes(64, 250, 128) == 0 and w4.w4_gptq_workspace_bytes(0, 256, 128) == 0
    assert w4.w4_gptq_workspace_bytes(64, 32768, 128) == 0          # past the supported K

    def gp(W=FAKE, X=FAKE, N=64, K=256, M=8, g=128, mode=0, q=FAKE, sc=FAKE, z=None, ws=FAKE, wsb=need):
        return w4.w4_gptq(P(W) if W else None, P(X) if X else None, N, K, M, g, mode, P(q) if q else None,
                          P(sc) if sc else None, P(z) if z else None, P(ws) if ws else None, wsb, None)
    for kw in ("W", "X", "q", "sc", "ws"):
        assert gp(**{kw: 0}) == E
    assert gp(g=48) == E and gp(mode=2) == E
    assert gp(N=0) == E and gp(M=0) == E and gp(K=16) == E and gp(K=320) == E
    assert gp(mode=1) == E                        # asymmetric needs qzeros
    assert gp(z=FAKE) == E                        # symmetric must not get qzeros
    assert gp(ws=FAKE + 64) == E and gp(wsb=need - 1) == E
    assert gp(W=FAKE + 1) == E and gp(q=FAKE + 2) == E


def test_repack_arguments(w4):
    assert w4.w4_repacked_words(4096, 4096) == 4096 * 512
    assert w4.w4_repacked_words(1000, 4096) == 1008 * 512        # N padded to whole 16-channel boxes
    assert w4.w4_repacked_words(16, 384) == 0                    # K not a multiple of 256
    E, U = w4.W4_ERR_INVALID_ARG, w4.W4_ERR_UNSUPPORTED
    rp = lambda q=FAKE, N=16, K=512, out=FAKE: w4.w4_repack(P(q) if q else None, N, K, P(out) if out else None, None)
    assert rp(q=0) == E and rp(out=0) == E and rp(N=0) == E and rp(K=128) == E
    assert rp(K=384) == U
    assert rp(q=FAKE + 4) == E and rp(out=FAKE + 8) == E
    # the repacked layout is served by the GEMV only, with whole 256-k boxes
    assert mm(w4, K=384, g=128, mode=w4.REPACKED) == U
    assert mm(w4, mode=w4.REPACKED | 0x800) == E
