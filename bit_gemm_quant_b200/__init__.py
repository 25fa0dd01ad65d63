"""B200-native group-wise INT4 weight quantization and the W4A16 GEMV/GEMM.

A thin ctypes binding over the C ABI of ``libw4.so`` (declared in
``include/w4.h``).  The raw entry points keep their C names and take device
pointers as integers; the tensor helpers ``quant_pack`` and ``gemm`` only
allocate outputs with torch, pass ``data_ptr()`` values and the current CUDA
stream, and raise ``W4Error`` on a nonzero status.  Every step of the path
runs in the library's kernels; there is no fallback: if ``libw4.so`` is
missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

SYM, ASYM = 0, 1
# OR-ed into the mode of w4a16_gemm / w4a16_gemm_noalloc: the packed weight is
# not written by the kernel right before the call on the stream (include/w4.h)
WEIGHTS_STATIC = 0x100
# OR-ed into the mode: Y is fp32 (the sums before their bf16 rounding)
OUT_F32 = 0x200
# OR-ed into the mode: qweight is in the w4_repack layout (GEMV, M <= 16)
REPACKED = 0x400
NVFP4, MXFP4 = 0, 1
FP4_BLOCK = {NVFP4: 16, MXFP4: 32}
MX_SCALES_ROWS, MX_SCALES_MMA = 0, 1
W4_OK, W4_ERR_INVALID_ARG, W4_ERR_UNSUPPORTED, W4_ERR_CUDA = 0, 1, 2, 3

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libw4.so")
_lib = None


class W4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__("%s failed: %s" % (what, w4_status_string(status) if _lib else status))
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libw4.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError("libw4.so is not built; run `python -m bit_gemm_quant_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        P, I64, I, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        L.w4_quant_pack.argtypes = [P, I64, I64, I, I, P, P, P, P, P]
        L.w4_quant_pack.restype = I
        L.w4a16_workspace_bytes.argtypes = [I64, I64, I64, I]
        L.w4a16_workspace_bytes.restype = SZ
        L.w4a16_gemm.argtypes = [P, I64, I64, I64, P, P, P, I, I, P, P, SZ, P]
        L.w4a16_gemm.restype = I
        L.w4a16_gemm_noalloc.argtypes = [P, I64, I64, I64, P, P, P, I, I, P, P]
        L.w4a16_gemm_noalloc.restype = I
        L.w4_awq_workspace_bytes.argtypes = [I64, I64, I64, I, I, I]
        L.w4_awq_workspace_bytes.restype = SZ
        L.w4_awq_search.argtypes = [P, P, I64, I64, I64, I, I, I, P, P, P, P, SZ, P]
        L.w4_awq_search.restype = I
        L.w4_fp4_quant.argtypes = [P, I64, I64, I, P, P, P]
        L.w4_fp4_quant.restype = I
        L.w4_repacked_words.argtypes = [I64, I64]
        L.w4_repacked_words.restype = SZ
        L.w4_repack.argtypes = [P, I64, I64, P, P]
        L.w4_repack.restype = I
        L.w4_gptq_workspace_bytes.argtypes = [I64, I64, I]
        L.w4_gptq_workspace_bytes.restype = SZ
        L.w4_gptq.argtypes = [P, P, I64, I64, I64, I, I, P, P, P, P, SZ, P]
        L.w4_gptq.restype = I
        L.w4_f32_to_bf16.argtypes = [P, I64, P, P]
        L.w4_f32_to_bf16.restype = I
        L.w4_mxfp8_quant.argtypes = [P, I64, I64, P, P, I, P]
        L.w4_mxfp8_quant.restype = I
        L.w4_mx_scale_layout.argtypes = [P, I64, I64, P, P]
        L.w4_mx_scale_layout.restype = I
        L.w4_mx_gemm.argtypes = [P, P, I64, I64, I64, P, P, P, I, P]
        L.w4_mx_gemm.restype = I
        L.w4_status_string.argtypes = [I]
        L.w4_status_string.restype = ctypes.c_char_p
        L.w4_layout_version.argtypes = []
        L.w4_layout_version.restype = I
        L.w4_device_error.argtypes = [ctypes.POINTER(I)]
        L.w4_device_error.restype = I
        L.w4_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        L.w4_set_wait_limit_ns.restype = None
        L.w4_test_stall_first_wait.argtypes = [I]
        L.w4_test_stall_first_wait.restype = None
        _lib = L
    return _lib


# --- raw C ABI, same names and argument order as include/w4.h ----------------

def w4_quant_pack(W, N, K, group, mode, s, qweight, scales, qzeros, stream) -> int:
    return lib().w4_quant_pack(W, N, K, group, mode, s, qweight, scales, qzeros, stream)


def w4a16_workspace_bytes(M, N, K, group) -> int:
    return int(lib().w4a16_workspace_bytes(M, N, K, group))


def w4a16_gemm(X, M, N, K, qweight, scales, qzeros, group, mode, Y, workspace, workspace_bytes, stream) -> int:
    return lib().w4a16_gemm(X, M, N, K, qweight, scales, qzeros, group, mode, Y, workspace,
                            workspace_bytes, stream)


def w4a16_gemm_noalloc(X, M, N, K, qweight, scales, qzeros, group, mode, Y, stream) -> int:
    return lib().w4a16_gemm_noalloc(X, M, N, K, qweight, scales, qzeros, group, mode, Y, stream)


def w4_awq_workspace_bytes(M, N, K, group, mode, n_alpha) -> int:
    return int(lib().w4_awq_workspace_bytes(M, N, K, group, mode, n_alpha))


def w4_awq_search(W, X, N, K, M, group, mode, n_alpha, losses, best, s_best, workspace, workspace_bytes,
                  stream) -> int:
    return lib().w4_awq_search(W, X, N, K, M, group, mode, n_alpha, losses, best, s_best, workspace,
                               workspace_bytes, stream)


def w4_fp4_quant(W, N, K, kind, codes, scales, stream) -> int:
    return lib().w4_fp4_quant(W, N, K, kind, codes, scales, stream)


def w4_repacked_words(N, K) -> int:
    return int(lib().w4_repacked_words(N, K))


def w4_repack(qweight, N, K, out, stream) -> int:
    return lib().w4_repack(qweight, N, K, out, stream)


def w4_gptq_workspace_bytes(N, K, group) -> int:
    return int(lib().w4_gptq_workspace_bytes(N, K, group))


def w4_gptq(W, X, N, K, M, group, mode, qweight, scales, qzeros, workspace, workspace_bytes, stream) -> int:
    return lib().w4_gptq(W, X, N, K, M, group, mode, qweight, scales, qzeros, workspace, workspace_bytes, stream)


def w4_f32_to_bf16(src, n, dst, stream) -> int:
    return lib().w4_f32_to_bf16(src, n, dst, stream)


def w4_mxfp8_quant(X, M, K, codes, scales, scale_layout, stream) -> int:
    return lib().w4_mxfp8_quant(X, M, K, codes, scales, scale_layout, stream)


def w4_mx_scale_layout(src, R, K, dst, stream) -> int:
    return lib().w4_mx_scale_layout(src, R, K, dst, stream)


def w4_mx_gemm(x_codes, x_scales, M, N, K, w_codes, w_scales, Y, flags, stream) -> int:
    return lib().w4_mx_gemm(x_codes, x_scales, M, N, K, w_codes, w_scales, Y, flags, stream)


def w4_status_string(status: int) -> str:
    return lib().w4_status_string(int(status)).decode()


def w4_layout_version() -> int:
    return int(lib().w4_layout_version())


def w4_set_wait_limit_ns(ns: int) -> None:
    lib().w4_set_wait_limit_ns(int(ns))


def w4_test_stall_first_wait(on: int) -> None:
    lib().w4_test_stall_first_wait(int(on))


def w4_device_error() -> int:
    code = ctypes.c_int(0)
    st = lib().w4_device_error(ctypes.byref(code))
    if st != W4_OK:
        raise W4Error(st, "w4_device_error")
    return code.value


# --- torch tensor helpers (argument marshalling only) -------------------------

def _stream_handle(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def packed_shapes(N: int, K: int, group: int):
    G = K // group
    return (N, K // 8), (N, G), (N, (G + 7) // 8)


def quant_pack(W, group: int = 128, mode: int = SYM, s=None, stream=None, out=None):
    """Quantize a bf16 CUDA tensor W[N,K]; returns (qweight, scales, qzeros or None)."""
    import torch
    N, K = W.shape
    qs, ss, zs = packed_shapes(N, K, group)
    if out is None:
        qweight = torch.empty(qs, dtype=torch.int32, device=W.device)
        scales = torch.empty(ss, dtype=torch.float16, device=W.device)
        qzeros = torch.empty(zs, dtype=torch.int32, device=W.device) if mode == ASYM else None
    else:
        qweight, scales, qzeros = out
    st = w4_quant_pack(_ptr(W), N, K, group, mode, _ptr(s), _ptr(qweight), _ptr(scales), _ptr(qzeros),
                       _stream_handle(stream))
    if st != W4_OK:
        raise W4Error(st, "w4_quant_pack")
    return qweight, scales, qzeros


def gemm(X, qweight, scales, qzeros, group: int, mode: int, N: int | None = None, workspace=None,
         out=None, stream=None, weights_static: bool = False, out_f32: bool = False, repacked: bool = False):
    """Y[M,N] = X . W^T from the packed weight; X bf16 CUDA tensor [M,K].
    ``weights_static`` passes W4_WEIGHTS_STATIC: the caller declares that the
    kernel right before this call on the stream does not write the packed
    weight (weights quantized once, earlier), so the weight stream may start
    before that kernel finishes.  ``out_f32`` passes W4_OUT_F32: Y is fp32,
    the sums before their bf16 rounding.  ``repacked`` passes W4_REPACKED:
    qweight comes from ``repack`` (give N then, the padded array has more
    rows)."""
    import torch
    M, K = X.shape
    if N is None:
        if repacked:
            raise ValueError("gemm(repacked=True) needs N: the repacked array's shape does not give it")
        N = qweight.shape[0]
    if out is not None:
        Y = out
    else:
        Y = torch.empty((M, N), dtype=torch.float32 if out_f32 else torch.bfloat16, device=X.device)
    if out_f32:
        mode |= OUT_F32
    if repacked:
        mode |= REPACKED
    need = w4a16_workspace_bytes(M, N, K, group)
    if need and workspace is None:
        workspace = torch.zeros(need, dtype=torch.uint8, device=X.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = w4a16_gemm(_ptr(X), M, N, K, _ptr(qweight), _ptr(scales), _ptr(qzeros), group,
                    mode | (WEIGHTS_STATIC if weights_static else 0), _ptr(Y), _ptr(workspace), wbytes,
                    _stream_handle(stream))
    if st != W4_OK:
        raise W4Error(st, "w4a16_gemm")
    return Y


def gemm_noalloc(X, qweight, scales, qzeros, group: int, mode: int, N: int | None = None, out=None, stream=None):
    """Like ``gemm`` for callers that cannot allocate device scratch: the
    split-K scratch is the library's own fixed array (shapes that need more
    than it holds raise W4Error with W4_ERR_UNSUPPORTED).  Only the output is
    allocated here, and only when ``out`` is None."""
    import torch
    M, K = X.shape
    if N is None:
        N = qweight.shape[0]
    Y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    st = w4a16_gemm_noalloc(_ptr(X), M, N, K, _ptr(qweight), _ptr(scales), _ptr(qzeros), group, mode, _ptr(Y),
                            _stream_handle(stream))
    if st != W4_OK:
        raise W4Error(st, "w4a16_gemm_noalloc")
    return Y


def awq_search(W, X, group: int = 128, mode: int = SYM, n_alpha: int = 20, stream=None):
    """AWQ scale search over bf16 CUDA tensors W[N,K] and calibration X[M,K].
    Returns (losses fp64 [n_alpha], best index tensor, s_best fp32 [K])."""
    import torch
    N, K = W.shape
    M = X.shape[0]
    need = w4_awq_workspace_bytes(M, N, K, group, mode, n_alpha)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=W.device)
    losses = torch.empty(n_alpha, dtype=torch.float64, device=W.device)
    best = torch.empty(1, dtype=torch.int32, device=W.device)
    s_best = torch.empty(K, dtype=torch.float32, device=W.device)
    st = w4_awq_search(_ptr(W), _ptr(X), N, K, M, group, mode, n_alpha, _ptr(losses), _ptr(best), _ptr(s_best),
                       _ptr(ws), ws.numel(), _stream_handle(stream))
    if st != W4_OK:
        raise W4Error(st, "w4_awq_search")
    return losses, best, s_best


def fp4_quant(W, kind: int = NVFP4, stream=None, out=None):
    """Block-scaled FP4 quantization of a bf16 CUDA tensor W[N,K].
    Returns (codes uint8 [N, K/2], scales uint8 [N, K/block])."""
    import torch
    N, K = W.shape
    B = FP4_BLOCK.get(kind, 16)
    if out is None:
        codes = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
        scales = torch.empty((N, max(K // B, 1)), dtype=torch.uint8, device=W.device)
    else:
        codes, scales = out
    st = w4_fp4_quant(_ptr(W), N, K, kind, _ptr(codes), _ptr(scales), _stream_handle(stream))
    if st != W4_OK:
        raise W4Error(st, "w4_fp4_quant")
    return codes, scales


def repack(qweight, N: int, K: int, stream=None, out=None):
    """The GEMV's box order of a packed weight (int32 [N, K/8] CUDA tensor):
    a flat int32 tensor of w4_repacked_words(N, K) words."""
    import torch
    n = w4_repacked_words(N, K)
    dst = out if out is not None else torch.empty(max(n, 4), dtype=torch.int32, device=qweight.device)
    st = w4_repack(_ptr(qweight), N, K, _ptr(dst), _stream_handle(stream))
    if st != W4_OK:
        raise W4Error(st, "w4_repack")
    return dst


def gptq(W, X, group: int = 128, mode: int = SYM, stream=None):
    """GPTQ of a bf16 CUDA tensor W[N,K] with calibration rows X[M,K] (bf16
    CUDA); returns (qweight, scales, qzeros or None) as quant_pack does."""
    import torch
    N, K = W.shape
    M = X.shape[0]
    qs, ss, zs = packed_shapes(N, K, group)
    qweight = torch.empty(qs, dtype=torch.int32, device=W.device)
    scales = torch.empty(ss, dtype=torch.float16, device=W.device)
    qzeros = torch.empty(zs, dtype=torch.int32, device=W.device) if mode == ASYM else None
    need = w4_gptq_workspace_bytes(N, K, group)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=W.device)
    st = w4_gptq(_ptr(W), _ptr(X), N, K, M, group, mode, _ptr(qweight), _ptr(scales), _ptr(qzeros), _ptr(ws),
                 ws.numel(), _stream_handle(stream))
    if st != W4_OK:
        raise W4Error(st, "w4_gptq")
    return qweight, scales, qzeros


def f32_to_bf16(src, out=None, stream=None):
    """bf16 (round to nearest even) copy of an fp32 CUDA tensor."""
    import torch
    dst = out if out is not None else torch.empty(src.shape, dtype=torch.bfloat16, device=src.device)
    st = w4_f32_to_bf16(_ptr(src), src.numel(), _ptr(dst), _stream_handle(stream))
    if st != W4_OK:
        raise W4Error(st, "w4_f32_to_bf16")
    return dst


def mx_scale_bytes(R: int, K: int) -> int:
    """Bytes of E8M0 scales for R rows x K columns in the tensor-core layout."""
    return (R + 127) // 128 * 128 * (K // 32)


def mxfp8_quant(X, scale_layout: int = MX_SCALES_MMA, stream=None, out=None):
    """MXFP8 quantization of a bf16 CUDA tensor X[M,K].
    Returns (codes uint8 [M, K], scales uint8: [M, K/32] for MX_SCALES_ROWS,
    flat [mx_scale_bytes(M, K)] for MX_SCALES_MMA)."""
    import torch
    M, K = X.shape
    if out is None:
        codes = torch.empty((M, K), dtype=torch.uint8, device=X.device)
        if scale_layout == MX_SCALES_ROWS:
            scales = torch.empty((M, max(K // 32, 1)), dtype=torch.uint8, device=X.device)
        else:
            scales = torch.empty(max(mx_scale_bytes(M, K), 1), dtype=torch.uint8, device=X.device)
    else:
        codes, scales = out
    st = w4_mxfp8_quant(_ptr(X), M, K, _ptr(codes), _ptr(scales), scale_layout, _stream_handle(stream))
    if st != W4_OK:
        raise W4Error(st, "w4_mxfp8_quant")
    return codes, scales


def mx_scale_layout(scales_rows, K: int, stream=None, out=None):
    """E8M0 scales uint8 [R, K/32] (CUDA) to the tensor-core layout (flat uint8)."""
    import torch
    R = scales_rows.shape[0]
    dst = out if out is not None else torch.empty(mx_scale_bytes(R, K), dtype=torch.uint8,
                                                  device=scales_rows.device)
    st = w4_mx_scale_layout(_ptr(scales_rows), R, K, _ptr(dst), _stream_handle(stream))
    if st != W4_OK:
        raise W4Error(st, "w4_mx_scale_layout")
    return dst


def mx_gemm(x_codes, x_scales, w_codes, w_scales, out=None, stream=None, weights_static: bool = False):
    """Y[M,N] bf16 = X^ . W^^T from MXFP8 activations (codes [M,K], tensor-core
    layout scales) and MXFP4 weights (codes [N,K/2], tensor-core layout scales).
    ``weights_static`` passes W4_WEIGHTS_STATIC (see ``gemm``)."""
    import torch
    M, K = x_codes.shape
    N = w_codes.shape[0]
    Y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=x_codes.device)
    st = w4_mx_gemm(_ptr(x_codes), _ptr(x_scales), M, N, K, _ptr(w_codes), _ptr(w_scales), _ptr(Y),
                    WEIGHTS_STATIC if weights_static else 0, _stream_handle(stream))
    if st != W4_OK:
        raise W4Error(st, "w4_mx_gemm")
    return Y
