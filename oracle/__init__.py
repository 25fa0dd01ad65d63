"""CPU oracle for group-wise INT4 weight quantization and the W4A16 product.

TEST INFRASTRUCTURE ONLY.  The arithmetic lives in ``w4_oracle.c`` (plain C,
IEEE binary32 without FMA contraction, fp64 product); this module compiles it
with gcc and marshals numpy arrays through ctypes.  Only ``tests/``, the smoke
check in ``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may use
it.  It shares no code with the CUDA library and never imports it.

Every function cites the passage it restates; see the header comment of
``w4_oracle.c`` for the readings taken where the pages leave a step open.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "w4_oracle.c")
_SO = os.path.join(_HERE, "libw4oracle.so")
_lib = None

SYM, ASYM = 0, 1
NVFP4, MXFP4 = 0, 1          # block-scaled FP4 kinds: 16-weight blocks with E4M3 scales, 32 with E8M0
FP4_BLOCK = {NVFP4: 16, MXFP4: 32}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
               "-frounding-math", "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _SO)
    return _SO


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.orc_f32_to_f16.argtypes, L.orc_f32_to_f16.restype = [ctypes.c_float], ctypes.c_uint16
        L.orc_f16_to_f32.argtypes, L.orc_f16_to_f32.restype = [ctypes.c_uint16], ctypes.c_float
        L.orc_f32_to_bf16.argtypes, L.orc_f32_to_bf16.restype = [ctypes.c_float], ctypes.c_uint16
        L.orc_bf16_to_f32.argtypes, L.orc_bf16_to_f32.restype = [ctypes.c_uint16], ctypes.c_float
        L.orc_quant_group.argtypes = [P, I64, I, P, P, P]
        L.orc_quant_group.restype = None
        L.orc_quant_pack_rows.argtypes = [P, I64, I64, I64, I, P, I64, I64, P, P, P]
        L.orc_quant_pack_rows.restype = I
        L.orc_dequant_rows.argtypes = [P, P, P, I64, I64, I64, I, I64, I64, P]
        L.orc_dequant_rows.restype = I
        L.orc_dequant_rows_f32.argtypes = [P, P, P, I64, I64, I64, I, I64, I64, P]
        L.orc_dequant_rows_f32.restype = I
        L.orc_gemm_f64.argtypes = [P, I64, I64, P, I64, P]
        L.orc_gemm_f64.restype = None
        L.orc_e2m1_decode.argtypes, L.orc_e2m1_decode.restype = [I], ctypes.c_float
        L.orc_f32_to_e2m1_sat.argtypes, L.orc_f32_to_e2m1_sat.restype = [ctypes.c_float], I
        L.orc_e4m3_decode.argtypes, L.orc_e4m3_decode.restype = [I], ctypes.c_float
        L.orc_f32_to_e4m3_sat.argtypes, L.orc_f32_to_e4m3_sat.restype = [ctypes.c_float], I
        L.orc_e8m0_decode.argtypes, L.orc_e8m0_decode.restype = [I], ctypes.c_float
        L.orc_fp4_quant_rows.argtypes = [P, I64, I64, I, P, P]
        L.orc_fp4_quant_rows.restype = I
        L.orc_fp4_dequant_rows.argtypes = [P, P, I64, I64, I, P]
        L.orc_fp4_dequant_rows.restype = I
        L.orc_mxfp8_quant_rows.argtypes = [P, I64, I64, P, P]
        L.orc_mxfp8_quant_rows.restype = I
        L.orc_mxfp8_dequant_rows.argtypes = [P, P, I64, I64, P]
        L.orc_mxfp8_dequant_rows.restype = I
        _lib = L
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# --- format conversions (IEEE binary16 / bfloat16 definitions) --------------

def f32_to_f16_bits(x: float) -> int:
    return int(lib().orc_f32_to_f16(float(x)))


def f16_bits_to_f32(h: int) -> float:
    return float(lib().orc_f16_to_f32(int(h)))


def f32_to_bf16_bits(x: float) -> int:
    return int(lib().orc_f32_to_bf16(float(x)))


def bf16_bits_to_f32(b: int) -> float:
    return float(lib().orc_bf16_to_f32(int(b)))


# --- one group (page 5, section 2.2 formulas; b = 4) -------------------------

def quant_group(w: np.ndarray, mode: int):
    """Quantize one group of fp32 values w' -> (s16 bits, zp, codes u[g])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    u = np.zeros(w.size, dtype=np.uint8)
    s16 = ctypes.c_uint16(0)
    zp = ctypes.c_int(0)
    lib().orc_quant_group(_ptr(w), w.size, int(mode), ctypes.byref(s16), ctypes.byref(zp), _ptr(u))
    return int(s16.value), int(zp.value), u


# --- whole matrices -----------------------------------------------------------

def packed_shapes(N: int, K: int, g: int):
    G = K // g
    return (N, K // 8), (N, G), (N, (G + 7) // 8)


def _chunks(r0: int, r1: int, threads: int):
    n = max(1, min(threads, r1 - r0))
    step = (r1 - r0 + n - 1) // n
    return [(a, min(a + step, r1)) for a in range(r0, r1, step)]


def quant_pack(W_bits: np.ndarray, g: int, mode: int, s: np.ndarray | None = None,
               rows: tuple[int, int] | None = None, threads: int = 1):
    """Fold (page 5 section 2.4, page 3 section 5.3), group-quantize (page 5
    section 2.2, page 2 group quantization) and pack rows [r0, r1) of a bf16
    weight W[N,K] given as uint16 bit patterns.

    Returns (qweight uint32 [N,K/8], scales uint16 fp16-bits [N,G],
    qzeros uint32 [N,ceil(G/8)] or None); rows outside [r0, r1) stay zero.
    """
    W_bits = np.ascontiguousarray(W_bits, dtype=np.uint16)
    N, K = W_bits.shape
    if s is not None:
        s = np.ascontiguousarray(s, dtype=np.float32)
        assert s.shape == (K,)
    r0, r1 = rows if rows is not None else (0, N)
    qs, ss, zs = packed_shapes(N, K, g)
    qweight = np.zeros(qs, dtype=np.uint32)
    scales = np.zeros(ss, dtype=np.uint16)
    qzeros = np.zeros(zs, dtype=np.uint32) if mode == ASYM else None
    L = lib()

    def run(span):
        rc = L.orc_quant_pack_rows(_ptr(W_bits), N, K, g, int(mode), _ptr(s), span[0], span[1],
                                   _ptr(qweight), _ptr(scales), _ptr(qzeros))
        if rc != 0:
            raise ValueError("oracle quant_pack rejected its arguments (code %d)" % rc)

    spans = _chunks(r0, r1, threads)
    if len(spans) == 1:
        run(spans[0])
    else:
        with ThreadPoolExecutor(len(spans)) as ex:
            list(ex.map(run, spans))
    return qweight, scales, qzeros


def dequant(qweight: np.ndarray, scales: np.ndarray, qzeros: np.ndarray | None, K: int, g: int,
            mode: int, rows: tuple[int, int] | None = None, exact_f32: bool = False,
            threads: int = 1) -> np.ndarray:
    """w^ = bf16_rne(float(u - zp) * float(s16)) (page 5 section 2.2, x^ = (q-zp)*s)
    for rows [r0, r1).  Returns bf16 bit patterns (uint16), or with
    ``exact_f32`` the exact fp32 product before the bf16 rounding."""
    N = qweight.shape[0]
    r0, r1 = rows if rows is not None else (0, N)
    qweight = np.ascontiguousarray(qweight, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    if qzeros is not None:
        qzeros = np.ascontiguousarray(qzeros, dtype=np.uint32)
    L = lib()
    out = np.zeros((r1 - r0, K), dtype=np.float32 if exact_f32 else np.uint16)
    fn = L.orc_dequant_rows_f32 if exact_f32 else L.orc_dequant_rows

    def run(span):
        dst = out[span[0] - r0:span[1] - r0]       # rows of a C-contiguous array: contiguous
        rc = fn(_ptr(qweight), _ptr(scales), _ptr(qzeros), N, K, g, int(mode), span[0], span[1], _ptr(dst))
        if rc != 0:
            raise ValueError("oracle dequant rejected its arguments (code %d)" % rc)

    spans = _chunks(r0, r1, threads)
    if len(spans) == 1:
        run(spans[0])
    else:
        with ThreadPoolExecutor(len(spans)) as ex:
            list(ex.map(run, spans))
    return out


def gemm_f64(X_bits: np.ndarray, What_bits: np.ndarray, threads: int = 1) -> np.ndarray:
    """Y[m][c] = sum_k x[m][k] * w^[c][k] in fp64 (X bf16 [M,K], W^ bf16 [C,K])."""
    X_bits = np.ascontiguousarray(X_bits, dtype=np.uint16)
    What_bits = np.ascontiguousarray(What_bits, dtype=np.uint16)
    M, K = X_bits.shape
    C, K2 = What_bits.shape
    assert K == K2
    Y = np.zeros((M, C), dtype=np.float64)
    L = lib()
    spans = _chunks(0, C, threads)

    def run(span):
        a, b = span
        part = np.zeros((M, b - a), dtype=np.float64)
        L.orc_gemm_f64(_ptr(X_bits), M, K, _ptr(np.ascontiguousarray(What_bits[a:b])), b - a, _ptr(part))
        Y[:, a:b] = part

    if len(spans) == 1:
        run(spans[0])
    else:
        with ThreadPoolExecutor(len(spans)) as ex:
            list(ex.map(run, spans))
    return Y


def w4a16_reference(X_bits, qweight, scales, qzeros, K, g, mode, channels=None, threads=1):
    """Y_ref = X . W^T in fp64 for all output channels or for a listed subset
    (the dequantized rows are produced by ``dequant``)."""
    N = qweight.shape[0]
    if channels is None:
        What = dequant(qweight, scales, qzeros, K, g, mode)
    else:
        channels = np.asarray(channels, dtype=np.int64)
        What = np.stack([dequant(qweight, scales, qzeros, K, g, mode, rows=(int(c), int(c) + 1))[0]
                         for c in channels]) if len(channels) else np.zeros((0, K), np.uint16)
    return gemm_f64(X_bits, What, threads=threads)


def w4a16_abs_reference(X_bits, qweight, scales, qzeros, K, g, mode, threads=1):
    """sum_k |x[m][k]| * |w^[n][k]| in fp64: the scale of the rounding error of
    any order of accumulating Y[m][n]."""
    What = dequant(qweight, scales, qzeros, K, g, mode)
    return gemm_f64(np.ascontiguousarray(X_bits, dtype=np.uint16) & 0x7FFF, What & 0x7FFF, threads=threads)


def e2m1_decode(code: int) -> float:
    """Value of a 4-bit E2M1 code (page 5 section 2.1)."""
    return float(lib().orc_e2m1_decode(int(code)))


# --- block-scaled FP4 (NVFP4 / MXFP4) ----------------------------------------
# Page 2 (learn.longtimenohack.com .../quantization.html, the Blackwell FP4
# paragraph): E2M1 values with one FP8 E4M3 scale per 16 weights, amax mapped
# to 6; page 3 (blog.freezetheflame.cc .../quantization-deep-dive.html, section
# 4.3): MXFP4, one E8M0 scale per 32 weights; page 5 (ai-infra.cypggs.com
# .../02-core-ideas, section 2.1): the E2M1 value set and the E4M3 format.  The
# readings are stated in w4_oracle.c.

def f32_to_e2m1(x: float) -> int:
    """E2M1 code of x: nearest value, ties to the even fraction bit, |x| > 6 saturating."""
    return int(lib().orc_f32_to_e2m1_sat(float(x)))


def e4m3_decode(code: int) -> float:
    """Value of an FP8 E4M3 code (1+4+3, bias 7, max 448, S.1111.111 NaN)."""
    return float(lib().orc_e4m3_decode(int(code)))


def f32_to_e4m3(x: float) -> int:
    """E4M3 code of x, round to nearest even, finite overflow saturating to 448."""
    return int(lib().orc_f32_to_e4m3_sat(float(x)))


def e8m0_decode(code: int) -> float:
    """Value of an E8M0 scale: 2^(code - 127)."""
    return float(lib().orc_e8m0_decode(int(code)))


def fp4_quant(W_bits: np.ndarray, kind: int):
    """Block-scaled FP4 quantization of bf16 W [N, K] (bit patterns).

    Returns (codes uint8 [N, K/2], two per byte with element 2i in the low
    nibble; scales uint8 [N, K/block]: E4M3 codes for NVFP4, E8M0 for MXFP4)."""
    W_bits = np.ascontiguousarray(W_bits, dtype=np.uint16)
    N, K = W_bits.shape
    B = FP4_BLOCK[kind]
    codes = np.zeros((N, K // 2), dtype=np.uint8)
    scales = np.zeros((N, K // B), dtype=np.uint8)
    if lib().orc_fp4_quant_rows(_ptr(W_bits), N, K, kind, _ptr(codes), _ptr(scales)) != 0:
        raise ValueError("K must be a multiple of the block")
    return codes, scales


def fp4_dequant(codes: np.ndarray, scales: np.ndarray, kind: int) -> np.ndarray:
    """w^ = e2m1(code) * scale as fp32 [N, K] (exact)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    N, K = codes.shape[0], codes.shape[1] * 2
    out = np.zeros((N, K), dtype=np.float32)
    if lib().orc_fp4_dequant_rows(_ptr(codes), _ptr(scales), N, K, kind, _ptr(out)) != 0:
        raise ValueError("K must be a multiple of the block")
    return out


def fp4_reference(X_bits: np.ndarray, codes: np.ndarray, scales: np.ndarray, kind: int, threads: int = 1) -> np.ndarray:
    """Y[m][n] = sum_k x[m][k] * w^[n][k] in fp64 with the FP4-dequantized weights
    (X bf16 [M, K]).  w^ is exact in bf16, so this is gemm_f64 of its bf16 bits."""
    What = fp4_dequant(codes, scales, kind)
    What_bits = (What.view(np.uint32) >> 16).astype(np.uint16)
    return gemm_f64(X_bits, What_bits, threads=threads)


def mxfp8_quant(X_bits: np.ndarray):
    """MXFP8 activations (page 3 section 4.3: activations kept at FP8, MX blocks
    of 32 with an E8M0 scale): returns (codes uint8 [M, K] E4M3, scales uint8
    [M, K/32] E8M0).  The scale rule is stated in w4_oracle.c."""
    X_bits = np.ascontiguousarray(X_bits, dtype=np.uint16)
    M, K = X_bits.shape
    codes = np.zeros((M, K), dtype=np.uint8)
    scales = np.zeros((M, K // 32), dtype=np.uint8)
    if lib().orc_mxfp8_quant_rows(_ptr(X_bits), M, K, _ptr(codes), _ptr(scales)) != 0:
        raise ValueError("K must be a multiple of 32")
    return codes, scales


def mxfp8_dequant(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """x^ = e4m3(code) * scale as fp32 [M, K] (exact)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    M, K = codes.shape
    out = np.zeros((M, K), dtype=np.float32)
    if lib().orc_mxfp8_dequant_rows(_ptr(codes), _ptr(scales), M, K, _ptr(out)) != 0:
        raise ValueError("K must be a multiple of 32")
    return out


def mx_reference(x_codes, x_scales, w_codes, w_scales) -> np.ndarray:
    """Y[m][n] = sum_k x^[m][k] * w^[n][k] in fp64 for MXFP8 activations and
    MXFP4 weights (both factors exact in fp32)."""
    Xd = mxfp8_dequant(x_codes, x_scales).astype(np.float64)
    Wd = fp4_dequant(w_codes, w_scales, MXFP4).astype(np.float64)
    return Xd @ Wd.T
