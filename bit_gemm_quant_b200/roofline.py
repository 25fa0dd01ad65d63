"""Algorithmic work per launch, the denominators of every throughput figure.

Bytes are the compulsory HBM traffic of one call, counted from the tensors it
must read and write once (not DRAM counters):

  w4_quant_pack(N, K, g):  read W (2NK) [+ s (4K)], write qweight (NK/2),
                           scales (2 N K/g) [+ qzeros (4 N ceil(K/g/8)) asym]
  w4a16_gemm(M, N, K, g):  read qweight (NK/2), scales, qzeros (asym), X (2MK),
                           write Y (2MN)
  FLOPs of w4a16_gemm:     2 M N K
  w4_fp4_quant(N, K, B):   read W (2NK), write codes (NK/2) and one scale byte
                           per block of B (N K/B)
  w4_mxfp8_quant(M, K):    read X (2MK), write codes (MK) and scales (MK/32)
  w4_mx_gemm(M, N, K):     read weight codes (NK/2) and scales (NK/32),
                           activation codes (MK) and scales (MK/32), write Y (2MN)
  FLOPs of w4_mx_gemm:     2 M N K
"""
from __future__ import annotations

import json
import os

SYM, ASYM = 0, 1


def packed_bytes(N: int, K: int, g: int, mode: int) -> int:
    G = K // g
    b = N * K // 2 + 2 * N * G
    if mode == ASYM:
        b += 4 * N * ((G + 7) // 8)
    return b


def quant_pack_bytes(N: int, K: int, g: int, mode: int, smooth: bool = False) -> int:
    return 2 * N * K + (4 * K if smooth else 0) + packed_bytes(N, K, g, mode)


def gemm_bytes(M: int, N: int, K: int, g: int, mode: int) -> int:
    return packed_bytes(N, K, g, mode) + 2 * M * K + 2 * M * N


def fp4_quant_bytes(N: int, K: int, block: int) -> int:
    return 2 * N * K + N * K // 2 + N * (K // block)


def mxfp8_quant_bytes(M: int, K: int) -> int:
    return 2 * M * K + M * K + M * K // 32


def mx_gemm_bytes(M: int, N: int, K: int) -> int:
    return N * K // 2 + N * K // 32 + M * K + M * K // 32 + 2 * M * N


def gemm_flops(M: int, N: int, K: int) -> int:
    return 2 * M * N * K


_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks(root: str) -> dict:
    """Measured HBM copy bandwidth and bf16 GEMM throughput of this machine's
    B200s (MEASURED_PEAKS.json at the repository root), else the fallback
    figures; ``source`` says which."""
    path = os.path.join(root, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(_FALLBACK, source="fallback")
