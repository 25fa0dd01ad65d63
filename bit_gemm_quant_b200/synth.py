"""Seeded synthetic inputs for the W4A16 path.

This module draws the inputs that both the CUDA library and the CPU oracle
consume: bf16 weights and activations with outlier channels, and the smoothing
vector handed to the quantizer.  It holds none of the quantization arithmetic;
it only draws random numbers (numpy ``default_rng``, PCG64) and rounds them to
bf16 with torch's CPU conversion.  The same seed gives the same bit patterns on
every machine.

Workloads (shapes from the Llama-style layers the pages discuss; outlier
channels follow the "1% of channels are salient" observation of the AWQ and
SmoothQuant sections of the pages):

  tiny        W[256,512] ~ N(0,0.02), symmetric g=128; X[4,512] ~ N(0,1) with
              channels 0 and 1 scaled x40 and x10.
  decode      M=1, K=4096, N in {4096, 11008, 12288}, asymmetric g=128;
              W ~ N(0,0.02) with 1% of input columns x5; X ~ N(0,1) with 1% of
              channels x40.
  smallbatch  M in {2,4,8,16,32}, K=8192, N=28672, symmetric g=128;
              W ~ N(0,0.015); X ~ N(0,1) with 0.5% of channels x30.
  prefill     M in {512,2048,8192}, K=4096, N=14336, asymmetric g=128;
              W ~ N(0,0.02); X ~ N(0,1) with 1% of channels x40.
  quantizer   W[28672,8192] ~ N(0,0.02); g in {32,64,128} x {sym, asym}; plus
              the smoothing fold with s = act^0.5/mean(act^0.5),
              act = |N(0,1)| with 1% of channels x20.
  decodequant the decode workload's three weights, quantized (no product).
  mxdecode    the decode workload's layers (same seeds and distributions) for
              the block-scaled product: MXFP4 weights, MXFP8 activations.

"p% outlier channels" are the first round(p*K) entries of a seeded
permutation of 0..K-1; weight columns and activation channels are drawn
independently.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

SYM, ASYM = 0, 1

# tags that separate the random streams of the tensors of one workload
_TAG_W, _TAG_WCOLS, _TAG_X, _TAG_XCOLS, _TAG_ACT, _TAG_ACTCOLS = 11, 12, 21, 22, 31, 32


def _rng(seed: int, tag: int, *extra: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(tag)] + [int(e) for e in extra])


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round an fp32 array to bf16 (torch CPU conversion) and return the bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def outlier_channels(seed: int, tag: int, K: int, frac: float) -> np.ndarray:
    n = int(round(frac * K))
    return _rng(seed, tag, K).permutation(K)[:n]


def weights(seed: int, N: int, K: int, std: float, outlier_frac: float = 0.0,
            outlier_mult: float = 1.0) -> np.ndarray:
    """bf16 bit patterns of W[N,K] ~ N(0, std^2), with a fraction of input
    columns multiplied by ``outlier_mult``."""
    w = _rng(seed, _TAG_W, N, K).standard_normal((N, K), dtype=np.float32)
    w *= np.float32(std)
    if outlier_frac > 0:
        cols = outlier_channels(seed, _TAG_WCOLS, K, outlier_frac)
        w[:, cols] *= np.float32(outlier_mult)
    return to_bf16_bits(w)


def activations(seed: int, M: int, K: int, outlier_frac: float = 0.0, outlier_mult: float = 1.0,
                fixed_channels: dict | None = None) -> np.ndarray:
    """bf16 bit patterns of X[M,K] ~ N(0,1) with outlier channels."""
    x = _rng(seed, _TAG_X, M, K).standard_normal((M, K), dtype=np.float32)
    if outlier_frac > 0:
        cols = outlier_channels(seed, _TAG_XCOLS, K, outlier_frac)
        x[:, cols] *= np.float32(outlier_mult)
    if fixed_channels:
        for c, mult in fixed_channels.items():
            x[:, c] *= np.float32(mult)
    return to_bf16_bits(x)


def smoothing_vector(seed: int, K: int, alpha: float = 0.5, outlier_frac: float = 0.01,
                     outlier_mult: float = 20.0) -> np.ndarray:
    """The per-input-channel smoothing vector the quantizer folds into W.

    Input recipe: mean activation magnitudes act = |N(0,1)| with 1% of the
    channels x20, and s = act^alpha / mean(act^alpha) evaluated in fp64 and
    rounded to fp32.  The library takes s as given; this is only how the
    synthetic s is drawn.
    """
    act = np.abs(_rng(seed, _TAG_ACT, K).standard_normal(K))
    if outlier_frac > 0:
        act[outlier_channels(seed, _TAG_ACTCOLS, K, outlier_frac)] *= outlier_mult
    p = act ** alpha
    return (p / p.mean()).astype(np.float32)


@dataclass
class Problem:
    """One quantize + multiply problem of a workload."""
    name: str
    M: int
    N: int
    K: int
    group: int
    mode: int
    w_std: float
    w_outlier: tuple = (0.0, 1.0)
    x_outlier: tuple = (0.0, 1.0)
    x_fixed: dict = field(default_factory=dict)
    smooth: bool = False
    seed: int = 0

    def W(self) -> np.ndarray:
        return weights(self.seed, self.N, self.K, self.w_std, *self.w_outlier)

    def X(self) -> np.ndarray:
        return activations(self.seed, self.M, self.K, *self.x_outlier, fixed_channels=self.x_fixed)

    def s(self):
        return smoothing_vector(self.seed, self.K) if self.smooth else None


def workload(name: str) -> list[Problem]:
    """The problems of a named workload (see the module docstring)."""
    if name == "tiny":
        return [Problem("tiny", 4, 256, 512, 128, SYM, 0.02, x_fixed={0: 40.0, 1: 10.0}, seed=0)]
    if name == "decode":
        return [Problem("decode_N%d" % N, 1, N, 4096, 128, ASYM, 0.02, (0.01, 5.0), (0.01, 40.0), seed=1)
                for N in (4096, 11008, 12288)]
    if name == "smallbatch":
        return [Problem("smallbatch_M%d" % M, M, 28672, 8192, 128, SYM, 0.015, (0.0, 1.0), (0.005, 30.0), seed=2)
                for M in (2, 4, 8, 16, 32)]
    if name == "prefill":
        return [Problem("prefill_M%d" % M, M, 14336, 4096, 128, ASYM, 0.02, (0.0, 1.0), (0.01, 40.0), seed=3)
                for M in (512, 2048, 8192)]
    if name == "decodequant":
        # the decode layers' weights (same seeds as the decode workload), quantized
        return [Problem("decode_N%d" % N, 0, N, 4096, 128, ASYM, 0.02, (0.01, 5.0), seed=1)
                for N in (4096, 11008, 12288)]
    if name == "mxdecode":
        return [Problem("mxdecode_N%d" % N, 1, N, 4096, 128, ASYM, 0.02, (0.01, 5.0), (0.01, 40.0), seed=1)
                for N in (4096, 11008, 12288)]
    if name == "quantizer":
        probs = []
        for g in (32, 64, 128):
            for mode in (SYM, ASYM):
                probs.append(Problem("quantizer_g%d_%s" % (g, "sym" if mode == SYM else "asym"),
                                     0, 28672, 8192, g, mode, 0.02, seed=4))
        probs.append(Problem("quantizer_g128_sym_smooth", 0, 28672, 8192, 128, SYM, 0.02, smooth=True, seed=4))
        return probs
    raise KeyError(name)


WORKLOADS = ("tiny", "decode", "smallbatch", "prefill", "quantizer", "decodequant", "mxdecode")
