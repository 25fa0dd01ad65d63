"""Pins of the oracle's block-scaled FP4 quantizers (NVFP4, MXFP4) and of the
formats they use (E2M1, FP8 E4M3, E8M0).

Each expected value is printed on a page (tests/golden/fp4_formats.json, cited
there), comes from an independent library routine (torch's float8_e4m3fn), or
from brute force in exact arithmetic over the formats' value sets.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

from conftest import golden

NVFP4, MXFP4 = 0, 1

E2M1_VALUES = {0: 0.0, 1: 0.5, 2: 1.0, 3: 1.5, 4: 2.0, 5: 3.0, 6: 4.0, 7: 6.0}   # code & 7 -> magnitude


def e2m1_nearest(x: float) -> float:
    """Nearest E2M1 value to x in exact arithmetic, ties to the even fraction
    bit (the low bit of the code), by brute force over the eight magnitudes."""
    fx = Fraction(abs(x))
    best = None
    for code, v in E2M1_VALUES.items():
        d = abs(fx - Fraction(v))
        key = (d, code & 1)
        if best is None or key < best[0]:
            best = (key, v)
    v = best[1]
    return -v if x < 0 else v


def bf16(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns of fp32 values (torch's round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_value(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


# ------------------------------------------------------------------ E2M1 --

def test_e2m1_encode_is_nearest_value_ties_to_even(oracle_mod):
    xs = [i / 64 for i in range(-640, 641)] + [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 7.0, 100.0, 1e-30]
    xs += list(np.random.default_rng(3).standard_normal(2000) * 3)
    for x in xs:
        x = float(np.float32(x))
        got = oracle_mod.e2m1_decode(oracle_mod.f32_to_e2m1(x))
        assert got == e2m1_nearest(x), (x, got, e2m1_nearest(x))


def test_e2m1_encode_inverts_decode(oracle_mod):
    for c in range(16):
        assert oracle_mod.f32_to_e2m1(oracle_mod.e2m1_decode(c)) == c


# ------------------------------------------------------------------ E4M3 --

def test_e4m3_format_facts(oracle_mod):
    fx = golden("fp4_formats.json")["e4m3"]
    vals = [oracle_mod.e4m3_decode(c) for c in range(256)]
    finite = [v for v in vals if v == v]
    assert max(finite) == fx["max"] and min(finite) == -fx["max"]
    assert oracle_mod.e4m3_decode(1 << fx["fraction_bits"]) == fx["min_normal"]
    assert [c for c in range(256) if vals[c] != vals[c]] == fx["nan_codes"]


def test_e4m3_decode_matches_torch(oracle_mod):
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    for c in range(256):
        got = oracle_mod.e4m3_decode(c)
        assert (got == ref[c]) or (got != got and ref[c] != ref[c]), (c, got, ref[c])


def test_e4m3_encode_matches_torch_in_range(oracle_mod):
    finite = sorted({oracle_mod.e4m3_decode(c) for c in range(128) if c != 127})
    mids = [(a + b) / 2 for a, b in zip(finite, finite[1:])]
    rng = np.random.default_rng(7)
    xs = np.array(finite + mids + list(rng.uniform(-448, 448, 4000)) +
                  list(rng.standard_normal(4000) * 2.0 ** rng.integers(-12, 8, 4000)), dtype=np.float32)
    xs = np.concatenate([xs, -xs])
    xs = xs[np.abs(xs) <= 448]
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle_mod.f32_to_e4m3(float(x)) for x in xs], dtype=np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (xs[bad[:5]], got[bad[:5]], ref[bad[:5]])


def test_e4m3_saturates(oracle_mod):
    assert oracle_mod.f32_to_e4m3(1e6) == 0x7E and oracle_mod.f32_to_e4m3(-1e6) == 0xFE
    assert oracle_mod.f32_to_e4m3(479.0) == 0x7E          # rounds to 480 > 448
    assert oracle_mod.f32_to_e4m3(float("inf")) == 0x7E


def test_e8m0_is_a_power_of_two(oracle_mod):
    for c in (0, 1, 100, 127, 128, 254):
        assert oracle_mod.e8m0_decode(c) == 2.0 ** (c - 127)


# ---------------------------------------------------------- block quant --

@pytest.mark.parametrize("kind", [NVFP4, MXFP4])
def test_bits_per_weight_from_buffer_sizes(oracle_mod, kind):
    fx = golden("fp4_formats.json")
    N, K = 8, 256
    codes, scales = oracle_mod.fp4_quant(bf16(np.ones((N, K), np.float32)), kind)
    bits = (codes.nbytes + scales.nbytes) * 8 / (N * K)
    if kind == NVFP4:
        assert bits == fx["nvfp4"]["bits_per_weight"]               # printed on page 2
    else:
        assert bits == 4 + fx["mxfp4"]["scale_bits"] / fx["mxfp4"]["block"]


@pytest.mark.parametrize("kind", [NVFP4, MXFP4])
@pytest.mark.parametrize("sigma", [1.0, 0.02])
def test_block_quant_follows_definition(oracle_mod, kind, sigma):
    """Every scale and every code against the definitions, computed here in
    exact arithmetic: the scale from the block's amax (E4M3 of fl32(amax/6) by
    torch's conversion for NVFP4; 2^(floor(log2 amax) - 2) for MXFP4) and each
    code as the nearest E2M1 value of fl32(w / scale), ties to even, saturated."""
    rng = np.random.default_rng(11 + kind)
    N, K = 6, 128
    Wb = bf16((rng.standard_normal((N, K)) * sigma).astype(np.float32))
    W = bf16_value(Wb)
    codes, scales = oracle_mod.fp4_quant(Wb, kind)
    B = 16 if kind == NVFP4 else 32
    for n in range(N):
        for b in range(K // B):
            blk = W[n, b * B:(b + 1) * B]
            amax = float(np.max(np.abs(blk)))
            if kind == NVFP4:
                t = np.float32(np.float32(amax) / np.float32(6.0))
                sc_ref = int(torch.tensor([t]).to(torch.float8_e4m3fn).view(torch.uint8)[0])
                s = float(torch.tensor([sc_ref], dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).float()[0])
            else:
                e = max(-127, min(127, int(np.floor(np.log2(amax))) - 2)) if amax > 0 else -127
                sc_ref, s = e + 127, 2.0 ** e
            assert scales[n, b] == sc_ref, (n, b)
            for i in range(B):
                k = b * B + i
                q = (codes[n, k // 2] >> (4 * (k & 1))) & 15
                want = 0.0 if s == 0 else e2m1_nearest(float(np.float32(np.float32(blk[i]) / np.float32(s))))
                assert oracle_mod.e2m1_decode(q) == want, (n, k, blk[i], s)


def test_nvfp4_block_maximum_maps_to_six(oracle_mod):
    """With a normal E4M3 scale, amax / s lies within 6 (1 -+ 2^-4)^-1, which
    rounds (or saturates) to 6: every block holds a code of magnitude 6."""
    rng = np.random.default_rng(21)
    Wb = bf16((rng.standard_normal((16, 256)) * 2.0).astype(np.float32))
    codes, scales = oracle_mod.fp4_quant(Wb, NVFP4)
    vals = oracle_mod.fp4_dequant(codes, scales, NVFP4)
    for n in range(16):
        for b in range(16):
            s = oracle_mod.e4m3_decode(int(scales[n, b]))
            assert s >= golden("fp4_formats.json")["e4m3"]["min_normal"]
            assert np.max(np.abs(vals[n, b * 16:(b + 1) * 16])) == 6.0 * s


def test_mxfp4_block_maximum_maps_to_four_or_six(oracle_mod):
    """amax / 2^(floor(log2 amax) - 2) lies in [4, 8): the block maximum's code
    is 4 or 6 (values of 7 and above saturate to 6)."""
    rng = np.random.default_rng(22)
    Wb = bf16((rng.standard_normal((16, 256)) * 0.02).astype(np.float32))
    codes, scales = oracle_mod.fp4_quant(Wb, MXFP4)
    W = bf16_value(Wb)
    for n in range(16):
        for b in range(8):
            s = oracle_mod.e8m0_decode(int(scales[n, b]))
            r = np.max(np.abs(W[n, b * 32:(b + 1) * 32])) / s
            assert 4.0 <= r < 8.0
            q = [(codes[n, k // 2] >> (4 * (k & 1))) & 15 for k in range(b * 32, (b + 1) * 32)]
            assert max(abs(oracle_mod.e2m1_decode(c)) for c in q) in (4.0, 6.0)


@pytest.mark.parametrize("kind", [NVFP4, MXFP4])
def test_dequant_is_the_exact_product_and_fits_bf16(oracle_mod, kind):
    rng = np.random.default_rng(23)
    Wb = bf16((rng.standard_normal((4, 64)) * 0.5).astype(np.float32))
    codes, scales = oracle_mod.fp4_quant(Wb, kind)
    got = oracle_mod.fp4_dequant(codes, scales, kind)
    B = 16 if kind == NVFP4 else 32
    for n in range(4):
        for k in range(64):
            q = (codes[n, k // 2] >> (4 * (k & 1))) & 15
            sc = int(scales[n, k // B])
            s = oracle_mod.e4m3_decode(sc) if kind == NVFP4 else oracle_mod.e8m0_decode(sc)
            assert float(got[n, k]) == oracle_mod.e2m1_decode(q) * s
    assert np.array_equal(bf16_value(bf16(got)), got)


def test_packing_puts_the_even_element_in_the_low_nibble(oracle_mod):
    # a 16-weight block with amax 3: s = e4m3(0.5) = 0.5, so w = 3 -> 6 (code 0b0111) and
    # w = -1 -> -2 (code 0b1100)
    w = np.zeros((1, 16), np.float32)
    w[0, 0], w[0, 1], w[0, 2] = 3.0, -1.0, 0.5
    codes, scales = oracle_mod.fp4_quant(bf16(w), NVFP4)
    assert oracle_mod.e4m3_decode(int(scales[0, 0])) == 0.5
    assert codes[0, 0] == (0xC << 4) | 0x7          # element 0 low nibble, element 1 high nibble
    assert codes[0, 1] == 0x2                       # element 2 = 0.5 / 0.5 = 1.0 -> code 2


def test_zero_block_gives_zero_codes(oracle_mod):
    for kind in (NVFP4, MXFP4):
        codes, scales = oracle_mod.fp4_quant(np.zeros((2, 64), np.uint16), kind)
        assert not codes.any()
        assert np.all(oracle_mod.fp4_dequant(codes, scales, kind) == 0.0)


@pytest.mark.parametrize("kind", [NVFP4, MXFP4])
def test_product_reference_selects_dequantized_columns(oracle_mod, kind):
    """One-hot activation rows pick columns of w^ (the product's orientation),
    and a dense product equals a plain fp64 matrix product of the decoded
    weights (decoded here from the codes and scales, not by the oracle)."""
    rng = np.random.default_rng(31 + kind)
    N, K = 12, 64
    Wb = bf16((rng.standard_normal((N, K)) * 0.5).astype(np.float32))
    codes, scales = oracle_mod.fp4_quant(Wb, kind)
    B = 16 if kind == NVFP4 else 32
    Wd = np.zeros((N, K))
    for n in range(N):
        for k in range(K):
            q = int((codes[n, k // 2] >> (4 * (k & 1))) & 15)
            mag = E2M1_VALUES[q & 7] * (-1.0 if q & 8 else 1.0)
            sc = int(scales[n, k // B])
            if kind == NVFP4:
                s = float(torch.tensor([sc], dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).float()[0])
            else:
                s = 2.0 ** (sc - 127)
            Wd[n, k] = mag * s
    ks = [0, 17, 63]
    X = np.zeros((len(ks), K), np.float32)
    for m, k in enumerate(ks):
        X[m, k] = 1.0
    Y = oracle_mod.fp4_reference(bf16(X), codes, scales, kind)
    for m, k in enumerate(ks):
        assert np.array_equal(Y[m], Wd[:, k])
    Xr = bf16((rng.standard_normal((5, K))).astype(np.float32))
    Y = oracle_mod.fp4_reference(Xr, codes, scales, kind)
    assert np.allclose(Y, bf16_value(Xr).astype(np.float64) @ Wd.T, rtol=1e-12, atol=1e-12)


# ------------------------------------------------- MXFP8 activations --

def _e4m3_code_torch(t: float) -> int:
    """torch's E4M3 code of t after saturation to +-448 (torch's own conversion
    gives NaN above the range; rounding never takes a value <= 448 above it)."""
    t = max(-448.0, min(448.0, t))
    return int(torch.tensor([t], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)[0])


@pytest.mark.parametrize("sigma", [1.0, 40.0, 1e-3])
def test_mxfp8_follows_definition(oracle_mod, sigma):
    """Scale 2^(floor(log2 amax) - 8) per 32 activations, codes E4M3 of
    fl32(x / scale) saturated at 448 (torch's conversion), checked one by one."""
    rng = np.random.default_rng(41)
    M, K = 4, 128
    Xb = bf16((rng.standard_normal((M, K)) * sigma).astype(np.float32))
    X = bf16_value(Xb)
    codes, scales = oracle_mod.mxfp8_quant(Xb)
    for m in range(M):
        for b in range(K // 32):
            blk = X[m, b * 32:(b + 1) * 32]
            amax = float(np.max(np.abs(blk)))
            e = max(-127, min(127, int(np.floor(np.log2(amax))) - 8)) if amax > 0 else -127
            assert scales[m, b] == e + 127
            for i in range(32):
                t = float(np.float32(np.float32(blk[i]) / np.float32(2.0 ** e)))
                assert codes[m, b * 32 + i] == _e4m3_code_torch(t), (m, b, i)


def test_mxfp8_block_maximum_and_exact_dequant(oracle_mod):
    """amax / scale lies in [256, 512): the block maximum's code is at least
    256 (448 when saturated), and x^ = e4m3(code) * scale exactly."""
    rng = np.random.default_rng(42)
    Xb = bf16((rng.standard_normal((8, 256)) * 3.0).astype(np.float32))
    codes, scales = oracle_mod.mxfp8_quant(Xb)
    d = oracle_mod.mxfp8_dequant(codes, scales)
    for m in range(8):
        for b in range(8):
            s = oracle_mod.e8m0_decode(int(scales[m, b]))
            vals = [oracle_mod.e4m3_decode(int(c)) for c in codes[m, b * 32:(b + 1) * 32]]
            assert 256.0 <= max(abs(v) for v in vals) <= 448.0
            assert all(float(d[m, b * 32 + i]) == vals[i] * s for i in range(32))


def test_mx_product_reference(oracle_mod):
    """One-hot activation rows are exact in MXFP8 (1.0 = 256 * 2^-8) and pick
    columns of w^; a dense product equals the fp64 product of the two
    dequantized operands."""
    rng = np.random.default_rng(43)
    N, K = 10, 96
    Wb = bf16((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    wc, ws = oracle_mod.fp4_quant(Wb, MXFP4)
    Wd = oracle_mod.fp4_dequant(wc, ws, MXFP4).astype(np.float64)
    ks = [3, 40, 95]
    X = np.zeros((len(ks), K), np.float32)
    for m, k in enumerate(ks):
        X[m, k] = 1.0
    xc, xs = oracle_mod.mxfp8_quant(bf16(X))
    Y = oracle_mod.mx_reference(xc, xs, wc, ws)
    for m, k in enumerate(ks):
        assert np.array_equal(Y[m], Wd[:, k])
    xc, xs = oracle_mod.mxfp8_quant(bf16((rng.standard_normal((6, K))).astype(np.float32)))
    Xd = oracle_mod.mxfp8_dequant(xc, xs).astype(np.float64)
    assert np.allclose(oracle_mod.mx_reference(xc, xs, wc, ws), Xd @ Wd.T, rtol=1e-12, atol=1e-15)
