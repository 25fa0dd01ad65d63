"""Pins of the CPU oracle against facts the pages and the mathematics fix.

None of these compares the oracle with itself: each expected value is printed
on a page (fixtures under tests/golden/, cited there), follows from a closed
form, comes from an independent library routine (numpy/torch format
conversions, scipy quadrature, exact rational arithmetic), or is a literal
derived by hand from the documented packed layout.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from conftest import golden

SYM, ASYM = 0, 1


# ---------------------------------------------------------------- formats --

def _interesting_f32(rng, n):
    """fp32 values around fp16 rounding boundaries, subnormals and overflow."""
    vals = [0.0, -0.0, 65504.0, 65519.99, 65520.0, 65536.0, 1e-8, 2.0 ** -24, 2.0 ** -25,
            3 * 2.0 ** -26, 2.0 ** -14, 6.1e-5, 1.0, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11]
    base = rng.standard_normal(n).astype(np.float32) * np.float32(4.0) ** rng.integers(-14, 9, n)
    # halfway points between consecutive fp16 values
    h = rng.integers(1, 0x7BFF, n // 4).astype(np.uint16)
    lo = h.view(np.float16).astype(np.float32)
    hi = (h + 1).view(np.float16).astype(np.float32)
    mid = ((lo.astype(np.float64) + hi.astype(np.float64)) / 2).astype(np.float32)
    return np.concatenate([np.array(vals, np.float32), base, mid, -mid])


def test_f16_conversion_matches_numpy(oracle_mod):
    rng = np.random.default_rng(5)
    xs = _interesting_f32(rng, 20000)
    with np.errstate(over="ignore"):
        ref = xs.astype(np.float16).view(np.uint16)
    got = np.array([oracle_mod.f32_to_f16_bits(x) for x in xs], dtype=np.uint16)
    assert np.array_equal(got, ref)
    back = np.array([oracle_mod.f16_bits_to_f32(h) for h in ref[np.isfinite(ref.view(np.float16))]],
                    dtype=np.float32)
    assert np.array_equal(back, ref[np.isfinite(ref.view(np.float16))].view(np.float16).astype(np.float32))


def test_bf16_conversion_matches_torch(oracle_mod):
    rng = np.random.default_rng(6)
    xs = np.concatenate([rng.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** rng.integers(-38, 38, 20000).astype(np.float32),
                         (rng.integers(0, 1 << 16, 5000).astype(np.uint32) << 16 | 0x8000).view(np.float32)])
    xs = xs[np.isfinite(xs)]
    ref = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle_mod.f32_to_bf16_bits(x) for x in xs], dtype=np.uint16)
    assert np.array_equal(got, ref)


# ------------------------------------------------------- worked example ----

def test_worked_example_page1(oracle_mod):
    """Range [-3.2, 3.2] on 16 levels: step 0.427, w = 0.21 lands on 0 (error 0.21, x100 -> 21)."""
    ex = golden("worked_example_uniform_int4.json")
    lo, hi = ex["range"]
    w = np.zeros(32, np.float32)
    w[0], w[1], w[2] = lo, hi, ex["w"]
    s16, zp, u = oracle_mod.quant_group(w, ASYM)
    step32 = np.float32(np.float32(hi) - np.float32(lo)) / np.float32(ex["levels"] - 1)
    assert round(float(step32), 3) == ex["step_printed"]
    d = oracle_mod.f16_bits_to_f32(s16)
    assert abs(d - ex["step_printed"]) < 5e-4
    w_hat = (int(u[2]) - zp) * d
    assert w_hat == ex["w_quantized_printed"]
    err = abs(ex["w"] - w_hat)
    assert round(err, 2) == ex["error_printed"]
    assert round(err * ex["activation"], 6) == ex["output_error_printed"]
    # the extremes take the end codes
    assert u[0] == 0 and u[1] in (14, 15)
    # symmetric reading of the same group also sends 0.21 to 0
    s16s, zps, us = oracle_mod.quant_group(w, SYM)
    assert (int(us[2]) - zps) == 0


# ---------------------------------------------------------- bits/weight ----

def test_bits_per_weight_from_buffers(oracle_mod):
    fx = golden("bits_per_weight.json")
    N, K = 64, 1024
    W = (np.arange(N * K, dtype=np.uint32) % 251).astype(np.uint16) + 0x3C00
    W = W.reshape(N, K)
    for case in fx["cases"]:
        mode = SYM if case["mode"] == "sym" else ASYM
        g = case["group"]
        q, s, z = oracle_mod.quant_pack(W, g, mode)
        bits = (q.nbytes + s.nbytes) * 8 / (N * K)
        if mode == SYM:
            assert z is None
            assert bits == case["bits_per_weight"]
        else:
            assert bits == case["bits_per_weight_scale_only"]
            zbits = z.nbytes * 8 / (N * K)
            assert zbits == case["zp_bits"] / g


# ---------------------------------------------------- error bound & codes --

def _groups(rng, n, g, scale_pow):
    out = []
    for i in range(n):
        v = rng.standard_normal(g).astype(np.float32) * np.float32(2.0 ** rng.integers(-scale_pow, scale_pow))
        if i % 3 == 1:
            v = np.abs(v)                    # single-signed group
        if i % 3 == 2:
            v[rng.integers(0, g)] *= 30       # an outlier
        out.append(v)
    return out


@pytest.mark.parametrize("mode", [SYM, ASYM])
def test_rounding_error_at_most_half_step(oracle_mod, mode):
    """Page 5 section 2.2: rounding error is at most half a step inside the clip range."""
    rng = np.random.default_rng(7)
    for w in _groups(rng, 300, 32, 12):
        s16, zp, u = oracle_mod.quant_group(w, mode)
        d = oracle_mod.f16_bits_to_f32(s16)
        n = np.array([round(Fraction(float(x)) / Fraction(d)) if d else 0 for x in w], dtype=np.int64)
        inside = (n + zp >= 0) & (n + zp <= 15)
        err = np.abs(w.astype(np.float64) - (u.astype(np.float64) - zp) * d)
        assert np.all(err[inside] <= d / 2)
        if mode == SYM:
            assert inside.all(), "symmetric codes are never clipped"
            assert (u.astype(int) - 8).min() >= -7, "q = -8 never occurs with s = amax/7"
        else:
            # clipping only ever touches the top code, by a sliver beyond half a step
            assert np.all(err[~inside] <= d / 2 * (1 + 2.0 ** -5))


def _brute_force_code(x, d, zp):
    """argmin over the 16 codes of |x - (c - zp) d| in exact arithmetic; ties go
    to the even integer c - zp (round half to even, page 5 section 2.2)."""
    X, D = Fraction(float(x)), Fraction(float(d))
    best = None
    for c in range(16):
        e = abs(X - (c - zp) * D)
        key = (e, (c - zp) % 2)
        if best is None or key < best[0]:
            best = (key, c)
    return best[1]


@pytest.mark.parametrize("mode", [SYM, ASYM])
def test_codes_equal_brute_force_over_16_codes(oracle_mod, mode):
    rng = np.random.default_rng(8)
    groups = _groups(rng, 120, 32, 6)
    # engineered ties and neighbours of ties: scale fixed by the amax element
    for dt in (0.6, 0.15, 1.0 / 3, 0.0123):
        amax = np.float32(7 * dt)
        s16 = oracle_mod.f32_to_f16_bits(np.float32(amax / np.float32(7)))
        d = oracle_mod.f16_bits_to_f32(s16)
        v = [amax, -amax]
        for n in range(-7, 7):
            b = np.float32((n + 0.5) * d)          # exact: b*d has <= 16 significant bits
            v += [b, np.nextafter(b, np.float32(np.inf)), np.nextafter(b, np.float32(-np.inf))]
        v = np.array(v, np.float32)
        for i in range(0, len(v), 30):
            grp = np.zeros(32, np.float32)
            chunk = v[i:i + 30]
            grp[:len(chunk)] = chunk
            grp[30], grp[31] = amax, -amax
            groups.append(grp)
    for w in groups:
        s16, zp, u = oracle_mod.quant_group(w, mode)
        d = oracle_mod.f16_bits_to_f32(s16)
        if d == 0:
            continue
        expect = [_brute_force_code(x, d, zp) for x in w]
        assert list(u) == expect


def test_invariants_and_degenerate_groups(oracle_mod):
    rng = np.random.default_rng(9)
    for w in _groups(rng, 200, 64, 8):
        s16, zp, u = oracle_mod.quant_group(w, ASYM)
        assert 0 <= zp <= 15
        mn, mx = min(w.min(), 0), max(w.max(), 0)
        if mn < 0:
            assert u[np.argmin(w)] == 0, "min maps to code 0"
        if mx > 0:
            assert u[np.argmax(w)] in (14, 15), "max maps to the top codes"
    # all-zero group: zero scale and zero codes
    s16, zp, u = oracle_mod.quant_group(np.zeros(32, np.float32), SYM)
    assert s16 == 0 and zp == 8 and np.all(u == 8)
    s16, zp, u = oracle_mod.quant_group(np.zeros(32, np.float32), ASYM)
    assert s16 == 0 and zp == 0 and np.all(u == 0)
    # fp16 underflow of the scale
    tiny = np.full(32, 1e-8, np.float32)
    s16, zp, u = oracle_mod.quant_group(tiny, SYM)
    assert s16 == 0 and np.all(u == 8)
    # scale saturates at the largest finite fp16
    big = np.zeros(32, np.float32)
    big[0], big[1] = 1e6, -3e5
    s16, zp, u = oracle_mod.quant_group(big, SYM)
    assert s16 == 0x7BFF and u[0] == 15 and u[1] == 8 - 5
    s16, zp, u = oracle_mod.quant_group(big, ASYM)
    assert s16 == 0x7BFF and u[0] == 15


# ----------------------------------------------------- layout literals -----

def test_packed_layout_literals(oracle_mod):
    """Word c holds even elements 8c,8c+2,.. in its low half and odd elements
    in its high half; zero-points are nibble j%8 of word j/8."""
    # a bf16 row whose codes are 0,1,...,15 in the first 16 positions (asymmetric,
    # 16 distinct levels 0..15 -> min 0 gives zp 0, step 1)
    K, g = 32, 32
    row = np.zeros((1, K), np.float32)
    row[0, :16] = np.arange(16)
    W = torch.from_numpy(row).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q, s, z = oracle_mod.quant_pack(W, g, ASYM)
    assert oracle_mod.f16_bits_to_f32(s[0, 0]) == 1.0
    assert z[0, 0] == 0
    assert q[0, 0] == 0x75316420
    assert q[0, 1] == 0xFDB9ECA8
    assert q[0, 2] == 0 and q[0, 3] == 0
    # zero-points of 9 groups: group j gets zp = j (values shifted so min = -j)
    K, g = 9 * 32, 32
    row = np.zeros((1, K), np.float32)
    for j in range(9):
        row[0, j * g] = -j
        row[0, j * g + 1] = 15 - j
    W = torch.from_numpy(row).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q, s, z = oracle_mod.quant_pack(W, g, ASYM)
    assert z.shape == (1, 2)
    assert z[0, 0] == 0x76543210 and z[0, 1] == 0x8


# ---------------------------------------------------------------- dequant --

def test_dequant_is_single_bf16_rounding_of_exact_product(oracle_mod):
    rng = np.random.default_rng(10)
    N, K, g = 8, 256, 64
    W = torch.from_numpy(rng.standard_normal((N, K)).astype(np.float32) * 0.02).to(torch.bfloat16)
    Wb = W.view(torch.int16).numpy().view(np.uint16)
    for mode in (SYM, ASYM):
        q, s, z = oracle_mod.quant_pack(Wb, g, mode)
        what = oracle_mod.dequant(q, s, z, K, g, mode)
        exact = oracle_mod.dequant(q, s, z, K, g, mode, exact_f32=True)
        # exact product recomputed here from codes read with numpy shifts
        shifts = np.array([0, 16, 4, 20, 8, 24, 12, 28], np.uint32)
        codes = ((q[:, :, None] >> shifts[None, None, :]) & 0xF).reshape(N, K).astype(np.int64)
        if mode == SYM:
            zps = np.full((N, K // g), 8)
        else:
            zps = ((z[:, :, None] >> (4 * np.arange(8, dtype=np.uint32))) & 0xF).reshape(N, -1)[:, :K // g]
        sc = s.view(np.float16).astype(np.float64)
        prod = (codes - np.repeat(zps, g, axis=1)) * np.repeat(sc, g, axis=1)
        assert np.array_equal(exact.astype(np.float64), prod)
        ref = torch.from_numpy(prod).to(torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(what, ref)


# ------------------------------------------------------------------ gemm --

def test_gemm_orientation_and_values(oracle_mod):
    rng = np.random.default_rng(11)
    K, C = 16, 3
    What = torch.from_numpy(rng.standard_normal((C, K)).astype(np.float32)).to(torch.bfloat16)
    Wb = What.view(torch.int16).numpy().view(np.uint16)
    # one-hot rows of X select columns k of W^: Y[m][c] = w^[c][k_m]
    ks = [0, 5, 15]
    X = np.zeros((len(ks), K), np.float32)
    for m, k in enumerate(ks):
        X[m, k] = 1.0
    Xb = torch.from_numpy(X).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    Y = oracle_mod.gemm_f64(Xb, Wb)
    assert Y.shape == (len(ks), C)
    wf = What.float().numpy().astype(np.float64)
    for m, k in enumerate(ks):
        assert np.array_equal(Y[m], wf[:, k])
    # a hand-sized product: x = (1, 2, 0, ...), w^ row c = (c+1, -1, ...)
    X = np.zeros((1, K), np.float32); X[0, 0], X[0, 1] = 1, 2
    W2 = np.zeros((C, K), np.float32)
    for c in range(C):
        W2[c, 0], W2[c, 1] = c + 1, -1
    Y = oracle_mod.gemm_f64(torch.from_numpy(X).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16),
                            torch.from_numpy(W2).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    assert Y.tolist() == [[-1.0, 0.0, 1.0]]


# ------------------------------------------------------------- smoothing --

def test_fold_multiplies_weights_along_input_channels(oracle_mod):
    """Page 5 section 2.4 / page 3 section 5.3: W' = W * diag(s), one factor per input channel k."""
    N, K, g = 4, 64, 32
    W = np.ones((N, K), np.float32)
    W[1] *= 0.5
    Wb = torch.from_numpy(W).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    s = np.ones(K, np.float32)
    s[3], s[40] = 4.0, 0.25
    q1, s1, _ = oracle_mod.quant_pack(Wb, g, SYM, s=s)
    Wf = (W * s[None, :]).astype(np.float32)
    # quantizing the pre-multiplied fp32 weights group by group gives the same codes
    for n in range(N):
        for j in range(K // g):
            s16, zp, u = oracle_mod.quant_group(Wf[n, j * g:(j + 1) * g], SYM)
            assert s1[n, j] == s16
    # element 3 is the largest of group 0: it takes code +7; element 40 is 1/4 of the rest of group 1
    d0 = oracle_mod.f16_bits_to_f32(s1[0, 0])
    assert d0 == oracle_mod.f16_bits_to_f32(oracle_mod.f32_to_f16_bits(np.float32(4.0) / np.float32(7.0)))
    what = oracle_mod.dequant(q1, s1, None, K, g, SYM, exact_f32=True)
    assert what[0, 3] == 7 * d0


def test_smoothing_identity_page4_demo():
    """(X/s)(W s)^T equals X W^T: to rounding in fp64, and within the page's 1e-5 in fp32."""
    fx = golden("smoothing_identity.json")
    rng = np.random.default_rng(239)
    x = rng.standard_normal((fx["tokens"], fx["hidden"]))
    for c, m in fx["x_channel_mult"].items():
        x[:, int(c)] *= m
    w = rng.standard_normal((fx["hidden"], fx["output"]))
    for r, m in fx["w_row_mult"].items():
        w[int(r)] *= m
    a = np.abs(x).max(0)
    b = np.abs(w).max(1)
    s = a ** fx["alpha"] / b ** (1 - fx["alpha"])
    ref = x @ w
    sm = (x / s) @ (w * s[:, None])
    assert np.abs(sm - ref).max() <= 1e-12 * np.abs(ref).max()
    x32, w32, s32 = x.astype(np.float32), w.astype(np.float32), s.astype(np.float32)
    sm32 = (x32 / s32) @ (w32 * s32[:, None])
    ref32 = x32 @ w32
    assert np.allclose(sm32, ref32, rtol=fx["tolerance_printed"], atol=fx["tolerance_printed"])
    assert np.abs(sm32 - ref32).max() < 10 * fx["max_abs_diff_printed"] * max(1.0, np.abs(ref32).max() / 100)


# --------------------------------------------------------- statistics ------

def test_scene1_relative_l2_statistics(oracle_mod):
    """Page 5 section 2.3 scene 1 (symmetric INT4, 256x512): the oracle's error
    statistics reproduce the printed table to within 2.5%."""
    fx = golden("scene1_relative_l2.json")
    N, K = fx["shape"]
    res = {"group_128": [], "group_32": [], "per_channel": [], "per_tensor": []}
    for seed in range(4):
        W = np.random.default_rng(100 + seed).standard_normal((N, K)).astype(np.float32)
        for key, g in (("group_128", 128), ("group_32", 32), ("per_channel", K), ("per_tensor", N * K)):
            flat = W.reshape(-1)
            deq = np.empty_like(flat, dtype=np.float64)
            for a in range(0, flat.size, g):
                s16, zp, u = oracle_mod.quant_group(flat[a:a + g], SYM)
                deq[a:a + g] = (u.astype(np.float64) - zp) * oracle_mod.f16_bits_to_f32(s16)
            res[key].append(np.linalg.norm(flat - deq) / np.linalg.norm(flat))
    for key, vals in res.items():
        printed = fx["int4"][key]
        # the per-tensor figure is set by the single largest of 131072 samples
        # (the printed INT8 and INT4 values both imply max|w| = 4.73, about one
        # standard deviation above the Gaussian mean of that maximum), so it gets
        # a wider band than the group and per-channel figures
        tol = 0.08 if key == "per_tensor" else 0.025
        assert abs(np.mean(vals) - printed) <= tol * printed, (key, np.mean(vals), printed)
    # ordering claims of the same section: finer groups cut the error (g128 -> g32 about 17%)
    cut = 1 - np.mean(res["group_32"]) / np.mean(res["group_128"])
    assert 0.12 < cut < 0.22


def test_scale_statistics_match_order_statistic(oracle_mod):
    """Statistics-consistency check (page 3 section 7.1): for Gaussian weights the
    mean symmetric scale equals E[max of g |N(0, sigma^2)|] / 7."""
    from scipy import integrate, special
    sigma, g = 0.02, 128
    rng = np.random.default_rng(12)
    W = (rng.standard_normal((512, 1024)) * sigma).astype(np.float32)
    Wb = torch.from_numpy(W).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q, s, _ = oracle_mod.quant_pack(Wb, g, SYM)
    mean_scale = s.view(np.float16).astype(np.float64).mean()
    # E[max |Z_i|] = int_0^inf 1 - P(|Z| <= t)^g dt with P(|Z| <= t) = erf(t / sqrt 2)
    emax, _ = integrate.quad(lambda t: 1 - special.erf(t / math.sqrt(2)) ** g, 0, 50)
    assert abs(mean_scale * 7 / sigma - emax) <= 0.01 * emax


# ------------------------------------------------------------------ E2M1 --

def test_e2m1_value_set(oracle_mod):
    fx = golden("e2m1_values.json")
    vals = {oracle_mod.e2m1_decode(c) for c in range(16)}
    assert vals == set(fx["values"]) | {-0.0}
    assert sorted(vals) == sorted(set(fx["values"]))


# ------------------------------------------------- rounding of quotients ---

def test_rint_of_fp32_quotient_equals_exact_rounding():
    """For fp32 x and an fp16-representable d > 0, rint(fl32(x/d)) equals the
    round-half-even of the exact quotient: the IEEE codes of page 5 section 2.2
    are the nearest codes in exact arithmetic.  Checked on a million quotients
    concentrated at and next to half-integers (exact comparison in fp64: b*d and
    x are exact there and the sign of x - b*d is exact)."""
    rng = np.random.default_rng(13)
    n = 1_000_000
    d = rng.integers(0x0001, 0x7BFF, n).astype(np.uint16).view(np.float16).astype(np.float32)
    b = rng.integers(-16, 16, n).astype(np.float64) + 0.5
    bd = (b * d.astype(np.float64)).astype(np.float32)            # exact: b*d has <= 16 bits
    ulps = rng.integers(-4, 5, n).astype(np.int32)
    x = (bd.view(np.int32) + ulps).view(np.float32)              # ties and their neighbours
    x[::7] = (rng.standard_normal(n // 7 + 1)[: x[::7].size] * 8 * d[::7]).astype(np.float32)
    ok = np.isfinite(x) & (d > 0)
    x, d = x[ok], d[ok]
    q32 = np.rint(x / d)                                          # numpy float32 division is IEEE
    X, D = x.astype(np.float64), d.astype(np.float64)
    f = np.floor(X / D)
    for _ in range(2):                                            # make f = floor(x/d) exactly
        f = np.where(X < f * D, f - 1, f)
        f = np.where(X >= (f + 1) * D, f + 1, f)
    h = (f + 0.5) * D                                             # exact in fp64
    exact = np.where(X > h, f + 1, np.where(X < h, f, np.where(f % 2 == 0, f, f + 1)))
    assert np.array_equal(q32.astype(np.float64), exact)
