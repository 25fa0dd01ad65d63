"""The arithmetic identities the quantizers' fast paths rest on, checked
on the CPU by exact emulation of the fp32 steps (numpy float64 holds every
product and residual exactly; the one sum that does not fit is resolved with
an error-free TwoSum).

1. Scale division by a constant (w4_quant_pack's s32 = fl32(amax / 7) and
   fl32((max - min) / 15)): q0 = fl(v * fl(1/c)), r = fma(-q0, c, v),
   q1 = fma(r, fl(1/c), q0) is the correctly rounded quotient for every one of
   the 2^23 significands of a binade.

2. The corrected quotient for rint (the codes and zero-points): for d > 0 an
   fp16 value and inv any fp32 within 2 ulp of 1/d (rcp.approx's bound),
   t0 = fl(x * inv), e = fma(-t0, d, x) (exact), t1 = fma(e, inv, t0) gives
   rint(t1) = rint(x / d) with ties to even -- for every bf16 x (unfolded
   weights, where exact ties are common) with a quotient below 32, and for
   fp32 x (folded weights, 24 significant bits) on the hardest cases: the 13
   floats nearest h * d for every half-integer h below 32.  Negative x mirror
   positive x (every step is odd in x).

3. The same quotient against the E2M1 rounding midpoints, for bf16 weights
   and E4M3 block scales (NVFP4): the identity an NVFP4 encoder without a
   division per weight would rest on.

Each check also runs on a planted mistake (no correction step) and must fail
there, so that it can fail at all.
"""
import numpy as np


def _f32(a):
    return np.asarray(a, dtype=np.float64).astype(np.float32)


def _next(a, direction):
    return np.nextafter(a, np.float32(direction)).astype(np.float64)


def _is_rn32(num64, den, q1):
    """q1 (float32) == RN32(num / den), exactly: den * (num/den - q1) = num - den
    * q1 is exact in float64 for the sizes used here."""
    q1d = q1.astype(np.float64)
    sd = num64 - den * q1d
    ulp = np.where(sd > 0, _next(q1, np.inf) - q1d, q1d - _next(q1, -np.inf))
    err, lim = np.abs(sd), den * ulp / 2
    return (err < lim) | ((err == lim) & ((q1.view(np.uint32) & 1) == 0))


def _const_div(v, c, corrected=True):
    z = np.float32(1.0) / np.float32(c)
    q0 = (v * z).astype(np.float32)
    if not corrected:
        return q0
    r64 = v.astype(np.float64) - q0.astype(np.float64) * c
    r = r64.astype(np.float32)
    assert np.array_equal(r.astype(np.float64), r64)          # the fma's residual is exact
    return _rn32_sum(q0.astype(np.float64), r.astype(np.float64) * np.float64(z))


def _rn32_sum(a, b):
    """RN32(a + b) for float64 a, b whose exact sum may not fit a float64."""
    s = a + b
    bb = s - a
    err = (a - (s - bb)) + (b - bb)                            # TwoSum: a + b = s + err exactly
    q = s.astype(np.float32)
    qd = q.astype(np.float64)
    up, dn = _next(q, np.inf), _next(q, -np.inf)
    # s exactly halfway between two floats: the error term decides (or ties to even)
    mid_up = s == (qd + up) / 2
    mid_dn = s == (qd + dn) / 2
    q = np.where(mid_up & (err > 0), _f32(up), q)
    q = np.where(mid_up & (err < 0), _f32(qd), q)
    q = np.where(mid_dn & (err < 0), _f32(dn), q)
    q = np.where(mid_dn & (err > 0), _f32(qd), q)
    return q.astype(np.float32)


def test_constant_division_is_correctly_rounded():
    m = np.arange(1 << 23, dtype=np.uint32)
    v = ((np.uint32(127) << 23) | m).view(np.float32)         # every significand of [1, 2)
    for c in (7.0, 15.0):
        assert _is_rn32(v.astype(np.float64), c, _const_div(v, c)).all(), c
        assert not _is_rn32(v.astype(np.float64), c, _const_div(v, c, corrected=False)).all()


def _exact_rint(x, d):
    """rint(x / d), ties to even, by exact comparisons (x, d float64 holding
    an fp32 and an fp16 value; x / d < 64)."""
    n = np.floor(x / d)
    n = np.where(x < n * d, n - 1, n)
    n = np.where(x >= (n + 1) * d, n + 1, n)
    frac = x - n * d                                           # exact
    half = 0.5 * d
    up = (frac > half) | ((frac == half) & (n % 2 == 1))
    return n + up


def _quot(x, d, inv, corrected=True):
    t0 = (x.astype(np.float64) * inv.astype(np.float64)).astype(np.float32)
    if not corrected:
        return t0
    e64 = x.astype(np.float64) - t0.astype(np.float64) * d.astype(np.float64)
    e = e64.astype(np.float32)
    assert np.array_equal(e.astype(np.float64), e64)          # the residual is exact
    return _rn32_sum(t0.astype(np.float64), e.astype(np.float64) * inv.astype(np.float64))


def _bf16_values(lo, hi):
    bits = np.arange(0, 1 << 15, dtype=np.uint32)
    v = (bits << 16).view(np.float32)
    return v[(v >= lo) & (v < hi)]


def test_corrected_quotient_rounds_like_the_exact_quotient():
    # every fp16 scale of [1, 2) (the identity is invariant under scaling x and
    # d by powers of two) and every bf16 weight with a quotient in [1/32, 32)
    d16 = np.arange(0x3C00, 0x4000, dtype=np.uint16).view(np.float16).astype(np.float32)
    x = _bf16_values(1.0 / 32, 64.0)
    X, D = np.meshgrid(x, d16, indexing="ij")
    X, D = X.ravel(), D.ravel()
    keep = X / D < 32
    X, D = X[keep], D[keep]
    want = _exact_rint(X.astype(np.float64), D.astype(np.float64))
    assert np.any(X.astype(np.float64) / D.astype(np.float64) % 1 == 0.5)   # exact ties occur
    rn = (np.float32(1.0) / D).astype(np.float32)
    for k in (-2, -1, 0, 1, 2):                               # rcp.approx within 2 ulp
        inv = rn.copy()
        for _ in range(abs(k)):
            inv = np.nextafter(inv, np.float32(np.inf if k > 0 else -np.inf)).astype(np.float32)
        got = np.rint(_quot(X, D, inv).astype(np.float64))    # the magic add: round half even
        assert np.array_equal(got, want), "inv off by %d ulp" % k
        if k == 1:
            bad = np.rint(_quot(X, D, inv, corrected=False).astype(np.float64))
            assert not np.array_equal(bad, want)


def test_corrected_quotient_on_fp32_weights_next_to_every_half_integer():
    d16 = np.arange(0x3C00, 0x4000, dtype=np.uint16).view(np.float16).astype(np.float32)
    D, H = np.meshgrid(d16, np.arange(32) + 0.5, indexing="ij")
    D, H = D.ravel(), H.ravel()
    centre = (H * D.astype(np.float64)).astype(np.float32)   # the float nearest h * d
    xs = [centre]
    for direction in (np.inf, -np.inf):
        v = centre
        for _ in range(6):
            v = np.nextafter(v, np.float32(direction)).astype(np.float32)
            xs.append(v)
    X = np.concatenate(xs)
    DD = np.tile(D, len(xs))
    want = _exact_rint(X.astype(np.float64), DD.astype(np.float64))
    rn = (np.float32(1.0) / DD).astype(np.float32)
    for k in (-2, -1, 0, 1, 2):
        inv = rn.copy()
        for _ in range(abs(k)):
            inv = np.nextafter(inv, np.float32(np.inf if k > 0 else -np.inf)).astype(np.float32)
        got = np.rint(_quot(X, DD, inv).astype(np.float64))
        assert np.array_equal(got, want), "inv off by %d ulp" % k
        bad = np.rint(_quot(X, DD, inv, corrected=False).astype(np.float64))
        assert not np.array_equal(bad, want)


def test_corrected_quotient_against_the_e2m1_midpoints():
    """The same corrected quotient for block-scaled FP4 (NVFP4: bf16 weight x,
    E4M3 block scale s with 4 significant bits): t1 lies on the exact
    quotient's side of every E2M1 rounding midpoint (0.25 ... 5) and equals
    the midpoint exactly when x / s does -- for every bf16 x with x / s < 8 and
    every E4M3 significand (the identity scales with powers of two, E4M3
    subnormals included), at every reciprocal error from -2 to +2 ulp."""
    s8 = (1.0 + np.arange(8) / 8.0).astype(np.float32)         # the 8 E4M3 significands of [1, 2)
    x = _bf16_values(1.0 / 64, 16.0)
    X, S = np.meshgrid(x, s8, indexing="ij")
    X, S = X.ravel(), S.ravel()
    keep = X.astype(np.float64) / S.astype(np.float64) < 8
    X, S = X[keep], S[keep]
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    # sign(q - m) exactly: x - m * s is exact in float64
    want = np.sign(X.astype(np.float64)[:, None] - mids[None, :] * S.astype(np.float64)[:, None])
    assert (want == 0).any()                                  # exact midpoints occur
    rn = (np.float32(1.0) / S).astype(np.float32)
    for k in (-2, -1, 0, 1, 2):
        inv = rn.copy()
        for _ in range(abs(k)):
            inv = np.nextafter(inv, np.float32(np.inf if k > 0 else -np.inf)).astype(np.float32)
        t1 = _quot(X, S, inv).astype(np.float64)
        assert np.array_equal(np.sign(t1[:, None] - mids[None, :]), want), "inv off by %d ulp" % k
    t0 = _quot(X, S, rn, corrected=False).astype(np.float64)  # a planted mistake fails
    assert not np.array_equal(np.sign(t0[:, None] - mids[None, :]), want)
