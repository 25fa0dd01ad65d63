"""The identity behind the kernels' exact dequantization, checked for every
finite fp16 scale and every code difference (no GPU involved).

The GEMV and the tensor-core path form w^ = bf16_rne((u - zp) * s16) with
bf16x2 arithmetic: D = (128 + u) - (128 + zp), s_hi = bf16_rne(s16),
s_lo = s16 - s_hi, c = D * s_lo and w^ = fma(D, s_hi, c). That is one
rounding of the exact product D * s16 provided that
  * 128 + u, 128 + zp and D are exact in bf16;
  * s_lo is exact in bf16 (so s_hi + s_lo == s16);
  * c = D * s_lo is exact in bf16 for every |D| <= 15;
since the fused multiply-add then rounds D * s_hi + D * s_lo = D * s16 once.
Output parity is checked against a tolerance, which would not notice a rare
(scale, code) pair where this failed; this test rules that out.
"""
import numpy as np
import torch


def bf16_exact(x: np.ndarray) -> np.ndarray:
    """True where the fp32 values x are representable in bf16."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return (t.to(torch.bfloat16).to(torch.float32) == t).numpy()


def test_offset_codes_and_differences_are_exact():
    u = np.arange(16, dtype=np.float32)
    assert bf16_exact(128 + u).all()
    D = np.arange(-15, 16, dtype=np.float32)
    assert bf16_exact(D).all()


def test_scale_split_is_exact_for_every_finite_fp16_scale():
    bits = np.arange(0x0000, 0x7C00, dtype=np.uint16)           # +0, subnormals, normals up to 65504
    s16 = bits.view(np.float16).astype(np.float32)
    s_hi = torch.from_numpy(s16).to(torch.bfloat16).to(torch.float32).numpy()
    s_lo = s16 - s_hi                                            # exact in fp32 (Sterbenz-like: s_hi ~ s16)
    assert np.array_equal(s_hi.astype(np.float64) + s_lo.astype(np.float64), s16.astype(np.float64))
    assert bf16_exact(s_lo).all()
    for D in range(-15, 16):
        c = np.float32(D) * s_lo                                 # |D| <= 15: at most 4 more bits
        assert bf16_exact(c).all(), D
        # the product D * s16 is exact in fp32 (<= 15 significant bits), so one
        # rounding of D * s_hi + c equals bf16_rne(D * s16)
        exact = np.float64(D) * s16.astype(np.float64)
        assert np.array_equal(np.float64(D) * s_hi.astype(np.float64) + c.astype(np.float64), exact)
        assert np.array_equal(exact.astype(np.float32).astype(np.float64), exact)
