"""Helpers shared by the GPU parity tests (device transfers and the output criteria)."""
import os

import numpy as np

# Output criteria for Y (bf16) against the oracle's fp64 product with the
# dequantized weights: relative Frobenius error and max error relative to max|Y_ref|.
REL_FRO_TOL = 2e-3
MAX_ABS_TOL = 1e-2

THREADS = max(1, min(32, os.cpu_count() or 1))


def dev_bf16(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def dev_f32(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def host_u32(t) -> np.ndarray:
    return t.cpu().numpy().view(np.uint32)


def host_u16(t) -> np.ndarray:
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def host_bf16_as_f64(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def assert_codes_equal(got, ref, what):
    if not np.array_equal(got, ref):
        bad = np.argwhere(got != ref)
        i = tuple(bad[0])
        raise AssertionError("%s: %d of %d entries differ; first at %s: got %#x, oracle %#x"
                             % (what, len(bad), ref.size, i, int(got[i]), int(ref[i])))


# Below this many outputs the Frobenius ratio is dominated by a handful of bf16
# output roundings (each up to 2^-8 relative), so small outputs are checked
# element by element against a rigorous bound instead.
MIN_OUTPUTS_FOR_NORM = 1024


def assert_y_elementwise(Y: np.ndarray, Y_ref: np.ndarray, Y_abs: np.ndarray, K: int, what: str = "Y"):
    """|Y - Y_ref| <= 2^-8 (|Y_ref| + e) + e with e = K 2^-22 sum_k |x w^|: one bf16
    rounding of an fp32 sum whose accumulation error is at most e."""
    e = K * 2.0 ** -22 * Y_abs
    bound = 2.0 ** -8 * (np.abs(Y_ref) + e) + e
    bad = ~(np.abs(Y - Y_ref) <= bound)          # NaN or Inf counts as outside
    assert np.isfinite(Y).all(), "%s: non-finite outputs" % what
    assert not bad.any(), "%s: %d outputs outside the rounding bound, first %s: got %r, ref %r, bound %r" % (
        what, int(bad.sum()), tuple(np.argwhere(bad)[0]), Y[bad][0], Y_ref[bad][0], bound[bad][0])


def assert_y_close(Y: np.ndarray, Y_ref: np.ndarray, what: str = "Y"):
    if Y.size < MIN_OUTPUTS_FOR_NORM:
        raise AssertionError("use assert_y_elementwise for outputs smaller than %d" % MIN_OUTPUTS_FOR_NORM)
    diff = Y - Y_ref
    ref_norm = np.linalg.norm(Y_ref)
    rel_fro = np.linalg.norm(diff) / ref_norm if ref_norm > 0 else np.linalg.norm(diff)
    ymax = np.abs(Y_ref).max()
    max_err = np.abs(diff).max()
    assert rel_fro <= REL_FRO_TOL, "%s: relative Frobenius error %.3e > %.0e" % (what, rel_fro, REL_FRO_TOL)
    assert max_err <= MAX_ABS_TOL * ymax, "%s: max error %.3e > %.0e * max|Y_ref| (%.3e)" % (
        what, max_err, MAX_ABS_TOL, ymax)
    return rel_fro, max_err / ymax if ymax else max_err
