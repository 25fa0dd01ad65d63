"""Pins for the oracle's AWQ scale search (page 2, AWQ section: the grid search
over alpha for s = act^alpha / mean(act^alpha)), checked against facts that do
not come from the search itself."""
import numpy as np

import oracle
from oracle import awq
from bit_gemm_quant_b200 import synth

SYM, ASYM = 0, 1


def small(seed=5, N=48, K=256, M=16, outliers=0.05):
    W = synth.weights(seed, N, K, 0.02)
    X = synth.activations(seed + 1, M, K, outliers, 40.0)
    return W, X


def test_alpha_grid_is_even_and_includes_both_ends():
    a = awq.alphas(20)
    assert a[0] == 0.0 and a[-1] == 1.0 and len(a) == 20
    assert np.allclose(np.diff(a), 1.0 / 19, rtol=0, atol=1e-15)


def test_act_is_the_mean_magnitude_per_input_channel():
    # hand-made 2 x 3 calibration block: exact in bf16
    X = np.array([[1.0, -2.0, 0.5], [-3.0, 2.0, 0.25]], dtype=np.float32)
    bits = (X.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(awq.act_magnitude(bits), [2.0, 2.0, 0.375])


def test_alpha_zero_is_plain_quantization():
    """At alpha = 0, s = 1 exactly, the fold is the identity and the loss is the
    plain RTN loss computed without any smoothing vector."""
    W, X = small()
    act = awq.act_magnitude(X)
    s0 = awq.smoothing(act, 0.0)
    assert np.all(s0 == 1.0)
    losses, _, _ = awq.awq_losses(W, X, 128, ASYM, n_alpha=3)
    q, sc, z = oracle.quant_pack(W, 128, ASYM)
    Y_ref = oracle.gemm_f64(X, W)
    Y_q = awq.f64_to_bf16_f64(oracle.w4a16_reference(X, q, sc, z, W.shape[1], 128, ASYM))
    assert losses[0] == np.mean((Y_ref - Y_q) ** 2)


def test_path_form_matches_the_listing_form():
    """The listing divides the dequantized weight by s; the oracle divides the
    activations (the W4A16 path's product).  The two agree up to the bf16
    roundings of X/s and of the output (smoothing identity, page 5 section 2.4)."""
    W, X = small(seed=9, N=32, K=256, M=8)
    K = W.shape[1]
    losses, _, _ = awq.awq_losses(W, X, 64, SYM, n_alpha=5)
    Xf = awq.bf16_bits_to_f64(X)
    Y_ref = Xf @ awq.bf16_bits_to_f64(W).T
    act = awq.act_magnitude(X)
    for i, a in enumerate(awq.alphas(5)):
        s = awq.smoothing(act, a)
        q, sc, z = oracle.quant_pack(W, 64, SYM, s=s)
        What = awq.bf16_bits_to_f64(oracle.dequant(q, sc, z, K, 64, SYM))
        Y_listing = (What / s.astype(np.float64)[None, :]) @ Xf.T
        loss_listing = np.mean((Y_ref - Y_listing.T) ** 2)
        assert abs(loss_listing - losses[i]) <= 2e-2 * loss_listing


def test_search_helps_when_activations_have_outlier_channels():
    """Page 2: a few input channels with large activations dominate the error;
    scaling them up in W before quantizing (alpha > 0) lowers the loss."""
    W, X = small(seed=13, N=64, K=512, M=32, outliers=0.02)
    losses, best, s = awq.awq_losses(W, X, 128, SYM, n_alpha=8)
    assert best > 0
    assert losses[best] < 0.9 * losses[0]
    assert abs(np.mean(s.astype(np.float64)) - 1.0) < 1e-6
