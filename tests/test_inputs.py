"""The seeded input generators: deterministic, right shapes, outliers where the recipe puts them."""
import numpy as np

from bit_gemm_quant_b200 import synth


def test_generators_are_deterministic():
    a = synth.weights(3, 64, 256, 0.02, 0.01, 5.0)
    b = synth.weights(3, 64, 256, 0.02, 0.01, 5.0)
    c = synth.weights(4, 64, 256, 0.02, 0.01, 5.0)
    assert a.dtype == np.uint16 and a.shape == (64, 256)
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    x1 = synth.activations(3, 2, 256, 0.01, 40.0)
    assert np.array_equal(x1, synth.activations(3, 2, 256, 0.01, 40.0))


def test_outlier_channels_follow_the_recipe():
    K = 4096
    cols = synth.outlier_channels(1, 22, K, 0.01)
    assert len(cols) == 41 and len(set(cols.tolist())) == 41
    x = synth.bf16_bits_to_f32(synth.activations(1, 8, K, 0.01, 40.0))
    rms = np.sqrt((x.astype(np.float64) ** 2).mean(0))
    assert rms[cols].mean() > 20 * np.delete(rms, cols).mean()


def test_smoothing_vector_recipe():
    s = synth.smoothing_vector(4, 8192)
    assert s.dtype == np.float32 and s.shape == (8192,)
    assert abs(float(s.astype(np.float64).mean()) - 1.0) < 1e-6
    assert s.min() > 0


def test_workloads_cover_the_named_configs():
    assert [p.N for p in synth.workload("decode")] == [4096, 11008, 12288]
    assert [p.M for p in synth.workload("smallbatch")] == [2, 4, 8, 16, 32]
    assert [p.M for p in synth.workload("prefill")] == [512, 2048, 8192]
    q = synth.workload("quantizer")
    assert {(p.group, p.mode) for p in q if not p.smooth} == {(g, m) for g in (32, 64, 128) for m in (0, 1)}
    assert any(p.smooth for p in q)
