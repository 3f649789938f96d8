"""The seeded generator: row ranges regenerate identically; moments are right."""
import numpy as np

from weight_only_quantized_fp6_b200 import inputs


def test_row_sampling_matches_full_matrix():
    full = inputs.weights(2003, 64, 320, outlier_p=0.001)
    rows = [0, 5, 6, 7, 40, 63]
    part = inputs.weights(2003, 64, 320, rows=rows, outlier_p=0.001)
    assert np.array_equal(full[rows], part)


def test_moments_and_outliers():
    W = inputs.weights(3000, 256, 1024)
    assert abs(W.std() - 0.02) < 0.0005 and abs(W.mean()) < 0.0005
    Wo = inputs.weights(3000, 256, 1024, outlier_p=0.001)
    ratio = Wo / np.where(W == 0, 1, W)
    frac8 = np.mean(np.isclose(ratio, 8.0))
    assert 0.0006 < frac8 < 0.0014
    x = inputs.activations(7, 64, 1024).view(np.float16).astype(np.float64)
    assert abs(x.std() - 1.0) < 0.02


def test_seeds_differ():
    assert not np.array_equal(inputs.weights(1, 8, 64), inputs.weights(2, 8, 64))
    assert inputs.activation_seed(inputs.weight_seed("llama70b_o_decode", 0), 16) == 2116
    assert inputs.weight_seed("tiny", 0) == 0 and inputs.weight_seed("opt30b", 3) == 4003


def test_parallel_generation_matches():
    a = inputs.weights(17, 300, 128, outlier_p=0.01)
    b = inputs.weights_parallel(17, 300, 128, outlier_p=0.01, threads=7)
    assert np.array_equal(a, b)
