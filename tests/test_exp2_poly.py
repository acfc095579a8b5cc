"""Accuracy pin of the cubic 2^x the tcgen05 softmax may use on the FMA pipe
(exp2_poly2 in the CUDA sources): 2^x = 2^floor(x) * p(x - floor(x)) with p a
cubic fitted to 2^f on [0, 1). Checked here against the float64 exponential:
its relative error stays below 8e-5 over the whole range a softmax feeds it
(x in [-126, 8]; rows are rescaled before P exceeds 2^8), far inside the bf16
rounding (2^-9) that P goes through before the PV product."""

import numpy as np

C = np.array([0.99992522, 0.69583354, 0.22606716, 0.07802452], dtype=np.float32)


def poly_exp2(x):
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    n = np.floor(x)
    f = (x - n).astype(np.float32)
    p = C[3]
    for c in (C[2], C[1], C[0]):
        p = (p * f + c).astype(np.float32)
    return p.astype(np.float64) * np.exp2(n.astype(np.float64))


def test_relative_error_over_the_softmax_range():
    x = np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float64).astype(np.float32)
    rel = np.abs(poly_exp2(x) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 8e-5, rel.max()


def test_integers_and_masked_keys():
    # exact powers of two up to the fit's value at f = 0; -inf (a masked key)
    # becomes a value below 2^-125, never a NaN
    for n in range(-20, 9):
        assert abs(poly_exp2(float(n)) / 2.0 ** n - 1) < 8e-5
    v = poly_exp2(-np.inf)
    assert np.isfinite(v) and 0 < v < 2.0 ** -125
