"""Pins for the oracle's fp64 GEMV over bf16 operands: exact rational sums on tiny shapes and an
independent library product (numpy float64 matmul) on larger ones."""
from fractions import Fraction

import numpy as np

import synth


def test_gemv_exact_on_tiny_shapes(orc):
    rng = np.random.default_rng(0)
    for rows, cols, batch in [(1, 1, 1), (3, 7, 2), (5, 33, 4), (2, 64, 16)]:
        w = synth.bf16_bits(rng.standard_normal((rows, cols)).astype(np.float32) * 0.02)
        x = synth.bf16_bits(rng.standard_normal((batch, cols)).astype(np.float32))
        y = orc.gemv_f64(w, x)
        wf, xf = orc.bf16_to_f32(w).astype(np.float64), orc.bf16_to_f32(x).astype(np.float64)
        for b in range(batch):
            for r in range(rows):
                exact = sum(Fraction(wf[r, c]) * Fraction(xf[b, c]) for c in range(cols))
                assert abs(Fraction(y[b, r]) - exact) <= abs(exact) * Fraction(1, 10 ** 13) + Fraction(1, 10 ** 30)


def test_gemv_matches_numpy_float64(orc):
    w = synth.bf16_normal(300, 2048, 0.02, 3)
    x = synth.activations(4, 2048, 3)
    y = orc.gemv_f64(w, x)
    ref = orc.bf16_to_f32(x).astype(np.float64) @ orc.bf16_to_f32(w).astype(np.float64).T
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))
