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


def _round_bf16_f64(v):
    """bf16 round-to-nearest-even of binary64 values in bf16's normal range, written from the
    format: 8 significant bits, ties to the even significand (numpy's round is half-to-even)."""
    m, e = np.frexp(v)
    return np.ldexp(np.round(m * 256.0) / 256.0, e)


def test_mlp_chain_matches_numpy(orc):
    """The oracle's MLP block (gate and up products, SiLU gate, hidden rounded once to bf16, down
    product) against the same chain written here from its definition with numpy float64."""
    rng = np.random.default_rng(5)
    hidden, inter, batch = 48, 160, 3
    wg = synth.bf16_bits(rng.standard_normal((inter, hidden)).astype(np.float32) * 0.2)
    wu = synth.bf16_bits(rng.standard_normal((inter, hidden)).astype(np.float32) * 0.2)
    wd = synth.bf16_bits(rng.standard_normal((hidden, inter)).astype(np.float32) * 0.2)
    x = synth.bf16_bits(rng.standard_normal((batch, hidden)).astype(np.float32))
    f = lambda b: orc.bf16_to_f32(b).astype(np.float64)  # noqa: E731
    g, u = f(x) @ f(wg).T, f(x) @ f(wu).T
    h = _round_bf16_f64(g * u / (1.0 + np.exp(-g)))
    ref = h @ f(wd).T
    y = orc.mlp_f64(wg, wu, wd, x)
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))
    # SiLU(0) = 0: an all-zero gate makes the hidden vector, and so y, exactly zero
    z = np.zeros_like(wg)
    assert np.all(orc.mlp_f64(z, wu, wd, x) == 0.0)
