"""Pins for the oracle's number formats, quantiser and dequantiser.

Each check ties the oracle to something other than itself: torch's own casts (an independent
library routine), exact rational arithmetic with ``fractions``, or figures the pages print.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rne_fraction_to_bf16(v: Fraction) -> int:
    """Exact round-to-nearest-even of a rational onto bf16 (binary32 exponent range)."""
    if v == 0:
        return 0
    sign = 0x8000 if v < 0 else 0
    a = abs(v)
    E = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** E > a:
        E -= 1
    E = max(E, -126)
    q = Fraction(2) ** (E - 7)
    k, rem = divmod(a, q)
    k = int(k)
    if rem * 2 > q or (rem * 2 == q and k % 2 == 1):
        k += 1
    r = k * q
    if r >= Fraction(2) ** 128:
        return sign | 0x7F80
    f = np.float32(float(r))
    return sign | int(np.array([f], dtype=np.float32).view(np.uint32)[0] >> 16)


def e4m3_fraction(b: int) -> Fraction:
    s, e, m = b >> 7, (b >> 3) & 15, b & 7
    v = Fraction(m, 512) if e == 0 else Fraction(8 + m, 8) * Fraction(2) ** (e - 7)
    return -v if s else v


def torch_bf16(a: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------------------------------------
# bf16
# ---------------------------------------------------------------------------------------------

def test_f32_to_bf16_matches_torch(orc):
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 2**32, 20000, dtype=np.uint64).astype(np.uint32)
    specials = np.array([0, 0x80000000, 0x7F800000, 0xFF800000, 0x7F7FFFFF, 0x00000001,
                         0x3F808000, 0x3F818000, 0x3F80FFFF, 0x00008000, 0x00018000],
                        dtype=np.uint32)
    a = np.concatenate([bits, specials]).view(np.float32)
    a = a[~np.isnan(a)]
    assert np.array_equal(orc.f32_to_bf16(a), torch_bf16(a))


def test_f32_to_bf16_nan_is_quiet_with_sign(orc):
    a = np.array([0x7FC00001, 0xFF800001], dtype=np.uint32).view(np.float32)
    assert orc.f32_to_bf16(a).tolist() == [0x7FC0, 0xFFC0]


def test_f64_to_bf16_exact_rationals(orc):
    rng = np.random.default_rng(1)
    vals = []
    for _ in range(3000):
        m = int(rng.integers(1, 2**20))
        e = int(rng.integers(-150, 130))
        s = -1 if rng.random() < 0.5 else 1
        vals.append(Fraction(s * m) * Fraction(2) ** e)
    got = orc.f64_to_bf16(np.array([float(v) for v in vals]))
    want = np.array([rne_fraction_to_bf16(v) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, want)


def test_bf16_exponent_field_of_pointer_range():
    """The pages' pointer exponents 240..255 are magnitudes 2^113..2^128 (bits 14..7, bias 127)."""
    fig = json.load(open(os.path.join(GOLDEN, "pages_figures.json")))["pointer_exponents"]
    lo, hi = fig["magnitude_log2"]
    b = torch_bf16(np.array([2.0 ** lo, -(2.0 ** 127) * 1.5], np.float32))
    assert ((b >> 7) & 0xFF).tolist() == [fig["range"][0], 254]
    assert ((torch_bf16(np.array([np.inf], np.float32)) >> 7) & 0xFF)[0] == fig["range"][1]


# ---------------------------------------------------------------------------------------------
# Float8 E4M3
# ---------------------------------------------------------------------------------------------

def test_e4m3_value_table_matches_torch_and_rationals(orc):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    got = np.array([orc.e4m3_value(c) for c in codes])
    nan = np.isnan(ref)
    assert nan.nonzero()[0].tolist() == [0x7F, 0xFF]
    assert np.isnan(got[nan]).all()
    assert np.array_equal(got[~nan], ref[~nan].astype(np.float64))
    for c in codes[~nan]:
        assert Fraction(got[c]) == e4m3_fraction(int(c))
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def test_f32_to_e4m3_matches_torch_in_range(orc):
    rng = np.random.default_rng(2)
    a = (rng.standard_normal(20000) * 10.0 ** rng.uniform(-4, 2.6, 20000)).astype(np.float32)
    a = a[np.abs(a) <= 448]
    # exact ties between neighbouring E4M3 values
    grid = np.array(sorted({abs(float(e4m3_fraction(c))) for c in range(0x7F)}), np.float64)
    ties = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)
    a = np.concatenate([a, ties, -ties, np.float32([0.0, -0.0, 448.0, 2.0 ** -10, 2.0 ** -11])])
    ref = torch.from_numpy(a).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(orc.f32_to_e4m3(a), ref)


def test_f32_to_e4m3_saturates(orc):
    a = np.float32([449.0, 463.9, 464.0, 1e6, np.inf, -500.0, -np.inf])
    assert orc.f32_to_e4m3(a).tolist() == [0x7E] * 5 + [0xFE] * 2


# ---------------------------------------------------------------------------------------------
# dequantisation: bf16(value(q) * scale), exhaustively against exact rationals
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("symfmt", [1, 2])
def test_dequant_exhaustive_exact(orc, symfmt):
    rng = np.random.default_rng(3 + symfmt)
    scales = np.concatenate([rng.integers(0x3000, 0x4100, 300), rng.integers(0x0001, 0x7F7F, 100),
                             [0x3F80, 0x0001, 0x7F7F, 0x8000 | 0x3C00]]).astype(np.uint16)
    syms = np.arange(256, dtype=np.uint8)
    sym = np.tile(syms, (scales.size, 1))
    got = orc.dequant(sym, scales, symfmt)
    for i, sb in enumerate(scales):
        s = Fraction(float(orc.bf16_to_f32(np.array([sb], np.uint16))[0]))
        for q in range(256):
            if symfmt == 1 and q in (0x7F, 0xFF):
                assert got[i, q] == (0xFFC0 if q & 0x80 else 0x7FC0)
                continue
            v = e4m3_fraction(q) if symfmt == 1 else Fraction(int(np.int8(np.uint8(q))))
            want = rne_fraction_to_bf16(v * s)
            if v == 0:  # signed zero: sign(value) xor sign(scale)
                neg = (symfmt == 1 and q == 0x80) ^ (float(s) < 0)
                want = 0x8000 if neg else 0
            assert got[i, q] == want, (symfmt, hex(sb), q)


# ---------------------------------------------------------------------------------------------
# quantiser
# ---------------------------------------------------------------------------------------------

def test_quantize_e4m3_matches_torch(orc):
    w = synth.normal(64, 1024, 0.02, 11)
    sym, sc = orc.quantize(w, orc.E4M3)
    amax = np.abs(w).max(axis=1)
    assert np.array_equal(sc, torch_bf16(amax / np.float32(448.0)))
    s = orc.bf16_to_f32(sc)
    ref = torch.from_numpy(np.clip(w / s[:, None], -448, 448)).to(torch.float8_e4m3fn)
    assert np.array_equal(sym, ref.view(torch.uint8).numpy())


def test_quantize_int8_definition(orc):
    w = synth.laplace_clipped(64, 1024, 0.01, 0.06, 12)
    sym, sc = orc.quantize(w, orc.INT8, 4.2281)
    s = orc.bf16_to_f32(sc)
    q = np.clip(np.rint(w / s[:, None]), -127, 127).astype(np.int8)
    assert np.array_equal(sym.view(np.int8), q)


def test_e4m3_entropy_matches_pages(orc):
    """Float8 entropy-coded at about 6.5 bits/param (EntQuant abstract page, Figure 4 caption)."""
    fig = json.load(open(os.path.join(GOLDEN, "pages_figures.json")))
    f = fig["float8_entropy_coded_bits_per_param"]
    w = synth.WORKLOADS["e4m3_1k"].tensors[0].generate()
    sym, _ = orc.quantize(w, orc.E4M3)
    assert abs(orc.entropy_bits(sym) - f["value"]) <= f["tolerance"]


def test_int8_divisor_gives_two_bits(orc):
    g = json.load(open(os.path.join(GOLDEN, "int8_div.json")))
    assert g["int8_div"] == synth.INT8_DIV_LAPLACE_8K
    spec = synth.WORKLOADS["int8_8k"].tensors[0]
    w = spec.generate(row_lo=0, row_hi=1024)
    sym, _ = orc.quantize(w, orc.INT8, synth.INT8_DIV_LAPLACE_8K)
    assert abs(orc.entropy_bits(sym) - 2.0) < 0.01
    assert set(np.unique(sym.view(np.int8)).tolist()) <= set(range(-5, 6))


def test_synth_row_blocks_are_independent():
    spec = synth.WORKLOADS["mlp_13b"].tensors[2]
    full = synth.normal(100, spec.cols, 0.02, spec.seed, spec.tensor)
    part = synth.normal(100, spec.cols, 0.02, spec.seed, spec.tensor, row_lo=37, row_hi=71)
    assert np.array_equal(full[37:71], part)
