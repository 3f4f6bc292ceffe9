"""Pins for the oracle's EntroLLM-style integer weights (EntroLLM page, "Metodologia": per-tensor
unsigned or asymmetric integer quantisation, Huffman-coded, decoded in parallel) in the DFloat11
layout: grid points round-trip exactly, the reconstruction error stays within half a step, the
code entropy of Gaussian weights matches the high-resolution closed form, and the coded stream's
Gaps / block positions and independent segments follow from the code lengths alone."""
import math

import numpy as np
import pytest

import synth


@pytest.mark.parametrize("bits", [8, 4])
def test_grid_points_round_trip_exactly(orc, bits):
    """w = (k - z) s with k covering 0 .. L-1: the asymmetric quantiser recovers s, z and every k,
    and the decoded weight is w rounded once to bf16."""
    L = 1 << bits
    rng = np.random.default_rng(bits)
    s = float(orc.bf16_to_f32(np.array([0x3C23], np.uint16))[0])  # a bf16 step (~0.00995)
    z = L // 3
    k = rng.integers(0, L, 5000)
    k[:2] = [0, L - 1]
    w = ((k - z) * s).astype(np.float32)
    sym, sc, zero = orc.intq_quantize(w, bits, orc.INTQ_ASYM)
    assert sc == 0x3C23 and zero == z
    assert np.array_equal(sym.astype(np.int64), k)
    # (k - z) s is exact in binary32; the decoded value is its bf16 rounding (torch's cast)
    assert np.array_equal(orc.intq_dequant(sym, sc, zero), synth.bf16_bits(w))


@pytest.mark.parametrize("bits,scheme", [(8, 0), (8, 1), (4, 0), (4, 1)])
def test_codes_in_range_and_error_within_half_a_step(orc, bits, scheme):
    w = synth.normal_with_outliers(64, 1024, 0.02, 0.01, 8.0, 7 + bits)
    sym, sc, zero = orc.intq_quantize(w, bits, scheme)
    L = 1 << bits
    assert sym.max() <= L - 1 and 0 <= zero <= L
    s = float(orc.bf16_to_f32(np.array([sc], np.uint16))[0])
    rec = orc.bf16_to_f32(orc.intq_dequant(sym, sc, zero)).astype(np.float64)
    err = np.abs(rec - w.astype(np.float64))
    # half a step (s itself is rounded to bf16, so the grid may fall a step short at one end)
    # plus the final bf16 rounding of the value
    bound = 0.5 * s * (1 + 2 ** -7) + np.abs(w) * 2 ** -8 + (s if scheme == 0 else 0.0) * (
        np.abs(w - w.mean()) > 0.99 * np.abs(w - w.mean()).max())
    assert np.all(err <= bound + 1e-12)


def test_gaussian_code_entropy_matches_closed_form(orc):
    """High-resolution quantisation of N(0, sigma) with step s: H = log2(sigma sqrt(2 pi e) / s)."""
    sigma = 0.02
    w = synth.normal(1024, 1024, sigma, 11)
    sym, sc, _ = orc.intq_quantize(w, 8, orc.INTQ_ASYM)
    s = float(orc.bf16_to_f32(np.array([sc], np.uint16))[0])
    sd = float(w.astype(np.float64).std())
    want = math.log2(sd * math.sqrt(2 * math.pi * math.e) / s)
    assert abs(orc.entropy_bits(sym) - want) < 0.02


def test_scheme_choice_takes_the_lower_entropy(orc):
    rng = np.random.default_rng(12)
    for w in (synth.normal(64, 512, 0.02, 13),
              np.abs(rng.standard_normal((64, 512))).astype(np.float32) * 0.02,
              (rng.standard_normal((64, 512)) * 0.02 + 0.05).astype(np.float32)):
        for bits in (8, 4):
            hs = [orc.entropy_bits(orc.intq_quantize(w, bits, sch)[0]) for sch in (0, 1)]
            _, _, _, chosen = orc.entrollm_quantize(w, bits)
            assert chosen == (1 if hs[1] < hs[0] else 0)


def _starts(lengths, sym):
    ln = lengths[sym].astype(np.int64)
    return np.concatenate([[0], np.cumsum(ln)[:-1]]), int(ln.sum())


@pytest.mark.parametrize("n,tpb", [(1, 256), (5000, 256), (40000, 32), (777, 4)])
def test_gaps_and_block_out_from_code_starts(orc, n, tpb):
    w = synth.normal(1, n, 0.02, 20 + n)
    sym, sc, z, _ = orc.entrollm_quantize(w, 8)
    h = orc.huff_encode_sym(sym, 8, sc, z, threads_per_block=tpb)
    starts, total = _starts(h.lengths, sym.ravel())
    assert h.total_bits == total
    T = h.threads
    gaps = orc.gaps_unpack(h.gaps, T)
    first = np.searchsorted(starts, 64 * np.arange(T), side="left")
    first_pos = np.where(first < n, starts[np.minimum(first, n - 1)], total)
    assert np.array_equal(gaps, first_pos - 64 * np.arange(T))
    blocks = (T + tpb - 1) // tpb
    want = np.searchsorted(starts, 64 * tpb * np.arange(blocks), side="left")
    assert np.array_equal(h.block_out[:-1], want) and h.block_out[-1] == n


def test_thread_segments_decode_independently(orc):
    w = synth.normal(1, 3000, 0.02, 30)
    sym, sc, z, _ = orc.entrollm_quantize(w, 4)
    h = orc.huff_encode_sym(sym, 4, sc, z, threads_per_block=8)
    codes = orc.huff_canonical(h.lengths)
    table = {format(int(codes[s]), f"0{int(h.lengths[s])}b"): s for s in range(256) if h.lengths[s]}
    bits = "".join(format(int(b), "08b") for b in h.enc)
    gaps = orc.gaps_unpack(h.gaps, h.threads)
    out = []
    for t in range(h.threads):
        pos, end = 64 * t + int(gaps[t]), min(64 * t + 64, h.total_bits)
        while pos < end:
            ln = next(ln for ln in range(1, 33) if bits[pos:pos + ln] in table)
            out.append(table[bits[pos:pos + ln]])
            pos += ln
    assert np.array_equal(np.array(out), sym.ravel())


def test_roundtrip_random_tiny_streams(orc):
    rng = np.random.default_rng(31)
    for _ in range(300):
        n = int(rng.integers(0, 200))
        alphabet = rng.choice(256, int(rng.integers(1, 6)), replace=False)
        sym = rng.choice(alphabet, n).astype(np.uint8)
        h = orc.huff_encode_sym(sym, 8, 0x3F80, 0, threads_per_block=int(rng.choice([1, 4, 256])))
        rc, out = orc.huff_decode_sym(h)
        assert rc == 0 and np.array_equal(out, sym)
        rc, vals = orc.entrollm_decode_bf16(h)
        assert rc == 0 and np.array_equal(orc.bf16_to_f32(vals), sym.astype(np.float32))
