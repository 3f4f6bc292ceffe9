"""The library's host compressor (include/eq_encode.h) against the oracle: same symbols, scales,
frequency tables, rANS containers and DFloat11 containers, bit for bit (the formats leave no
freedom once the tables are fixed)."""
import numpy as np
import pytest

import synth


@pytest.fixture(scope="module")
def eq():
    import decoding_interleaved_rans_b200 as m
    m.lib()
    return m


@pytest.mark.parametrize("name", ["e4m3_1k", "int8_8k", "mlp_13b"])
def test_quantize_matches_oracle(eq, orc, name):
    wl = synth.WORKLOADS[name]
    spec = wl.tensors[0]
    w = spec.generate(row_lo=0, row_hi=min(spec.rows, 300))
    fmt = 1 if wl.symfmt == "e4m3" else 2
    a = eq.codec.quantize(w, fmt, wl.int8_div)
    b = orc.quantize(w, fmt, wl.int8_div)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_quantize_edge_values(eq, orc):
    rng = np.random.default_rng(1)
    w = (rng.standard_normal((40, 300)) * 10.0 ** rng.uniform(-8, 3, (40, 300))).astype(np.float32)
    w[0] = 0.0
    w[1, :5] = [448.0 * 3, -1e-30, 1e-40, -0.0, 7.0]
    for fmt in (1, 2):
        a = eq.codec.quantize(w, fmt, 3.7)
        b = orc.quantize(w, fmt, 3.7)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


@pytest.mark.parametrize("chunk,S,G", [(16384, 32, 8), (65536, 128, 8), (0, 64, 8), (999, 32, 1),
                                       (4096, 256, 8)])
def test_rans_encode_matches_oracle(eq, orc, chunk, S, G):
    w = synth.normal_with_outliers(96, 1024, 0.02, 0.01, 8.0, 5)
    sym, sc = orc.quantize(w, orc.E4M3)
    fa = eq.codec.rans_freqs(sym)
    assert np.array_equal(fa, orc.rans_freqs(sym))
    a = eq.codec.rans_encode(sym, sc, 1, chunk, S, G)
    b = orc.rans_encode(sym, sc, 1, chunk, S, G)
    assert np.array_equal(a.states, b.states)
    assert np.array_equal(a.word_off, b.word_off)
    assert np.array_equal(a.words, b.words)


@pytest.mark.parametrize("pb", [8, 7])
@pytest.mark.parametrize("chunk,S,G", [(65536, 128, 8), (999, 32, 1), (0, 64, 8), (4096, 32, 3)])
def test_rans_encode_8bit_matches_oracle(eq, orc, chunk, S, G, pb):
    w = synth.laplace_clipped(96, 1024, 0.01, 0.06, 7)
    sym, sc = orc.quantize(w, orc.INT8, synth.INT8_DIV_LAPLACE_8K)
    f = orc.rans_freqs(sym, pb)
    assert np.array_equal(eq.codec.rans_freqs(sym, pb), f)
    a = eq.codec.rans_encode(sym, sc, 2, chunk, S, G, prob_bits=pb)
    b = orc.rans_encode(sym, sc, 2, chunk, S, G, prob_bits=pb)
    assert np.array_equal(a.states, b.states)
    assert np.array_equal(a.word_off, b.word_off)
    assert np.array_equal(a.words, b.words)


def test_choose_prob_bits(eq, orc):
    """7-bit tables for the 2-bit Int8 workload, 12-bit ones for ~6.5-bit Float8 weights, 8-bit
    ones where 7 bits would lose too much."""
    wl = synth.WORKLOADS["int8_8k"]
    sym, _ = orc.quantize(wl.tensors[0].generate(row_lo=0, row_hi=256), orc.INT8, wl.int8_div)
    assert eq.codec.choose_prob_bits(np.bincount(sym.ravel(), minlength=256)) == wl.prob_bits == 7
    assert eq.codec.choose_prob_bits(np.bincount(sym.ravel(), minlength=256), 0.002) == 8
    sym, _ = orc.quantize(synth.WORKLOADS["e4m3_1k"].tensors[0].generate(), orc.E4M3)
    assert eq.codec.choose_prob_bits(np.bincount(sym.ravel(), minlength=256)) == 12


def test_rans_freqs_edge_cases(eq, orc):
    for sym in [np.zeros(0, np.uint8), np.full(10, 3, np.uint8), np.arange(256, dtype=np.uint8),
                np.repeat(np.arange(256, dtype=np.uint8), np.arange(1, 257))]:
        assert np.array_equal(eq.codec.rans_freqs(sym), orc.rans_freqs(sym))


@pytest.mark.parametrize("tpb", [256, 32, 1])
def test_huff_encode_matches_oracle(eq, orc, tpb):
    w = synth.bf16_normal(32, 4096, 0.015, 6)
    a = eq.codec.huff_encode(w, tpb)
    b = orc.huff_encode_bf16(w, tpb)
    assert np.array_equal(a.lengths, b.lengths)
    assert a.total_bits == b.total_bits
    for f in ("enc_exp", "sign_mant", "gaps", "block_out"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f


def test_huff_lengths_optimal_and_capped(eq, orc):
    rng = np.random.default_rng(2)
    for _ in range(100):
        counts = np.zeros(256, np.uint64)
        k = int(rng.integers(1, 80))
        counts[rng.choice(256, k, replace=False)] = rng.integers(1, 10 ** 6, k).astype(np.uint64)
        a = eq.codec.huff_lengths(counts).astype(np.int64)
        b = orc.huff_lengths(counts).astype(np.int64)
        assert (a * counts.astype(np.int64)).sum() == (b * counts.astype(np.int64)).sum()
    fib = [1, 1]
    while len(fib) < 40:
        fib.append(fib[-1] + fib[-2])
    counts = np.zeros(256, np.uint64)
    counts[:40] = fib
    a = eq.codec.huff_lengths(counts, 32)
    b = orc.huff_lengths(counts, 32)
    assert a.max() <= 32 and np.array_equal(a, b.astype(np.uint32))


def test_normalize_from_counts_matches_oracle(eq, orc):
    rng = np.random.default_rng(3)
    for _ in range(50):
        counts = np.zeros(256, np.uint64)
        k = int(rng.integers(1, 257))
        counts[rng.choice(256, k, replace=False)] = rng.integers(1, 10 ** 7, k).astype(np.uint64)
        f = np.zeros(256, np.uint32)
        assert orc.lib().orc_rans_normalize(counts.ctypes.data, 12, f.ctypes.data) == 0
        assert np.array_equal(eq.normalize_freqs(counts), f)


def test_super_weights_and_excluding_quantiser_match_oracle(eq, orc):
    w = synth.laplace_clipped(300, 1024, 0.01, 0.06, 8)
    synth.plant_super_weights(w, 9, 8)
    ia, va = eq.codec.super_weights(w)
    ib, vb = orc.super_weights(w)
    assert ia.size == 9 and np.array_equal(ia, ib) and np.array_equal(va, vb)
    for fmt in (1, 2):
        a = eq.codec.quantize_excluding(w, fmt, synth.INT8_DIV_LAPLACE_8K, ia)
        b = orc.quantize_excluding(w, fmt, synth.INT8_DIV_LAPLACE_8K, ib)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    with pytest.raises(eq.EqError):  # the list must increase
        eq.codec.quantize_excluding(w, 2, 4.0, ia[::-1].copy())


@pytest.mark.parametrize("bits", [8, 4])
def test_integer_quantiser_and_byte_huffman_match_oracle(eq, orc, bits):
    rng = np.random.default_rng(bits)
    for w in (synth.normal(128, 1024, 0.02, 9),
              np.abs(rng.standard_normal((64, 700))).astype(np.float32) * 0.03,
              synth.normal_with_outliers(50, 333, 0.02, 0.01, 8.0, 10)):
        for scheme in (0, 1):
            a = eq.codec.intq_quantize(w, bits, scheme)
            b = orc.intq_quantize(w, bits, scheme)
            assert np.array_equal(a[0], b[0]) and a[1:] == b[1:]
        for tpb in (256, 32):
            h = eq.codec.entrollm_encode(w, bits, threads_per_block=tpb)
            sym, sc, z, _ = orc.entrollm_quantize(w, bits)
            o = orc.huff_encode_sym(sym, bits, sc, z, threads_per_block=tpb)
            assert (h.scale, h.zero, h.total_bits) == (o.scale, o.zero, o.total_bits)
            assert np.array_equal(h.lengths, o.lengths)
            for f in ("enc", "gaps", "block_out"):
                assert np.array_equal(getattr(h, f), getattr(o, f)), f
