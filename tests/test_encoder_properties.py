"""Property test of the library's host compressor against the oracle: for random shapes, chunk
lengths, stream counts, run lengths, table sizes (12-, 8- and 7-bit) and symbol distributions
(one symbol, two, a few, skewed, uniform over the alphabet the table can hold), the frequency
table and the rANS container (final states, word offsets, words) are the same bit for bit."""
import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings, strategies as st


@pytest.fixture(scope="module")
def eq():
    import decoding_interleaved_rans_b200 as m
    m.lib()
    return m


def symbols(rng, rows, cols, pb, kind):
    """A [rows, cols] uint8 matrix whose alphabet fits a 2^pb-slot table."""
    limit = min(256, 1 << (pb - 1))
    if kind == "one":
        return np.full((rows, cols), rng.integers(0, 256), np.uint8)
    if kind == "two":
        a, b = rng.choice(256, 2, replace=False)
        return np.where(rng.random((rows, cols)) < 0.9, a, b).astype(np.uint8)
    alphabet = rng.choice(256, limit, replace=False)
    if kind == "skewed":
        idx = np.minimum(rng.geometric(0.3, (rows, cols)) - 1, limit - 1)
    elif kind == "few":
        idx = rng.integers(0, min(5, limit), (rows, cols))
    else:
        idx = rng.integers(0, limit, (rows, cols))
    return alphabet[idx].astype(np.uint8)


@settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(rows=st.integers(1, 12), cols=st.integers(1, 300), pb=st.sampled_from([12, 8, 7]),
       run=st.sampled_from([1, 2, 3, 8]), streams=st.sampled_from([32, 64, 96, 160]),
       chunk=st.one_of(st.just(0), st.integers(1, 5000)),
       kind=st.sampled_from(["one", "two", "few", "skewed", "uniform"]),
       seed=st.integers(0, 2**31 - 1))
def test_host_encoder_matches_oracle(eq, orc, rows, cols, pb, run, streams, chunk, kind, seed):
    rng = np.random.default_rng(seed)
    sym = symbols(rng, rows, cols, pb, kind)
    sc = np.full(rows, 0x3F80, np.uint16)
    freqs = orc.rans_freqs(sym, pb)
    assert np.array_equal(eq.codec.rans_freqs(sym, pb), freqs)
    a = eq.codec.rans_encode(sym, sc, 1, chunk, streams, run, prob_bits=pb)
    b = orc.rans_encode(sym, sc, 1, chunk, streams, run, prob_bits=pb)
    assert np.array_equal(a.states, b.states)
    assert np.array_equal(a.word_off, b.word_off)
    assert np.array_equal(a.words, b.words)


def bf16_weights(rng, rows, cols, kind):
    """bf16 bit patterns [rows, cols] with exponent distributions from one exponent to all 256."""
    if kind == "normal":
        w = (rng.standard_normal((rows, cols)) * 0.015).astype(np.float32)
        return (w.view(np.uint32) >> 16).astype(np.uint16)
    if kind == "one_exponent":
        e = int(rng.integers(1, 255))
        return ((rng.integers(0, 2, (rows, cols)) << 15) | (e << 7)
                | rng.integers(0, 128, (rows, cols))).astype(np.uint16)
    if kind == "wide":  # magnitudes over many decades: long codes
        w = (rng.standard_normal((rows, cols)) * 10.0 ** rng.uniform(-30, 30, (rows, cols)))
        return (w.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    return rng.integers(0, 1 << 16, (rows, cols)).astype(np.uint16)  # every pattern, NaN and inf too


@settings(max_examples=40, deadline=None, suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(rows=st.integers(1, 40), cols=st.integers(1, 700), tpb=st.sampled_from([1, 32, 256]),
       kind=st.sampled_from(["normal", "one_exponent", "wide", "any"]), seed=st.integers(0, 2**31 - 1))
def test_host_df11_encoder_matches_oracle(eq, orc, rows, cols, tpb, kind, seed):
    w = bf16_weights(np.random.default_rng(seed), rows, cols, kind)
    a = eq.codec.huff_encode(w, tpb)
    b = orc.huff_encode_bf16(w, tpb)
    assert np.array_equal(a.lengths, b.lengths)
    assert a.total_bits == b.total_bits
    for f in ("enc_exp", "sign_mant", "gaps", "block_out"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f


@settings(max_examples=30, deadline=None, suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(rows=st.integers(1, 30), cols=st.integers(1, 500), bits=st.sampled_from([8, 4]),
       tpb=st.sampled_from([1, 32, 256]), spread=st.floats(1e-6, 10.0), shift=st.floats(-1.0, 1.0),
       seed=st.integers(0, 2**31 - 1))
def test_host_integer_code_encoder_matches_oracle(eq, orc, rows, cols, bits, tpb, spread, shift,
                                                  seed):
    """EntroLLM-style integer codes: the per-tensor quantiser and the byte-stream Huffman coder."""
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((rows, cols)) * spread + shift * spread).astype(np.float32)
    for scheme in (0, 1):
        a = eq.codec.intq_quantize(w, bits, scheme)
        b = orc.intq_quantize(w, bits, scheme)
        assert np.array_equal(a[0], b[0]) and a[1:] == b[1:]
    h = eq.codec.entrollm_encode(w, bits, threads_per_block=tpb)
    sym, sc, z, _ = orc.entrollm_quantize(w, bits)
    o = orc.huff_encode_sym(sym, bits, sc, z, threads_per_block=tpb)
    assert (h.scale, h.zero, h.total_bits) == (o.scale, o.zero, o.total_bits)
    assert np.array_equal(h.lengths, o.lengths)
    for f in ("enc", "gaps", "block_out"):
        assert np.array_equal(getattr(h, f), getattr(o, f)), f
