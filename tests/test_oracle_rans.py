"""Pins for the oracle's interleaved rANS coder.

The pages say only that the flattened symbol stream is ANS-coded and decoded in parallel on the
GPU ("Float8@2bits" summary, sections "Codificacion de Pesos" and "Decodificacion en Tiempo de
Inferencia").  The coder here is pinned by: brute-force round trips on every short sequence, a
closed form for the uniform table, the single-symbol table, an independent arbitrary-precision
ANS, the stream-assignment rule recomputed by slicing, and the Shannon bound the pages' rate
claims rest on.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
M = 4096


def table(freq_of: dict) -> np.ndarray:
    f = np.zeros(256, np.uint32)
    for s, v in freq_of.items():
        f[s] = v
    assert f.sum() == M
    return f


TABLES = [
    table({0: 2048, 1: 1024, 2: 1024}),
    table({7: 1, 128: 4094, 255: 1}),
    table({0: 1365, 100: 1365, 200: 1366}),
    table({3: 4000, 4: 95, 250: 1}),
]


@pytest.mark.parametrize("ti", range(len(TABLES)))
def test_bruteforce_roundtrip_all_short_sequences(orc, ti):
    f = TABLES[ti]
    alphabet = np.nonzero(f)[0]
    for S, G in [(1, 1), (2, 1), (2, 8), (32, 1), (32, 8), (3, 2), (40, 1), (64, 8)]:
        for n in range(0, 8):
            for seq in itertools.product(alphabet, repeat=n):
                sym = np.array(seq, np.uint8)
                st, words, cnt = orc.rans_encode_chunk(sym, f, S, G)
                rc, out = orc.rans_decode_chunk(words, st, n, f, S, G, cnt)
                assert rc == 0 and np.array_equal(out, sym), (ti, S, G, seq)
            if n >= 5 and S >= 32:
                break


def test_uniform_table_closed_form(orc):
    """f_s = 16 for every byte: each symbol is exactly 8 bits.  A stream holding n_s symbols emits
    floor(n_s / 2) words and ends with a state of bit length 17 + 8 (n_s mod 2).  Coding s maps
    x = [h | l] (l = low 4 bits) to [h | s | l], so the stream's first symbol sits in bits 4..11
    of its final state."""
    f = np.full(256, 16, np.uint32)
    rng = np.random.default_rng(5)
    for S, G, n in [(1, 1, 9), (32, 8, 1000), (32, 1, 777), (4, 8, 333), (64, 8, 100)]:
        sym = rng.integers(0, 256, n, dtype=np.uint8)
        st, words, _ = orc.rans_encode_chunk(sym, f, S, G)
        stream = (np.arange(n) // G) % S
        expect_words = 0
        for s in range(S):
            mine = sym[stream == s]
            ns = mine.size
            expect_words += ns // 2
            x = int(st[s])
            assert x.bit_length() == 17 + 8 * (ns % 2)
            if ns:
                assert ((x >> 4) & 0xFF) == int(mine[0])
            else:
                assert x == 1 << 16
        assert words.size == expect_words


def test_single_symbol_table_emits_nothing(orc):
    f = table({42: M})
    for S, G in [(1, 1), (32, 8), (128, 8)]:
        sym = np.full(5000, 42, np.uint8)
        st, words, cnt = orc.rans_encode_chunk(sym, f, S, G)
        assert words.size == 0 and (st == 1 << 16).all() and (cnt == 0).all()
        rc, out = orc.rans_decode_chunk(words, st, sym.size, f, S, G, cnt)
        assert rc == 0 and (out == 42).all()


def test_stream_assignment_matches_slicing(orc):
    """Stream s codes exactly the symbols j with floor(j / G) mod S == s, in increasing j: its final
    state and word count equal those of a one-stream coder fed that slice."""
    f = orc.rans_freqs(synth.symbols_from_pmf(np.exp(-np.arange(256) / 9.0), 100000, 3))
    sym = synth.symbols_from_pmf(np.exp(-np.arange(256) / 9.0), 5000, 4)
    sym = sym[f[sym] > 0]
    n = sym.size
    for S, G in [(32, 8), (64, 1), (5, 3), (96, 8)]:
        st, words, cnt = orc.rans_encode_chunk(sym, f, S, G)
        total = 0
        for s in range(S):
            sl = sym[((np.arange(n) // G) % S) == s]
            st1, w1, _ = orc.rans_encode_chunk(sl, f, 1, 1)
            assert st1[0] == st[s]
            total += w1.size
        assert total == words.size == cnt.sum()


def test_group_substream_is_a_32_stream_chunk(orc):
    """Group g of a chunk (streams 32g .. 32g+31) codes the runs r with r mod S in its range; its
    substream and states are exactly those of a 32-stream chunk made of those runs in order."""
    sym = synth.symbols_from_pmf(np.exp(-np.arange(256) / 4.0), 30000, 11)
    f = orc.rans_freqs(sym)
    for S, G in [(64, 8), (128, 8), (96, 1)]:
        n = sym.size - sym.size % 7
        s = sym[:n]
        st, words, cnt = orc.rans_encode_chunk(s, f, S, G)
        offs = np.concatenate([[0], np.cumsum(cnt)])
        runs = np.arange(n) // G
        for g in range(S // 32):
            mine = s[((runs % S) // 32) == g]
            st1, w1, c1 = orc.rans_encode_chunk(mine, f, 32, G)
            assert np.array_equal(st1, st[32 * g:32 * g + 32])
            assert np.array_equal(w1, words[offs[g]:offs[g + 1]])


def big_ans_encode(sym, f, cum):
    """Arbitrary-precision ANS without renormalisation (the textbook C(s, x))."""
    x = 1 << 16
    for s in reversed(sym.tolist()):
        x = (x // int(f[s])) * M + (x % int(f[s])) + int(cum[s])
    return x


def big_ans_decode(x, n, f, cum):
    slot_sym = np.repeat(np.arange(256), f)
    out = []
    for _ in range(n):
        slot = x % M
        s = int(slot_sym[slot])
        x = int(f[s]) * (x // M) + slot - int(cum[s])
        out.append(s)
    return np.array(out, np.uint8), x


def test_size_matches_arbitrary_precision_ans(orc):
    f = TABLES[3]
    cum = np.concatenate([[0], np.cumsum(f)[:-1]])
    rng = np.random.default_rng(8)
    sym = rng.choice(np.nonzero(f)[0], 3000, p=f[np.nonzero(f)[0]] / M).astype(np.uint8)
    X = big_ans_encode(sym, f, cum)
    back, x0 = big_ans_decode(X, sym.size, f, cum)
    assert np.array_equal(back, sym) and x0 == 1 << 16
    ideal = sum(math.log2(M / f[s]) for s in sym.tolist())
    assert abs((math.log2(X) - 16) - ideal) < 1.0
    st, words, _ = orc.rans_encode_chunk(sym, f, 1, 1)
    coded = 16 * words.size + math.log2(int(st[0])) - 16
    assert abs(coded - (math.log2(X) - 16)) <= 0.002 * ideal + 1


def test_corruption_is_reported(orc):
    sym = synth.symbols_from_pmf(np.exp(-np.arange(256) / 5.0), 20000, 9)
    f = orc.rans_freqs(sym)
    st, words, cnt = orc.rans_encode_chunk(sym, f, 32, 8)
    assert orc.rans_decode_chunk(words[:-1], st, sym.size, f, 32, 8)[0] != 0   # truncated
    bad = st.copy()
    bad[3] ^= 0x40
    assert orc.rans_decode_chunk(words, bad, sym.size, f, 32, 8)[0] != 0       # wrong state
    bad = st.copy()
    bad[0] = 5                                                                   # state below L
    assert orc.rans_decode_chunk(words, bad, sym.size, f, 32, 8)[0] != 0
    st2, w2, c2 = orc.rans_encode_chunk(sym, f, 64, 8)                         # words of the
    assert orc.rans_decode_chunk(w2, st2, sym.size, f, 64, 8, c2[::-1])[0] != 0  # other group
    flipped = 0
    for k in range(40):
        w = words.copy()
        w[(k * 997) % w.size] ^= 1 << (k % 16)
        flipped += orc.rans_decode_chunk(w, st, sym.size, f, 32, 8)[0] != 0
    assert flipped >= 38


def test_normalize_properties(orc):
    rng = np.random.default_rng(10)
    for trial in range(200):
        k = int(rng.integers(1, 257))
        counts = np.zeros(256, np.uint64)
        idx = rng.choice(256, k, replace=False)
        counts[idx] = rng.integers(1, 10 ** int(rng.integers(1, 9)), k).astype(np.uint64)
        f = np.zeros(256, np.uint32)
        assert orc.lib().orc_rans_normalize(counts.ctypes.data, 12, f.ctypes.data) == 0
        assert f.sum() == M
        assert ((f > 0) == (counts > 0)).all()
        if k == 1:
            assert f[idx[0]] == M
        ideal = counts.astype(np.float64) * M / counts.sum()
        big = counts > 0
        # every symbol but the most frequent one stays within one unit of its ideal share
        top = int(np.argmax(counts))
        others = big.copy()
        others[top] = False
        if f.sum() == M and np.floor(ideal[big]).clip(min=1).sum() <= M:
            assert (np.abs(f[others] - ideal[others]) <= 1.0).all()


@pytest.mark.parametrize("name", ["e4m3_1k", "int8_8k"])
def test_container_size_near_shannon(orc, name):
    """Compressed words within 1% of N * H / 8, where H is the symbol histogram's Shannon entropy;
    states, offsets, scales and the table are the overhead (EntQuant: lossless ANS on the symbol
    stream, Float8 at about 6.5 bits/param)."""
    wl = synth.WORKLOADS[name]
    spec = wl.tensors[0]
    rows = spec.rows if spec.numel <= (1 << 21) else 512
    w = spec.generate(row_lo=0, row_hi=rows)
    fmt = orc.E4M3 if wl.symfmt == "e4m3" else orc.INT8
    sym, sc = orc.quantize(w, fmt, wl.int8_div)
    t = orc.rans_encode(sym, sc, fmt, wl.chunk_symbols, wl.streams, wl.run)
    H = orc.entropy_bits(sym)
    shannon_bytes = t.numel * H / 8
    assert t.payload_bytes <= 1.01 * shannon_bytes
    overhead = t.states.nbytes + t.word_off.nbytes + t.scales.nbytes + 256 * 2
    assert t.compressed_bytes <= 1.01 * shannon_bytes + overhead
    counts = np.bincount(sym.ravel(), minlength=256)
    assert orc.cross_entropy_bits(counts, t.freqs) - H < 0.05
    rc, out = orc.rans_decode_bf16(t, threads=4)
    assert rc == 0
    assert np.array_equal(out.reshape(sym.shape), orc.dequant(sym, sc, fmt))


def test_partial_last_chunk_and_row_chunks(orc):
    w = synth.normal(37, 200, 0.02, 21)
    sym, sc = orc.quantize(w, orc.E4M3)
    for chunk, S, G in [(1000, 32, 8), (0, 32, 8), (999, 64, 1), (7400, 32, 8)]:
        t = orc.rans_encode(sym, sc, orc.E4M3, chunk, S, G)
        rc, out = orc.rans_decode_bf16(t)
        assert rc == 0
        assert np.array_equal(out.reshape(sym.shape), orc.dequant(sym, sc, orc.E4M3))
        assert t.words.size % 8 == 0


def test_int8_golden_divisor_roundtrip(orc):
    g = json.load(open(os.path.join(GOLDEN, "int8_div.json")))
    w = synth.WORKLOADS["int8_8k"].tensors[0].generate(row_lo=0, row_hi=64)
    sym, sc = orc.quantize(w, orc.INT8, g["int8_div"])
    t = orc.rans_encode(sym, sc, orc.INT8, 65536, 128, 8)
    rc, out = orc.rans_decode_bf16(t)
    assert rc == 0 and np.array_equal(out.reshape(sym.shape), orc.dequant(sym, sc, orc.INT8))
