"""Pins for the oracle's renormalisation interval.  With 2^prob_bits slots a stream renormalises
after every k-th of its own steps (and after its last), k = floor(16 / prob_bits): 8-bit tables
renormalise once per pair of steps.  The pins: brute-force round trips, a closed form for the
uniform 8-bit table that fixes the pairing, the flush bound and the word order, an independent
arbitrary-precision ANS for the size, and the Shannon bound on the Int8 workload."""
import itertools
import math

import numpy as np
import pytest

import synth


def tbl(bits, freq_of):
    f = np.zeros(256, np.uint32)
    for s, v in freq_of.items():
        f[s] = v
    assert f.sum() == 1 << bits
    return f


TABLES = [(8, tbl(8, {0: 128, 1: 64, 2: 64})), (8, tbl(8, {5: 1, 9: 254, 77: 1})),
          (8, tbl(8, {0: 85, 1: 85, 2: 86})), (7, tbl(7, {0: 1, 1: 126, 200: 1})),
          (7, tbl(7, {3: 43, 4: 42, 5: 43})), (5, tbl(5, {0: 3, 1: 13, 2: 16})),
          (4, tbl(4, {0: 1, 1: 5, 2: 10}))]


@pytest.mark.parametrize("ti", range(len(TABLES)))
def test_bruteforce_roundtrip_all_short_sequences(orc, ti):
    bits, f = TABLES[ti]
    alphabet = np.nonzero(f)[0]
    for S, G in [(1, 1), (2, 1), (2, 8), (32, 8), (3, 2), (40, 1), (1, 3)]:
        for n in range(0, 8):
            for seq in itertools.product(alphabet, repeat=n):
                sym = np.array(seq, np.uint8)
                st, words, cnt = orc.rans_encode_chunk(sym, f, S, G, prob_bits=bits)
                rc, out = orc.rans_decode_chunk(words, st, n, f, S, G, cnt, prob_bits=bits)
                assert rc == 0 and np.array_equal(out, sym), (ti, S, G, seq)
            if n >= 5 and S >= 32:
                break


def stream_symbols(sym, S, G):
    """Each stream's symbols in its own step order: stream s takes runs s, s + S, ..."""
    runs = np.arange(sym.size) // G
    return [sym[(runs % S) == s] for s in range(S)]


def test_uniform_8bit_closed_form(orc):
    """f_s = 1 for all 256 bytes: coding s maps x to 256 x + s, so a stream's steps pair up into
    16-bit words.  With the renormalisation point after every second step, a stream of T symbols
    s_0 .. s_{T-1} ends in the state (T odd ? 256 : 1) * 2^16 + 256 s_1 + s_0 (T >= 2), or
    2^24 + s_0 (T = 1), and reads floor(T / 2) words: 256 s_3 + s_2, 256 s_5 + s_4, ..., then
    s_{T-1} (T odd) or 0 (T even)."""
    f = np.ones(256, np.uint32)
    rng = np.random.default_rng(12)
    for T in range(0, 12):
        sym = rng.integers(0, 256, T, dtype=np.uint8)
        st, words, _ = orc.rans_encode_chunk(sym, f, 1, 1, prob_bits=8)
        s = [int(v) for v in sym]
        if T == 0:
            assert st[0] == 1 << 16 and words.size == 0
            continue
        if T == 1:
            assert st[0] == (1 << 24) + s[0] and words.size == 0
            continue
        assert st[0] == ((256 if T % 2 else 1) << 16) + 256 * s[1] + s[0]
        expect = [s[i] + 256 * s[i + 1] for i in range(2, T - 1, 2)]
        expect.append(s[T - 1] if T % 2 else 0)
        assert words.tolist() == expect, T
    for S, G, n in [(32, 8, 1000), (4, 8, 333), (32, 1, 777), (5, 3, 200)]:
        sym = rng.integers(0, 256, n, dtype=np.uint8)
        st, words, _ = orc.rans_encode_chunk(sym, f, S, G, prob_bits=8)
        total = 0
        for s, mine in enumerate(stream_symbols(sym, S, G)):
            T = mine.size
            total += T // 2
            if T >= 2:
                assert st[s] == ((256 if T % 2 else 1) << 16) + 256 * int(mine[1]) + int(mine[0])
        assert words.size == total


def test_12bit_keeps_one_renormalisation_per_step(orc):
    """12-bit tables (k = 1): the uniform 12-bit table f_s = 16 costs 8 bits per symbol, so a
    stream's 16-bit words come once per two steps but its renormalisation test runs every step,
    and its state has bit length 17 + 8 (T mod 2) (a pair-renormalising coder would differ)."""
    f = np.full(256, 16, np.uint32)
    sym = np.random.default_rng(13).integers(0, 256, 9, dtype=np.uint8)
    st, words, _ = orc.rans_encode_chunk(sym, f, 1, 1, prob_bits=12)
    assert int(st[0]).bit_length() == 25 and words.size == 4


def test_size_matches_arbitrary_precision_ans_8bit(orc):
    bits, f = TABLES[0]
    M = 1 << bits
    cum = np.concatenate([[0], np.cumsum(f)[:-1]])
    rng = np.random.default_rng(14)
    sym = rng.choice(np.nonzero(f)[0], 4000, p=f[np.nonzero(f)[0]] / M).astype(np.uint8)
    x = 1 << 16
    for s in reversed(sym.tolist()):
        x = (x // int(f[s])) * M + (x % int(f[s])) + int(cum[s])
    ideal = sum(math.log2(M / f[s]) for s in sym.tolist())
    assert abs((math.log2(x) - 16) - ideal) < 1.0
    st, words, _ = orc.rans_encode_chunk(sym, f, 1, 1, prob_bits=bits)
    coded = 16 * words.size + math.log2(int(st[0])) - 16
    assert abs(coded - ideal) <= 0.002 * ideal + 16
    rc, out = orc.rans_decode_chunk(words, st, sym.size, f, 1, 1, prob_bits=bits)
    assert rc == 0 and np.array_equal(out, sym)


def test_int8_workload_8bit_table_near_shannon(orc):
    """The Int8 workload (entropy about 2 bits over 9 values) in 8-bit tables: words within 1% of
    N H / 8, the table's cross-entropy within 0.01 bits of H, and a lossless round trip."""
    wl = synth.WORKLOADS["int8_8k"]
    w = wl.tensors[0].generate(row_lo=0, row_hi=256)
    sym, sc = orc.quantize(w, orc.INT8, wl.int8_div)
    t = orc.rans_encode(sym, sc, orc.INT8, 65536, 128, 8, prob_bits=8)
    H = orc.entropy_bits(sym)
    assert t.payload_bytes <= 1.01 * t.numel * H / 8
    counts = np.bincount(sym.ravel(), minlength=256)
    assert orc.cross_entropy_bits(counts, t.freqs, 8) - H < 0.01
    rc, out = orc.rans_decode_bf16(t, threads=4)
    assert rc == 0 and np.array_equal(out.reshape(sym.shape), orc.dequant(sym, sc, orc.INT8))


def test_8bit_corruption_is_reported(orc):
    sym = synth.symbols_from_pmf(np.exp(-np.arange(256) / 2.0), 20000, 15)
    f = orc.rans_freqs(sym, 8)
    st, words, cnt = orc.rans_encode_chunk(sym, f, 32, 8, prob_bits=8)
    assert orc.rans_decode_chunk(words[:-1], st, sym.size, f, 32, 8, prob_bits=8)[0] != 0
    bad = st.copy()
    bad[7] ^= 0x100
    assert orc.rans_decode_chunk(words, bad, sym.size, f, 32, 8, prob_bits=8)[0] != 0


def test_uniform_7bit_closed_form(orc):
    """f_s = 1 for bytes 0..127 (7-bit table): coding s maps x to 128 x + s, so a pair of steps
    adds exactly 14 bits (2^14 x + 128 s_b + s_a) and a flush removes 16.  The pair's flush
    bound is 2^(32 - 14) = 2^18: the encoder flushes before a pair iff x has at least 19 bits.
    So the word count follows from bit lengths alone (start 2^16: 17 bits), and the final state's
    low 14 bits are 128 s_1 + s_0."""
    f = np.zeros(256, np.uint32)
    f[:128] = 1
    rng = np.random.default_rng(16)
    for T in range(2, 60, 2):
        sym = rng.integers(0, 128, T, dtype=np.uint8)
        st, words, _ = orc.rans_encode_chunk(sym, f, 1, 1, prob_bits=7)
        bits, flushes = 17, 0
        for _ in range(T // 2):
            if bits >= 19:
                bits -= 16
                flushes += 1
            bits += 14
        assert words.size == flushes, T
        assert int(st[0]).bit_length() == bits, T
        assert int(st[0]) & 0x3FFF == 128 * int(sym[1]) + int(sym[0])
        rc, out = orc.rans_decode_chunk(words, st, T, f, 1, 1, prob_bits=7)
        assert rc == 0 and np.array_equal(out, sym)


def test_int8_workload_7bit_table_near_shannon(orc):
    wl = synth.WORKLOADS["int8_8k"]
    w = wl.tensors[0].generate(row_lo=0, row_hi=256)
    sym, sc = orc.quantize(w, orc.INT8, wl.int8_div)
    t = orc.rans_encode(sym, sc, orc.INT8, 65536, 128, 8, prob_bits=7)
    H = orc.entropy_bits(sym)
    counts = np.bincount(sym.ravel(), minlength=256)
    ce = orc.cross_entropy_bits(counts, t.freqs, 7)
    assert ce - H < 0.012  # 7-bit probabilities cost about 0.4% on this alphabet
    assert t.payload_bytes <= 1.01 * t.numel * ce / 8
    rc, out = orc.rans_decode_bf16(t, threads=4)
    assert rc == 0 and np.array_equal(out.reshape(sym.shape), orc.dequant(sym, sc, orc.INT8))
