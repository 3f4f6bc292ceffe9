"""Pins for the oracle's DFloat11 coder (DFloat11 page: "Formato DFloat11", "Decodificacion basada
en LUT jerarquicas", "Kernels GPU de 2 etapas y metadatos auxiliares").

Huffman lengths are pinned by the Kraft equality, the Shannon bounds and brute-force optimality on
small alphabets; canonical codes by the prefix property and their order; the thread/Gap/block
metadata by recomputing code start positions with a cumulative sum and decoding thread segments
independently; the bf16 statistics by the figures the DFloat11 page prints.
"""
import itertools
import json
import os

import numpy as np
import pytest

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
FIG = json.load(open(os.path.join(GOLDEN, "pages_figures.json")))


def kraft(lens):
    return sum(2.0 ** -int(l) for l in lens if l)


def test_kraft_and_shannon_bounds(orc):
    rng = np.random.default_rng(0)
    for _ in range(300):
        k = int(rng.integers(2, 257))
        counts = np.zeros(256, np.uint64)
        counts[rng.choice(256, k, replace=False)] = rng.integers(1, 10 ** 6, k).astype(np.uint64)
        lens = orc.huff_lengths(counts)
        assert ((lens > 0) == (counts > 0)).all()
        assert abs(kraft(lens) - 1.0) < 1e-12
        p = counts[counts > 0] / counts.sum()
        H = float(-(p * np.log2(p)).sum())
        mean = float((lens[counts > 0] * p).sum())
        assert H - 1e-9 <= mean < H + 1


def test_optimal_by_brute_force(orc):
    """For up to 6 symbols, no length vector satisfying Kraft costs less than the oracle's."""
    rng = np.random.default_rng(1)
    for _ in range(60):
        k = int(rng.integers(2, 7))
        c = rng.integers(1, 50, k)
        counts = np.zeros(256, np.uint64)
        counts[:k] = c
        lens = orc.huff_lengths(counts)[:k].astype(int)
        best = min(sum(int(ci) * li for ci, li in zip(c, L))
                   for L in itertools.product(range(1, k), repeat=k) if kraft(L) <= 1.0)
        assert sum(int(ci) * li for ci, li in zip(c, lens)) == best


def test_length_limit_package_merge(orc):
    """Fibonacci counts force depth > 32; the capped code is still complete, within the cap, and
    no worse than any cap-respecting code found by a simple greedy repair."""
    fib = [1, 1]
    while len(fib) < 40:
        fib.append(fib[-1] + fib[-2])
    counts = np.zeros(256, np.uint64)
    counts[:40] = fib
    free = orc.huff_lengths(counts, max_len=64)
    assert free.max() > 32
    capped = orc.huff_lengths(counts, max_len=32)
    assert capped.max() <= 32 and abs(kraft(capped) - 1.0) < 1e-12
    cost = lambda L: int((counts.astype(np.int64) * L.astype(np.int64)).sum())  # noqa: E731
    assert cost(capped) >= cost(free)
    # with a generous cap package-merge gives an optimal code, same cost as the tree
    gen = orc.huff_lengths(counts, max_len=40)
    assert gen.max() <= 40 and cost(gen) == cost(free)


def test_canonical_codes(orc):
    rng = np.random.default_rng(2)
    counts = np.zeros(256, np.uint64)
    counts[rng.choice(256, 50, replace=False)] = rng.integers(1, 10 ** 5, 50).astype(np.uint64)
    lens = orc.huff_lengths(counts)
    codes = orc.huff_canonical(lens)
    used = [s for s in range(256) if lens[s]]
    order = sorted(used, key=lambda s: (lens[s], s))
    strs = [format(int(codes[s]), f"0{int(lens[s])}b") for s in order]
    for a, b in itertools.combinations(strs, 2):
        assert not b.startswith(a) and not a.startswith(b)
    # canonical: left-justified code values increase along (length, byte) order
    vals = [int(codes[s]) << (32 - int(lens[s])) for s in order]
    assert vals == sorted(vals) and len(set(vals)) == len(vals)
    assert strs[0] == "0" * int(lens[order[0]])


def _code_starts(h, w):
    e = (w >> 7) & 0xFF
    L = h.lengths[e].astype(np.int64)
    return np.concatenate([[0], np.cumsum(L)[:-1]]), int(L.sum())


@pytest.mark.parametrize("seed,n,tpb", [(3, 1, 256), (4, 5000, 256), (5, 40000, 32), (6, 777, 4)])
def test_gaps_and_block_out_from_code_starts(orc, seed, n, tpb):
    w = synth.bf16_normal(1, n, 0.015, seed)[0]
    h = orc.huff_encode_bf16(w, threads_per_block=tpb)
    starts, total = _code_starts(h, w)
    assert h.total_bits == total
    T = h.threads
    assert T == (total + 63) // 64
    gaps = orc.gaps_unpack(h.gaps, T)
    first = np.searchsorted(starts, 64 * np.arange(T), side="left")
    first_pos = np.where(first < n, starts[np.minimum(first, n - 1)], total)
    assert np.array_equal(gaps, first_pos - 64 * np.arange(T))
    assert gaps.max(initial=0) <= FIG["gap_bits"]["range"][1]
    blocks = (T + tpb - 1) // tpb
    want = np.searchsorted(starts, 64 * tpb * np.arange(blocks), side="left")
    assert np.array_equal(h.block_out[:-1], want) and h.block_out[-1] == n


def test_thread_segments_decode_independently(orc):
    """Decode every 64-bit thread segment on its own, starting at its Gap and keeping the codes
    that start inside it (the page's two-stage kernel); the concatenation is the exponent stream."""
    w = synth.bf16_normal(1, 3000, 0.015, 7)[0]
    h = orc.huff_encode_bf16(w, threads_per_block=8)
    codes = orc.huff_canonical(h.lengths)
    table = {format(int(codes[s]), f"0{int(h.lengths[s])}b"): s for s in range(256) if h.lengths[s]}
    bits = "".join(format(int(b), "08b") for b in h.enc_exp)
    gaps = orc.gaps_unpack(h.gaps, h.threads)
    out, counts = [], []
    for t in range(h.threads):
        pos, end, k = 64 * t + int(gaps[t]), min(64 * t + 64, h.total_bits), 0
        while pos < end:
            for ln in range(1, 33):
                if bits[pos:pos + ln] in table:
                    out.append(table[bits[pos:pos + ln]])
                    pos += ln
                    k += 1
                    break
            else:
                raise AssertionError("no code")
        counts.append(k)
    assert np.array_equal(np.array(out), (w >> 7) & 0xFF)
    assert np.array_equal(np.cumsum([0] + counts)[::8][:h.blocks], h.block_out[:-1])


def test_roundtrip_random_tiny_streams(orc):
    rng = np.random.default_rng(8)
    for trial in range(300):
        n = int(rng.integers(0, 200))
        k = int(rng.integers(1, 6))
        exps = rng.choice(256, k, replace=False)
        e = rng.choice(exps, n)
        w = ((rng.integers(0, 2, n) << 15) | (e << 7) | rng.integers(0, 128, n)).astype(np.uint16)
        h = orc.huff_encode_bf16(w, threads_per_block=int(rng.choice([1, 4, 256])))
        rc, out = orc.huff_decode_bf16(h)
        assert rc == 0 and np.array_equal(out, w)


def test_df11_statistics_match_pages(orc):
    """bf16 exponent of N(0, 0.015) weights: a few bits of entropy, tens of values used, about
    11 bits/weight after coding, about 70% of the bf16 size (DFloat11 page)."""
    spec = synth.WORKLOADS["df11_8k"].tensors[0]
    w = spec.generate(row_lo=0, row_hi=256)
    counts = orc.exponent_counts(w)
    H = orc.shannon(counts)
    f = FIG["bf16_exponent_entropy_bits"]
    assert abs(H - f["value"]) <= f["tolerance"]
    lo, hi = FIG["bf16_exponent_values_used"]["range"]
    assert lo <= int((counts > 0).sum()) <= hi
    h = orc.huff_encode_bf16(w)
    bpw = h.compressed_bytes * 8 / h.n
    assert abs(bpw - FIG["df11_bits_per_weight"]["value"]) <= FIG["df11_bits_per_weight"]["tolerance"]
    frac = h.compressed_bytes / (2 * h.n)
    assert abs(frac - FIG["df11_size_fraction"]["value"]) <= FIG["df11_size_fraction"]["tolerance"]
    assert h.lengths.max() <= FIG["max_code_len"]["value"]
    rc, out = orc.huff_decode_bf16(h)
    assert rc == 0 and np.array_equal(out, w.ravel())


def test_decode_reports_corruption(orc):
    w = synth.bf16_normal(1, 4000, 0.015, 9)[0]
    h = orc.huff_encode_bf16(w)
    h.total_bits -= 3
    assert orc.huff_decode_bf16(h)[0] != 0
