"""GPU parity: eq_huff_bf16_decode (DFloat11) against the original bf16 bits, bit for bit."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def eq():
    import decoding_interleaved_rans_b200 as m
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    m.lib()
    return m


def run(eq, h):
    d = eq.DeviceHuff.upload(h)
    out, st = eq.huff_bf16_decode(d)
    torch.cuda.synchronize()
    return eq.bf16_bits(out).ravel(), int(st.item())


def test_df11_8k_full_size(eq, orc):
    """The 8192x28672 bf16 workload (N(0, 0.015)), every element."""
    w = synth.WORKLOADS["df11_8k"].tensors[0].generate().ravel()
    h = orc.huff_encode_bf16(w)
    out, st = run(eq, h)
    assert st == 0 and np.array_equal(out, w)


@pytest.mark.parametrize("n,tpb,std", [(1, 256, 0.015), (7, 32, 0.015), (1000, 64, 1.0),
                                       (123457, 256, 0.015), (300000, 512, 3e-5),
                                       (50000, 128, 100.0)])
def test_shapes_and_block_sizes(eq, orc, n, tpb, std):
    w = synth.bf16_normal(1, n, std, n)[0]
    h = orc.huff_encode_bf16(w, threads_per_block=tpb)
    out, st = run(eq, h)
    assert st == 0 and np.array_equal(out, w)


def test_all_exponents_and_long_codes(eq, orc):
    """Every exponent value 0..255 (240..255 included, which the page's 8-bit tables would reserve)
    with Fibonacci-like frequencies so that codes reach the 32-bit cap and four table levels."""
    rng = np.random.default_rng(4)
    fib = [1, 1]
    while len(fib) < 40:
        fib.append(fib[-1] + fib[-2])
    counts = np.ones(256, np.int64)
    perm = rng.permutation(256)
    counts[perm[:40]] = np.array(fib[::-1]) // 1000 + 1
    e = np.repeat(np.arange(256), counts)
    rng.shuffle(e)
    w = ((rng.integers(0, 2, e.size) << 15) | (e << 7) | rng.integers(0, 128, e.size)).astype(np.uint16)
    h = orc.huff_encode_bf16(w)
    assert h.lengths.max() >= 12  # three table levels
    out, st = run(eq, h)
    assert st == 0 and np.array_equal(out, w)
    fibc = np.zeros(256, np.uint64)
    fibc[:40] = fib
    lens = orc.huff_lengths(fibc, 32)
    assert lens.max() == 32
    e = np.repeat(np.arange(40), [min(int(c), 3) for c in fib])
    w = ((e << 7) | 0x35).astype(np.uint16)
    h = orc.huff_encode_bf16(w, lengths=lens)
    out, st = run(eq, h)
    assert st == 0 and np.array_equal(out, w)


def test_warps_with_short_and_long_segments(eq, orc):
    """Regions of ~2.6-bit exponent codes (about 24 values a 64-bit segment) alternate with runs
    of one exponent (1-bit codes, 64 values a segment), so some warps stage at most 32 values per
    lane and others more, and the boundaries fall inside warps and blocks."""
    rng = np.random.default_rng(44)
    parts = []
    for i in range(9):
        n = int(rng.integers(3000, 40000))
        if i % 2 == 0:
            parts.append(synth.bf16_normal(1, n, 0.015, 440 + i)[0])
        else:
            parts.append(np.full(n, 0x3C10, np.uint16) | (rng.integers(0, 2, n).astype(np.uint16) << 15))
    w = np.concatenate(parts)
    for tpb in (64, 256):
        h = orc.huff_encode_bf16(w, threads_per_block=tpb)
        out, st = run(eq, h)
        assert st == 0 and np.array_equal(out, w), tpb


def test_single_exponent(eq, orc):
    w = np.full(5000, 0x3F80, np.uint16)
    w[::3] = 0xBF81
    h = orc.huff_encode_bf16(w)
    out, st = run(eq, h)
    assert st == 0 and np.array_equal(out, w)


def test_product_encoder_container(eq, orc):
    w = synth.bf16_normal(64, 28672, 0.015, 9).ravel()
    h = eq.codec.huff_encode(w)
    out, st = run(eq, h)
    assert st == 0 and np.array_equal(out, w)


def test_corruption_sets_status(eq, orc):
    w = synth.bf16_normal(1, 200000, 0.015, 10)[0]
    h = orc.huff_encode_bf16(w)
    h.block_out = h.block_out.copy()
    h.block_out[3] += 5
    _, st = run(eq, h)
    assert st & 8
    h = orc.huff_encode_bf16(w)
    h.gaps = h.gaps.copy()
    h.gaps[100] ^= 0x5A
    _, st = run(eq, h)
    assert st & (4 | 8)
