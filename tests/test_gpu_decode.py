"""GPU parity: eq_decode (interleaved rANS -> bf16) against the oracle, bit for bit.

The expected output is the oracle's dequantisation of the quantised symbols (a lossless decoder
must reproduce exactly those); the coded input is the oracle's encoding of the same symbols.
"""
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


def quantized(orc, spec, symfmt, int8_div=0.0, row_lo=0, row_hi=None):
    w = spec.generate(row_lo=row_lo, row_hi=row_hi)
    return orc.quantize(w, symfmt, int8_div)


def run_decode(eq, hosts):
    dev = [eq.DeviceRans.upload(h) for h in hosts]
    outs, status = eq.decode(dev)
    torch.cuda.synchronize()
    return [eq.bf16_bits(o).ravel() for o in outs], int(status.item())


def expect(orc, sym, sc, fmt):
    return orc.dequant(sym, sc, fmt).ravel()


@pytest.mark.parametrize("streams,run", [(32, 8), (32, 1), (64, 8), (128, 8), (256, 8), (128, 1)])
def test_e4m3_1k_all_layouts(eq, orc, streams, run):
    wl = synth.WORKLOADS["e4m3_1k"]
    sym, sc = quantized(orc, wl.tensors[0], orc.E4M3)
    h = orc.rans_encode(sym, sc, orc.E4M3, wl.chunk_symbols, streams, run)
    (out,), st = run_decode(eq, [h])
    assert st == 0
    assert np.array_equal(out, expect(orc, sym, sc, orc.E4M3))


def test_int8_8k_full_size(eq, orc):
    """The 8192x8192 Int8 workload in the bench's launch configuration, every element."""
    wl = synth.WORKLOADS["int8_8k"]
    sym, sc = quantized(orc, wl.tensors[0], orc.INT8, wl.int8_div)
    h = orc.rans_encode(sym, sc, orc.INT8, wl.chunk_symbols, wl.streams, wl.run,
                        prob_bits=wl.prob_bits)
    (out,), st = run_decode(eq, [h])
    assert st == 0
    assert np.array_equal(out, expect(orc, sym, sc, orc.INT8))


@pytest.mark.parametrize("rows,cols,chunk,streams,run", [
    (1, 8, 8, 32, 8),            # one run, one chunk
    (3, 200, 1000, 32, 8),       # chunks cut rows, ragged last chunk
    (37, 200, 7400, 64, 8),      # one chunk holding everything, ragged last round
    (5, 104, 104, 128, 8),       # one row per chunk, mostly idle streams
    (17, 333, 999, 32, 1),       # run 1, odd sizes
    (64, 1024, 65536, 256, 8),   # exactly one full chunk
    (1, 1, 1, 32, 1),            # a single symbol
])
def test_ragged_shapes(eq, orc, rows, cols, chunk, streams, run):
    w = synth.normal(rows, cols, 0.02, 40 + rows)
    sym, sc = orc.quantize(w, orc.E4M3)
    h = orc.rans_encode(sym, sc, orc.E4M3, chunk, streams, run)
    (out,), st = run_decode(eq, [h])
    assert st == 0
    assert np.array_equal(out, expect(orc, sym, sc, orc.E4M3))


def test_special_symbols(eq, orc):
    """E4M3 NaN codes and signed zeros, Int8 -128 and 127: every byte value decodes."""
    rng = np.random.default_rng(3)
    for fmt in (orc.E4M3, orc.INT8):
        sym = rng.integers(0, 256, (64, 512), dtype=np.uint8)
        sc = synth.bf16_bits(rng.uniform(1e-4, 2.0, 64).astype(np.float32))
        sc[0] = 0xBC00  # a negative scale
        h = orc.rans_encode(sym, sc, fmt, 4096, 64, 8)
        (out,), st = run_decode(eq, [h])
        assert st == 0
        assert np.array_equal(out, expect(orc, sym, sc, fmt))


def test_single_symbol_table(eq, orc):
    sym = np.full((16, 256), 0x38, np.uint8)
    sc = np.full(16, 0x3F80, np.uint16)
    h = orc.rans_encode(sym, sc, orc.E4M3, 1024, 32, 8)
    assert h.word_off[-1] == 0
    (out,), st = run_decode(eq, [h])
    assert st == 0 and np.array_equal(out, expect(orc, sym, sc, orc.E4M3))


def test_grouped_launch_mixed(eq, orc):
    """Several tensors of different formats and layouts in one eq_decode call."""
    hosts, want = [], []
    specs = [(orc.E4M3, 256, 1024, 16384, 128, 8), (orc.INT8, 100, 800, 8000, 64, 8),
             (orc.E4M3, 33, 512, 512, 32, 1), (orc.INT8, 64, 4096, 65536, 128, 8),
             (orc.E4M3, 128, 4096, 65536, 128, 8)]
    for i, (fmt, r, c, chunk, S, G) in enumerate(specs):
        w = synth.laplace_clipped(r, c, 0.01, 0.06, 60 + i) if fmt == orc.INT8 else \
            synth.normal_with_outliers(r, c, 0.02, 0.01, 8.0, 60 + i)
        sym, sc = orc.quantize(w, fmt, 4.2281)
        hosts.append(orc.rans_encode(sym, sc, fmt, chunk, S, G))
        want.append(expect(orc, sym, sc, fmt))
    outs, st = run_decode(eq, hosts)
    assert st == 0
    for o, e in zip(outs, want):
        assert np.array_equal(o, e)


def test_llama_layer_grouped(eq, orc):
    """One LLaMA-2-7B-shaped layer (7 tensors, 1% outliers x8) decoded in one launch."""
    wl = synth.scaled(synth.WORKLOADS["llama2_7b"], layers=1)
    hosts, want = [], []
    for spec in wl.tensors:
        sym, sc = quantized(orc, spec, orc.E4M3)
        hosts.append(orc.rans_encode(sym, sc, orc.E4M3, wl.chunk_symbols, wl.streams, wl.run))
        want.append(expect(orc, sym, sc, orc.E4M3))
    outs, st = run_decode(eq, hosts)
    assert st == 0
    for o, e in zip(outs, want):
        assert np.array_equal(o, e)


def test_product_encoder_stream_decodes(eq, orc):
    """The library's own compressor (used by the bench) produces streams the kernel decodes to the
    oracle's values."""
    wl = synth.WORKLOADS["int8_8k"]
    w = wl.tensors[0].generate(row_lo=0, row_hi=512)
    sym, sc = eq.codec.quantize(w, eq.EQ_SYM_INT8, wl.int8_div)
    h = eq.codec.rans_encode(sym, sc, eq.EQ_SYM_INT8, wl.chunk_symbols, wl.streams, wl.run,
                             prob_bits=wl.prob_bits)
    (out,), st = run_decode(eq, [h])
    osym, osc = orc.quantize(w, orc.INT8, wl.int8_div)
    assert st == 0 and np.array_equal(out, expect(orc, osym, osc, orc.INT8))


def test_corruption_sets_status(eq, orc):
    w = synth.normal(64, 1024, 0.02, 70)
    sym, sc = orc.quantize(w, orc.E4M3)
    h = orc.rans_encode(sym, sc, orc.E4M3, 16384, 32, 8)
    # wrong final state in chunk 1
    h.states = h.states.copy()
    h.states[40] ^= 0x1234
    _, st = run_decode(eq, [h])
    assert st & 3  # the stream ends in a wrong state or runs past its words
    # truncated chunk: drop its last word (offsets shifted, stream shorter than it needs)
    h = orc.rans_encode(sym, sc, orc.E4M3, 16384, 32, 8)
    h.word_off = h.word_off.copy()
    h.word_off[1:] -= 1
    h.words = np.concatenate([h.words[:int(h.word_off[1])], h.words[int(h.word_off[1]) + 1:]])
    _, st = run_decode(eq, [h])
    assert st & 3
    # state below 2^16
    h = orc.rans_encode(sym, sc, orc.E4M3, 16384, 32, 8)
    h.states = h.states.copy()
    h.states[0] = 7
    _, st = run_decode(eq, [h])
    assert st != 0


def test_host_validation(eq, orc):
    w = synth.normal(8, 64, 0.02, 71)
    sym, sc = orc.quantize(w, orc.E4M3)
    h = orc.rans_encode(sym, sc, orc.E4M3, 512, 32, 8)
    t = eq.DeviceRans.upload(h)
    for field, val in [("streams", 48), ("run", 4), ("prob_bits", 11), ("num_chunks", 3)]:
        bad = eq.DeviceRans(**{**t.__dict__, field: val})
        with pytest.raises(eq.EqError):
            eq.decode([bad])
