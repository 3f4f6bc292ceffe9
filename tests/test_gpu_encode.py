"""GPU parity: the device compressor (quantise, histogram, rANS plan + encode) against the oracle's
compressor, bit for bit, and its containers through the decoder."""
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


def cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_bits(t):
    return t.cpu().numpy().view(np.uint16) if t.dtype == torch.int16 else t.cpu().numpy()


@pytest.mark.parametrize("fmt", [1, 2])
def test_quantize_matches_oracle(eq, orc, fmt):
    w = synth.WORKLOADS["e4m3_1k"].tensors[0].generate() if fmt == 1 else \
        synth.WORKLOADS["int8_8k"].tensors[0].generate(row_lo=0, row_hi=256)
    sym, sc = eq.quantize_device(cuda(w), fmt, synth.INT8_DIV_LAPLACE_8K)
    osym, osc = orc.quantize(w, fmt, synth.INT8_DIV_LAPLACE_8K)
    assert np.array_equal(sym.cpu().numpy(), osym)
    assert np.array_equal(host_bits(sc), osc)


def test_quantize_edge_values(eq, orc):
    rng = np.random.default_rng(1)
    w = (rng.standard_normal((40, 300)) * 10.0 ** rng.uniform(-8, 3, (40, 300))).astype(np.float32)
    w[0] = 0.0
    w[1, :5] = [448.0 * 3, -1e-30, 1e-40, -0.0, 7.0]
    for fmt in (1, 2):
        sym, sc = eq.quantize_device(cuda(w), fmt, 3.7)
        osym, osc = orc.quantize(w, fmt, 3.7)
        assert np.array_equal(sym.cpu().numpy(), osym) and np.array_equal(host_bits(sc), osc)


def test_histogram(eq):
    rng = np.random.default_rng(2)
    for n in (0, 1, 15, 4097, 1 << 20, (1 << 20) + 7):
        a = rng.integers(0, 256, n, dtype=np.uint8)
        c = eq.histogram_device(cuda(a) if n else torch.zeros(1, dtype=torch.uint8, device="cuda")[:0])
        assert np.array_equal(c.cpu().numpy(), np.bincount(a, minlength=256))


@pytest.mark.parametrize("rows,cols,chunk,S,G", [
    (64, 1024, 16384, 32, 8), (256, 4096, 65536, 128, 8), (37, 200, 1000, 64, 8),
    (17, 333, 999, 32, 1), (8, 512, 4096, 256, 8), (5, 104, 0, 96, 8)])
def test_encode_matches_oracle(eq, orc, rows, cols, chunk, S, G):
    w = synth.normal_with_outliers(rows, cols, 0.02, 0.01, 8.0, rows + S)
    osym, osc = orc.quantize(w, orc.E4M3)
    h = orc.rans_encode(osym, osc, orc.E4M3, chunk, S, G)
    t = eq.rans_encode_device(cuda(osym), cuda(osc.view(np.int16)), 1, chunk, S, G)
    torch.cuda.synchronize()
    assert np.array_equal(t.word_off.cpu().numpy().view(np.uint64), h.word_off)
    assert np.array_equal(t.states.cpu().numpy().view(np.uint32), h.states)
    total = int(h.word_off[-1])
    assert np.array_equal(t.words.cpu().numpy().view(np.uint16)[:total], h.words[:total])
    (out,), st = eq.decode([t])
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(eq.bf16_bits(out).ravel(), orc.dequant(osym, osc, orc.E4M3).ravel())


@pytest.mark.parametrize("rows,cols,chunk,S", [
    (64, 1024, 16384, 32), (256, 4096, 65536, 128), (37, 200, 1000, 64), (8, 512, 4096, 256),
    (5, 104, 0, 96)])
def test_encode_8bit_matches_oracle(eq, orc, rows, cols, chunk, S):
    w = synth.laplace_clipped(rows, cols, 0.01, 0.06, rows + S)
    osym, osc = orc.quantize(w, orc.INT8, synth.INT8_DIV_LAPLACE_8K)
    h = orc.rans_encode(osym, osc, orc.INT8, chunk, S, 8, prob_bits=8)
    t = eq.rans_encode_device(cuda(osym), cuda(osc.view(np.int16)), 2, chunk, S, 8, prob_bits=8)
    torch.cuda.synchronize()
    assert np.array_equal(t.word_off.cpu().numpy().view(np.uint64), h.word_off)
    assert np.array_equal(t.states.cpu().numpy().view(np.uint32), h.states)
    total = int(h.word_off[-1])
    assert np.array_equal(t.words.cpu().numpy().view(np.uint16)[:total], h.words[:total])
    (out,), st = eq.decode([t])
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(eq.bf16_bits(out).ravel(), orc.dequant(osym, osc, orc.INT8).ravel())


def test_full_pipeline_int8_workload(eq, orc):
    """fp32 weights on the GPU -> quantise -> histogram -> frequencies -> encode -> decode, in the
    workload's own table size."""
    wl = synth.WORKLOADS["int8_8k"]
    w = wl.tensors[0].generate(row_lo=0, row_hi=1024)
    sym, sc = eq.quantize_device(cuda(w), 2, wl.int8_div)
    t = eq.rans_encode_device(sym, sc, 2, wl.chunk_symbols, wl.streams, wl.run,
                              prob_bits=wl.prob_bits)
    osym, osc = orc.quantize(w, orc.INT8, wl.int8_div)
    h = orc.rans_encode(osym, osc, orc.INT8, wl.chunk_symbols, wl.streams, wl.run,
                        prob_bits=wl.prob_bits)
    assert np.array_equal(t.word_off.cpu().numpy().view(np.uint64), h.word_off)
    assert np.array_equal(t.states.cpu().numpy().view(np.uint32), h.states)
    (out,), st = eq.decode([t])
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(eq.bf16_bits(out).ravel(), orc.dequant(osym, osc, orc.INT8).ravel())


def test_single_symbol_and_missing_symbol(eq, orc):
    sym = np.full((4, 256), 0x38, np.uint8)
    sc = np.full(4, 0x3F80, np.uint16)
    t = eq.rans_encode_device(cuda(sym), cuda(sc.view(np.int16)), 1, 512, 32, 8)
    (out,), st = eq.decode([t])
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(t.word_off[-1].item()) == 0
    assert np.array_equal(eq.bf16_bits(out).ravel(), orc.dequant(sym, sc, 1).ravel())
    f = np.zeros(256, np.uint32)
    f[0x30] = 4096  # the table lacks the symbol actually present
    st = eq.new_status("cuda")
    eq.rans_encode_device(cuda(sym), cuda(sc.view(np.int16)), 1, 512, 32, 8, freqs=f, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & 4
