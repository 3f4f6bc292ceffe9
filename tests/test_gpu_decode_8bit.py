"""GPU parity for 8-bit rANS tables (streams renormalise after every second step): eq_decode
against the oracle, bit for bit, on the Int8 workload, ragged shapes, every byte value, one-symbol
tables, launches that mix 8- and 12-bit tensors, and corrupted streams."""
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


def run_decode(eq, hosts):
    dev = [eq.DeviceRans.upload(h) for h in hosts]
    outs, status = eq.decode(dev)
    torch.cuda.synchronize()
    return [eq.bf16_bits(o).ravel() for o in outs], int(status.item())


def int8_syms(orc, rows, cols, seed):
    w = synth.laplace_clipped(rows, cols, 0.01, 0.06, seed)
    return orc.quantize(w, orc.INT8, synth.INT8_DIV_LAPLACE_8K)


@pytest.mark.parametrize("streams", [32, 64, 128, 256])
def test_int8_layouts(eq, orc, streams):
    sym, sc = int8_syms(orc, 512, 2048, 80)
    h = orc.rans_encode(sym, sc, orc.INT8, 65536, streams, 8, prob_bits=8)
    (out,), st = run_decode(eq, [h])
    assert st == 0 and np.array_equal(out, orc.dequant(sym, sc, orc.INT8).ravel())


@pytest.mark.parametrize("rows,cols,chunk,streams", [
    (1, 8, 8, 32), (3, 200, 1000, 32), (37, 200, 7400, 64), (5, 104, 104, 128),
    (64, 1024, 65536, 256), (9, 4096, 4104, 32)])
def test_ragged_shapes(eq, orc, rows, cols, chunk, streams):
    sym, sc = int8_syms(orc, rows, cols, 81 + rows)
    h = orc.rans_encode(sym, sc, orc.INT8, chunk, streams, 8, prob_bits=8)
    (out,), st = run_decode(eq, [h])
    assert st == 0 and np.array_equal(out, orc.dequant(sym, sc, orc.INT8).ravel())


def test_every_byte_value_both_formats(eq, orc):
    """All 256 bytes present, so the 8-bit table is the uniform one (f = 1 each)."""
    rng = np.random.default_rng(82)
    for fmt in (orc.E4M3, orc.INT8):
        sym = rng.integers(0, 256, (64, 512), dtype=np.uint8)
        sc = synth.bf16_bits(rng.uniform(1e-4, 2.0, 64).astype(np.float32))
        sc[1] = 0xBC00
        h = orc.rans_encode(sym, sc, fmt, 4096, 64, 8, prob_bits=8)
        assert (h.freqs == 1).all()
        (out,), st = run_decode(eq, [h])
        assert st == 0 and np.array_equal(out, orc.dequant(sym, sc, fmt).ravel())


def test_e4m3_normal_weights(eq, orc):
    wl = synth.WORKLOADS["e4m3_1k"]
    sym, sc = orc.quantize(wl.tensors[0].generate(), orc.E4M3)
    h = orc.rans_encode(sym, sc, orc.E4M3, 16384, 32, 8, prob_bits=8)
    (out,), st = run_decode(eq, [h])
    assert st == 0 and np.array_equal(out, orc.dequant(sym, sc, orc.E4M3).ravel())


def test_single_symbol_table(eq, orc):
    sym = np.full((16, 256), 0x02, np.uint8)
    sc = np.full(16, 0x3F80, np.uint16)
    h = orc.rans_encode(sym, sc, orc.INT8, 1024, 32, 8, prob_bits=8)
    assert h.word_off[-1] == 0
    (out,), st = run_decode(eq, [h])
    assert st == 0 and np.array_equal(out, orc.dequant(sym, sc, orc.INT8).ravel())


def test_mixed_table_sizes_in_one_call(eq, orc):
    hosts, want = [], []
    for i, (fmt, pb, r, c, chunk, S, G) in enumerate([
            (orc.INT8, 8, 100, 800, 8000, 64, 8), (orc.INT8, 12, 64, 4096, 65536, 128, 8),
            (orc.E4M3, 12, 33, 512, 512, 32, 1), (orc.E4M3, 8, 128, 1024, 16384, 32, 8),
            (orc.INT8, 8, 256, 2048, 65536, 128, 8)]):
        w = synth.laplace_clipped(r, c, 0.01, 0.06, 90 + i) if fmt == orc.INT8 else \
            synth.normal(r, c, 0.02, 90 + i)
        sym, sc = orc.quantize(w, fmt, synth.INT8_DIV_LAPLACE_8K)
        hosts.append(orc.rans_encode(sym, sc, fmt, chunk, S, G, prob_bits=pb))
        want.append(orc.dequant(sym, sc, fmt).ravel())
    outs, st = run_decode(eq, hosts)
    assert st == 0
    for o, e in zip(outs, want):
        assert np.array_equal(o, e)


def test_corruption_and_mismatched_table(eq, orc):
    sym, sc = int8_syms(orc, 64, 1024, 95)
    h = orc.rans_encode(sym, sc, orc.INT8, 16384, 32, 8, prob_bits=8)
    h.states = h.states.copy()
    h.states[40] ^= 0x1234
    assert run_decode(eq, [h])[1] & 3
    h = orc.rans_encode(sym, sc, orc.INT8, 16384, 32, 8, prob_bits=8)
    h.word_off = h.word_off.copy()
    h.word_off[1:] -= 1
    h.words = np.concatenate([h.words[:int(h.word_off[1])], h.words[int(h.word_off[1]) + 1:]])
    assert run_decode(eq, [h])[1] & 3
    # a 12-bit table, or an 8-bit one of the other symbol format, under an 8-bit Int8
    # descriptor: caught on the device, nothing decoded from it
    h = orc.rans_encode(sym, sc, orc.INT8, 16384, 32, 8, prob_bits=8)
    for kind, pb in ((eq.EQ_TABLE_RANS, 12), (eq.EQ_TABLE_RANS8_E4M3, 8)):
        t = eq.DeviceRans.upload(h)
        t.tables = torch.zeros(eq.table_bytes(kind), dtype=torch.uint8, device="cuda")
        eq.build_tables(kind, orc.rans_freqs(sym, pb), pb, t.tables)
        outs, status = eq.decode([t])
        torch.cuda.synchronize()
        assert int(status.item()) & eq.EQ_DEV_CORRUPT_STATE


def test_8bit_needs_runs_of_8(eq, orc):
    sym, sc = int8_syms(orc, 8, 64, 96)
    h = orc.rans_encode(sym, sc, orc.INT8, 512, 32, 1, prob_bits=8)
    with pytest.raises(eq.EqError):
        run_decode(eq, [h])
