"""GPU parity for 7-bit rANS tables decoded through pair tables (one lookup per pair of steps):
eq_decode against the oracle, bit for bit, on the Int8 workload at full size, many layouts, warps
that decode several units in turn, E4M3 symbols, one-symbol tables, launches mixing table sizes,
and corrupted or mismatched inputs."""
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


@pytest.mark.parametrize("streams", [None, 128, 96])
def test_int8_full_size(eq, orc, streams):
    """The bench weight in the bench's layout, and with 128 / 96 streams per chunk."""
    wl = synth.WORKLOADS["int8_8k"]
    sym, sc = orc.quantize(wl.tensors[0].generate(), orc.INT8, wl.int8_div)
    h = orc.rans_encode(sym, sc, orc.INT8, wl.chunk_symbols, streams or wl.streams, wl.run, prob_bits=7)
    (out,), st = run_decode(eq, [h])
    assert st == 0 and np.array_equal(out, orc.dequant(sym, sc, orc.INT8).ravel())


@pytest.mark.parametrize("streams", [32, 64, 96, 128, 192, 256, 1024])
def test_layouts(eq, orc, streams):
    sym, sc = int8_syms(orc, 512, 2048, 400 + streams)
    h = orc.rans_encode(sym, sc, orc.INT8, 65536 * (1 + streams // 256), streams, 8, prob_bits=7)
    (out,), st = run_decode(eq, [h])
    assert st == 0 and np.array_equal(out, orc.dequant(sym, sc, orc.INT8).ravel())


@pytest.mark.parametrize("rows,cols,chunk,streams", [
    (1, 8, 8, 32), (3, 200, 1000, 32), (37, 200, 7400, 64), (5, 104, 104, 128),
    (9, 4096, 4104, 32), (1024, 8192, 1024, 32)])  # the last: ~8 units per warp slot
def test_ragged_shapes_and_unit_loops(eq, orc, rows, cols, chunk, streams):
    sym, sc = int8_syms(orc, rows, cols, 410 + rows)
    h = orc.rans_encode(sym, sc, orc.INT8, chunk, streams, 8, prob_bits=7)
    (out,), st = run_decode(eq, [h])
    assert st == 0 and np.array_equal(out, orc.dequant(sym, sc, orc.INT8).ravel())


@pytest.mark.parametrize("streams", [32, 64])
def test_e4m3_symbols_and_nan_codes(eq, orc, streams):
    rng = np.random.default_rng(420)
    alphabet = rng.choice(256, 120, replace=False).astype(np.uint8)
    alphabet[:2] = [0x7F, 0xFF]  # NaN codes decode to the signed quiet NaN
    sym = rng.choice(alphabet, (64, 1024)).astype(np.uint8)
    sc = synth.bf16_bits(rng.uniform(1e-3, 2.0, 64).astype(np.float32))
    h = orc.rans_encode(sym, sc, orc.E4M3, 16384, streams, 8, prob_bits=7)
    (out,), st = run_decode(eq, [h])
    assert st == 0 and np.array_equal(out, orc.dequant(sym, sc, orc.E4M3).ravel())


@pytest.mark.parametrize("streams", [32, 64])
def test_single_symbol_table(eq, orc, streams):
    sym = np.full((16, 256), 0x03, np.uint8)
    sc = np.full(16, 0x3F80, np.uint16)
    h = orc.rans_encode(sym, sc, orc.INT8, 1024, streams, 8, prob_bits=7)
    (out,), st = run_decode(eq, [h])
    assert st == 0 and np.array_equal(out, orc.dequant(sym, sc, orc.INT8).ravel())


def test_mixed_table_sizes_in_one_call(eq, orc):
    hosts, want = [], []
    for i, (pb, r, c, S) in enumerate([(7, 100, 800, 64), (8, 64, 4096, 128), (12, 33, 512, 32),
                                       (7, 256, 2048, 128), (7, 8, 64, 32)]):
        sym, sc = int8_syms(orc, r, c, 430 + i)
        hosts.append(orc.rans_encode(sym, sc, orc.INT8, 8000 if i == 0 else 65536, S, 8,
                                     prob_bits=pb))
        want.append(orc.dequant(sym, sc, orc.INT8).ravel())
    outs, st = run_decode(eq, hosts)
    assert st == 0
    for o, e in zip(outs, want):
        assert np.array_equal(o, e)


def test_corruption_and_mismatched_tables(eq, orc):
    sym, sc = int8_syms(orc, 64, 1024, 440)
    h = orc.rans_encode(sym, sc, orc.INT8, 16384, 32, 8, prob_bits=7)
    h.states = h.states.copy()
    h.states[40] ^= 0x1234
    assert run_decode(eq, [h])[1] & 3
    # a 16 KiB slot table under a 7-bit descriptor: the header is checked before the table is
    # read, nothing past the table is touched, and the tensor is reported
    h = orc.rans_encode(sym, sc, orc.INT8, 16384, 32, 8, prob_bits=7)
    t = eq.DeviceRans.upload(h)
    small = torch.zeros(eq.table_bytes(eq.EQ_TABLE_RANS8_INT8), dtype=torch.uint8, device="cuda")
    eq.build_tables(eq.EQ_TABLE_RANS8_INT8, orc.rans_freqs(sym, 8), 8, small)
    t.tables = small
    _, status = eq.decode([t])
    torch.cuda.synchronize()
    assert int(status.item()) & eq.EQ_DEV_CORRUPT_STATE


def test_device_encoder_matches_oracle(eq, orc):
    sym, sc = int8_syms(orc, 256, 4096, 450)
    h = orc.rans_encode(sym, sc, orc.INT8, 65536, 128, 8, prob_bits=7)
    t = eq.rans_encode_device(torch.from_numpy(sym).cuda(), torch.from_numpy(sc.view(np.int16)).cuda(),
                              2, 65536, 128, 8, prob_bits=7)
    torch.cuda.synchronize()
    assert np.array_equal(t.word_off.cpu().numpy().view(np.uint64), h.word_off)
    assert np.array_equal(t.states.cpu().numpy().view(np.uint32), h.states)
    total = int(h.word_off[-1])
    assert np.array_equal(t.words.cpu().numpy().view(np.uint16)[:total], h.words[:total])
    (out,), st = eq.decode([t])
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(eq.bf16_bits(out).ravel(), orc.dequant(sym, sc, orc.INT8).ravel())
