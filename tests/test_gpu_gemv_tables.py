"""GPU parity: eq_decode_gemv on 8- and 7-bit tables (the 7-bit ones through pair tables) against
the oracle's fp64 product of the decoded bf16 weights, within the GEMV bar of 1e-3 relative L2 and
held to 1e-5 as in the 12-bit tests: the 2-bit Int8 weight at full size, ragged shapes, CTAs whose
warps take several chunks in turn (CUDA-core and tensor-core paths), E4M3 symbols, one-symbol
tables, super weights, and a table whose size the descriptor does not match."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu
BAR = 1e-3
TIGHT = 1e-5


@pytest.fixture(scope="module")
def eq():
    import decoding_interleaved_rans_b200 as m
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    m.lib()
    return m


def rel_l2(y, ref):
    return float(np.linalg.norm(y - ref) / np.linalg.norm(ref))


def gemv(eq, h, x_bits):
    t = eq.DeviceRans.upload(h)
    x = torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).cuda().view(torch.bfloat16)
    y, st = eq.decode_gemv(t, x)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64), int(st.item())


def int8_syms(orc, rows, cols, seed):
    w = synth.laplace_clipped(rows, cols, 0.01, 0.06, seed)
    return orc.quantize(w, orc.INT8, synth.INT8_DIV_LAPLACE_8K)


@pytest.mark.parametrize("pb", [7, 8])
def test_int8_2bit_weight_full_size(eq, orc, pb):
    """The 8192 x 8192 Int8 weight of about 2 bits per parameter, one row per chunk (8192 warps'
    worth of chunks), batch 1, 4 and 16."""
    wl = synth.WORKLOADS["int8_8k"]
    spec = wl.tensors[0]
    sym, sc = orc.quantize(spec.generate(), orc.INT8, wl.int8_div)
    h = orc.rans_encode(sym, sc, orc.INT8, spec.cols, 32, 8, prob_bits=pb)
    wbf = orc.dequant(sym, sc, orc.INT8)
    for batch in (1, 4, 16):
        x = synth.activations(batch, spec.cols, 500 + pb, tensor=batch)
        y, st = gemv(eq, h, x)
        assert st == 0
        err = rel_l2(y, orc.gemv_f64(wbf, x))
        assert err <= BAR and err <= TIGHT, (pb, batch, err)


@pytest.mark.parametrize("pb", [7, 8])
@pytest.mark.parametrize("rows,cols,chunk_rows", [
    (1, 8, 1), (37, 200, 1), (50, 1024, 4), (9, 4096, 3), (64, 512, 2), (7, 13824, 1),
    (8192, 64, 1),    # 7-bit, batch < 8: more chunks than the SMs' warps, each warp loops
    (8192, 256, 1)])  # 7-bit, batch >= 8: more 16-chunk groups than CTA halves, each loops
@pytest.mark.parametrize("batch", [1, 3, 8, 16])
def test_shapes_and_batches(eq, orc, pb, rows, cols, chunk_rows, batch):
    sym, sc = int8_syms(orc, rows, cols, 510 + rows + cols)
    h = orc.rans_encode(sym, sc, orc.INT8, chunk_rows * cols, 32, 8, prob_bits=pb)
    x = synth.activations(batch, cols, 511)
    y, st = gemv(eq, h, x)
    assert st == 0
    assert rel_l2(y, orc.gemv_f64(orc.dequant(sym, sc, orc.INT8), x)) <= TIGHT


@pytest.mark.parametrize("pb", [7, 8])
def test_e4m3_symbols(eq, orc, pb):
    rng = np.random.default_rng(520 + pb)
    alphabet = rng.choice([s for s in range(256) if s & 0x7F != 0x7F], 100, replace=False)
    sym = rng.choice(alphabet.astype(np.uint8), (48, 1024)).astype(np.uint8)
    sc = synth.bf16_bits(rng.uniform(1e-3, 1.0, 48).astype(np.float32))
    h = orc.rans_encode(sym, sc, orc.E4M3, 2048, 32, 8, prob_bits=pb)
    for batch in (2, 8):
        x = synth.activations(batch, 1024, 521)
        y, st = gemv(eq, h, x)
        assert st == 0 and rel_l2(y, orc.gemv_f64(orc.dequant(sym, sc, orc.E4M3), x)) <= TIGHT


@pytest.mark.parametrize("pb", [7, 8])
@pytest.mark.parametrize("batch", [1, 8])
def test_single_symbol_table(eq, orc, pb, batch):
    sym = np.full((16, 256), 0x05, np.uint8)
    sc = np.full(16, 0x3F80, np.uint16)
    h = orc.rans_encode(sym, sc, orc.INT8, 256, 32, 8, prob_bits=pb)
    x = synth.activations(batch, 256, 530)
    y, st = gemv(eq, h, x)
    assert st == 0 and rel_l2(y, orc.gemv_f64(orc.dequant(sym, sc, orc.INT8), x)) <= TIGHT


@pytest.mark.parametrize("pb", [7, 8])
@pytest.mark.parametrize("batch", [1, 16])
def test_super_weights(eq, orc, pb, batch):
    rows, cols = 96, 2048
    w = synth.laplace_clipped(rows, cols, 0.01, 0.06, 540 + pb)
    synth.plant_super_weights(w, 10, 541)
    idx, val = orc.super_weights(w)
    sym, sc = orc.quantize_excluding(w, orc.INT8, synth.INT8_DIV_LAPLACE_8K, idx)
    h = orc.rans_encode(sym, sc, orc.INT8, cols, 32, 8, prob_bits=pb)
    h.patch_idx, h.patch_val = idx, val
    want = orc.patch_bf16(orc.dequant(sym, sc, orc.INT8), idx, val)
    x = synth.activations(batch, cols, 542, tensor=batch)
    y, st = gemv(eq, h, x)
    assert st == 0 and rel_l2(y, orc.gemv_f64(want.reshape(rows, cols), x)) <= TIGHT


@pytest.mark.parametrize("batch", [1, 8])
def test_table_of_another_size_is_reported(eq, orc, batch):
    """A 1 KiB 8-bit slot table under a 7-bit descriptor: the header is checked before the table
    is read, nothing past it is touched, and the launch reports the tensor."""
    sym, sc = int8_syms(orc, 64, 1024, 550)
    t = eq.DeviceRans.upload(orc.rans_encode(sym, sc, orc.INT8, 1024, 32, 8, prob_bits=7))
    small = torch.zeros(eq.table_bytes(eq.EQ_TABLE_RANS8_INT8), dtype=torch.uint8, device="cuda")
    eq.build_tables(eq.EQ_TABLE_RANS8_INT8, orc.rans_freqs(sym, 8), 8, small)
    t.tables = small
    x = torch.zeros(batch, 1024, dtype=torch.bfloat16, device="cuda")
    _, status = eq.decode_gemv(t, x)
    torch.cuda.synchronize()
    assert int(status.item()) & eq.EQ_DEV_CORRUPT_STATE


def test_corrupted_state_is_reported(eq, orc):
    sym, sc = int8_syms(orc, 64, 1024, 560)
    h = orc.rans_encode(sym, sc, orc.INT8, 1024, 32, 8, prob_bits=7)
    h.states = h.states.copy()
    h.states[40] ^= 0x1234
    x = synth.activations(4, 1024, 561)
    _, st = gemv(eq, h, x)
    assert st & 3
