"""GPU parity for the tables that carry the symbols' values as bf16 (8-bit slot tables, 7-bit pair
tables), so that the decoder dequantises two symbols with one bf16x2 multiply by the row scale.
Checked exhaustively against the oracle's dequantisation (the exact product in binary64, one
rounding to bf16): every symbol code of both formats, the E4M3 NaN codes included, times every
finite bf16 scale, so subnormal scales and products and overflow to infinity are all covered; and
a table built for the other symbol format is reported, by the decoder and by the fused GEMV."""
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


def finite_bf16_scales() -> np.ndarray:
    b = np.arange(65536, dtype=np.uint32)
    return b[(b & 0x7F80) != 0x7F80].astype(np.uint16)  # exponent field not all ones


@pytest.mark.parametrize("pb,half", [(7, 0), (7, 1), (8, None)])
@pytest.mark.parametrize("fmt", [1, 2])
def test_every_code_times_every_finite_scale(eq, orc, fmt, pb, half):
    """Row r holds the codes (7-bit tables: one half of the byte range, 8-bit ones: all 256),
    rotated by r, and has the r-th finite bf16 pattern as its scale: every (code, scale) pair
    occurs once.  The codes are equally frequent, so each owns one slot of the table."""
    sc = finite_bf16_scales()
    rows = sc.size
    k = 1 << pb
    codes = np.arange(k, dtype=np.uint16) + (128 * half if half else 0)
    sym = codes[(np.arange(k)[None, :] + np.arange(rows)[:, None]) % k].astype(np.uint8)
    h = orc.rans_encode(sym, sc, fmt, 16384, 32, 8, prob_bits=pb)
    assert np.all(h.freqs[codes] == 1)
    t = eq.DeviceRans.upload(h)
    (out,), st = eq.decode([t])
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = eq.bf16_bits(out)
    want = orc.dequant(sym, sc, fmt)
    bad = np.argwhere(got != want)
    assert bad.size == 0, [(int(sym[r, c]), hex(int(sc[r])), hex(int(got[r, c])), hex(int(want[r, c])))
                           for r, c in bad[:8]]


@pytest.mark.parametrize("pb", [7, 8])
def test_table_of_the_other_format_is_reported(eq, orc, pb):
    w = synth.laplace_clipped(64, 1024, 0.01, 0.06, 610)
    sym, sc = orc.quantize(w, orc.INT8, synth.INT8_DIV_LAPLACE_8K)
    t = eq.DeviceRans.upload(orc.rans_encode(sym, sc, orc.INT8, 1024, 32, 8, prob_bits=pb))
    kind = eq.EQ_TABLE_RANS_PAIR_E4M3 if pb == 7 else eq.EQ_TABLE_RANS8_E4M3
    other = torch.zeros(eq.table_bytes(kind), dtype=torch.uint8, device="cuda")
    eq.build_tables(kind, orc.rans_freqs(sym, pb), pb, other)
    t.tables = other
    _, status = eq.decode([t])
    torch.cuda.synchronize()
    assert int(status.item()) & eq.EQ_DEV_CORRUPT_STATE
    for batch in (1, 8):
        x = torch.zeros(batch, 1024, dtype=torch.bfloat16, device="cuda")
        _, status = eq.decode_gemv(t, x)
        torch.cuda.synchronize()
        assert int(status.item()) & eq.EQ_DEV_CORRUPT_STATE


def finite_e4m3_codes() -> np.ndarray:
    c = np.arange(256, dtype=np.uint16)
    return c[(c & 0x7F) != 0x7F]  # 254 codes: all but the two NaN patterns


@pytest.mark.parametrize("case", ["e4m3_finite_rows", "e4m3_finite_ragged", "e4m3_with_nan",
                                  "int8"])
def test_12bit_every_code_times_every_finite_scale(eq, orc, case):
    """12-bit tables carry no values: E4M3 tables without NaN codes take the exponent-offset
    dequantisation (the code's bits placed in a bf16 scaled by 2^-120, times scale * 2^120),
    which the decoder chooses per unit of rows only while every row scale is below 2^8 in
    magnitude; other units, tables holding a NaN code and Int8 take the per-symbol product.
    Rows are sorted by scale bit pattern, so units of small scales, units of large scales and
    units holding both all occur, and every (code, finite scale) pair is compared with the
    oracle's one-rounding product.  The 256-column cases take the whole-row loop, the 264-column
    one (chunks cutting rows) the general loop."""
    sc = finite_bf16_scales()
    rows = sc.size
    fmt = orc.INT8 if case == "int8" else orc.E4M3
    if case == "e4m3_finite_ragged":  # 264 columns: a multiple of the run, not of a round
        codes = np.concatenate([finite_e4m3_codes(), finite_e4m3_codes()[:10]])
    elif case == "e4m3_finite_rows":
        codes = np.concatenate([finite_e4m3_codes(), np.array([0x00, 0x80], np.uint16)])
    else:
        codes = np.arange(256, dtype=np.uint16)
    k = codes.size
    sym = codes[(np.arange(k)[None, :] + np.arange(rows)[:, None]) % k].astype(np.uint8)
    h = orc.rans_encode(sym, sc, fmt, 16384, 32, 8, prob_bits=12)
    t = eq.DeviceRans.upload(h)
    (out,), st = eq.decode([t])
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = eq.bf16_bits(out)
    want = orc.dequant(sym, sc, fmt)
    bad = np.argwhere(got != want)
    assert bad.size == 0, [(int(sym[r, c]), hex(int(sc[r])), hex(int(got[r, c])), hex(int(want[r, c])))
                           for r, c in bad[:8]]


@pytest.mark.parametrize("chunk_rows", [1, 4])
def test_12bit_e4m3_gemv_one_hot_every_code_times_every_finite_scale(eq, orc, chunk_rows):
    """The fused GEMV's exponent-offset path (12-bit E4M3 tables without NaN codes, per row while
    the scale is below 2^8 in magnitude) against the oracle's dequantisation: with one-hot
    activations each output is one decoded weight (every other product is an exact zero and one
    is the weight times one), so over all columns every (code, finite scale) pair is compared
    exactly, at batch 1 (one row per chunk: the one-row loop), 4 and 16 (tensor-core kernel).
    Rows whose products overflow to infinity turn into NaN through infinity times zero; the
    oracle's dequantisation of those rows holds an infinity, and the kernel's outputs there are NaN."""
    sc = finite_bf16_scales()
    rows = sc.size
    codes = np.concatenate([finite_e4m3_codes(), np.array([0x00, 0x80], np.uint16)])
    cols = codes.size
    sym = codes[(np.arange(cols)[None, :] + np.arange(rows)[:, None]) % cols].astype(np.uint8)
    h = orc.rans_encode(sym, sc, orc.E4M3, cols * chunk_rows, 32, 8, prob_bits=12)
    t = eq.DeviceRans.upload(h)
    want = orc.dequant(sym, sc, orc.E4M3).astype(np.uint32) << 16
    wantf = want.view(np.float32)
    finite = np.isfinite(wantf).all(axis=1)
    assert 0 < finite.sum() < rows
    for batch in (1, 4, 16):
        for j0 in range(0, cols, batch):
            x = torch.zeros(batch, cols, dtype=torch.bfloat16, device="cuda")
            x[torch.arange(batch), j0 + torch.arange(batch)] = 1.0
            y, st = eq.decode_gemv(t, x)
            torch.cuda.synchronize()
            assert int(st.item()) == 0
            y = y.cpu().numpy()
            ref = wantf[:, j0:j0 + batch].T
            ok = np.equal(y[:, finite], ref[:, finite])
            assert ok.all(), (batch, j0, np.argwhere(~ok)[:4])
            assert np.isnan(y[:, ~finite]).all(), (batch, j0)
