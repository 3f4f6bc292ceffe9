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
