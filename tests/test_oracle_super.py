"""Pins for the oracle's super-weight exclusion ("Float8@2bits" summary, "Manejo de Pesos
Superiores": with an Int8 base, extreme outliers are kept out of the entropy optimisation so they
do not crush their channel).  Reading: |w| > tau * rms(w) marks a super weight; it is stored
exactly (bf16) and left out of its row's AbsMax scale; its symbol is 0; decoding writes it back.
Checked against numpy/torch recomputations and against the collapse the pages describe."""
import numpy as np
import pytest

import synth

TAU = 20.0


def planted(rows=256, cols=2048, n=6, seed=3):
    w = synth.laplace_clipped(rows, cols, 0.01, 0.06, seed)
    pos = synth.plant_super_weights(w, n, seed)
    return w, pos


def test_detection_matches_numpy_threshold(orc):
    w, pos = planted()
    idx, val = orc.super_weights(w, TAU)
    w64 = w.astype(np.float64)
    limit = TAU * np.sqrt(np.mean(w64 * w64))
    expect = np.nonzero(np.abs(w64.ravel()) > limit)[0]
    assert np.array_equal(idx, expect.astype(np.uint64))
    assert idx.tolist() == pos  # exactly the planted ones: the clipped Laplace body stays below
    assert np.array_equal(val, synth.bf16_bits(w.ravel()[expect]))
    assert np.all(np.diff(idx.astype(np.int64)) > 0)


def test_no_super_weights_in_plain_tensors(orc):
    for w in (synth.laplace_clipped(64, 1024, 0.01, 0.06, 4), synth.normal(64, 1024, 0.02, 5)):
        idx, _ = orc.super_weights(w, TAU)
        assert idx.size == 0


def test_excluded_rows_keep_their_own_scale(orc):
    w, pos = planted()
    idx, _ = orc.super_weights(w, TAU)
    div = synth.INT8_DIV_LAPLACE_8K
    sym, sc = orc.quantize_excluding(w, orc.INT8, div, idx)
    plain_sym, plain_sc = orc.quantize(w, orc.INT8, div)
    rows_sw = sorted({p // w.shape[1] for p in pos})
    mask = np.zeros(w.size, bool)
    mask[idx.astype(np.int64)] = True
    mask = mask.reshape(w.shape)
    for r in range(w.shape[0]):
        if r in rows_sw:
            others = np.abs(w[r][~mask[r]]).max()
            assert sc[r] == synth.bf16_bits(np.array([np.float32(others) / np.float32(div)]))[0]
            assert (sym[r][mask[r]] == 0).all()
        else:
            assert sc[r] == plain_sc[r] and np.array_equal(sym[r], plain_sym[r])


def test_exclusion_avoids_the_collapse(orc):
    """Without exclusion a row holding a super weight quantises almost every other weight to 0;
    with it, the row looks like the others, and its reconstruction error drops by far."""
    w, pos = planted()
    cols = w.shape[1]
    div = synth.INT8_DIV_LAPLACE_8K
    idx, val = orc.super_weights(w, TAU)
    sym_p, sc_p = orc.quantize(w, orc.INT8, div)
    sym_x, sc_x = orc.quantize_excluding(w, orc.INT8, div, idx)
    zero_avg = float((sym_x == 0).mean())
    f32 = lambda b: orc.bf16_to_f32(b).astype(np.float64)  # noqa: E731
    rec_p = f32(orc.dequant(sym_p, sc_p, orc.INT8))
    rec_x = f32(orc.patch_bf16(orc.dequant(sym_x, sc_x, orc.INT8), idx, val))
    def err(rec, r, keep):  # relative error over the row's ordinary weights
        return np.linalg.norm(rec[r][keep] - w[r][keep]) / np.linalg.norm(w[r][keep])

    all_cols = np.ones(cols, bool)
    typical = np.median([err(rec_x, r, all_cols) for r in range(0, w.shape[0], 17)])
    for p in pos:
        r = p // cols
        keep = np.arange(cols) != p % cols
        assert (sym_p[r] == 0).mean() > 0.95
        assert abs((sym_x[r] == 0).mean() - zero_avg) < 0.05
        assert err(rec_p, r, keep) > 0.95                 # the channel collapsed to zero
        assert err(rec_x, r, keep) < 1.5 * typical        # as good as any other row
        assert rec_x[r][p % cols] == f32(synth.bf16_bits(w[r][p % cols:p % cols + 1]))[0]


@pytest.mark.parametrize("prob_bits", [12, 8])
def test_rans_round_trip_with_patch(orc, prob_bits):
    w, pos = planted(rows=128, cols=4096)
    idx, val = orc.super_weights(w, TAU)
    sym, sc = orc.quantize_excluding(w, orc.INT8, synth.INT8_DIV_LAPLACE_8K, idx)
    t = orc.rans_encode(sym, sc, orc.INT8, 65536, 128, 8, prob_bits=prob_bits)
    t.patch_idx, t.patch_val = idx, val
    rc, out = orc.rans_decode_bf16(t, threads=4)
    assert rc == 0
    want = orc.patch_bf16(orc.dequant(sym, sc, orc.INT8), idx, val).ravel()
    assert np.array_equal(out, want)
    assert np.array_equal(out[idx.astype(np.int64)], synth.bf16_bits(w.ravel()[idx.astype(np.int64)]))
