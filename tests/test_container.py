"""On-disk coded tensors: the library's writer and reader round-trip every array, and the
oracle's own reader (written separately from the format description) decodes the files to the
original weights."""
import os

import numpy as np
import pytest

import synth


@pytest.fixture(scope="module")
def eq():
    import decoding_interleaved_rans_b200 as m
    m.lib()
    return m


def test_rans_file_round_trip(eq, orc, tmp_path):
    w = synth.laplace_clipped(64, 1024, 0.01, 0.06, 3)
    synth.plant_super_weights(w, 3, 3)
    idx, val = eq.codec.super_weights(w)
    sym, sc = eq.codec.quantize_excluding(w, 2, synth.INT8_DIV_LAPLACE_8K, idx)
    for pb in (7, 8, 12):
        h = eq.codec.rans_encode(sym, sc, 2, 65536, 128, 8, prob_bits=pb)
        h.patch_idx, h.patch_val = idx, val
        p = os.path.join(tmp_path, f"w{pb}.eqrt")
        eq.codec.save(p, h)
        g = eq.codec.load(p)
        assert type(g) is type(h) and g.prob_bits == pb
        for f in ("freqs", "states", "word_off", "words", "scales", "patch_idx", "patch_val"):
            assert np.array_equal(getattr(g, f), getattr(h, f)), f
        o = orc.load_container(p)
        rc, out = orc.rans_decode_bf16(o, threads=2)
        assert rc == 0
        want = orc.patch_bf16(orc.dequant(sym, sc, orc.INT8), idx, val).ravel()
        assert np.array_equal(out, want)


def test_huffman_files(eq, orc, tmp_path):
    wb = synth.bf16_normal(16, 4096, 0.015, 5)
    h = eq.codec.huff_encode(wb)
    p = os.path.join(tmp_path, "w.eqhf")
    eq.codec.save(p, h)
    rc, out = orc.huff_decode_bf16(orc.load_container(p))
    assert rc == 0 and np.array_equal(out, wb.ravel())
    g = eq.codec.load(p)
    assert g.total_bits == h.total_bits and np.array_equal(g.enc_exp, h.enc_exp)
    w = synth.normal(32, 1024, 0.02, 6)
    hi = eq.codec.entrollm_encode(w, 4)
    p = os.path.join(tmp_path, "w.eqhi")
    eq.codec.save(p, hi)
    rc, vals = orc.entrollm_decode_bf16(orc.load_container(p))
    sym, sc, z, _ = orc.entrollm_quantize(w, 4)
    assert rc == 0 and np.array_equal(vals, orc.intq_dequant(sym, sc, z).ravel())


def test_bad_files_are_refused(eq, tmp_path):
    p = os.path.join(tmp_path, "bad")
    with open(p, "wb") as f:
        f.write(b"NOPE" + bytes(12))
    with pytest.raises(ValueError):
        eq.codec.load(p)
    h = eq.codec.rans_encode(np.zeros((2, 8), np.uint8), np.full(2, 0x3F80, np.uint16), 2, 0, 32, 8)
    eq.codec.save(p, h)
    raw = bytearray(open(p, "rb").read())
    raw[4] = 9  # a future version
    open(p, "wb").write(bytes(raw))
    with pytest.raises(ValueError):
        eq.codec.load(p)
