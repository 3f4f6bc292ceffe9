"""GPU parity for eq_decode_from_host: a coded weight decoded straight from pinned host memory, its
arrays copied piece by piece (runs of whole chunks covering whole rows) while the pieces already
copied decode.  The device container is cleared first, so every array the decoder reads must
have been copied; the output must equal the oracle's bit for bit for any number of pieces, chunk
sizes that do or do not end on row boundaries, both symbol formats and table sizes, super
weights (decoded in one piece), and repeated calls on the same container."""
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


def streamed(eq, h, pieces, repeats=1):
    t = eq.DeviceRans.upload(h)
    for a in (t.states, t.word_off, t.words, t.scales):
        a.zero_()
    src = eq.PinnedRans.from_host(h)
    out = torch.empty(h.rows, h.cols, dtype=torch.bfloat16, device="cuda")
    for _ in range(repeats):
        out.fill_(7.0)
        _, st = eq.decode_from_host(t, src, out, pieces=pieces)
        torch.cuda.synchronize()
        yield eq.bf16_bits(out).ravel(), int(st.item())


@pytest.mark.parametrize("pieces", [1, 2, 3, 4, 7])
def test_int8_7bit(eq, orc, pieces):
    w = synth.laplace_clipped(1024, 8192, 0.01, 0.06, 700)
    sym, sc = orc.quantize(w, orc.INT8, synth.INT8_DIV_LAPLACE_8K)
    h = orc.rans_encode(sym, sc, orc.INT8, 65536, 128, 8, prob_bits=7)
    want = orc.dequant(sym, sc, orc.INT8).ravel()
    for got, st in streamed(eq, h, pieces, repeats=2):
        assert st == 0 and np.array_equal(got, want)


@pytest.mark.parametrize("rows,cols,chunk,streams,run,pb", [
    (300, 304, 1000, 32, 8, 12),   # every 38th chunk ends on a row boundary
    (37, 200, 999, 64, 1, 12),     # chunks never end on one before the last: one piece
    (257, 512, 4096, 64, 8, 8),    # a partial last chunk
])
def test_e4m3_layouts(eq, orc, rows, cols, chunk, streams, run, pb):
    w = synth.normal(rows, cols, 0.02, 710 + rows)
    sym, sc = orc.quantize(w, orc.E4M3)
    h = orc.rans_encode(sym, sc, orc.E4M3, chunk, streams, run, prob_bits=pb)
    want = orc.dequant(sym, sc, orc.E4M3).ravel()
    for pieces in (1, 3, 5):
        for got, st in streamed(eq, h, pieces):
            assert st == 0 and np.array_equal(got, want), pieces


def test_super_weights_decode_in_one_piece(eq, orc):
    rows, cols = 256, 2048
    w = synth.laplace_clipped(rows, cols, 0.01, 0.06, 720)
    synth.plant_super_weights(w, 5, 721)
    idx, val = orc.super_weights(w)
    sym, sc = orc.quantize_excluding(w, orc.INT8, synth.INT8_DIV_LAPLACE_8K, idx)
    h = orc.rans_encode(sym, sc, orc.INT8, 16384, 64, 8, prob_bits=7)
    h.patch_idx, h.patch_val = idx, val
    want = orc.patch_bf16(orc.dequant(sym, sc, orc.INT8), idx, val).ravel()
    for got, st in streamed(eq, h, 4):
        assert st == 0 and np.array_equal(got, want)


def test_host_arguments_checked_before_anything_runs(eq, orc):
    w = synth.laplace_clipped(64, 1024, 0.01, 0.06, 730)
    sym, sc = orc.quantize(w, orc.INT8, synth.INT8_DIV_LAPLACE_8K)
    h = orc.rans_encode(sym, sc, orc.INT8, 16384, 64, 8, prob_bits=7)
    t = eq.DeviceRans.upload(h)
    src = eq.PinnedRans.from_host(h)
    out = torch.empty(64, 1024, dtype=torch.bfloat16, device="cuda")
    import ctypes as C
    L = eq.lib()
    d = t.desc()
    st = eq.new_status("cuda")
    cur = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    # a word count below the last offset, and a null host array: rejected on the host
    assert L.eq_decode_from_host(C.byref(d), C.c_void_p(src.states.data_ptr()), C.c_void_p(src.word_off.data_ptr()),
                                 C.c_void_p(src.words.data_ptr()), 1, C.c_void_p(src.scales.data_ptr()), 2,
                                 C.c_void_p(out.data_ptr()), C.c_void_p(st.data_ptr()), cur, cur) == 1
    assert L.eq_decode_from_host(C.byref(d), None, C.c_void_p(src.word_off.data_ptr()),
                                 C.c_void_p(src.words.data_ptr()), src.words.numel(),
                                 C.c_void_p(src.scales.data_ptr()), 2, C.c_void_p(out.data_ptr()),
                                 C.c_void_p(st.data_ptr()), cur, cur) == 1
    # copy_stream == stream: nothing overlaps, the result is the same
    _, st2 = eq.decode_from_host(t, src, out, pieces=3, copy_stream=torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    assert np.array_equal(eq.bf16_bits(out).ravel(), orc.dequant(sym, sc, orc.INT8).ravel())
