"""The C-ABI library loads, exports every function its headers declare, and rejects bad
arguments on the host before touching a GPU (these calls fail validation, so they launch nothing
and run without a device)."""
import ctypes as C
import glob
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def eq():
    import decoding_interleaved_rans_b200 as m
    m.lib()
    return m


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        txt = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\b(eq_[a-z0-9_]+)\s*\(", txt))
    return sorted(names)


def test_every_declared_symbol_is_exported(eq):
    names = declared_functions()
    assert {"eq_build_tables", "eq_decode", "eq_decode_gemv", "eq_huff_bf16_decode"} <= set(names)
    L = eq.lib()
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(eq.EXPORTS)


def test_version_and_strings(eq):
    L = eq.lib()
    assert L.eq_abi_version() == 3
    for code in range(5):
        assert L.eq_status_string(code)
    assert eq.table_bytes(1) >= 4096 * 4 and eq.table_bytes(2) > 0 and eq.table_bytes(7) == 0
    # 7-bit pair tables, one kind per symbol format: 16384 entries of 8 bytes behind the header;
    # 8-bit slot tables likewise: 256 entries of 4 bytes
    assert eq.table_bytes(eq.EQ_TABLE_RANS_PAIR_E4M3) == eq.table_bytes(eq.EQ_TABLE_RANS_PAIR_INT8) \
        == 16 + 16384 * 8
    assert eq.table_bytes(eq.EQ_TABLE_RANS8_E4M3) == eq.table_bytes(eq.EQ_TABLE_RANS8_INT8) == 16 + 256 * 4


def test_build_tables_rejects_bad_input_on_host(eq):
    L = eq.lib()
    fake = C.c_void_p(1 << 20)  # never dereferenced: validation fails first
    bad_sum = (C.c_uint32 * 256)(*([16] * 255 + [15]))
    assert L.eq_build_tables(1, bad_sum, 12, fake, None) == 2
    ok = (C.c_uint32 * 256)(*([16] * 256))
    assert L.eq_build_tables(1, ok, 11, fake, None) == 3
    assert L.eq_build_tables(1, ok, 12, C.c_void_p((1 << 20) + 4), None) == 1  # misaligned
    too_long = (C.c_uint32 * 256)(*([33] + [0] * 255))
    assert L.eq_build_tables(2, too_long, 0, fake, None) == 2
    over_kraft = (C.c_uint32 * 256)(*([1, 1, 1] + [0] * 253))
    assert L.eq_build_tables(2, over_kraft, 0, fake, None) == 2
    # pair tables (both symbol formats) take 7-bit frequencies only
    seven = (C.c_uint32 * 256)(*([1] * 128 + [0] * 128))
    for kind in (eq.EQ_TABLE_RANS_PAIR_E4M3, eq.EQ_TABLE_RANS_PAIR_INT8):
        assert L.eq_build_tables(kind, ok, 12, fake, None) == 3
        assert L.eq_build_tables(kind, bad_sum, 7, fake, None) == 2
        assert L.eq_build_tables(kind, seven, 7, C.c_void_p((1 << 20) + 8), None) == 1
    # 8-bit slot tables (both formats) take 8-bit frequencies only; the 12-bit kind 12-bit ones
    eight = (C.c_uint32 * 256)(*([1] * 256))
    for kind in (eq.EQ_TABLE_RANS8_E4M3, eq.EQ_TABLE_RANS8_INT8):
        assert L.eq_build_tables(kind, ok, 12, fake, None) == 3
        assert L.eq_build_tables(kind, seven, 7, fake, None) == 3
    assert L.eq_build_tables(eq.EQ_TABLE_RANS, eight, 8, fake, None) == 3
    assert L.eq_build_tables(7, seven, 7, fake, None) == 1  # no such kind


def test_decode_rejects_bad_descriptors_on_host(eq):
    L = eq.lib()
    d = eq._lib.RansTensorDesc(eq._lib.EQ_ABI_VERSION, 1, 4, 64, 12, 256, 32, 8, 1, 1 << 20,
                               1 << 20, 1 << 20, 1 << 20, 1 << 20)
    out = (C.c_void_p * 1)(1 << 20)
    st = C.c_void_p(1 << 20)
    for field, val, code in [("version", 0, 1), ("symfmt", 3, 1), ("streams", 40, 3),
                             ("run", 2, 3), ("prob_bits", 10, 3), ("num_chunks", 2, 1),
                             ("chunk_symbols", 100, 1), ("words", (1 << 20) + 2, 1),
                             ("n_patch", 3, 1), ("n_patch", 1 << 40, 1), ("prob_bits", 8, 0)]:
        bad = eq._lib.RansTensorDesc.from_buffer_copy(d)
        setattr(bad, field, val)
        if code == 0:
            continue  # valid on the host; would launch
        assert L.eq_decode(C.byref(bad), 1, out, st, None) == code, field
    bad = eq._lib.RansTensorDesc.from_buffer_copy(d)
    bad.n_patch, bad.patch_idx, bad.patch_val = 2, (1 << 20) + 4, 1 << 20  # misaligned list
    assert L.eq_decode(C.byref(bad), 1, out, st, None) == 1
    assert L.eq_decode(C.byref(d), 1, out, None, None) == 1
    assert L.eq_decode(None, 0, None, None, None) == 0


def test_gemv_and_huff_reject_bad_input_on_host(eq):
    L = eq.lib()
    d = eq._lib.RansTensorDesc(eq._lib.EQ_ABI_VERSION, 1, 4, 64, 12, 100, 32, 8, 3, 1 << 20,
                               1 << 20, 1 << 20, 1 << 20, 1 << 20)  # chunks do not hold whole rows
    assert L.eq_decode_gemv(C.byref(d), C.c_void_p(1 << 20), 1, C.c_void_p(1 << 20),
                            C.c_void_p(1 << 20), None) in (1, 3)
    h = eq._lib.HuffTensorDesc(10, 30, 8, 256, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20)
    h.bytes_per_thread = 4
    assert L.eq_huff_bf16_decode(C.byref(h), C.c_void_p(1 << 20), C.c_void_p(1 << 20), None) in (1, 3)


def test_decode_from_host_rejects_bad_input_on_host(eq):
    """Argument checks before any copy or launch: no descriptor, a descriptor of another ABI
    version, missing host arrays, a word count below the last offset (read from the host
    offsets), a misaligned output."""
    import numpy as np
    L = eq.lib()
    fake = C.c_void_p(1 << 20)
    good = eq._lib.RansTensorDesc(eq._lib.EQ_ABI_VERSION, 2, 4, 64, 7, 64, 32, 8, 4, 1 << 20,
                                  1 << 20, 1 << 20, 1 << 20, 1 << 20)
    states = np.zeros(4 * 32, np.uint32)
    word_off = np.arange(5, dtype=np.uint64) * 8  # four substreams of 8 words
    words = np.zeros(32, np.uint16)
    scales = np.zeros(4, np.uint16)
    ptr = lambda a: C.c_void_p(a.ctypes.data)  # noqa: E731
    args = lambda d, st, wo, w, nw, sc, out: (C.byref(d) if d is not None else None, st, wo, w, nw,  # noqa: E731
                                              sc, 1, out, fake, None, None)
    assert L.eq_decode_from_host(*args(None, ptr(states), ptr(word_off), ptr(words), 32, ptr(scales), fake)) == 1
    bad = eq._lib.RansTensorDesc(eq._lib.EQ_ABI_VERSION + 1, 2, 4, 64, 7, 64, 32, 8, 4, 1 << 20,
                                 1 << 20, 1 << 20, 1 << 20, 1 << 20)
    assert L.eq_decode_from_host(*args(bad, ptr(states), ptr(word_off), ptr(words), 32, ptr(scales), fake)) == 1
    assert L.eq_decode_from_host(*args(good, None, ptr(word_off), ptr(words), 32, ptr(scales), fake)) == 1
    assert L.eq_decode_from_host(*args(good, ptr(states), ptr(word_off), ptr(words), 31, ptr(scales), fake)) == 1
    assert L.eq_decode_from_host(*args(good, ptr(states), ptr(word_off), ptr(words), 32, ptr(scales),
                                       C.c_void_p((1 << 20) + 2))) == 1


class _FakeDev:
    """Stands in for a device tensor: only its address is used, and only by host validation."""

    def __init__(self, n_elems):
        self._n = n_elems

    def data_ptr(self):
        return 1 << 24

    def numel(self):
        return self._n


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="launches would run on fake pointers; host-only check")
@pytest.mark.parametrize("chunk,streams,run", [(16384, 32, 8), (65536, 128, 8), (0, 64, 8),
                                               (999, 96, 1)])
def test_binding_descriptors_pass_host_validation(eq, orc, chunk, streams, run):
    """Descriptors built by the Python binding from a real container pass every host check; with
    no CUDA device the call then stops at the first CUDA query (EQ_ERR_CUDA), never earlier."""
    import synth
    w = synth.normal(40, 1024, 0.02, 3)
    sym, sc = orc.quantize(w, orc.E4M3)
    for h in (orc.rans_encode(sym, sc, 1, chunk, streams, run),
              eq.codec.rans_encode(sym, sc, 1, chunk, streams, run)):
        nchunks = (h.rows * h.cols + (chunk or h.cols) - 1) // (chunk or h.cols)
        t = eq.DeviceRans(h.rows, h.cols, h.symfmt, h.prob_bits, h.chunk_symbols, h.streams,
                          h.run, nchunks, *[_FakeDev(1) for _ in range(5)])
        assert len(h.word_off) == nchunks * (streams // 32) + 1
        d = t.desc()
        out = (C.c_void_p * 1)(1 << 24)
        assert eq.lib().eq_decode(C.byref(d), 1, out, C.c_void_p(1 << 24), None) == 4


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="launches would run on fake pointers; host-only check")
def test_binding_gemv_and_huff_descriptors_pass_host_validation(eq, orc):
    import synth
    wl = synth.WORKLOADS["mlp_13b"]
    w = synth.normal(8, 5120, 0.02, 4)
    sym, sc = orc.quantize(w, orc.E4M3)
    h = eq.codec.rans_encode(sym, sc, 1, wl.chunk_rows * 5120, wl.streams, wl.run)
    nchunks = (h.rows * h.cols) // h.chunk_symbols
    t = eq.DeviceRans(h.rows, h.cols, 1, 12, h.chunk_symbols, h.streams, h.run, nchunks,
                      *[_FakeDev(1) for _ in range(5)])
    d = t.desc()
    fake = C.c_void_p(1 << 24)
    assert eq.lib().eq_decode_gemv(C.byref(d), fake, 4, fake, fake, None) == 4
    hb = eq.codec.huff_encode(synth.bf16_normal(4, 4096, 0.015, 5))
    th = eq.DeviceHuff(hb.n, hb.total_bits, 8, hb.threads_per_block,
                       *[_FakeDev(1) for _ in range(5)])
    dh = th.desc()
    assert eq.lib().eq_huff_bf16_decode(C.byref(dh), fake, fake, None) == 4
