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
    assert L.eq_abi_version() == 1
    for code in range(5):
        assert L.eq_status_string(code)
    assert eq.table_bytes(1) >= 4096 * 4 and eq.table_bytes(2) > 0 and eq.table_bytes(7) == 0


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


def test_decode_rejects_bad_descriptors_on_host(eq):
    L = eq.lib()
    d = eq._lib.RansTensorDesc(1, 1, 4, 64, 12, 256, 32, 8, 1, 1 << 20, 1 << 20, 1 << 20,
                               1 << 20, 1 << 20)
    out = (C.c_void_p * 1)(1 << 20)
    st = C.c_void_p(1 << 20)
    for field, val, code in [("version", 0, 1), ("symfmt", 3, 1), ("streams", 40, 3),
                             ("run", 2, 3), ("prob_bits", 10, 3), ("num_chunks", 2, 1),
                             ("chunk_symbols", 100, 1), ("words", (1 << 20) + 2, 1)]:
        bad = eq._lib.RansTensorDesc.from_buffer_copy(d)
        setattr(bad, field, val)
        assert L.eq_decode(C.byref(bad), 1, out, st, None) == code, field
    assert L.eq_decode(C.byref(d), 1, out, None, None) == 1
    assert L.eq_decode(None, 0, None, None, None) == 0


def test_gemv_and_huff_reject_bad_input_on_host(eq):
    L = eq.lib()
    d = eq._lib.RansTensorDesc(1, 1, 4, 64, 12, 100, 32, 8, 3, 1 << 20, 1 << 20, 1 << 20,
                               1 << 20, 1 << 20)  # chunks do not hold whole rows
    assert L.eq_decode_gemv(C.byref(d), C.c_void_p(1 << 20), 1, C.c_void_p(1 << 20),
                            C.c_void_p(1 << 20), None) in (1, 3)
    h = eq._lib.HuffTensorDesc(10, 30, 8, 256, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20)
    h.bytes_per_thread = 4
    assert L.eq_huff_bf16_decode(C.byref(h), C.c_void_p(1 << 20), C.c_void_p(1 << 20), None) in (1, 3)
