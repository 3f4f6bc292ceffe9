"""GPU parity for EntroLLM-style integer weights (eq_huff_int_decode): Huffman-coded 8- and
4-bit codes decoded by the two-stage kernel to bf16((q - zero) * scale), bit for bit against the
oracle's sequential decoder."""
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


def run(eq, h):
    t = eq.DeviceHuffInt.upload(h)
    out, st = eq.huff_int_decode(t)
    torch.cuda.synchronize()
    return eq.bf16_bits(out).ravel(), int(st.item())


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("rows,cols,tpb", [(1024, 1024, 256), (37, 999, 32), (3, 7, 512),
                                           (512, 3072, 128), (1, 1, 256)])
def test_decode_matches_oracle(eq, orc, bits, rows, cols, tpb):
    w = synth.normal(rows, cols, 0.02, rows + cols + bits)
    sym, sc, z, _ = orc.entrollm_quantize(w, bits)
    h = orc.huff_encode_sym(sym, bits, sc, z, threads_per_block=tpb)
    rc, want = orc.entrollm_decode_bf16(h)
    assert rc == 0
    out, st = run(eq, h)
    assert st == 0 and np.array_equal(out, want.ravel())


def test_product_encoder_streams(eq, orc):
    """The library's own compressor; skewed and outlier-heavy weights pick different schemes."""
    rng = np.random.default_rng(5)
    for w in (np.abs(rng.standard_normal((256, 1024))).astype(np.float32) * 0.02,
              synth.normal_with_outliers(256, 1024, 0.02, 0.01, 8.0, 6)):
        for bits in (8, 4):
            h = eq.codec.entrollm_encode(w, bits)
            sym, sc, z, _ = orc.entrollm_quantize(w, bits)
            out, st = run(eq, h)
            assert st == 0 and np.array_equal(out, orc.intq_dequant(sym, sc, z).ravel())


def test_single_code_and_code_above_the_limit(eq, orc):
    sym = np.full(5000, 9, np.uint8)
    h = orc.huff_encode_sym(sym, 4, 0x3F80, 3)
    out, st = run(eq, h)
    assert st == 0 and np.array_equal(out, orc.intq_dequant(sym, 0x3F80, 3))
    # a 4-bit tensor whose stream holds the code 17: decoded, but reported
    sym = np.random.default_rng(7).integers(0, 16, 3000).astype(np.uint8)
    sym[1234] = 17
    h = orc.huff_encode_sym(sym, 4, 0x3F80, 8)
    assert run(eq, h)[1] & eq.EQ_DEV_BAD_CODE
