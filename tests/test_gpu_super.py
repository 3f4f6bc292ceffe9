"""GPU parity for super weights (the sorted (index, bf16) list written over the decoded weights):
eq_decode bit for bit and eq_decode_gemv within the GEMV bar, against the oracle."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu
TIGHT = 1e-5


@pytest.fixture(scope="module")
def eq():
    import decoding_interleaved_rans_b200 as m
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    m.lib()
    return m


def coded(orc, rows, cols, fmt, chunk, S, G, pb, n_super, seed):
    w = synth.laplace_clipped(rows, cols, 0.01, 0.06, seed) if fmt == orc.INT8 else \
        synth.normal(rows, cols, 0.02, seed)
    synth.plant_super_weights(w, n_super, seed)
    idx, val = orc.super_weights(w)
    assert idx.size == n_super
    sym, sc = orc.quantize_excluding(w, fmt, synth.INT8_DIV_LAPLACE_8K, idx)
    h = orc.rans_encode(sym, sc, fmt, chunk, S, G, prob_bits=pb)
    h.patch_idx, h.patch_val = idx, val
    want = orc.patch_bf16(orc.dequant(sym, sc, fmt), idx, val)
    return h, want


def decode(eq, hosts):
    outs, st = eq.decode([eq.DeviceRans.upload(h) for h in hosts])
    torch.cuda.synchronize()
    return [eq.bf16_bits(o).ravel() for o in outs], int(st.item())


@pytest.mark.parametrize("fmt,chunk,S,G,pb", [(2, 65536, 128, 8, 8), (2, 65536, 128, 8, 12),
                                              (1, 16384, 32, 8, 12), (2, 999, 64, 1, 12),
                                              (2, 4096, 256, 8, 8)])
def test_decode_with_super_weights(eq, orc, fmt, chunk, S, G, pb):
    h, want = coded(orc, 200, 2048, fmt, chunk, S, G, pb, 12, 100 + S)
    (out,), st = decode(eq, [h])
    assert st == 0 and np.array_equal(out, want.ravel())


def test_grouped_launch_mixed_patched_and_plain(eq, orc):
    hosts, wants = [], []
    for i, (n_super, pb) in enumerate([(5, 8), (0, 8), (17, 12), (1, 8)]):
        if n_super:
            h, want = coded(orc, 128, 4096, orc.INT8, 65536, 128, 8, pb, n_super, 110 + i)
        else:
            w = synth.laplace_clipped(64, 1024, 0.01, 0.06, 110 + i)
            sym, sc = orc.quantize(w, orc.INT8, synth.INT8_DIV_LAPLACE_8K)
            h = orc.rans_encode(sym, sc, orc.INT8, 65536, 128, 8, prob_bits=pb)
            want = orc.dequant(sym, sc, orc.INT8)
        hosts.append(h)
        wants.append(want.ravel())
    outs, st = decode(eq, hosts)
    assert st == 0
    for o, w in zip(outs, wants):
        assert np.array_equal(o, w)


def test_all_zero_tensor_with_super_weights(eq, orc):
    """Every ordinary weight zero: a one-symbol table plus the list."""
    w = np.zeros((64, 512), np.float32)
    synth.plant_super_weights(w, 4, 120)
    idx, val = orc.super_weights(w, 1.0)
    sym, sc = orc.quantize_excluding(w, orc.INT8, 4.0, idx)
    h = orc.rans_encode(sym, sc, orc.INT8, 4096, 32, 8, prob_bits=8)
    h.patch_idx, h.patch_val = idx, val
    (out,), st = decode(eq, [h])
    assert st == 0 and np.array_equal(out, orc.patch_bf16(orc.dequant(sym, sc, orc.INT8), idx, val).ravel())


def test_bad_lists_are_reported(eq, orc):
    h, _ = coded(orc, 64, 1024, orc.INT8, 65536, 128, 8, 8, 6, 130)
    bad = h.patch_idx.copy()
    bad[2], bad[3] = bad[3], bad[2]  # not increasing
    h.patch_idx = bad
    assert decode(eq, [h])[1] & eq.EQ_DEV_CORRUPT_STATE
    h, _ = coded(orc, 64, 1024, orc.INT8, 65536, 128, 8, 8, 6, 131)
    sym = np.zeros((64, 1024), np.uint8)
    sym[:] = 1  # every weight codes a nonzero value, so no listed position decodes to zero
    h2 = orc.rans_encode(sym, h.scales, orc.INT8, 65536, 128, 8, prob_bits=8)
    h2.patch_idx, h2.patch_val = h.patch_idx, h.patch_val
    assert decode(eq, [h2])[1] & eq.EQ_DEV_CORRUPT_STATE


@pytest.mark.parametrize("batch", [1, 4, 16])
@pytest.mark.parametrize("fmt", [1, 2])
def test_gemv_with_super_weights(eq, orc, fmt, batch):
    rows, cols = 96, 2048
    h, want = coded(orc, rows, cols, fmt, cols, 32, 8, 12, 10, 140 + fmt)
    x = synth.activations(batch, cols, 141, tensor=batch)
    t = eq.DeviceRans.upload(h)
    xt = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    y, st = eq.decode_gemv(t, xt)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = orc.gemv_f64(want.reshape(rows, cols), x)
    got = y.cpu().numpy().astype(np.float64)
    assert np.linalg.norm(got - ref) <= TIGHT * np.linalg.norm(ref)
