"""GPU parity: eq_decode_gemv (decode + GEMV fused) against the oracle's fp64 product of the
decoded bf16 weights.  The bar is a relative L2 error of at most 1e-3 over the whole [batch, rows]
output.  The kernel multiplies the exact bf16 weights by the bf16 activations (each product exact
in fp32) and sums in fp32, so its error is fp32 summation error, far inside the bar; the tests
also hold it to 1e-5 so that a wrong weight or activation cannot hide under the 1e-3 bar."""
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


@pytest.mark.parametrize("name", ["gate", "up", "down"])
def test_mlp_13b_full_size(eq, orc, name):
    """The 13B MLP weights at full size, batch 1, 4 and 16, in the bench's layout."""
    wl = synth.WORKLOADS["mlp_13b"]
    spec = next(t for t in wl.tensors if t.name == name)
    sym, sc = orc.quantize(spec.generate(), orc.E4M3)
    h = orc.rans_encode(sym, sc, orc.E4M3, wl.chunk_for(spec), wl.streams, wl.run)
    wbf = orc.dequant(sym, sc, orc.E4M3)
    for batch in wl.batches:
        x = synth.activations(batch, spec.cols, 4, tensor=100 + batch)
        y, st = gemv(eq, h, x)
        ref = orc.gemv_f64(wbf, x)
        assert st == 0
        err = rel_l2(y, ref)
        assert err <= BAR and err <= TIGHT, (name, batch, err)


@pytest.mark.parametrize("rows,cols,chunk_rows,streams", [
    (1, 8, 1, 32), (37, 200, 1, 32), (50, 1024, 4, 32), (9, 4096, 3, 32), (64, 512, 2, 32),
    (7, 13824, 1, 32), (13, 5120, 4, 32)])
@pytest.mark.parametrize("batch", [1, 3, 8, 16])
def test_shapes_and_batches(eq, orc, rows, cols, chunk_rows, streams, batch):
    w = synth.normal(rows, cols, 0.02, rows + cols)
    sym, sc = orc.quantize(w, orc.E4M3)
    h = orc.rans_encode(sym, sc, orc.E4M3, chunk_rows * cols, streams, 8)
    x = synth.activations(batch, cols, 5)
    y, st = gemv(eq, h, x)
    ref = orc.gemv_f64(orc.dequant(sym, sc, orc.E4M3), x)
    assert st == 0
    assert rel_l2(y, ref) <= TIGHT


def test_int8_and_special_symbols(eq, orc):
    rng = np.random.default_rng(6)
    for fmt in (orc.E4M3, orc.INT8):
        sym = rng.integers(0, 256, (40, 512), dtype=np.uint8)
        if fmt == orc.E4M3:
            sym[(sym & 0x7F) == 0x7F] = 0x00  # NaN weights would make the product NaN
        sc = synth.bf16_bits(rng.uniform(1e-3, 1.0, 40).astype(np.float32))
        h = orc.rans_encode(sym, sc, fmt, 512, 32, 8)
        x = synth.activations(4, 512, 7)
        y, st = gemv(eq, h, x)
        ref = orc.gemv_f64(orc.dequant(sym, sc, fmt), x)
        assert st == 0 and rel_l2(y, ref) <= TIGHT


def test_single_symbol_table(eq, orc):
    sym = np.full((8, 256), 0x40, np.uint8)
    sc = np.full(8, 0x3C00, np.uint16)
    h = orc.rans_encode(sym, sc, orc.E4M3, 256, 32, 8)
    x = synth.activations(2, 256, 8)
    y, st = gemv(eq, h, x)
    ref = orc.gemv_f64(orc.dequant(sym, sc, orc.E4M3), x)
    assert st == 0 and rel_l2(y, ref) <= TIGHT


def test_unsupported_layouts_rejected(eq, orc):
    w = synth.normal(8, 200, 0.02, 9)
    sym, sc = orc.quantize(w, orc.E4M3)
    x = torch.zeros(1, 200, dtype=torch.bfloat16, device="cuda")
    for chunk, S, G in [(300, 32, 8), (400, 32, 8), (200, 32, 1), (200, 64, 8)]:
        t = eq.DeviceRans.upload(orc.rans_encode(sym, sc, orc.E4M3, chunk, S, G))
        with pytest.raises(eq.EqError):
            eq.decode_gemv(t, x)


def test_every_batch_width_after_another_on_a_large_tensor(eq, orc):
    """Each kernel instance opts into its own shared-memory size: on a tensor with enough chunks
    for 16-warp CTAs (whose shared memory exceeds the default limit), every batch width runs
    after the others, the CUDA-core batch 9..16 kernel included (chunks not a multiple of 256)."""
    w = synth.normal(16384, 64, 0.02, 10)
    sym, sc = orc.quantize(w, orc.E4M3)
    h = orc.rans_encode(sym, sc, orc.E4M3, 64, 32, 8)
    wbf = orc.dequant(sym, sc, orc.E4M3)
    for batch in (8, 16, 5, 2, 1, 12):
        x = synth.activations(batch, 64, 11, tensor=200 + batch)
        y, st = gemv(eq, h, x)
        assert st == 0, batch
        assert rel_l2(y, orc.gemv_f64(wbf, x)) <= TIGHT, batch
