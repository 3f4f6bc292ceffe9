"""GPU parity at full size: the LLaMA-2-7B-shaped stack (32 layers x 7 tensors, 6.48 G weights,
Float8-E4M3 with 1% x8 outliers), all 224 tensors decoded in ONE eq_decode call, the call the
bench times (the pages decode a transformer block's weights together; one call over the whole
model is the same launch with more descriptors).  Coded by the oracle tensor by tensor; every
output of one tensor per layer is compared, plus 4 sampled chunks of every other tensor, whose
expected values come from regenerating just those rows (the quantiser's scales are per row)."""
import numpy as np
import pytest
import torch

import synth

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def test_llama2_7b_full_stack_one_call(orc):
    import decoding_interleaved_rans_b200 as eq
    assert torch.cuda.is_available()
    wl = synth.WORKLOADS["llama2_7b"]
    assert len(wl.tensors) == 224
    dev, kept = [], {}
    for i, spec in enumerate(wl.tensors):
        sym, sc = orc.quantize(spec.generate(), orc.E4M3)
        h = orc.rans_encode(sym, sc, orc.E4M3, wl.chunk_symbols, wl.streams, wl.run)
        dev.append(eq.DeviceRans.upload(h))
        layer, k = divmod(i, 7)
        if k == layer % 7:  # compared in full
            kept[i] = (sym, sc)
        del h
    outs, st = eq.decode(dev)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, int(st.item())
    rng = np.random.default_rng(0)
    checked = 0
    chunk = wl.chunk_symbols
    for i, (spec, o, t) in enumerate(zip(wl.tensors, outs, dev)):
        got = eq.bf16_bits(o).ravel()
        if i in kept:
            sym, sc = kept.pop(i)
            assert np.array_equal(got, orc.dequant(sym, sc, orc.E4M3).ravel()), spec.name
            checked += got.size
            continue
        for c in rng.choice(t.num_chunks, 4, replace=False):
            j0, j1 = int(c) * chunk, min(t.numel, (int(c) + 1) * chunk)
            r0, r1 = j0 // t.cols, (j1 - 1) // t.cols + 1
            sym, sc = orc.quantize(spec.generate(row_lo=r0, row_hi=r1), orc.E4M3)
            want = orc.dequant(sym, sc, orc.E4M3).ravel()[j0 - r0 * t.cols:j1 - r0 * t.cols]
            assert np.array_equal(got[j0:j1], want), (spec.name, int(c))
            checked += j1 - j0
    assert checked > 6.48e9 / 7 * 0.9
