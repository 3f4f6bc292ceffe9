"""GPU parity at full size: the LLaMA-2-7B-shaped stack (32 layers x 7 tensors, 6.48 G weights,
Float8-E4M3 with 1% x8 outliers) decoded one transformer block per eq_decode call, the way the
pages decode weights block by block.  Coded by the oracle layer by layer; every output of one
tensor per layer is compared, plus 4 sampled chunks of every other tensor."""
import numpy as np
import pytest
import torch

import synth

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def test_llama2_7b_full_stack(orc):
    import decoding_interleaved_rans_b200 as eq
    assert torch.cuda.is_available()
    wl = synth.WORKLOADS["llama2_7b"]
    rng = np.random.default_rng(0)
    checked = 0
    for layer in range(32):
        specs = [t for t in wl.tensors if t.name.startswith(f"layers.{layer}.")]
        hosts, syms, scs = [], [], []
        for spec in specs:
            sym, sc = orc.quantize(spec.generate(), orc.E4M3)
            hosts.append(orc.rans_encode(sym, sc, orc.E4M3, wl.chunk_symbols, wl.streams, wl.run))
            syms.append(sym)
            scs.append(sc)
        dev = [eq.DeviceRans.upload(h) for h in hosts]
        outs, st = eq.decode(dev)
        torch.cuda.synchronize()
        assert int(st.item()) == 0, (layer, int(st.item()))
        full = layer % 7
        for i, (o, sym, sc, h) in enumerate(zip(outs, syms, scs, hosts)):
            got = eq.bf16_bits(o).ravel()
            if i == full:
                assert np.array_equal(got, orc.dequant(sym, sc, orc.E4M3).ravel()), (layer, i)
                checked += got.size
                continue
            chunk = wl.chunk_symbols
            for c in rng.choice(h.num_chunks, 4, replace=False):
                j0, j1 = int(c) * chunk, min(h.numel, (int(c) + 1) * chunk)
                r0, r1 = j0 // h.cols, (j1 - 1) // h.cols + 1
                want = orc.dequant(sym[r0:r1], sc[r0:r1], orc.E4M3).ravel()
                want = want[j0 - r0 * h.cols:j1 - r0 * h.cols]
                assert np.array_equal(got[j0:j1], want), (layer, i, int(c))
                checked += j1 - j0
        del dev, outs, hosts, syms, scs
        torch.cuda.empty_cache()
    assert checked > 6.48e9 / 7 * 0.9
