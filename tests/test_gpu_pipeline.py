"""GPU: block-by-block decode overlapped with compute gives exactly the sequential result, and the
decoded weights equal the oracle's."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def test_overlapped_equals_sequential(orc):
    import decoding_interleaved_rans_b200 as eq
    from decoding_interleaved_rans_b200.pipeline import BlockPipeline
    wl = synth.scaled(synth.WORKLOADS["llama2_7b"], row_div=16, layers=4)
    blocks, want = [], []
    for layer in range(4):
        specs = [t for t in wl.tensors if t.name.startswith(f"layers.{layer}.")]
        hs, ws = [], []
        for spec in specs:
            sym, sc = orc.quantize(spec.generate(), orc.E4M3)
            hs.append(eq.DeviceRans.upload(orc.rans_encode(sym, sc, orc.E4M3, 16384, 64, 8)))
            ws.append(orc.dequant(sym, sc, orc.E4M3))
        blocks.append(hs)
        want.append(ws)
    pipe = BlockPipeline(blocks)
    x = torch.randn(64, max(t.cols for t in blocks[0]), device="cuda").to(torch.bfloat16)
    results = {}
    for overlap in (False, True):
        outs = []

        def compute(i, weights):
            ys = [x[:, :w.shape[1]] @ w.t() for w in weights]
            outs.append(torch.cat([y.float().sum(1, keepdim=True) for y in ys], 1))
            if i == 2:  # keep a copy of one block's decoded weights
                outs.append([w.clone() for w in weights])
        pipe.run(compute, overlap=overlap)
        torch.cuda.synchronize()
        results[overlap] = outs
    assert int(pipe.status.item()) == 0
    for a, b in zip(results[False], results[True]):
        if isinstance(a, list):
            for wa, wb, wo in zip(a, b, want[2]):
                assert torch.equal(wa, wb)
                assert np.array_equal(eq.bf16_bits(wa).ravel(), wo.ravel())
        else:
            assert torch.equal(a, b)
