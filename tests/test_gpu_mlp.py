"""GPU parity: eq_mlp_decode (gate/up decode-GEMVs, SiLU gate, down decode-GEMV) against the
oracle's binary64 chain over the decoded bf16 weights, relative L2 <= 1e-3.  The hidden vector is
rounded to bf16 on both sides; an element whose fp32 value sits next to a bf16 rounding boundary
may round the other way, which moves y by far less than the bar."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu
BAR = 1e-3


def rel_l2(y, ref):
    return float(np.linalg.norm(y - ref) / np.linalg.norm(ref))


def coded(orc, w, chunk_rows=1):
    sym, sc = orc.quantize(w, orc.E4M3)
    h = orc.rans_encode(sym, sc, orc.E4M3, chunk_rows * w.shape[1], 32, 8)
    return h, orc.dequant(sym, sc, orc.E4M3)


@pytest.mark.parametrize("hidden,inter,batch", [(512, 1024, 1), (1024, 2816, 4), (256, 512, 16),
                                                (5120, 13824, 1), (5120, 13824, 16)])
def test_mlp_chain(orc, hidden, inter, batch):
    import decoding_interleaved_rans_b200 as eq
    hg, wg = coded(orc, synth.normal(inter, hidden, 0.02, 81, 0))
    hu, wu = coded(orc, synth.normal(inter, hidden, 0.02, 81, 1))
    hd, wd = coded(orc, synth.normal(hidden, inter, 0.02, 81, 2))
    x = synth.activations(batch, hidden, 82)
    tg, tu, td = (eq.DeviceRans.upload(h) for h in (hg, hu, hd))
    xt = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    y, st = eq.mlp_decode(tg, tu, td, xt)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = orc.mlp_f64(wg, wu, wd, x)
    assert rel_l2(y.cpu().numpy().astype(np.float64), ref) <= BAR


def test_mlp_rejects_bad_shapes_and_scratch(orc):
    import decoding_interleaved_rans_b200 as eq
    hg, _ = coded(orc, synth.normal(64, 256, 0.02, 83))
    hd, _ = coded(orc, synth.normal(256, 64, 0.02, 84))
    tg, td = eq.DeviceRans.upload(hg), eq.DeviceRans.upload(hd)
    x = torch.zeros(2, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(eq.EqError):
        eq.mlp_decode(tg, tg, tg, x)  # down has the wrong shape
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(eq.EqError):
        eq.mlp_decode(tg, tg, td, x, scratch=small)
