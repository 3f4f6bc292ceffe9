"""Failure reporting on the GPU: a bounded wait that runs out (a copy that is never issued)
ends the kernel with EQ_DEV_TIMEOUT after about a second, and the context stays usable; corrupt
streams are reported in the status word, never by a trap (the decode tests cover those)."""
import time

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_reports_timeout(orc):
    import decoding_interleaved_rans_b200 as eq
    t0 = time.perf_counter()
    st = eq.selftest_bounded_wait()
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(st.item()) == eq.EQ_DEV_TIMEOUT
    assert 0.5 < dt < 30.0
    # the context still works: an ordinary decode right after
    w = synth.normal(16, 512, 0.02, 7)
    sym, sc = orc.quantize(w, orc.E4M3)
    (out,), st = eq.decode([eq.DeviceRans.upload(orc.rans_encode(sym, sc, orc.E4M3, 4096, 32, 8))])
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(eq.bf16_bits(out).ravel(), orc.dequant(sym, sc, orc.E4M3).ravel())
