"""eq_mlp_decode_noalloc (library-held scratch) against eq_mlp_decode (caller scratch), through
the C ABI, on two calls in a row of different sizes so that the second reuses the shared array.
Same relative L2 bar as the other MLP tests; both run the same kernels in the same order, so the
outputs are expected to agree exactly as well.  Its defining property is checked too: a call
leaves the device's free memory and torch's reserved pool exactly as they were."""
import ctypes as C

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu
BAR = 1e-3


@pytest.fixture(scope="module")
def eq():
    import decoding_interleaved_rans_b200 as m
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    m.lib()
    return m


def upload(eq, w):
    sym, sc = eq.codec.quantize(w, eq.EQ_SYM_E4M3)
    h = eq.codec.rans_encode(sym, sc, eq.EQ_SYM_E4M3, w.shape[1], 32, 8)
    return eq.DeviceRans.upload(h)


def noalloc(eq, g, u, d, x):
    y = torch.empty(x.shape[0], d.rows, dtype=torch.float32, device=x.device)
    st = eq.new_status(x.device)
    dg, du, dd = g.desc(), u.desc(), d.desc()
    code = eq.lib().eq_mlp_decode_noalloc(C.byref(dg), C.byref(du), C.byref(dd), x.data_ptr(),
                                          x.shape[0], y.data_ptr(), st.data_ptr(),
                                          torch.cuda.current_stream().cuda_stream)
    return code, y, st


def test_noalloc_matches_caller_scratch_two_calls(eq):
    hidden, inter = 1024, 2816
    g = upload(eq, synth.normal(inter, hidden, 0.02, 91, 0))
    u = upload(eq, synth.normal(inter, hidden, 0.02, 91, 1))
    d = upload(eq, synth.normal(hidden, inter, 0.02, 91, 2))
    for call, batch in enumerate((16, 3)):
        x = torch.from_numpy(synth.activations(batch, hidden, 92 + call).view(np.int16))
        x = x.cuda().view(torch.bfloat16)
        code, y, st = noalloc(eq, g, u, d, x)
        assert code == 0
        ref, st_ref = eq.mlp_decode(g, u, d, x)
        torch.cuda.synchronize()
        assert int(st.item()) == 0 and int(st_ref.item()) == 0
        a, b = y.cpu().double().numpy(), ref.cpu().double().numpy()
        assert np.linalg.norm(a - b) <= BAR * np.linalg.norm(b), call
        assert np.array_equal(a, b), call


def test_noalloc_call_allocates_nothing(eq):
    hidden, inter, batch = 512, 1408, 4
    g = upload(eq, synth.normal(inter, hidden, 0.02, 94, 0))
    u = upload(eq, synth.normal(inter, hidden, 0.02, 94, 1))
    d = upload(eq, synth.normal(hidden, inter, 0.02, 94, 2))
    x = torch.from_numpy(synth.activations(batch, hidden, 95).view(np.int16))
    x = x.cuda().view(torch.bfloat16)
    y = torch.empty(batch, hidden, dtype=torch.float32, device="cuda")
    st = eq.new_status(x.device)
    dg, du, dd = g.desc(), u.desc(), d.desc()
    stream = torch.cuda.current_stream().cuda_stream

    def call():
        code = eq.lib().eq_mlp_decode_noalloc(C.byref(dg), C.byref(du), C.byref(dd),
                                              x.data_ptr(), batch, y.data_ptr(), st.data_ptr(),
                                              stream)
        torch.cuda.synchronize()
        assert code == 0 and int(st.item()) == 0

    call()  # the first call on the device may load the library's code there
    free0, reserved0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_reserved()
    call()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_reserved() == reserved0


def test_noalloc_rejects_sizes_beyond_its_array(eq):
    hidden, inter = 16, 32776  # inter * 16 > EQ_MLP_NOALLOC_MAX_ELEMS (524288)
    g = upload(eq, synth.normal(inter, hidden, 0.02, 93, 0))
    d = upload(eq, synth.normal(hidden, inter, 0.02, 93, 2))
    x = torch.zeros(16, hidden, dtype=torch.bfloat16, device="cuda")
    code, _, _ = noalloc(eq, g, g, d, x)
    assert code == 3  # EQ_ERR_UNSUPPORTED, nothing launched
    code, y, st = noalloc(eq, g, g, d, x[:15])  # 15 * 32776 fits
    torch.cuda.synchronize()
    assert code == 0 and int(st.item()) == 0 and bool(torch.isfinite(y).all())
