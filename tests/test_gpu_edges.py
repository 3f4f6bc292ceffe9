"""GPU parity at the format's limits: the largest stream count (1024 = 32 groups per chunk), one
group's word substream far longer than its ring (thousands of refills), empty tensors inside a
grouped call, more tensors of one kernel variant in one call than one launch's descriptor table
holds (256: the call is split into launches, each sized from its own tensors), a LLaMA-2-7B-shaped
set of 224 tensors in one call, and a tensor whose chunks hold a single run."""
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


def decode(eq, hosts):
    outs, st = eq.decode([eq.DeviceRans.upload(h) for h in hosts])
    torch.cuda.synchronize()
    return [eq.bf16_bits(o).ravel() for o in outs], int(st.item())


@pytest.mark.parametrize("pb,fmt", [(12, 1), (8, 2)])
def test_max_streams(eq, orc, pb, fmt):
    w = synth.normal(256, 4096, 0.02, 200) if fmt == 1 else \
        synth.laplace_clipped(256, 4096, 0.01, 0.06, 200)
    sym, sc = orc.quantize(w, fmt, synth.INT8_DIV_LAPLACE_8K)
    h = orc.rans_encode(sym, sc, fmt, 65536 * 4, 1024, 8, prob_bits=pb)
    (out,), st = decode(eq, [h])
    assert st == 0 and np.array_equal(out, orc.dequant(sym, sc, fmt).ravel())


def test_long_substream(eq, orc):
    """One 2^21-symbol chunk on 32 streams: a 1.7 MB substream through a 2 KiB ring."""
    w = synth.normal(512, 4096, 0.02, 201)
    sym, sc = orc.quantize(w, orc.E4M3)
    h = orc.rans_encode(sym, sc, orc.E4M3, 1 << 21, 32, 8)
    assert int(h.word_off[1]) * 2 > 1_000_000
    (out,), st = decode(eq, [h])
    assert st == 0 and np.array_equal(out, orc.dequant(sym, sc, orc.E4M3).ravel())


def test_empty_tensors_in_a_grouped_call(eq, orc):
    hosts, want = [], []
    for i, (r, c) in enumerate([(0, 64), (16, 512), (0, 0), (8, 1024)]):
        w = synth.normal(max(r, 1), max(c, 8), 0.02, 210 + i)[:r, :c]
        sym, sc = orc.quantize(np.ascontiguousarray(w), orc.E4M3)
        hosts.append(orc.rans_encode(sym, sc, orc.E4M3, 4096, 32, 8))
        want.append(orc.dequant(sym, sc, orc.E4M3).ravel())
    outs, st = decode(eq, hosts)
    assert st == 0
    for o, e in zip(outs, want):
        assert np.array_equal(o, e)


def test_mixed_variants_in_one_call(eq, orc):
    """200 tensors spread over four kernel variants (symbol format x table size)."""
    hosts, want = [], []
    for i in range(200):
        fmt = orc.INT8 if i % 3 else orc.E4M3
        w = synth.normal(4, 256, 0.02, 300 + i)
        sym, sc = orc.quantize(w, fmt, 20.0)
        hosts.append(orc.rans_encode(sym, sc, fmt, 512, 32, 8, prob_bits=8 if i % 2 else 12))
        want.append(orc.dequant(sym, sc, fmt).ravel())
    outs, st = decode(eq, hosts)
    assert st == 0
    for o, e in zip(outs, want):
        assert np.array_equal(o, e)


@pytest.mark.parametrize("pb,fmt,count", [(12, 1, 300), (7, 2, 290), (8, 2, 270)])
def test_split_launch_of_one_variant(eq, orc, pb, fmt, count):
    """More tensors of ONE kernel variant than a launch holds (256), so eq_decode splits them.
    Sizes vary (1 to 40 chunks of 2 to 4 groups) so that each launch's warps per CTA and each
    tensor's CTA share come from that launch's own units; every output is compared in full."""
    hosts, want = [], []
    rng = np.random.default_rng(count)
    for i in range(count):
        rows = int(rng.integers(1, 41)) * 16
        w = synth.normal(rows, 1024, 0.02, 400 + i) if fmt == 1 else \
            synth.laplace_clipped(rows, 1024, 0.01, 0.06, 400 + i)
        sym, sc = orc.quantize(w, fmt, synth.INT8_DIV_LAPLACE_8K)
        streams = 32 * int(rng.integers(2, 5))
        hosts.append(orc.rans_encode(sym, sc, fmt, 16384, streams, 8, prob_bits=pb))
        want.append(orc.dequant(sym, sc, fmt).ravel())
    outs, st = decode(eq, hosts)
    assert st == 0
    for i, (o, e) in enumerate(zip(outs, want)):
        assert np.array_equal(o, e), i


def test_llama_shaped_224_tensors_in_one_call(eq, orc):
    """The LLaMA-2-7B-shaped stack's 224 tensors (32 layers x q, k, v, o, gate, up, down) with
    their rows cut by 64, coded as the full stack is (E4M3, 12-bit tables, 64 KiB chunks, 128
    streams), decoded in one eq_decode call and compared in full."""
    wl = synth.scaled(synth.WORKLOADS["llama2_7b"], row_div=64)
    assert len(wl.tensors) == 224
    hosts, want = [], []
    for spec in wl.tensors:
        sym, sc = orc.quantize(spec.generate(), orc.E4M3)
        hosts.append(orc.rans_encode(sym, sc, orc.E4M3, wl.chunk_symbols, wl.streams, wl.run))
        want.append(orc.dequant(sym, sc, orc.E4M3).ravel())
    outs, st = decode(eq, hosts)
    assert st == 0
    for i, (o, e) in enumerate(zip(outs, want)):
        assert np.array_equal(o, e), wl.tensors[i].name


def test_chunks_of_a_single_run(eq, orc):
    w = synth.normal(64, 64, 0.02, 220)
    sym, sc = orc.quantize(w, orc.E4M3)
    for G, pb in [(8, 12), (8, 8), (1, 12)]:
        h = orc.rans_encode(sym, sc, orc.E4M3, G, 32, G, prob_bits=pb)
        (out,), st = decode(eq, [h])
        assert st == 0 and np.array_equal(out, orc.dequant(sym, sc, orc.E4M3).ravel())
