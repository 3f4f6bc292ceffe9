"""Seeded synthetic inputs for the entropy-coded weight workloads.

This module is the one piece that both sides use: the CPU oracle (through the
tests) and the GPU library (through the tests and the bench).  It draws random
weight and activation tensors with the shapes and value distributions of the
workloads, and nothing else: no quantiser, no scale, no entropy coder and no
table lives here.

Determinism: every tensor is generated in blocks of ``ROW_BLOCK`` rows, each
block from its own PCG64 stream keyed by ``SeedSequence([seed, tensor, block])``.
Any block can therefore be regenerated alone, which lets a test check sampled
rows of a multi-gigabyte workload without drawing all of it.

Workloads (the shapes follow the pages' model families):
  * ``e4m3_1k``     one 1024x1024 weight, N(0, 0.02)                       (EntQuant Float8 base)
  * ``int8_8k``     8192x8192, Laplace(0, 0.01) clipped at +-0.06            (EntQuant Int8 base)
  * ``llama2_7b``   32 layers x {q,k,v,o 4096x4096; gate,up 11008x4096; down 4096x11008},
                    N(0, 0.02) with 1% of entries multiplied by 8          (LLaMA-2-7B shapes)
  * ``mlp_13b``     gate, up 13824x5120 and down 5120x13824, N(0, 0.02);
                    activations bf16 N(0, 1) with batch 1, 4, 16           (LLaMA-2-13B MLP)
  * ``df11_8k``     8192x28672 bf16 weights from N(0, 0.015)               (DFloat11 bf16 weights)
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

ROW_BLOCK = 16

# ----------------------------------------------------------------------------------------------
# block-keyed generators
# ----------------------------------------------------------------------------------------------


def _rng(seed: int, tensor: int, block: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor, block])))


def _fill_blocks(rows: int, cols: int, seed: int, tensor: int, draw, row_lo: int = 0,
                 row_hi: int | None = None, threads: int | None = None) -> np.ndarray:
    """Fill rows [row_lo, row_hi) of a rows x cols fp32 tensor, block by block.

    ``draw(rng, n)`` returns n fp32 values.  Blocks are aligned to ROW_BLOCK rows of the full
    tensor, so the values of a row do not depend on which slice is requested.
    """
    row_hi = rows if row_hi is None else row_hi
    assert 0 <= row_lo <= row_hi <= rows
    out = np.empty((row_hi - row_lo, cols), dtype=np.float32)
    b_lo, b_hi = row_lo // ROW_BLOCK, (row_hi + ROW_BLOCK - 1) // ROW_BLOCK

    def one(b: int) -> None:
        r0, r1 = b * ROW_BLOCK, min(rows, (b + 1) * ROW_BLOCK)
        vals = draw(_rng(seed, tensor, b), (r1 - r0) * cols).reshape(r1 - r0, cols)
        s0, s1 = max(r0, row_lo), min(r1, row_hi)
        out[s0 - row_lo:s1 - row_lo] = vals[s0 - r0:s1 - r0]

    nblk = b_hi - b_lo
    nthr = threads if threads is not None else min(len(os.sched_getaffinity(0)), 32)
    if nblk * cols < (1 << 22) or nthr <= 1:
        for b in range(b_lo, b_hi):
            one(b)
    else:
        with ThreadPoolExecutor(nthr) as ex:
            list(ex.map(one, range(b_lo, b_hi)))
    return out


def normal(rows: int, cols: int, std: float, seed: int, tensor: int = 0, **kw) -> np.ndarray:
    """fp32 weights ~ N(0, std^2)."""
    def draw(g, n):
        v = g.standard_normal(n, dtype=np.float32)
        v *= np.float32(std)
        return v
    return _fill_blocks(rows, cols, seed, tensor, draw, **kw)


def normal_with_outliers(rows: int, cols: int, std: float, frac: float, mult: float, seed: int,
                         tensor: int = 0, **kw) -> np.ndarray:
    """fp32 weights ~ N(0, std^2); each entry independently (prob ``frac``) multiplied by ``mult``."""
    def draw(g, n):
        v = g.standard_normal(n, dtype=np.float32)
        v *= np.float32(std)
        hit = g.random(n, dtype=np.float32) < np.float32(frac)
        v[hit] *= np.float32(mult)
        return v
    return _fill_blocks(rows, cols, seed, tensor, draw, **kw)


def laplace_clipped(rows: int, cols: int, b: float, clip: float, seed: int, tensor: int = 0,
                    **kw) -> np.ndarray:
    """fp32 weights ~ Laplace(0, b), clipped to [-clip, clip]."""
    def draw(g, n):
        return np.clip(g.laplace(0.0, b, n), -clip, clip).astype(np.float32)
    return _fill_blocks(rows, cols, seed, tensor, draw, **kw)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round an fp32 array to bf16 with torch's own cast; returns the raw uint16 bit patterns."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_normal(rows: int, cols: int, std: float, seed: int, tensor: int = 0, **kw) -> np.ndarray:
    """bf16 weights (uint16 bit patterns) drawn as fp32 N(0, std^2) and cast to bf16."""
    return bf16_bits(normal(rows, cols, std, seed, tensor, **kw))


def activations(batch: int, cols: int, seed: int, tensor: int = 1000) -> np.ndarray:
    """bf16 activations x ~ N(0, 1), shape [batch][cols], as uint16 bit patterns."""
    return bf16_normal(batch, cols, 1.0, seed, tensor)


def plant_super_weights(w: np.ndarray, n: int, seed: int, lo: float = 0.5,
                        hi: float = 2.0) -> list:
    """Overwrite n seeded positions of w (in place, distinct rows) with super weights: magnitude
    uniform in [lo, hi), random sign; LLaMA's super weights sit about 100x above the typical
    weight.  Returns the flat indices, sorted."""
    rows, cols = w.shape
    g = _rng(seed, 0, 7)
    rs = g.choice(rows, size=min(n, rows), replace=False)
    cs = g.integers(0, cols, size=rs.size)
    mags = g.uniform(lo, hi, size=rs.size) * np.where(g.integers(0, 2, size=rs.size) > 0, 1, -1)
    w[rs, cs] = mags.astype(np.float32)
    return sorted(int(r) * cols + int(c) for r, c in zip(rs, cs))


def random_bytes(n: int, seed: int) -> np.ndarray:
    """Uniform random bytes (used by fault-injection tests)."""
    return _rng(seed, 0, 0).integers(0, 256, n, dtype=np.uint8)


def symbols_from_pmf(pmf: np.ndarray, n: int, seed: int) -> np.ndarray:
    """n i.i.d. byte symbols drawn from a 256-entry probability vector."""
    pmf = np.asarray(pmf, dtype=np.float64)
    pmf = pmf / pmf.sum()
    return _rng(seed, 0, 1).choice(256, size=n, p=pmf).astype(np.uint8)


# ----------------------------------------------------------------------------------------------
# workload descriptions (shapes, distributions, seeds, container choices)
# ----------------------------------------------------------------------------------------------


@dataclass(frozen=True)
class TensorSpec:
    name: str
    rows: int
    cols: int
    dist: str            # "normal" | "normal_outliers" | "laplace_clipped" | "bf16_normal"
    seed: int
    tensor: int          # key of the tensor inside its seed's stream family
    std: float = 0.02
    b: float = 0.01
    clip: float = 0.06
    frac: float = 0.01
    mult: float = 8.0

    @property
    def numel(self) -> int:
        return self.rows * self.cols

    def generate(self, row_lo: int = 0, row_hi: int | None = None, threads: int | None = None):
        kw = dict(row_lo=row_lo, row_hi=row_hi, threads=threads)
        if self.dist == "normal":
            return normal(self.rows, self.cols, self.std, self.seed, self.tensor, **kw)
        if self.dist == "normal_outliers":
            return normal_with_outliers(self.rows, self.cols, self.std, self.frac, self.mult,
                                        self.seed, self.tensor, **kw)
        if self.dist == "laplace_clipped":
            return laplace_clipped(self.rows, self.cols, self.b, self.clip, self.seed,
                                   self.tensor, **kw)
        if self.dist == "bf16_normal":
            return bf16_normal(self.rows, self.cols, self.std, self.seed, self.tensor, **kw)
        raise ValueError(self.dist)


@dataclass(frozen=True)
class Workload:
    name: str
    tensors: tuple
    symfmt: str = "e4m3"          # "e4m3" | "int8" | "bf16"
    chunk_symbols: int = 65536     # rANS chunk length in symbols; 0 = one row per chunk
    streams: int = 128             # interleaved rANS streams per chunk (multiple of 32)
    run: int = 8                   # consecutive symbols a stream decodes before the next stream
    int8_div: float = 0.0          # Int8: scale = absmax(row) / int8_div
    batches: tuple = field(default=())
    chunk_rows: int = 0            # > 0: chunks of this many whole rows (overrides chunk_symbols)
    prob_bits: int = 12            # rANS table precision: 12, or 8 / 7 for low-entropy alphabets

    def chunk_for(self, spec: "TensorSpec") -> int:
        """Chunk length in symbols for one tensor of the workload."""
        if self.chunk_rows:
            return self.chunk_rows * spec.cols
        return self.chunk_symbols if self.chunk_symbols else spec.cols

    @property
    def numel(self) -> int:
        return sum(t.numel for t in self.tensors)


# Int8 divisor for the Laplace workload: the per-row scale is absmax/INT8_DIV, and this value puts
# the empirical symbol entropy of the 8192x8192 tensor at 2.00 bits.  It was found by bisection
# with the oracle's quantiser (tests/golden/make_golden.py writes and checks it).
INT8_DIV_LAPLACE_8K = 4.2281


def _llama2_7b(layers: int = 32) -> tuple:
    shapes = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
              ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]
    out = []
    for layer in range(layers):
        for ti, (nm, r, c) in enumerate(shapes):
            out.append(TensorSpec(f"layers.{layer}.{nm}", r, c, "normal_outliers", 3 + layer, ti))
    return tuple(out)


WORKLOADS = {
    "e4m3_1k": Workload("e4m3_1k", (TensorSpec("w", 1024, 1024, "normal", 1, 0),),
                        symfmt="e4m3", chunk_symbols=16384, streams=32, run=8),
    "int8_8k": Workload("int8_8k", (TensorSpec("w", 8192, 8192, "laplace_clipped", 2, 0),),
                        symfmt="int8", chunk_symbols=65536, streams=128, run=8,
                        int8_div=INT8_DIV_LAPLACE_8K, prob_bits=7),
    "llama2_7b": Workload("llama2_7b", _llama2_7b(), symfmt="e4m3", chunk_symbols=65536,
                          streams=128, run=8),
    "mlp_13b": Workload("mlp_13b", (TensorSpec("gate", 13824, 5120, "normal", 4, 0),
                                    TensorSpec("up", 13824, 5120, "normal", 4, 1),
                                    TensorSpec("down", 5120, 13824, "normal", 4, 2)),
                        symfmt="e4m3", chunk_symbols=0, streams=32, run=8, batches=(1, 4, 16),
                        chunk_rows=1),
    "df11_8k": Workload("df11_8k", (TensorSpec("w", 8192, 28672, "bf16_normal", 5, 0,
                                               std=0.015),), symfmt="bf16"),
}


def scaled(w: Workload, row_div: int = 1, layers: int | None = None) -> Workload:
    """A smaller copy of a workload for quick tests: fewer rows and/or fewer layers."""
    ts = w.tensors
    if layers is not None:
        keep = {f"layers.{i}." for i in range(layers)}
        ts = tuple(t for t in ts if any(t.name.startswith(k) for k in keep))
    ts = tuple(TensorSpec(t.name, max(1, t.rows // row_div), t.cols, t.dist, t.seed, t.tensor,
                          t.std, t.b, t.clip, t.frac, t.mult) for t in ts)
    return Workload(w.name + (f"/rows{row_div}" if row_div > 1 else "")
                    + (f"/layers{layers}" if layers is not None else ""), ts, w.symfmt,
                    w.chunk_symbols, w.streams, w.run, w.int8_div, w.batches, w.chunk_rows,
                    w.prob_bits)
