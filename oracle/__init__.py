"""CPU oracle for entropy-coded LLM weights -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package.  The library under ``decoding_interleaved_rans_b200`` never does, and the two share
no code: the oracle is plain C (``eq_oracle.c``, loaded through ctypes) plus the numpy glue below.

Every function cites the passage of the pages it follows; see the header of ``eq_oracle.c``.
The pins that tie the oracle to the pages and to mathematics (rather than to itself) are in
``tests/test_oracle_*.py``.  No function here is "parity unpinned".
"""
from __future__ import annotations

import ctypes as C
import math
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "eq_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle.so")

E4M3, INT8 = 1, 2
PROB_BITS = 12
RANS_L = 1 << 16

ERRORS = {0: "ok", -1: "bad argument", -2: "symbol missing from table", -3: "corrupt stream",
          -4: "word overrun", -5: "no code matches"}


def build(force: bool = False) -> str:
    """Compile eq_oracle.c into oracle/_build/liboracle.so (plain gcc, no CUDA)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    os.makedirs(_LIB_DIR, exist_ok=True)
    tmp = _LIB + f".{os.getpid()}.tmp"
    subprocess.check_call(["gcc", "-O2", "-std=gnu11", "-ffp-contract=off", "-fPIC", "-shared",
                           "-Wall", "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> C.CDLL:
    global _lib
    if _lib is None:
        L = C.CDLL(build())
        p = C.c_void_p
        i64, u64, u32, i32 = C.c_int64, C.c_uint64, C.c_uint32, C.c_int
        sig = {
            "orc_bf16_to_f32": (C.c_float, [C.c_uint16]),
            "orc_f32_to_bf16": (C.c_uint16, [C.c_float]),
            "orc_f64_to_bf16": (C.c_uint16, [C.c_double]),
            "orc_e4m3_value": (C.c_double, [C.c_uint8]),
            "orc_f32_to_e4m3": (C.c_uint8, [C.c_float]),
            "orc_quantize_e4m3": (None, [p, i64, i64, p, p]),
            "orc_quantize_int8": (None, [p, i64, i64, C.c_float, p, p]),
            "orc_super_weights": (i64, [p, i64, i64, C.c_double, i64, p, p]),
            "orc_quantize_excluding": (None, [p, i64, i64, i32, C.c_float, p, i64, p, p]),
            "orc_dequant_one": (C.c_uint16, [C.c_uint8, C.c_uint16, i32]),
            "orc_dequant": (None, [p, p, i64, i64, i32, p]),
            "orc_rans_normalize": (i32, [p, u32, p]),
            "orc_rans_groups": (i64, [u32]),
            "orc_rans_encode_chunk": (i64, [p, i64, p, u32, u32, u32, p, p, p]),
            "orc_rans_decode_chunk": (i32, [p, p, p, i64, p, u32, u32, u32, p]),
            "orc_rans_decode_bf16": (i32, [p, p, p, p, p, i64, i64, i32, u32, i64, u32, u32,
                                           i64, i64, p]),
            "orc_gemv_f64": (None, [p, p, i64, i64, i64, p]),
            "orc_huff_lengths": (i32, [p, i32, p]),
            "orc_intq_quantize": (i32, [p, i64, i32, i32, p, p, p]),
            "orc_intq_dequant": (None, [p, i64, C.c_uint16, C.c_int32, p]),
            "orc_huff_total_bits_sym": (u64, [p, i64, p]),
            "orc_huff_encode_sym": (i32, [p, i64, p, p, u32, p, p, p, u64]),
            "orc_huff_decode_sym": (i32, [p, u64, i64, p, p]),
            "orc_huff_canonical": (None, [p, p]),
            "orc_huff_total_bits": (u64, [p, i64, p]),
            "orc_huff_encode": (i32, [p, i64, p, p, u32, p, p, p, p, u64]),
            "orc_huff_decode": (i32, [p, u64, p, i64, p, p]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _p(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _threads(n: int | None) -> int:
    return n if n else len(os.sched_getaffinity(0))


# ----------------------------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------------------------

def f32_to_bf16(a) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32).ravel()
    f = lib().orc_f32_to_bf16
    return np.fromiter((f(float(v)) for v in a), dtype=np.uint16, count=a.size)


def f64_to_bf16(a) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float64).ravel()
    f = lib().orc_f64_to_bf16
    return np.fromiter((f(float(v)) for v in a), dtype=np.uint16, count=a.size)


def bf16_to_f32(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def e4m3_value(sym: int) -> float:
    return lib().orc_e4m3_value(int(sym))


def f32_to_e4m3(a) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32).ravel()
    f = lib().orc_f32_to_e4m3
    return np.fromiter((f(float(v)) for v in a), dtype=np.uint8, count=a.size)


# ----------------------------------------------------------------------------------------------
# quantisation (per-output-channel AbsMax scale, Float8-E4M3 / Int8 base alphabets)
# ----------------------------------------------------------------------------------------------

def quantize(w: np.ndarray, symfmt: int, int8_div: float = 0.0):
    """Returns (symbols uint8 [rows, cols], scales bf16-bits uint16 [rows])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, cols = w.shape
    sym = np.empty((rows, cols), dtype=np.uint8)
    sc = np.empty(rows, dtype=np.uint16)
    nthr = _threads(None)
    step = max(1, (rows + nthr - 1) // nthr)

    def part(r0):
        r1 = min(rows, r0 + step)
        if symfmt == E4M3:
            lib().orc_quantize_e4m3(_p(w[r0:r1]), r1 - r0, cols, _p(sym[r0:r1]), _p(sc[r0:r1]))
        else:
            lib().orc_quantize_int8(_p(w[r0:r1]), r1 - r0, cols, float(int8_div),
                                    _p(sym[r0:r1]), _p(sc[r0:r1]))
    if rows * cols < (1 << 20):
        part_all = [part(r0) for r0 in range(0, rows, step)]
        del part_all
    else:
        with ThreadPoolExecutor(nthr) as ex:
            list(ex.map(part, range(0, rows, step)))
    return sym, sc


def dequant(sym: np.ndarray, scales: np.ndarray, symfmt: int) -> np.ndarray:
    """bf16( value(q) * scale[row] ), exact product, one rounding.  Returns uint16 [rows, cols]."""
    sym = np.ascontiguousarray(sym, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    rows, cols = sym.shape
    out = np.empty((rows, cols), dtype=np.uint16)
    lib().orc_dequant(_p(sym), _p(scales), rows, cols, symfmt, _p(out))
    return out


def dequant_one(q: int, scale_bits: int, symfmt: int) -> int:
    return lib().orc_dequant_one(int(q), int(scale_bits), symfmt)


def entropy_bits(sym: np.ndarray) -> float:
    """Empirical Shannon entropy (bits/symbol) of a byte array."""
    c = np.bincount(np.asarray(sym, dtype=np.uint8).ravel(), minlength=256).astype(np.float64)
    p = c[c > 0] / c.sum()
    return float(-(p * np.log2(p)).sum())


# ----------------------------------------------------------------------------------------------
# rANS containers
# ----------------------------------------------------------------------------------------------

def rans_groups(streams: int) -> int:
    """Streams form groups of 32, each with its own word substream."""
    return (streams + 31) // 32


@dataclass
class RansTensor:
    """One interleaved-rANS-coded weight (format of the library's eq_rans_tensor).

    word_off has num_chunks * groups + 1 entries (one substream per chunk and group of 32
    streams); words are padded with zeros to a multiple of 8 (16 bytes)."""
    rows: int
    cols: int
    symfmt: int
    prob_bits: int
    chunk_symbols: int
    streams: int
    run: int
    freqs: np.ndarray     # uint32[256], sums to 2^prob_bits
    states: np.ndarray    # uint32[num_chunks * streams]
    word_off: np.ndarray  # uint64[num_chunks * groups + 1]
    words: np.ndarray     # uint16
    scales: np.ndarray    # uint16[rows] (bf16 bits)
    # super weights written back over the decoded values: flat indices (sorted) and bf16 bits
    patch_idx: np.ndarray = field(default_factory=lambda: np.zeros(0, np.uint64))
    patch_val: np.ndarray = field(default_factory=lambda: np.zeros(0, np.uint16))

    @property
    def numel(self) -> int:
        return self.rows * self.cols

    @property
    def groups(self) -> int:
        return rans_groups(self.streams)

    @property
    def num_chunks(self) -> int:
        return (len(self.word_off) - 1) // self.groups

    @property
    def payload_bytes(self) -> int:
        """Words actually used (without the alignment padding)."""
        return int(self.word_off[-1]) * 2

    @property
    def compressed_bytes(self) -> int:
        """Everything the decoder reads: words, states, offsets, scales, frequency table and the
        super-weight list."""
        return (self.payload_bytes + self.states.nbytes + self.word_off.nbytes
                + self.scales.nbytes + 256 * 2 + self.patch_idx.nbytes + self.patch_val.nbytes)


def rans_freqs(sym: np.ndarray, prob_bits: int = PROB_BITS) -> np.ndarray:
    counts = np.bincount(np.asarray(sym, dtype=np.uint8).ravel(), minlength=256).astype(np.uint64)
    freqs = np.zeros(256, dtype=np.uint32)
    rc = lib().orc_rans_normalize(_p(counts), prob_bits, _p(freqs))
    if rc:
        raise ValueError(ERRORS.get(rc, rc))
    return freqs


def rans_encode_chunk(sym: np.ndarray, freqs: np.ndarray, streams: int, run: int,
                      prob_bits: int = PROB_BITS):
    """Encode one chunk; returns (states uint32[S], words uint16 (group substreams one after the
    other, decoder order), per-group word counts int64[ceil(S / 32)])."""
    sym = np.ascontiguousarray(sym, dtype=np.uint8).ravel()
    freqs = np.ascontiguousarray(freqs, dtype=np.uint32)
    states = np.empty(streams, dtype=np.uint32)
    words = np.empty(max(1, sym.size), dtype=np.uint16)
    counts = np.zeros(rans_groups(streams), dtype=np.int64)
    nw = lib().orc_rans_encode_chunk(_p(sym) if sym.size else _p(np.zeros(1, np.uint8)),
                                     sym.size, _p(freqs), prob_bits, streams, run, _p(states),
                                     _p(words), _p(counts))
    if nw < 0:
        raise ValueError(ERRORS.get(nw, nw))
    return states, words[:nw].copy(), counts


def rans_decode_chunk(words: np.ndarray, states: np.ndarray, n: int, freqs: np.ndarray,
                      streams: int, run: int, counts=None, prob_bits: int = PROB_BITS):
    """Decode one chunk; returns (status, symbols uint8[n]).  counts: words per group (default:
    all words belong to the one group)."""
    words = np.ascontiguousarray(words, dtype=np.uint16)
    states = np.ascontiguousarray(states, dtype=np.uint32)
    freqs = np.ascontiguousarray(freqs, dtype=np.uint32)
    if counts is None:
        assert rans_groups(streams) == 1
        counts = [words.size]
    goff = np.zeros(len(counts) + 1, dtype=np.int64)
    np.cumsum(np.asarray(counts, dtype=np.int64), out=goff[1:])
    out = np.zeros(max(1, n), dtype=np.uint8)
    wp = _p(words) if words.size else _p(np.zeros(1, np.uint16))
    rc = lib().orc_rans_decode_chunk(wp, _p(goff), _p(states), n, _p(freqs), prob_bits,
                                     streams, run, _p(out))
    return rc, out[:n]


def rans_encode(sym: np.ndarray, scales: np.ndarray, symfmt: int, chunk_symbols: int,
                streams: int, run: int, prob_bits: int = PROB_BITS, freqs=None,
                threads: int | None = None) -> RansTensor:
    """Encode a [rows, cols] symbol matrix.  chunk_symbols == 0 means one row per chunk."""
    sym = np.ascontiguousarray(sym, dtype=np.uint8)
    rows, cols = sym.shape
    flat = sym.ravel()
    N = flat.size
    chunk = cols if chunk_symbols == 0 else chunk_symbols
    if freqs is None:
        freqs = rans_freqs(flat, prob_bits)
    nchunks = (N + chunk - 1) // chunk
    ng = rans_groups(streams)
    states = np.empty(nchunks * streams, dtype=np.uint32)
    pieces = [None] * nchunks
    counts = np.zeros((nchunks, ng), dtype=np.uint64)

    def one(c):
        j0 = c * chunk
        st, w, cnt = rans_encode_chunk(flat[j0:j0 + chunk], freqs, streams, run, prob_bits)
        states[c * streams:(c + 1) * streams] = st
        pieces[c] = w
        counts[c] = cnt

    if nchunks <= 4 or N < (1 << 20):
        for c in range(nchunks):
            one(c)
    else:
        with ThreadPoolExecutor(_threads(threads)) as ex:
            list(ex.map(one, range(nchunks)))
    word_off = np.zeros(nchunks * ng + 1, dtype=np.uint64)
    np.cumsum(counts.ravel(), out=word_off[1:])
    total = int(word_off[-1])
    words = np.zeros(((total + 7) // 8) * 8 if total else 8, dtype=np.uint16)
    if nchunks and total:
        words[:total] = np.concatenate(pieces)
    return RansTensor(rows, cols, symfmt, prob_bits, chunk_symbols, streams, run,
                      np.ascontiguousarray(freqs, dtype=np.uint32), states, word_off, words,
                      np.ascontiguousarray(scales, dtype=np.uint16))


def rans_decode_bf16(t: RansTensor, chunks=None, threads: int | None = 1):
    """Decode chunks (default: all), dequantise to bf16 and write the super weights back.
    Returns (status, uint16 [rows*cols]).

    Only the decoded chunks' spans of the output are written (the rest stays zero)."""
    out = np.zeros(t.numel, dtype=np.uint16)
    chunk = t.cols if t.chunk_symbols == 0 else t.chunk_symbols
    if chunks is None:
        chunks = range(t.num_chunks)
    chunks = list(chunks)
    words = t.words if t.words.size else np.zeros(8, np.uint16)

    def run(c0c1):
        c0, c1 = c0c1
        return lib().orc_rans_decode_bf16(_p(words), _p(t.word_off), _p(t.states), _p(t.freqs),
                                          _p(t.scales), t.rows, t.cols, t.symfmt, t.prob_bits,
                                          chunk, t.streams, t.run, c0, c1, _p(out))
    spans = [(c, c + 1) for c in chunks]
    nthr = _threads(threads)
    if nthr <= 1:
        rcs = [run(s) for s in spans]
    else:
        with ThreadPoolExecutor(nthr) as ex:
            rcs = list(ex.map(run, spans))
    rc = next((r for r in rcs if r), 0)
    if t.patch_idx.size:
        done = np.zeros(t.num_chunks, bool)
        done[chunks] = True
        mine = done[(t.patch_idx // chunk).astype(np.int64)]
        out[t.patch_idx[mine].astype(np.int64)] = t.patch_val[mine]
    return rc, out


def super_weights(w: np.ndarray, tau: float = 20.0):
    """Super weights of a tensor: |w| > tau * rms(w).  Returns (flat indices uint64 sorted,
    bf16 bits uint16)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, cols = w.shape
    n = lib().orc_super_weights(_p(w), rows, cols, float(tau), 0, None, None)
    if n < 0:
        raise ValueError("bad arguments")
    idx = np.zeros(max(1, n), np.uint64)
    val = np.zeros(max(1, n), np.uint16)
    lib().orc_super_weights(_p(w), rows, cols, float(tau), n, _p(idx), _p(val))
    return idx[:n], val[:n]


def quantize_excluding(w: np.ndarray, symfmt: int, int8_div: float, idx: np.ndarray):
    """AbsMax quantisation with the listed positions left out of their rows' scales (symbol 0).
    Returns (symbols uint8 [rows, cols], scales uint16 [rows])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, cols = w.shape
    idx = np.ascontiguousarray(idx, dtype=np.uint64)
    sym = np.empty((rows, cols), np.uint8)
    sc = np.empty(rows, np.uint16)
    lib().orc_quantize_excluding(_p(w), rows, cols, symfmt, float(int8_div),
                                 _p(idx) if idx.size else None, idx.size, _p(sym), _p(sc))
    return sym, sc


def patch_bf16(out: np.ndarray, idx: np.ndarray, val: np.ndarray) -> np.ndarray:
    """Decoded bf16 weights with the super weights written back (a copy)."""
    o = np.array(out, dtype=np.uint16, copy=True)
    o.reshape(-1)[np.asarray(idx, np.int64)] = val
    return o


# ----------------------------------------------------------------------------------------------
# GEMV
# ----------------------------------------------------------------------------------------------

def gemv_f64(w_bf16: np.ndarray, x_bf16: np.ndarray) -> np.ndarray:
    """y[b][r] = sum_c W[r][c] x[b][c] in binary64.  Returns float64 [batch, rows]."""
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = w.shape
    batch = x.shape[0]
    assert x.shape[1] == cols
    y = np.empty((batch, rows), dtype=np.float64)
    nthr = _threads(None)
    step = max(1, (rows + nthr - 1) // nthr)

    def part(r0):
        r1 = min(rows, r0 + step)
        yb = np.empty((batch, r1 - r0), dtype=np.float64)
        lib().orc_gemv_f64(_p(w[r0:r1]), _p(x), r1 - r0, cols, batch, _p(yb))
        y[:, r0:r1] = yb
    if rows * cols * batch < (1 << 20):
        for r0 in range(0, rows, step):
            part(r0)
    else:
        with ThreadPoolExecutor(nthr) as ex:
            list(ex.map(part, range(0, rows, step)))
    return y


def mlp_f64(wg_bf16, wu_bf16, wd_bf16, x_bf16) -> np.ndarray:
    """y[b] = W_down h[b], h = bf16( silu(W_gate x[b]) * (W_up x[b]) ), silu(v) = v / (1 + e^-v);
    the products in binary64, h rounded once to bf16 (what the down projection reads)."""
    g = gemv_f64(wg_bf16, x_bf16)
    u = gemv_f64(wu_bf16, x_bf16)
    hv = g / (1.0 + np.exp(-g)) * u
    h = f64_to_bf16(hv.ravel()).reshape(hv.shape)
    return gemv_f64(wd_bf16, h)


# ----------------------------------------------------------------------------------------------
# DFloat11 (Huffman-coded bf16 exponent)
# ----------------------------------------------------------------------------------------------

@dataclass
class HuffTensor:
    """One DFloat11-coded bf16 weight (format of the library's eq_huff_tensor)."""
    n: int
    bytes_per_thread: int
    threads_per_block: int
    total_bits: int
    lengths: np.ndarray    # uint8[256] code length of each exponent value (0 = unused)
    enc_exp: np.ndarray    # uint8[threads * 8 + 16]  EncodedExponent, MSB-first, zero padded
    sign_mant: np.ndarray  # uint8[n]                 PackedSignMantissa
    gaps: np.ndarray       # uint8[ceil(5 threads / 8) + 8]  5-bit Gaps, LSB-first
    block_out: np.ndarray  # uint64[blocks + 1]        first output index of each block

    @property
    def threads(self) -> int:
        return (self.total_bits + 63) // 64

    @property
    def blocks(self) -> int:
        return len(self.block_out) - 1

    @property
    def compressed_bytes(self) -> int:
        return (self.threads * 8 + self.n + (5 * self.threads + 7) // 8
                + self.block_out.nbytes + 256)


def huff_lengths(counts: np.ndarray, max_len: int = 32) -> np.ndarray:
    counts = np.ascontiguousarray(counts, dtype=np.uint64)
    lens = np.zeros(256, dtype=np.uint8)
    rc = lib().orc_huff_lengths(_p(counts), max_len, _p(lens))
    if rc:
        raise ValueError(ERRORS.get(rc, rc))
    return lens


def huff_canonical(lengths: np.ndarray) -> np.ndarray:
    lengths = np.ascontiguousarray(lengths, dtype=np.uint8)
    codes = np.zeros(256, dtype=np.uint32)
    lib().orc_huff_canonical(_p(lengths), _p(codes))
    return codes


def exponent_counts(w_bf16: np.ndarray) -> np.ndarray:
    e = (np.asarray(w_bf16, dtype=np.uint16).ravel() >> 7) & 0xFF
    return np.bincount(e, minlength=256).astype(np.uint64)


def huff_encode_bf16(w_bf16: np.ndarray, threads_per_block: int = 256, max_len: int = 32,
                     lengths=None) -> HuffTensor:
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16).ravel()
    n = w.size
    if lengths is None:
        lengths = huff_lengths(exponent_counts(w), max_len)
    lengths = np.ascontiguousarray(lengths, dtype=np.uint8)
    codes = huff_canonical(lengths)
    total_bits = int(lib().orc_huff_total_bits(_p(w), n, _p(lengths)))
    threads = (total_bits + 63) // 64
    blocks = (threads + threads_per_block - 1) // threads_per_block
    enc = np.zeros(threads * 8 + 16, dtype=np.uint8)
    sm = np.zeros(max(1, n), dtype=np.uint8)
    gaps = np.zeros((5 * threads + 7) // 8 + 8, dtype=np.uint8)
    block_out = np.zeros(blocks + 1, dtype=np.uint64)
    wp = _p(w) if n else _p(np.zeros(1, np.uint16))
    rc = lib().orc_huff_encode(wp, n, _p(lengths), _p(codes), threads_per_block, _p(enc),
                               _p(sm), _p(gaps), _p(block_out), threads)
    if rc:
        raise ValueError(ERRORS.get(rc, rc))
    return HuffTensor(n, 8, threads_per_block, total_bits, lengths, enc, sm[:n].copy(), gaps,
                      block_out)


def huff_decode_bf16(h: HuffTensor):
    """Plain sequential canonical decode.  Returns (status, uint16[n])."""
    out = np.zeros(max(1, h.n), dtype=np.uint16)
    sm = h.sign_mant if h.n else np.zeros(1, np.uint8)
    rc = lib().orc_huff_decode(_p(h.enc_exp), h.total_bits, _p(sm), h.n, _p(h.lengths), _p(out))
    return rc, out[:h.n]


# ----------------------------------------------------------------------------------------------
# EntroLLM-style integer weights, Huffman-coded in the DFloat11 layout
# ----------------------------------------------------------------------------------------------

INTQ_ASYM, INTQ_UNSIGNED = 0, 1


def intq_quantize(w: np.ndarray, bits: int, scheme: int):
    """Per-tensor b-bit codes: returns (codes uint8, same shape as w), bf16 scale bits, zero)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    sym = np.empty(w.shape, np.uint8)
    sc, z = C.c_uint16(), C.c_int32()
    rc = lib().orc_intq_quantize(_p(w), w.size, bits, scheme, _p(sym), C.byref(sc), C.byref(z))
    if rc:
        raise ValueError(ERRORS.get(rc, rc))
    return sym, int(sc.value), int(z.value)


def intq_dequant(sym: np.ndarray, scale: int, zero: int) -> np.ndarray:
    """bf16( (q - z) * s ), one rounding.  Returns uint16 of sym's shape."""
    sym = np.ascontiguousarray(sym, dtype=np.uint8)
    out = np.empty(sym.shape, np.uint16)
    lib().orc_intq_dequant(_p(sym), sym.size, int(scale), int(zero), _p(out))
    return out


def entrollm_quantize(w: np.ndarray, bits: int):
    """EntroLLM's per-tensor choice between unsigned and asymmetric quantisation: the scheme
    whose codes have the lower entropy (ties: asymmetric).  Returns (codes, scale, zero, scheme)."""
    best = None
    for scheme in (INTQ_ASYM, INTQ_UNSIGNED):
        sym, sc, z = intq_quantize(w, bits, scheme)
        h = entropy_bits(sym)
        if best is None or h < best[0]:
            best = (h, sym, sc, z, scheme)
    return best[1], best[2], best[3], best[4]


@dataclass
class HuffSymTensor:
    """Huffman-coded integer weights (format of the library's eq_huff_int_tensor)."""
    n: int
    bits: int
    threads_per_block: int
    total_bits: int
    lengths: np.ndarray    # uint8[256] code length of each code byte (0 = unused)
    enc: np.ndarray        # uint8[threads * 8 + 16]  the coded stream, MSB-first, zero padded
    gaps: np.ndarray       # uint8[ceil(5 threads / 8) + 8]
    block_out: np.ndarray  # uint64[blocks + 1]
    scale: int             # bf16 bits
    zero: int

    @property
    def threads(self) -> int:
        return (self.total_bits + 63) // 64

    @property
    def compressed_bytes(self) -> int:
        return self.threads * 8 + (5 * self.threads + 7) // 8 + self.block_out.nbytes + 256 + 8


def huff_encode_sym(sym: np.ndarray, bits: int, scale: int, zero: int,
                    threads_per_block: int = 256, max_len: int = 32) -> HuffSymTensor:
    s = np.ascontiguousarray(sym, dtype=np.uint8).ravel()
    n = s.size
    lengths = huff_lengths(np.bincount(s, minlength=256).astype(np.uint64), max_len)
    codes = huff_canonical(lengths)
    total_bits = int(lib().orc_huff_total_bits_sym(_p(s) if n else None, n, _p(lengths)))
    threads = (total_bits + 63) // 64
    blocks = (threads + threads_per_block - 1) // threads_per_block
    enc = np.zeros(threads * 8 + 16, dtype=np.uint8)
    gaps = np.zeros((5 * threads + 7) // 8 + 8, dtype=np.uint8)
    block_out = np.zeros(blocks + 1, dtype=np.uint64)
    rc = lib().orc_huff_encode_sym(_p(s) if n else None, n, _p(lengths), _p(codes),
                                   threads_per_block, _p(enc), _p(gaps), _p(block_out), threads)
    if rc:
        raise ValueError(ERRORS.get(rc, rc))
    return HuffSymTensor(n, bits, threads_per_block, total_bits, lengths, enc, gaps, block_out,
                         int(scale), int(zero))


def huff_decode_sym(h: HuffSymTensor):
    """Sequential canonical decode.  Returns (status, codes uint8[n])."""
    out = np.zeros(max(1, h.n), dtype=np.uint8)
    rc = lib().orc_huff_decode_sym(_p(h.enc), h.total_bits, h.n, _p(h.lengths), _p(out))
    return rc, out[:h.n]


def entrollm_decode_bf16(h: HuffSymTensor):
    """Decode and dequantise: (status, bf16 bits uint16[n])."""
    rc, sym = huff_decode_sym(h)
    return rc, intq_dequant(sym, h.scale, h.zero)


def gaps_unpack(gaps: np.ndarray, threads: int) -> np.ndarray:
    """Read the 5-bit Gap of each thread (LSB-first bit packing)."""
    bits = np.unpackbits(np.asarray(gaps, dtype=np.uint8), bitorder="little")
    idx = 5 * np.arange(threads)[:, None] + np.arange(5)[None, :]
    return (bits[idx] << np.arange(5)).sum(axis=1).astype(np.uint8)


def shannon(counts) -> float:
    c = np.asarray(counts, dtype=np.float64)
    p = c[c > 0] / c.sum()
    return float(-(p * np.log2(p)).sum())


def cross_entropy_bits(counts, freqs, prob_bits: int = PROB_BITS) -> float:
    """Bits/symbol of an ideal coder using the quantised table freqs on data with these counts."""
    c = np.asarray(counts, dtype=np.float64)
    f = np.asarray(freqs, dtype=np.float64)
    m = c > 0
    return float(-(c[m] * np.log2(f[m] / (1 << prob_bits))).sum() / c.sum())


def int8_div_for_entropy(w: np.ndarray, target_bits: float, lo: float = 0.5, hi: float = 127.0,
                         iters: int = 40) -> float:
    """Bisection on the Int8 divisor so that the quantised tensor's entropy hits target_bits."""
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        s, _ = quantize(w, INT8, mid)
        if entropy_bits(s) < target_bits:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def log2_state_bits(x: int) -> float:
    return math.log2(x)


# ----------------------------------------------------------------------------------------------
# Coded-tensor files (read independently of the library's writer, to check the format):
# magic (4 bytes) | version u32 | header length u64 | JSON header | arrays at 16-aligned offsets
# after the header.  Returns the oracle's container for the magic.
# ----------------------------------------------------------------------------------------------

def load_container(path: str):
    import json
    import struct
    with open(path, "rb") as f:
        raw = f.read()
    magic = raw[:4]
    version, hlen = struct.unpack("<IQ", raw[4:16])
    if version != 1:
        raise ValueError("unknown container version")
    head = json.loads(raw[16:16 + hlen].decode("utf-8"))
    start = 16 + hlen
    start += (-start) % 16
    arr = {}
    for name, dtype, shape, off, nbytes in head["arrays"]:
        dt = np.dtype(dtype)
        arr[name] = np.frombuffer(raw[start + off:start + off + nbytes], dt).reshape(shape).copy()
    fl = head["fields"]
    if magic == b"EQRT":
        return RansTensor(fl["rows"], fl["cols"], fl["symfmt"], fl["prob_bits"],
                          fl["chunk_symbols"], fl["streams"], fl["run"], arr["freqs"],
                          arr["states"], arr["word_off"], arr["words"], arr["scales"],
                          arr["patch_idx"], arr["patch_val"])
    if magic == b"EQHF":
        return HuffTensor(fl["n"], 8, fl["threads_per_block"], fl["total_bits"], arr["lengths"],
                          arr["enc_exp"], arr["sign_mant"], arr["gaps"], arr["block_out"])
    if magic == b"EQHI":
        return HuffSymTensor(fl["n"], fl["bits"], fl["threads_per_block"], fl["total_bits"],
                             arr["lengths"], arr["enc"], arr["gaps"], arr["block_out"],
                             fl["scale"], fl["zero"])
    raise ValueError("unknown container magic")
