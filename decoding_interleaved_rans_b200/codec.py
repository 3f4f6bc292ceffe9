"""Host-side compressor (include/eq_encode.h): numpy in, host containers out.

The pages compress once, offline; this is that step, run by libeq.so on CPU threads.  The
containers hold exactly the arrays DeviceRans.upload / DeviceHuff.upload expect.
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass, field

import numpy as np

from . import _lib as L


def _p(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


@dataclass
class HostRans:
    rows: int
    cols: int
    symfmt: int
    prob_bits: int
    chunk_symbols: int
    streams: int
    run: int
    freqs: np.ndarray
    states: np.ndarray
    word_off: np.ndarray
    words: np.ndarray
    scales: np.ndarray
    # super weights written back after decoding: flat indices (sorted), bf16 bits
    patch_idx: np.ndarray = field(default_factory=lambda: np.zeros(0, np.uint64))
    patch_val: np.ndarray = field(default_factory=lambda: np.zeros(0, np.uint16))

    @property
    def numel(self) -> int:
        return self.rows * self.cols


@dataclass
class HostHuff:
    n: int
    total_bits: int
    threads_per_block: int
    lengths: np.ndarray
    enc_exp: np.ndarray
    sign_mant: np.ndarray
    gaps: np.ndarray
    block_out: np.ndarray


def quantize(w: np.ndarray, symfmt: int, int8_div: float = 0.0, threads: int = 0):
    """Per-row AbsMax quantisation -> (symbols uint8 [rows, cols], bf16 scales uint16 [rows])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, cols = w.shape
    sym = np.empty((rows, cols), np.uint8)
    sc = np.empty(rows, np.uint16)
    L.check(L.lib().eq_quantize_host(_p(w), rows, cols, symfmt, float(int8_div), _p(sym), _p(sc),
                                     threads), "eq_quantize_host")
    return sym, sc


def super_weights(w: np.ndarray, tau: float = 20.0):
    """Super weights (|w| > tau * rms(w)): (flat indices uint64 sorted, bf16 bits uint16)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, cols = w.shape
    n = C.c_uint64()
    L.check(L.lib().eq_super_weights_host(_p(w), rows, cols, float(tau), 0, None, None,
                                          C.byref(n)), "eq_super_weights_host")
    idx = np.zeros(max(1, n.value), np.uint64)
    val = np.zeros(max(1, n.value), np.uint16)
    L.check(L.lib().eq_super_weights_host(_p(w), rows, cols, float(tau), n.value, _p(idx),
                                          _p(val), C.byref(n)), "eq_super_weights_host")
    return idx[:n.value], val[:n.value]


def quantize_excluding(w: np.ndarray, symfmt: int, int8_div: float, idx: np.ndarray,
                       threads: int = 0):
    """AbsMax quantisation with the listed positions (sorted flat indices) left out of their
    rows' scales and coded as symbol 0."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, cols = w.shape
    idx = np.ascontiguousarray(idx, dtype=np.uint64)
    sym = np.empty((rows, cols), np.uint8)
    sc = np.empty(rows, np.uint16)
    L.check(L.lib().eq_quantize_excluding_host(_p(w), rows, cols, symfmt, float(int8_div),
                                               _p(idx) if idx.size else None, idx.size, _p(sym),
                                               _p(sc), threads), "eq_quantize_excluding_host")
    return sym, sc


def rans_freqs(sym: np.ndarray, prob_bits: int = 12) -> np.ndarray:
    sym = np.ascontiguousarray(sym, dtype=np.uint8).ravel()
    f = np.zeros(256, np.uint32)
    L.check(L.lib().eq_rans_freqs_host(_p(sym) if sym.size else None, sym.size, prob_bits, _p(f)),
            "eq_rans_freqs_host")
    return f


def rans_encode(sym: np.ndarray, scales: np.ndarray, symfmt: int, chunk_symbols: int,
                streams: int, run: int, freqs=None, threads: int = 0,
                prob_bits: int = 12) -> HostRans:
    """prob_bits 12, or 8 (streams renormalise once per two steps; needs run 8).  Given freqs
    must sum to 2^prob_bits."""
    sym = np.ascontiguousarray(sym, dtype=np.uint8)
    rows, cols = sym.shape
    if freqs is None:
        freqs = rans_freqs(sym, prob_bits)
    freqs = np.ascontiguousarray(freqs, dtype=np.uint32)
    if int(freqs.sum()) != 1 << prob_bits:
        raise ValueError("freqs do not sum to 2^prob_bits")
    chunk = chunk_symbols if chunk_symbols else cols
    nchunks = (rows * cols + chunk - 1) // chunk
    states = np.empty(max(1, nchunks * streams), np.uint32)
    word_off = np.zeros(nchunks * ((streams + 31) // 32) + 1, np.uint64)
    wp, nw = C.c_void_p(), C.c_uint64()
    L.check(L.lib().eq_rans_encode_host(_p(sym) if sym.size else None, rows, cols, _p(freqs),
                                        chunk_symbols, streams, run, threads, _p(states),
                                        _p(word_off), C.byref(wp), C.byref(nw)),
            "eq_rans_encode_host")
    try:
        words = np.ctypeslib.as_array(C.cast(wp, C.POINTER(C.c_uint16)), (nw.value,)).copy()
    finally:
        L.lib().eq_free_host(wp)
    return HostRans(rows, cols, symfmt, prob_bits, chunk_symbols, streams, run, freqs,
                    states[:nchunks * streams], word_off, words,
                    np.ascontiguousarray(scales, np.uint16))


def choose_prob_bits(counts, max_loss: float = 0.005) -> int:
    """The smallest table (7, then 8 bits) that codes these symbol counts within max_loss
    (relative) of the 12-bit table's rate, else 12.  7- and 8-bit tables halve the decoder's
    renormalisation work and 7-bit ones decode two symbols per lookup; they suit low-entropy
    alphabets (a few Int8 values), not the ~6.5-bit Float8 one.  A 7-bit table holds at most 128
    symbols, an 8-bit one 256."""
    c = np.asarray(counts, dtype=np.float64).ravel()
    used = int(np.count_nonzero(c))
    if c.sum() == 0:
        return 12
    cu = np.ascontiguousarray(c, dtype=np.uint64)
    rate = {}
    for pb in (7, 8, 12):
        if used > (1 << pb):
            continue
        f = np.zeros(256, np.uint32)
        L.check(L.lib().eq_rans_normalize_host(_p(cu), pb, _p(f)), "eq_rans_normalize_host")
        m = c > 0
        rate[pb] = float(-(c[m] * np.log2(f[m] / float(1 << pb))).sum() / c.sum())
    for pb in (7, 8):
        if pb in rate and rate[pb] <= rate[12] * (1 + max_loss):
            return pb
    return 12


@dataclass
class HostHuffInt:
    """EntroLLM-style integer weights, Huffman-coded (eq_huff_int_tensor's arrays)."""
    n: int
    bits: int
    zero: int
    scale: int  # bf16 bits
    total_bits: int
    threads_per_block: int
    lengths: np.ndarray
    enc: np.ndarray
    gaps: np.ndarray
    block_out: np.ndarray


def intq_quantize(w: np.ndarray, bits: int, scheme: int):
    """Per-tensor integer codes: (codes uint8 of w's shape, bf16 scale bits, zero point)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    sym = np.empty(w.shape, np.uint8)
    sc, z = C.c_uint16(), C.c_int32()
    L.check(L.lib().eq_intq_quantize_host(_p(w) if w.size else None, w.size, bits, scheme,
                                          _p(sym) if w.size else None, C.byref(sc), C.byref(z)),
            "eq_intq_quantize_host")
    return sym, int(sc.value), int(z.value)


def _entropy(sym: np.ndarray) -> float:
    c = np.bincount(np.asarray(sym, np.uint8).ravel(), minlength=256).astype(np.float64)
    p = c[c > 0] / max(1.0, c.sum())
    return float(-(p * np.log2(p)).sum())


def entrollm_encode(w: np.ndarray, bits: int, threads_per_block: int = 256,
                    max_len: int = 32) -> HostHuffInt:
    """EntroLLM's mixed per-tensor quantisation (of the unsigned and the asymmetric scheme, the
    one whose codes have the lower entropy; ties: asymmetric), then the codes Huffman-coded."""
    best = None
    for scheme in (L.EQ_INTQ_ASYM, L.EQ_INTQ_UNSIGNED):
        q = intq_quantize(w, bits, scheme)
        h = _entropy(q[0])
        if best is None or h < best[0]:
            best = (h, q)
    sym, scale, zero = best[1]
    s = np.ascontiguousarray(sym, np.uint8).ravel()
    n = s.size
    lengths = huff_lengths(np.bincount(s, minlength=256).astype(np.uint64), max_len)
    tb = C.c_uint64()
    sp = _p(s) if n else None
    L.check(L.lib().eq_huff_sym_plan_host(sp, n, _p(lengths), C.byref(tb)), "eq_huff_sym_plan_host")
    total_bits = tb.value
    threads = (total_bits + 63) // 64
    blocks = (threads + threads_per_block - 1) // threads_per_block
    enc = np.zeros(threads * 8 + 16, np.uint8)
    gaps = np.zeros((5 * threads + 7) // 8 + 8, np.uint8)
    block_out = np.zeros(blocks + 1, np.uint64)
    L.check(L.lib().eq_huff_sym_encode_host(sp, n, _p(lengths), threads_per_block, total_bits,
                                            _p(enc), _p(gaps), _p(block_out)),
            "eq_huff_sym_encode_host")
    return HostHuffInt(n, bits, zero, scale, total_bits, threads_per_block,
                       lengths.astype(np.uint8), enc, gaps, block_out)


def huff_lengths(counts: np.ndarray, max_len: int = 32) -> np.ndarray:
    counts = np.ascontiguousarray(counts, dtype=np.uint64)
    lens = np.zeros(256, np.uint32)
    L.check(L.lib().eq_huff_lengths_host(_p(counts), max_len, _p(lens)), "eq_huff_lengths_host")
    return lens


def exponent_counts(w_bf16: np.ndarray) -> np.ndarray:
    e = (np.asarray(w_bf16, dtype=np.uint16).ravel() >> 7) & 0xFF
    return np.bincount(e, minlength=256).astype(np.uint64)


def huff_encode(w_bf16: np.ndarray, threads_per_block: int = 256, lengths=None,
                max_len: int = 32) -> HostHuff:
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16).ravel()
    n = w.size
    if lengths is None:
        lengths = huff_lengths(exponent_counts(w), max_len)
    lengths = np.ascontiguousarray(lengths, dtype=np.uint32)
    tb = C.c_uint64()
    wp = _p(w) if n else None
    L.check(L.lib().eq_huff_plan_host(wp, n, _p(lengths), C.byref(tb)), "eq_huff_plan_host")
    total_bits = tb.value
    threads = (total_bits + 63) // 64
    blocks = (threads + threads_per_block - 1) // threads_per_block
    enc = np.zeros(threads * 8 + 16, np.uint8)
    sm = np.zeros(max(1, n), np.uint8)
    gaps = np.zeros((5 * threads + 7) // 8 + 8, np.uint8)
    block_out = np.zeros(blocks + 1, np.uint64)
    L.check(L.lib().eq_huff_encode_host(wp, n, _p(lengths), threads_per_block, total_bits,
                                        _p(enc), _p(sm), _p(gaps), _p(block_out)),
            "eq_huff_encode_host")
    return HostHuff(n, total_bits, threads_per_block, lengths.astype(np.uint8), enc, sm[:n],
                    gaps, block_out)


# ------------------------------------------------------------------------------------------------
# On-disk containers (the compressed weight is the checkpoint): a versioned file holding one
# coded tensor, loadable without re-encoding.
#   bytes 0..3   magic: b"EQRT" (rANS), b"EQHF" (DFloat11), b"EQHI" (Huffman-coded integers)
#   bytes 4..7   format version (little-endian u32, currently 1)
#   bytes 8..15  header length H (u64); then H bytes of UTF-8 JSON:
#                {"fields": {scalar fields}, "arrays": [[name, dtype, shape, offset, nbytes], ...]}
#   arrays at the listed byte offsets (16-byte aligned, little-endian)
# ------------------------------------------------------------------------------------------------
import json as _json

_MAGIC = {HostRans: b"EQRT", HostHuff: b"EQHF", HostHuffInt: b"EQHI"}
_KIND = {v: k for k, v in _MAGIC.items()}
_ARRAYS = {HostRans: ("freqs", "states", "word_off", "words", "scales", "patch_idx", "patch_val"),
           HostHuff: ("lengths", "enc_exp", "sign_mant", "gaps", "block_out"),
           HostHuffInt: ("lengths", "enc", "gaps", "block_out")}
CONTAINER_VERSION = 1


def save(path: str, h) -> None:
    """Write one coded tensor (HostRans, HostHuff or HostHuffInt) to `path`."""
    cls = type(h)
    if cls not in _MAGIC:
        raise TypeError(f"cannot save {cls.__name__}")
    names = _ARRAYS[cls]
    fields = {k: int(v) for k, v in vars(h).items() if k not in names}
    arrays, blobs, off = [], [], 0
    for nm in names:
        a = np.ascontiguousarray(getattr(h, nm))
        arrays.append([nm, a.dtype.str, list(a.shape), off, a.nbytes])
        blobs.append((off, a))
        off = (off + a.nbytes + 15) // 16 * 16
    head = _json.dumps({"fields": fields, "arrays": arrays}).encode()
    base = (16 + len(head) + 15) // 16 * 16
    with open(path, "wb") as f:
        f.write(_MAGIC[cls] + np.uint32(CONTAINER_VERSION).tobytes()
                + np.uint64(len(head)).tobytes() + head)
        f.write(b"\0" * (base - 16 - len(head)))
        for o, a in blobs:
            f.seek(base + o)
            f.write(a.tobytes())


def load(path: str):
    """Read a container written by save()."""
    with open(path, "rb") as f:
        raw = f.read()
    cls = _KIND.get(raw[:4])
    if cls is None:
        raise ValueError("not a coded-tensor file")
    ver = int(np.frombuffer(raw[4:8], np.uint32)[0])
    if ver != CONTAINER_VERSION:
        raise ValueError(f"container version {ver}, expected {CONTAINER_VERSION}")
    hl = int(np.frombuffer(raw[8:16], np.uint64)[0])
    head = _json.loads(raw[16:16 + hl].decode())
    base = (16 + hl + 15) // 16 * 16
    kw = dict(head["fields"])
    for nm, dt, shape, off, nb in head["arrays"]:
        kw[nm] = np.frombuffer(raw, dtype=np.dtype(dt), count=nb // np.dtype(dt).itemsize,
                               offset=base + off).reshape(shape).copy()
    return cls(**kw)
