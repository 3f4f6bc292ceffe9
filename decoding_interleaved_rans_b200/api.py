"""Python face of the C ABI: device-resident coded tensors and the four decode calls.

PyTorch supplies device memory and the current stream; the library's kernels do all the work.
Every wrapper passes raw pointers and the stream handle to libeq.so and checks the returned
status; nothing here computes a decoded value.
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass

import numpy as np
import torch

from . import _lib as L


def _stream(stream) -> C.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t: torch.Tensor | None) -> C.c_void_p:
    return C.c_void_p(0 if t is None else t.data_ptr())


def _dev(a: np.ndarray, device, as_dtype) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    return torch.from_numpy(a.view(as_dtype)).to(device, non_blocking=False)


def table_bytes(kind: int) -> int:
    return int(L.lib().eq_table_bytes(kind))


def build_tables(kind: int, host_in, prob_bits: int, d_tables: torch.Tensor, stream=None) -> None:
    """eq_build_tables: frequencies (rANS) or code lengths (Huffman) -> device tables."""
    arr = (C.c_uint32 * 256)(*[int(v) for v in np.asarray(host_in).ravel()[:256]])
    L.check(L.lib().eq_build_tables(kind, arr, prob_bits, _ptr(d_tables), _stream(stream)),
            "eq_build_tables")


def new_status(device) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def rans_table_kind(prob_bits: int, symfmt: int) -> int:
    """12-bit tables decode through a slot table of symbols; 8-bit ones through a slot table and
    7-bit ones through a pair table, both carrying the symbols' values (one kind per format)."""
    e4 = symfmt == L.EQ_SYM_E4M3
    if prob_bits == 7:
        return L.EQ_TABLE_RANS_PAIR_E4M3 if e4 else L.EQ_TABLE_RANS_PAIR_INT8
    if prob_bits == 8:
        return L.EQ_TABLE_RANS8_E4M3 if e4 else L.EQ_TABLE_RANS8_INT8
    return L.EQ_TABLE_RANS


@dataclass
class DeviceRans:
    """An interleaved-rANS-coded weight resident in device memory (eq_rans_tensor)."""
    rows: int
    cols: int
    symfmt: int
    prob_bits: int
    chunk_symbols: int
    streams: int
    run: int
    num_chunks: int
    states: torch.Tensor
    word_off: torch.Tensor
    words: torch.Tensor
    scales: torch.Tensor
    tables: torch.Tensor
    patch_idx: torch.Tensor | None = None  # super weights: int64 flat indices, sorted
    patch_val: torch.Tensor | None = None  # their bf16 bits (int16)

    @property
    def numel(self) -> int:
        return self.rows * self.cols

    @property
    def n_patch(self) -> int:
        return 0 if self.patch_idx is None else int(self.patch_idx.numel())

    @property
    def compressed_bytes(self) -> int:
        """Bytes the decoder reads from memory: words in use, states, offsets, scales, table and
        the super-weight list."""
        used_words = int(self.word_off[-1].item()) if self.num_chunks else 0
        return (2 * used_words + 4 * self.states.numel() + 8 * self.word_off.numel()
                + 2 * self.scales.numel() + 256 * 2 + 10 * self.n_patch)

    def desc(self) -> L.RansTensorDesc:
        chunk = self.chunk_symbols if self.chunk_symbols else self.cols
        npatch = self.n_patch
        return L.RansTensorDesc(L.EQ_ABI_VERSION, self.symfmt, self.rows, self.cols,
                                self.prob_bits, chunk, self.streams, self.run, self.num_chunks,
                                self.states.data_ptr(), self.word_off.data_ptr(),
                                self.words.data_ptr(), self.scales.data_ptr(),
                                self.tables.data_ptr(), npatch,
                                self.patch_idx.data_ptr() if npatch else None,
                                self.patch_val.data_ptr() if npatch else None)

    @classmethod
    def upload(cls, h, device="cuda", stream=None) -> "DeviceRans":
        """Copy a host container (fields rows, cols, symfmt, prob_bits, chunk_symbols, streams,
        run, freqs, states, word_off, words, scales) to the device and build its table."""
        words = np.ascontiguousarray(h.words, dtype=np.uint16)
        if words.size % 8:
            words = np.concatenate([words, np.zeros(8 - words.size % 8, np.uint16)])
        if words.size == 0:
            words = np.zeros(8, np.uint16)
        chunk = int(h.chunk_symbols) if h.chunk_symbols else int(h.cols)
        nchunks = (int(h.rows) * int(h.cols) + chunk - 1) // chunk
        assert len(h.word_off) == nchunks * ((int(h.streams) + 31) // 32) + 1, "word_off length"
        t = cls(int(h.rows), int(h.cols), int(h.symfmt), int(h.prob_bits), int(h.chunk_symbols),
                int(h.streams), int(h.run), nchunks,
                _dev(np.asarray(h.states, np.uint32), device, np.int32),
                _dev(np.asarray(h.word_off, np.uint64), device, np.int64),
                _dev(words, device, np.int16),
                _dev(np.asarray(h.scales, np.uint16), device, np.int16),
                torch.empty(table_bytes(rans_table_kind(int(h.prob_bits), int(h.symfmt))),
                            dtype=torch.uint8, device=device))
        build_tables(rans_table_kind(t.prob_bits, t.symfmt), h.freqs, t.prob_bits, t.tables, stream)
        pidx = getattr(h, "patch_idx", None)
        if pidx is not None and len(pidx):
            t.patch_idx = _dev(np.asarray(pidx, np.uint64), device, np.int64)
            t.patch_val = _dev(np.asarray(h.patch_val, np.uint16), device, np.int16)
        return t


@dataclass
class DeviceHuff:
    """A DFloat11-coded bf16 weight resident in device memory (eq_huff_tensor)."""
    n: int
    total_bits: int
    bytes_per_thread: int
    threads_per_block: int
    enc_exp: torch.Tensor
    sign_mant: torch.Tensor
    gaps: torch.Tensor
    block_out: torch.Tensor
    tables: torch.Tensor

    @property
    def threads(self) -> int:
        return (self.total_bits + 63) // 64

    @property
    def compressed_bytes(self) -> int:
        return (8 * self.threads + self.n + (5 * self.threads + 7) // 8
                + 8 * self.block_out.numel() + 256)

    def desc(self) -> L.HuffTensorDesc:
        return L.HuffTensorDesc(self.n, self.total_bits, self.bytes_per_thread,
                                self.threads_per_block, self.enc_exp.data_ptr(),
                                self.sign_mant.data_ptr(), self.gaps.data_ptr(),
                                self.block_out.data_ptr(), self.tables.data_ptr())

    @classmethod
    def upload(cls, h, device="cuda", stream=None) -> "DeviceHuff":
        """Copy a host container (fields n, total_bits, threads_per_block, lengths, enc_exp,
        sign_mant, gaps, block_out) to the device and build its tables."""
        sm = np.asarray(h.sign_mant, np.uint8)
        if sm.size == 0:
            sm = np.zeros(16, np.uint8)
        t = cls(int(h.n), int(h.total_bits), 8, int(h.threads_per_block),
                _dev(np.asarray(h.enc_exp, np.uint8), device, np.uint8),
                _dev(sm, device, np.uint8),
                _dev(np.asarray(h.gaps, np.uint8), device, np.uint8),
                _dev(np.asarray(h.block_out, np.uint64), device, np.int64),
                torch.empty(table_bytes(L.EQ_TABLE_HUFF), dtype=torch.uint8, device=device))
        build_tables(L.EQ_TABLE_HUFF, h.lengths, 0, t.tables, stream)
        return t


@dataclass
class DeviceHuffInt:
    """EntroLLM-style Huffman-coded integer weights resident in device memory
    (eq_huff_int_tensor)."""
    n: int
    total_bits: int
    threads_per_block: int
    bits: int
    zero: int
    scale: int  # bf16 bits
    enc: torch.Tensor
    gaps: torch.Tensor
    block_out: torch.Tensor
    tables: torch.Tensor

    @property
    def threads(self) -> int:
        return (self.total_bits + 63) // 64

    @property
    def compressed_bytes(self) -> int:
        return (8 * self.threads + (5 * self.threads + 7) // 8 + 8 * self.block_out.numel()
                + 256 + 8)

    def desc(self) -> L.HuffIntTensorDesc:
        return L.HuffIntTensorDesc(self.n, self.total_bits, 8, self.threads_per_block,
                                   self.enc.data_ptr(), self.gaps.data_ptr(),
                                   self.block_out.data_ptr(), self.tables.data_ptr(), self.bits,
                                   self.zero, self.scale, 0, 0)

    @classmethod
    def upload(cls, h, device="cuda", stream=None) -> "DeviceHuffInt":
        """Copy a host container (fields n, total_bits, threads_per_block, bits, zero, scale,
        lengths, enc, gaps, block_out) to the device and build its tables."""
        t = cls(int(h.n), int(h.total_bits), int(h.threads_per_block), int(h.bits), int(h.zero),
                int(h.scale), _dev(np.asarray(h.enc, np.uint8), device, np.uint8),
                _dev(np.asarray(h.gaps, np.uint8), device, np.uint8),
                _dev(np.asarray(h.block_out, np.uint64), device, np.int64),
                torch.empty(table_bytes(L.EQ_TABLE_HUFF), dtype=torch.uint8, device=device))
        build_tables(L.EQ_TABLE_HUFF, h.lengths, 0, t.tables, stream)
        return t


def huff_int_decode(h: DeviceHuffInt, out=None, status=None, stream=None):
    """eq_huff_int_decode: Huffman-coded integer codes -> bf16 [n]."""
    dev = h.enc.device
    if out is None:
        out = torch.empty(max(h.n, 1), dtype=torch.bfloat16, device=dev)[:h.n]
    if status is None:
        status = new_status(dev)
    d = h.desc()
    L.check(L.lib().eq_huff_int_decode(C.byref(d), _ptr(out), _ptr(status), _stream(stream)),
            "eq_huff_int_decode")
    return out, status


def decode(tensors, outs=None, status=None, stream=None):
    """eq_decode over a list of DeviceRans.  Returns (list of bf16 outputs, status tensor)."""
    tensors = list(tensors)
    dev = tensors[0].words.device
    if outs is None:
        outs = [torch.empty(t.rows, t.cols, dtype=torch.bfloat16, device=dev) for t in tensors]
    if status is None:
        status = new_status(dev)
    descs = (L.RansTensorDesc * len(tensors))(*[t.desc() for t in tensors])
    ptrs = (C.c_void_p * len(tensors))(*[o.data_ptr() for o in outs])
    L.check(L.lib().eq_decode(descs, len(tensors), ptrs, _ptr(status), _stream(stream)),
            "eq_decode")
    return outs, status


@dataclass
class PinnedRans:
    """A coded weight's arrays in pinned host memory, the source of decode_from_host."""
    states: torch.Tensor    # int32 [num_chunks * streams]
    word_off: torch.Tensor  # int64 [units + 1]
    words: torch.Tensor     # int16, padded to a multiple of 8 words
    scales: torch.Tensor    # int16 (bf16 bits) [rows]
    offsets: np.ndarray     # word_off as numpy, to find each piece's word range on the host

    @classmethod
    def from_host(cls, h) -> "PinnedRans":
        words = np.ascontiguousarray(h.words, dtype=np.uint16)
        if words.size % 8 or words.size == 0:
            words = np.concatenate([words, np.zeros(8 - words.size % 8, np.uint16)])
        pin = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a).view(dt)).pin_memory()  # noqa: E731
        return cls(pin(np.asarray(h.states, np.uint32), np.int32),
                   pin(np.asarray(h.word_off, np.uint64), np.int64), pin(words, np.int16),
                   pin(np.asarray(h.scales, np.uint16), np.int16),
                   np.asarray(h.word_off, np.uint64).copy())

    @classmethod
    def from_device(cls, t: "DeviceRans") -> "PinnedRans":
        """Pinned host copies of a device container's coded arrays."""
        def pin(x: torch.Tensor) -> torch.Tensor:
            h = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
            h.copy_(x)
            return h
        wo = pin(t.word_off)
        return cls(pin(t.states), wo, pin(t.words), pin(t.scales), wo.numpy().view(np.uint64).copy())

    def h2d_bytes(self) -> int:
        return sum(x.numel() * x.element_size() for x in (self.states, self.word_off, self.words, self.scales))


def decode_from_host(t: DeviceRans, src: PinnedRans, out: torch.Tensor, status=None, stream=None,
                     pieces: int = 1, copy_stream=None):
    """eq_decode_from_host: decode a coded weight straight from pinned host memory.  Its arrays
    are copied into the device container t (same layout, table already built) piece by piece on
    copy_stream, each piece a run of whole chunks ending on a row boundary, and each piece
    decodes on `stream` as soon as its copy has landed.  Returns (out, status)."""
    dev = t.words.device
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    if copy_stream is None:
        copy_stream = torch.cuda.Stream(dev)
    if status is None:
        status = new_status(dev)
    assert out.dtype == torch.bfloat16 and out.is_contiguous() and out.numel() == t.numel
    assert t.words.numel() >= src.words.numel()
    d = t.desc()
    L.check(L.lib().eq_decode_from_host(C.byref(d), _ptr(src.states), _ptr(src.word_off),
                                        _ptr(src.words), src.words.numel(), _ptr(src.scales),
                                        int(pieces), _ptr(out), _ptr(status), _stream(stream),
                                        _stream(copy_stream)), "eq_decode_from_host")
    return out, status


def decode_gemv(t: DeviceRans, x: torch.Tensor, y=None, status=None, stream=None):
    """eq_decode_gemv: y[b] = W x[b] with W decoded on chip.  x bf16 [batch, cols]."""
    assert x.dtype == torch.bfloat16 and x.is_contiguous() and x.shape[-1] == t.cols
    batch = x.shape[0]
    if y is None:
        y = torch.empty(batch, t.rows, dtype=torch.float32, device=x.device)
    if status is None:
        status = new_status(x.device)
    d = t.desc()
    L.check(L.lib().eq_decode_gemv(C.byref(d), _ptr(x), batch, _ptr(y), _ptr(status),
                                   _stream(stream)), "eq_decode_gemv")
    return y, status


def mlp_scratch_bytes(inter: int, batch: int) -> int:
    return int(L.lib().eq_mlp_scratch_bytes(inter, batch))


def mlp_decode(gate: DeviceRans, up: DeviceRans, down: DeviceRans, x: torch.Tensor, y=None,
               scratch=None, status=None, stream=None):
    """eq_mlp_decode: y[b] = W_down(silu(W_gate x[b]) * (W_up x[b])) from coded weights."""
    assert x.dtype == torch.bfloat16 and x.is_contiguous() and x.shape[-1] == gate.cols
    batch = x.shape[0]
    if y is None:
        y = torch.empty(batch, down.rows, dtype=torch.float32, device=x.device)
    nbytes = mlp_scratch_bytes(gate.rows, batch)
    if scratch is None:
        scratch = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
    if status is None:
        status = new_status(x.device)
    dg, du, dd = gate.desc(), up.desc(), down.desc()
    L.check(L.lib().eq_mlp_decode(C.byref(dg), C.byref(du), C.byref(dd), _ptr(x), batch, _ptr(y),
                                  _ptr(scratch), scratch.numel() * scratch.element_size(),
                                  _ptr(status), _stream(stream)), "eq_mlp_decode")
    return y, status


def selftest_bounded_wait(status=None, stream=None, device="cuda"):
    """eq_selftest_bounded_wait: a wait for a copy that never lands ends, after about a second,
    with EQ_DEV_TIMEOUT in the status word."""
    if status is None:
        status = new_status(device)
    L.check(L.lib().eq_selftest_bounded_wait(_ptr(status), _stream(stream)),
            "eq_selftest_bounded_wait")
    return status


def huff_bf16_decode(h: DeviceHuff, out=None, status=None, stream=None):
    """eq_huff_bf16_decode: DFloat11 -> bf16 [n]."""
    dev = h.enc_exp.device
    if out is None:
        out = torch.empty(max(h.n, 1), dtype=torch.bfloat16, device=dev)[:h.n]
    if status is None:
        status = new_status(dev)
    d = h.desc()
    L.check(L.lib().eq_huff_bf16_decode(C.byref(d), _ptr(out), _ptr(status), _stream(stream)),
            "eq_huff_bf16_decode")
    return out, status


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 patterns of a bf16 tensor (device or host)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


# ------------------------------------------------------------------------------------------------
# GPU compressor (include/eq_encode.h, *_device calls)
# ------------------------------------------------------------------------------------------------

def quantize_device(w: torch.Tensor, symfmt: int, int8_div: float = 0.0, stream=None):
    """Per-row AbsMax quantisation on the GPU: fp32 [rows, cols] -> (uint8 symbols, bf16 scales
    as int16 bits)."""
    assert w.dtype == torch.float32 and w.is_cuda and w.is_contiguous() and w.dim() == 2
    rows, cols = w.shape
    sym = torch.empty(rows, cols, dtype=torch.uint8, device=w.device)
    sc = torch.empty(rows, dtype=torch.int16, device=w.device)
    L.check(L.lib().eq_quantize_device(_ptr(w), rows, cols, symfmt, float(int8_div), _ptr(sym),
                                       _ptr(sc), _stream(stream)), "eq_quantize_device")
    return sym, sc


def histogram_device(sym: torch.Tensor, stream=None) -> torch.Tensor:
    counts = torch.zeros(256, dtype=torch.int32, device=sym.device)
    L.check(L.lib().eq_histogram_device(_ptr(sym), sym.numel(), _ptr(counts), _stream(stream)),
            "eq_histogram_device")
    return counts


def normalize_freqs(counts, prob_bits: int = 12) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(counts).astype(np.uint64))
    f = np.zeros(256, np.uint32)
    L.check(L.lib().eq_rans_normalize_host(c.ctypes.data, prob_bits, f.ctypes.data),
            "eq_rans_normalize_host")
    return f


def rans_encode_device(sym: torch.Tensor, scales: torch.Tensor, symfmt: int, chunk_symbols: int,
                       streams: int, run: int, freqs=None, status=None,
                       stream=None, prob_bits: int = 12) -> "DeviceRans":
    """Encode a device symbol matrix on the GPU into a DeviceRans (plan, offsets, encode).
    prob_bits 12, or 8 (needs run 8 and cols % 8 == 0)."""
    assert sym.dtype == torch.uint8 and sym.is_cuda and sym.is_contiguous() and sym.dim() == 2
    rows, cols = sym.shape
    dev = sym.device
    if freqs is None:
        freqs = normalize_freqs(histogram_device(sym, stream).cpu().numpy(), prob_bits)
    f = (C.c_uint32 * 256)(*[int(v) for v in np.asarray(freqs).ravel()[:256]])
    chunk = chunk_symbols if chunk_symbols else cols
    nchunks = (rows * cols + chunk - 1) // chunk
    units = nchunks * (streams // 32)
    states = torch.empty(max(1, nchunks * streams), dtype=torch.int32, device=dev)
    word_off = torch.empty(units + 1, dtype=torch.int64, device=dev)
    if status is None:
        status = new_status(dev)
    L.check(L.lib().eq_rans_plan_device(_ptr(sym), rows, cols, f, chunk_symbols, streams, run,
                                        _ptr(states), _ptr(word_off), _ptr(status),
                                        _stream(stream)), "eq_rans_plan_device")
    total = int(word_off[-1].item())
    words = torch.zeros(max(8, (total + 7) // 8 * 8), dtype=torch.int16, device=dev)
    L.check(L.lib().eq_rans_encode_device(_ptr(sym), rows, cols, f, chunk_symbols, streams, run,
                                          _ptr(word_off), _ptr(words), _ptr(status),
                                          _stream(stream)), "eq_rans_encode_device")
    t = DeviceRans(rows, cols, symfmt, prob_bits, chunk_symbols, streams, run, nchunks,
                   states[:nchunks * streams] if nchunks else states, word_off, words,
                   scales, torch.empty(table_bytes(rans_table_kind(prob_bits, symfmt)),
                                       dtype=torch.uint8, device=dev))
    build_tables(rans_table_kind(prob_bits, symfmt), freqs, prob_bits, t.tables, stream)
    return t
