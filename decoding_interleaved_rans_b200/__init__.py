"""B200-native decoding of entropy-coded LLM weights.

    eq_build_tables / eq_decode / eq_decode_gemv / eq_huff_bf16_decode   (include/eq.h)
    eq_mlp_decode / eq_huff_int_decode                                     (include/eq.h)

Two codecs from the pages: EntQuant-style interleaved rANS over Float8-E4M3 / Int8 symbols with
per-output-channel scales, and DFloat11-style bf16 with a canonical-Huffman-coded exponent.  The
decode kernels (sm_100a) live in libeq.so, built in-tree from csrc/; PyTorch only provides device
memory and streams.  The host-side compressor is in ``codec``.
"""
from ._lib import (EQ_DEV_BAD_CODE, EQ_DEV_CORRUPT_STATE, EQ_DEV_COUNT_MISMATCH,  # noqa: F401
                   EQ_DEV_OVERRUN, EQ_DEV_TIMEOUT, EQ_SYM_E4M3, EQ_SYM_INT8, EQ_TABLE_HUFF,
                   EQ_TABLE_RANS, EQ_TABLE_RANS8_E4M3, EQ_TABLE_RANS8_INT8, EQ_TABLE_RANS_PAIR_E4M3,
                   EQ_TABLE_RANS_PAIR_INT8, EXPORTS, EqError, lib)
from .api import (DeviceHuff, DeviceHuffInt, DeviceRans, PinnedRans, bf16_bits, build_tables,  # noqa: F401
                  decode, decode_from_host, decode_gemv, histogram_device, huff_bf16_decode, huff_int_decode,
                  mlp_decode, selftest_bounded_wait,
                  mlp_scratch_bytes, new_status, normalize_freqs,
                  quantize_device, rans_encode_device, table_bytes)
from . import codec  # noqa: F401
