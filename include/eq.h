/*
 * eq.h -- C ABI of the B200 (sm_100a) entropy-coded weight decoder.
 *
 * The library turns entropy-coded LLM weights that live in device memory back into bf16, or
 * multiplies them straight from their coded form:
 *
 *   eq_build_tables      frequency table or Huffman code lengths -> device decode tables
 *   eq_decode            interleaved-rANS Float8-E4M3 / Int8 symbols -> bf16 weights
 *   eq_decode_gemv       interleaved-rANS weights times activations, y = W x, W never in HBM
 *   eq_huff_bf16_decode  DFloat11 (Huffman-coded exponent + raw sign/mantissa) -> bf16
 *
 * Conventions shared by every call:
 *   - Every pointer inside a tensor descriptor is DEVICE memory owned by the caller; the library
 *     never allocates, frees or keeps device memory, and keeps no pointer after the call.
 *   - Descriptors and other host arguments are read during the call and may be freed when it
 *     returns.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL = legacy default
 *     stream).  Nothing synchronises the host.
 *   - Argument and format errors found on the host return an eq_status without launching.
 *     A failed launch returns EQ_ERR_CUDA.
 *   - Corrupt data is reported on the device: the kernels OR EQ_DEV_* bits into *d_status (a
 *     caller-zeroed uint32 in device memory) and never trap.  Output written for a chunk whose
 *     status bit is set is unspecified.
 *
 * Where the pages leave a format open, the reading used is stated at the field.
 */
#ifndef EQ_H
#define EQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define EQ_ABI_VERSION 3u

typedef enum {
  EQ_OK = 0,
  EQ_ERR_ARG = 1,         /* a pointer is NULL, a size is out of range, or fields disagree */
  EQ_ERR_FORMAT = 2,      /* a table or header violates the coded format                   */
  EQ_ERR_UNSUPPORTED = 3, /* valid format, but outside what this build decodes              */
  EQ_ERR_CUDA = 4         /* a CUDA call or launch failed                                   */
} eq_status;

/* device-side status bits, OR-ed into *d_status */
#define EQ_DEV_CORRUPT_STATE 1u  /* a rANS stream did not end in state 2^16                   */
#define EQ_DEV_OVERRUN 2u        /* a chunk asked for more words / bits than it holds         */
#define EQ_DEV_BAD_CODE 4u       /* Huffman: a bit pattern matches no code                    */
#define EQ_DEV_COUNT_MISMATCH 8u /* Huffman: codes found in a block differ from block_out     */
#define EQ_DEV_TIMEOUT 16u       /* a bounded wait on an asynchronous copy gave up            */

typedef enum { EQ_SYM_E4M3 = 1, EQ_SYM_INT8 = 2 } eq_symfmt;
typedef enum {
  EQ_TABLE_RANS = 1,
  EQ_TABLE_HUFF = 2,
  EQ_TABLE_RANS_PAIR_E4M3 = 3, /* 7-bit pair table carrying the symbols' Float8-E4M3 values */
  EQ_TABLE_RANS_PAIR_INT8 = 4, /* 7-bit pair table carrying the symbols' Int8 values         */
  EQ_TABLE_RANS8_E4M3 = 5,     /* 8-bit slot table carrying the symbols' Float8-E4M3 values */
  EQ_TABLE_RANS8_INT8 = 6      /* 8-bit slot table carrying the symbols' Int8 values         */
} eq_table_kind;

/*
 * One interleaved-rANS-coded weight W[rows][cols] ("Float8@2bits: Entropy Coding Enables
 * Data-Free Model Compression", summary sections "Codificacion de Pesos" and "Decodificacion en
 * Tiempo de Inferencia": the optimised weights, Float8-E4M3 or Int8 symbols with one scale per
 * output channel, are flattened into one symbol stream and ANS-coded; a parallel ANS decoder
 * restores them on the GPU before the layer runs).  The pages fix no rANS variant; this one is:
 *
 *   probabilities M = 2^prob_bits (prob_bits = 12, 8 or 7), state x in [2^16, 2^32), 16-bit words.
 *   The row-major symbol stream is cut into chunks of chunk_symbols symbols (the last one may be
 *   shorter); chunk c is coded on its own by `streams` interleaved rANS states.  Inside a chunk,
 *   symbol j belongs to run r = j / run, stream r % streams, round r / streams, position j % run;
 *   the decoder visits (round, position, stream) in increasing order and skips streams that hold
 *   no symbol at that step.  The streams form groups of 32 (group g = streams 32g .. 32g + 31);
 *   each group reads its own word substream, so the groups of a chunk decode independently.
 *   Decoding symbol s from x: slot = x mod M, s is the symbol with cum[s] <= slot < cum[s] +
 *   freq[s], x = freq[s] * (x / M) + slot - cum[s].  At a renormalisation point, if x < 2^16,
 *   x = x * 2^16 + the next word of the stream's group.  A 12-bit stream has a renormalisation
 *   point after each of its steps; an 8- or 7-bit stream after every second one of its own
 *   steps (and after its last), which is exact because two such steps shrink the state by at
 *   most 2^16; it halves the renormalisation work.  A 7-bit table also decodes both steps of a
 *   pair with one lookup (EQ_TABLE_RANS_PAIR_E4M3 / _INT8).  A well-formed chunk ends with every
 *   state at 2^16 and every word read.
 *   Dequantisation: out = bf16_rne( value(s) * scale[row] ), value(s) being the E4M3 value of the
 *   byte (NaN codes 0x7F/0xFF give the bf16 quiet NaN 0x7FC0 / 0xFFC0) or the byte read as int8.
 *   Scales are finite (the quantisers make them so); with an infinite or NaN scale a product that
 *   is NaN comes out as some bf16 NaN.
 *   Super weights ("Float8@2bits" summary, "Manejo de Pesos Superiores": extreme outliers of Int8
 *   weights kept out of the entropy coding): an optional sorted list of (flat index, bf16 value)
 *   written over the decoded weight.  The coded symbol at a listed position must dequantise to
 *   zero (the quantiser codes it as 0); eq_decode reports EQ_DEV_CORRUPT_STATE otherwise, and
 *   eq_decode_gemv adds value * x for each listed weight.
 */
typedef struct {
  uint32_t version;       /* EQ_ABI_VERSION                                                    */
  uint32_t symfmt;        /* eq_symfmt                                                         */
  uint32_t rows, cols;    /* W is rows x cols, row-major; rows*cols < 2^40                     */
  uint32_t prob_bits;     /* 12, or 8 or 7 (then run must be 8)                                 */
  uint32_t chunk_symbols; /* symbols per chunk (>= 1); a multiple of `run`                     */
  uint32_t streams;       /* interleaved states per chunk: a multiple of 32, at most 1024      */
  uint32_t run;           /* consecutive symbols per stream visit: 1 or 8; 8 needs cols % 8 == 0 */
  uint64_t num_chunks;    /* ceil(rows * cols / chunk_symbols)                                 */
  const uint32_t *states; /* [num_chunks][streams] final encoder states                         */
  const uint64_t *word_off; /* [num_chunks * streams / 32 + 1]: substream (c, g) is words
                             [word_off[c * streams / 32 + g], word_off[... + 1])                */
  const uint16_t *words;  /* all substreams, chunk-major, decoder order; allocation padded with
                             zeros to a multiple of 8 words (16 bytes); base 16-byte aligned    */
  const uint16_t *scales; /* [rows] bf16 per-output-channel scales                              */
  const void *tables;     /* from eq_build_tables: EQ_TABLE_RANS for 12-bit tables,
                             EQ_TABLE_RANS8_E4M3 / _INT8 for 8-bit ones and
                             EQ_TABLE_RANS_PAIR_E4M3 / _INT8 for 7-bit ones (the kind matching
                             symfmt); 16-byte aligned                                         */
  uint64_t n_patch;       /* super weights in the list (0: none)                               */
  const uint64_t *patch_idx; /* [n_patch] flat row-major indices, strictly increasing           */
  const uint16_t *patch_val; /* [n_patch] their bf16 values                                     */
} eq_rans_tensor;

/*
 * One DFloat11-coded bf16 weight (DFloat11 page, "Formato DFloat11": the 8-bit exponent is
 * Huffman-coded and bit-packed into EncodedExponent, sign and mantissa stay raw in
 * PackedSignMantissa; "Kernels GPU de 2 etapas y metadatos auxiliares": each thread owns 8
 * contiguous bytes of EncodedExponent and decodes the codes that start there, Gaps gives each
 * thread's first code offset in 5 bits, and one output position is stored per thread block).
 *
 *   exponent e = bits 14..7 of the bf16; PackedSignMantissa byte = sign << 7 | low 7 bits.
 *   Codes are canonical (symbols ordered by (length, value) get consecutive codes), written
 *   MSB-first from bit 0 of byte 0.  Thread t owns bits [64 t, 64 t + 64); Gap[t] is the offset
 *   from 64 t of the first code starting at or after 64 t (0..31, 5 bits, LSB-first packing).
 *   threads = ceil(total_bits / 64); blocks = ceil(threads / threads_per_block);
 *   block_out[b] = index of the first weight decoded by block b; block_out[blocks] = n.
 */
typedef struct {
  uint64_t n;                  /* number of bf16 weights                                      */
  uint64_t total_bits;         /* length of the code stream in bits                           */
  uint32_t bytes_per_thread;   /* 8                                                           */
  uint32_t threads_per_block;  /* 32..512, a multiple of 32 (256 is the usual choice)          */
  const uint8_t *enc_exp;      /* EncodedExponent, threads * 8 bytes + 16 zero bytes           */
  const uint8_t *sign_mant;    /* PackedSignMantissa [n]                                      */
  const uint8_t *gaps;         /* ceil(5 threads / 8) bytes + 8 zero bytes                    */
  const uint64_t *block_out;   /* [blocks + 1]                                                */
  const void *tables;          /* eq_table_bytes(EQ_TABLE_HUFF) bytes from eq_build_tables(HUFF) */
} eq_huff_tensor;

/*
 * EntroLLM-style integer weights (EntroLLM page, "Metodologia": per-tensor unsigned or
 * asymmetric integer quantisation, the codes Huffman-coded and decoded in parallel): n codes of
 * `bits` bits, Huffman-coded in the layout of eq_huff_tensor with the code bytes in place of the
 * exponents and no sign/mantissa stream.  Code q decodes to bf16_rne((q - zero) * scale); the
 * product is exact in fp32, so that is the only rounding.
 */
typedef struct {
  uint64_t n;                  /* number of weights                                            */
  uint64_t total_bits;         /* bits in the coded stream                                     */
  uint32_t bytes_per_thread;   /* 8                                                             */
  uint32_t threads_per_block;  /* 32 .. 512, a multiple of 32                                  */
  const uint8_t *enc;          /* the coded stream, MSB-first, threads * 8 + 16 bytes (zero
                                  padded), 8-byte aligned                                       */
  const uint8_t *gaps;         /* 5-bit Gap of each 64-bit thread segment, LSB-first packing   */
  const uint64_t *block_out;   /* first output index of each block of threads, then n          */
  const void *tables;          /* eq_build_tables(EQ_TABLE_HUFF) from the codes' lengths        */
  uint32_t bits;               /* 8 or 4; a decoded code above 2^bits - 1 sets EQ_DEV_BAD_CODE  */
  int32_t zero;                /* zero point, 0 .. 2^bits                                      */
  uint16_t scale;              /* bf16 scale                                                   */
  uint16_t reserved16;
  uint32_t reserved32;
} eq_huff_int_tensor;

/* Bytes of device memory eq_build_tables writes for `kind` (0 for an unknown kind). */
size_t eq_table_bytes(eq_table_kind kind);

/*
 * Build the device decode tables of one tensor into d_tables (eq_table_bytes(kind) bytes,
 * 16-byte aligned, caller-owned).  The table contents travel as kernel arguments: no host
 * buffer outlives the call and no copy engine is used.
 *   EQ_TABLE_RANS: host_in[256] = symbol frequencies, summing to 4096 (prob_bits = 12).
 *     Builds the slot table: one 32-bit entry per slot holding the slot's symbol, its frequency
 *     and slot - cum[symbol].
 *   EQ_TABLE_RANS8_E4M3 / EQ_TABLE_RANS8_INT8: host_in[256] = frequencies summing to 256
 *     (prob_bits = 8).  Builds the 8-bit slot table: one 32-bit entry per slot holding the
 *     frequency, slot - cum[symbol] and, instead of the symbol, its value as bf16 (exact) in the
 *     symbol format the kind names, so that two decoded symbols dequantise with one bf16x2
 *     multiply by the row scale.
 *   EQ_TABLE_RANS_PAIR_E4M3 / EQ_TABLE_RANS_PAIR_INT8: host_in[256] = frequencies summing to
 *     128 (prob_bits = 7).  Builds the pair table (16384 x 8 bytes): for each value of the
 *     state's low 14 bits, the values (as bf16, exact) of the two symbols the next two steps
 *     decode, in the symbol format the kind names, and the two steps' combined product and
 *     offset, so a pair of steps is one lookup and one multiply-add and its dequantisation one
 *     bf16x2 multiply by the row scale.  A tensor's table must be of its own symbol format
 *     (eq_decode reports EQ_DEV_CORRUPT_STATE otherwise).
 *   EQ_TABLE_HUFF: host_in[256] = code length of each exponent value (0 = absent), prob_bits
 *     ignored.  Builds the hierarchical lookup tables of the DFloat11 page ("Decodificacion
 *     basada en LUT jerarquicas": the code tree cut into height-8 subtrees, each a 256-entry
 *     table) and, from them, a 2048-entry window table that returns every code lying wholly in
 *     the next 11 bits (up to four) with one lookup.  EQ_ERR_FORMAT if a length exceeds 32 or the
 *     lengths violate the Kraft inequality; EQ_ERR_UNSUPPORTED if more than 32 subtables would
 *     be needed.
 */
eq_status eq_build_tables(eq_table_kind kind, const uint32_t *host_in, uint32_t prob_bits,
                          void *d_tables, void *stream);

/*
 * Decode n_tensors rANS-coded weights to bf16 (one launch per group of tensors that share
 * symfmt, run and prob_bits).  d_out[i] points to rows*cols bf16 values (16-byte aligned) for
 * tensor i; the array d_out itself is host memory.  Decoding all tensors of a transformer block
 * in one call follows the pages' block-wise decompression (DFloat11 page, "Descompresion por
 * bloque transformer"; "Float8@2bits" summary: decompression alternates with the forward
 * kernels block by block).
 */
eq_status eq_decode(const eq_rans_tensor *ts, uint32_t n_tensors, uint16_t *const *d_out,
                    uint32_t *d_status, void *stream);

/*
 * eq_decode of one tensor whose coded arrays are in host memory (pinned, for the copies to
 * overlap).  No counterpart in the pages, which keep the coded weights in GPU memory
 * ("Float8@2bits" summary, "Decodificacion en Tiempo de Inferencia"); this is the offloaded case
 * the DFloat11 page compares against.  The host arrays h_states [num_chunks * streams],
 * h_word_off [num_chunks * streams / 32 + 1], h_words [n_words] and h_scales [rows] are copied
 * into the device arrays *t points at (same layout; t->words must hold n_words words, the rest
 * as in eq_rans_tensor) piece by piece on copy_stream, each piece a run of whole chunks ending on
 * a row boundary; each piece decodes on `stream` as soon as its copy has landed, while the next
 * one is copied.  pieces: how many (1 = copy everything, then decode); a tensor with super
 * weights, or whose chunks end on a row boundary only at the end, goes in one piece.  copy_stream
 * may equal stream (nothing then overlaps).  The call returns once everything is enqueued; the
 * host arrays must stay valid until the stream's work is done.  Errors as eq_decode;
 * EQ_ERR_ARG for null host pointers or n_words below the last word offset.
 */
eq_status eq_decode_from_host(const eq_rans_tensor *t, const uint32_t *h_states,
                              const uint64_t *h_word_off, const uint16_t *h_words, uint64_t n_words,
                              const uint16_t *h_scales, uint32_t pieces, uint16_t *d_out,
                              uint32_t *d_status, void *stream, void *copy_stream);

/*
 * y[b][r] = sum_c W[r][c] * x[b][c] for b < batch, with W decoded from its rANS stream on chip
 * and never written to memory ("Float8@2bits" summary, closing section: fused decompression
 * kernels are the next step; the decoded values are consumed where they are produced).  W is
 * taken exactly as eq_decode would return it (bf16 of value * scale), products and sums in fp32.
 * x: bf16 [batch][cols], 16-byte aligned.  y: fp32 [batch][rows].  batch 1..16; for batch >= 8
 * (and chunk_symbols % 256 == 0) the product of each 16-row x 256-column decoded tile with x runs
 * on the tensor cores (mma, bf16 in, fp32 accumulate).
 * Takes 12-, 8- and 7-bit tables (the decode steps of eq_decode; a 7-bit table's pair table fills
 * most of an SM's shared memory, so one CTA per SM takes chunk after chunk).
 * Requires run == 8, streams == 32 (one warp owns a chunk, so its sums never leave the warp)
 * and whole rows per chunk (chunk_symbols a multiple of cols); a chunk of several rows also needs
 * cols % 256 == 0, so that one decode round never straddles two rows.  Otherwise
 * EQ_ERR_UNSUPPORTED.
 */
eq_status eq_decode_gemv(const eq_rans_tensor *t, const uint16_t *d_x, uint32_t batch, float *d_y,
                         uint32_t *d_status, void *stream);

/*
 * Reconstruct n bf16 weights from their DFloat11 coding, bit-exactly (DFloat11 page, "Kernels
 * GPU de 2 etapas y metadatos auxiliares": stage 1 decodes and counts, a block-wide prefix sum
 * gives every thread its output position, stage 2 decodes again into shared memory and the block
 * writes its span once, coalesced).  d_out: n bf16 values.
 */
eq_status eq_huff_bf16_decode(const eq_huff_tensor *h, uint16_t *d_out, uint32_t *d_status,
                              void *stream);

/*
 * Decode n EntroLLM-style Huffman-coded integer weights to bf16 with the two-stage kernel of
 * eq_huff_bf16_decode (same segments, Gaps, block scan and coalesced stores; the merge step
 * turns each code q into bf16((q - zero) * scale)).  d_out: n bf16 values, 16-byte aligned.
 */
eq_status eq_huff_int_decode(const eq_huff_int_tensor *h, uint16_t *d_out, uint32_t *d_status,
                             void *stream);

/*
 * Beyond the four calls: a LLaMA-style MLP block straight from coded weights,
 *   y[b] = W_down ( silu(W_gate x[b]) * (W_up x[b]) ),   silu(v) = v / (1 + e^-v),
 * with gate, up: inter x hidden and down: hidden x inter, all in eq_decode_gemv's layout; the
 * hidden activations are rounded to bf16 before the down projection.  The decoded weights never
 * reach memory ("Float8@2bits" summary, closing section: fused decompression + compute kernels).
 * d_x: bf16 [batch][hidden]; d_y: fp32 [batch][hidden]; batch 1..16; inter % 8 == 0.
 * d_scratch: device memory of at least eq_mlp_scratch_bytes(inter, batch) bytes, 256-byte
 * aligned, owned by the caller; it holds the two fp32 products and the bf16 hidden vector.
 */
size_t eq_mlp_scratch_bytes(uint32_t inter, uint32_t batch);
eq_status eq_mlp_decode(const eq_rans_tensor *gate, const eq_rans_tensor *up,
                        const eq_rans_tensor *down, const uint16_t *d_x, uint32_t batch,
                        float *d_y, void *d_scratch, size_t scratch_bytes, uint32_t *d_status,
                        void *stream);

/*
 * No counterpart in the pages: an addition for callers that cannot allocate device memory.
 * eq_mlp_decode with the scratch inside the library, for callers that can pass no scratch
 * buffer: an engine or framework that has reserved (nearly) all of HBM for its own allocator,
 * so a cudaMalloc from here would fail or eat into its pool, and hot loops that must not pay
 * for cudaMalloc / cudaFree, which can synchronise the device.  The scratch is one fixed device
 * array per device (placed by the CUDA runtime when it loads the library's code on that device)
 * sized for inter * batch <= EQ_MLP_NOALLOC_MAX_ELEMS (5 MiB); no allocating routine is called.
 * Larger sizes return EQ_ERR_UNSUPPORTED without launching.  `stream` must belong to the current
 * device (EQ_ERR_ARG otherwise): the array used is the current device's, and its address there is
 * looked up on every call (a host-side lookup that allocates nothing; it also stays right after a
 * device reset).  The first call on a device may load the library's code there, so make it before
 * any stream capture.  Every call on a device shares the array, so calls whose work may overlap
 * on the GPU (streams not ordered with one another) race: order them.  Nothing needs zeroing
 * beforehand.  Arguments, layouts and other errors as eq_mlp_decode.
 */
#define EQ_MLP_NOALLOC_MAX_ELEMS 524288u
eq_status eq_mlp_decode_noalloc(const eq_rans_tensor *gate, const eq_rans_tensor *up,
                                const eq_rans_tensor *down, const uint16_t *d_x, uint32_t batch,
                                float *d_y, uint32_t *d_status, void *stream);

/*
 * Not on the pages: a check of the library's own failure reporting.  The decode kernels wait only
 * for their own bulk copies, and every such wait gives up after about a second with
 * EQ_DEV_TIMEOUT in *d_status instead of hanging.  This launches one warp that waits, through
 * the same bounded wait, for a copy that is never issued: after about a second *d_status has
 * EQ_DEV_TIMEOUT and the context stays usable.  Nothing is left in flight.
 */
eq_status eq_selftest_bounded_wait(uint32_t *d_status, void *stream);

/* Human-readable name of a status code (static storage). */
const char *eq_status_string(eq_status s);

/* EQ_ABI_VERSION of the loaded library. */
uint32_t eq_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* EQ_H */
