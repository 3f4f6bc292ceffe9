/*
 * eq_encode.h -- host-side compressor of the library (the offline step that produces what the
 * decoders in eq.h consume).
 *
 * The pages compress once, offline, then keep the weights coded in GPU memory ("Float8@2bits"
 * summary, "Codificacion de Pesos": per-channel AbsMax scales, Float8/Int8 symbols, ANS over the
 * flattened stream; DFloat11 page, "Formato DFloat11": Huffman-coded bf16 exponents).  The *_host
 * calls run on the host CPU with worker threads and touch no GPU; the *_device calls at the end
 * run the rANS side on the GPU.  The formats are the ones defined in eq.h.  Arrays of the host
 * calls are host memory owned by the caller unless stated otherwise.
 */
#ifndef EQ_ENCODE_H
#define EQ_ENCODE_H

#include <stddef.h>
#include <stdint.h>

#include "eq.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Per-output-channel AbsMax quantisation of an fp32 weight w[rows][cols].
 *   E4M3: scale[r] = bf16(max_c |w[r][c]| / 448), sym = E4M3(w / scale[r]) (round to nearest even,
 *         saturating at 448).
 *   INT8: scale[r] = bf16(max_c |w[r][c]| / int8_div), sym = clamp(rne(w / scale[r]), -127, 127).
 * A row of zeros gets scale 1.0.  threads = 0 uses every available core.
 */
eq_status eq_quantize_host(const float *w, uint32_t rows, uint32_t cols, uint32_t symfmt,
                           float int8_div, uint8_t *sym, uint16_t *scales, uint32_t threads);

/*
 * Super weights ("Float8@2bits" summary, "Manejo de Pesos Superiores"): the weights with
 * |w| > tau * rms(w) (rms over the whole tensor).  Writes up to max_out flat indices (increasing)
 * and their bf16 values; *n_out = how many there are.  Call with max_out = 0 to count.
 */
eq_status eq_super_weights_host(const float *w, uint32_t rows, uint32_t cols, double tau,
                                uint64_t max_out, uint64_t *idx, uint16_t *val, uint64_t *n_out);

/*
 * eq_quantize_host with the listed positions (flat indices, strictly increasing) left out of
 * their rows' AbsMax scales; they are coded as symbol 0 (value zero), so the eq_rans_tensor
 * patch list can carry them exactly.
 */
eq_status eq_quantize_excluding_host(const float *w, uint32_t rows, uint32_t cols,
                                     uint32_t symfmt, float int8_div, const uint64_t *idx,
                                     uint64_t n_idx, uint8_t *sym, uint16_t *scales,
                                     uint32_t threads);

/*
 * Frequency table for rANS, summing to 2^prob_bits: f = 0 for absent symbols, else
 * max(1, floor(count * 2^prob_bits / n)); the remainder goes to the most frequent symbol (lowest
 * byte on ties); an excess is taken back one unit at a time from the largest f > 1 (lowest byte
 * on ties).  n = 0 gives f[0] = 2^prob_bits.
 */
eq_status eq_rans_freqs_host(const uint8_t *sym, uint64_t n, uint32_t prob_bits, uint32_t *freqs);

/* The same normalisation from 256 symbol counts (e.g. those of eq_histogram_device). */
eq_status eq_rans_normalize_host(const uint64_t *counts, uint32_t prob_bits, uint32_t *freqs);

/*
 * Interleaved-rANS encoding of a symbol matrix sym[rows][cols] in the format of eq_rans_tensor.
 * chunk_symbols = 0 means one row per chunk.  states: [num_chunks * streams]; word_off:
 * [num_chunks * ceil(streams / 32) + 1] (one word substream per chunk and group of 32 streams).
 * freqs sums to 4096 (12-bit table), or 256 / 128 (8- / 7-bit table, whose streams renormalise
 * after every second step).  The words are returned in a buffer the library allocates (*words, *n_words
 * words, zero-padded to a multiple of 8); release it with eq_free_host.
 */
eq_status eq_rans_encode_host(const uint8_t *sym, uint32_t rows, uint32_t cols,
                              const uint32_t *freqs, uint32_t chunk_symbols, uint32_t streams,
                              uint32_t run, uint32_t threads, uint32_t *states, uint64_t *word_off,
                              uint16_t **words, uint64_t *n_words);

/*
 * EntroLLM-style per-tensor integer quantisation of n weights to `bits`-bit codes (8 or 4):
 *   EQ_INTQ_ASYM:     scale = bf16((max - min) / (2^bits - 1)), zero = clamp(rne(-min / scale));
 *   EQ_INTQ_UNSIGNED: scale = bf16(max|w| / (2^(bits-1) - 1)), zero = 2^(bits-1);
 *   code = clamp(rne(w / scale) + zero, 0, 2^bits - 1); a zero scale becomes 1.
 */
#define EQ_INTQ_ASYM 0u
#define EQ_INTQ_UNSIGNED 1u
eq_status eq_intq_quantize_host(const float *w, uint64_t n, uint32_t bits, uint32_t scheme,
                                uint8_t *sym, uint16_t *scale, int32_t *zero);

/*
 * The eq_huff_tensor layout for any byte stream (eq_huff_int_tensor's coded codes): plan gives
 * total_bits; encode fills enc (threads * 8 + 16 bytes), gaps (ceil(5 threads / 8) + 8 bytes)
 * and block_out (blocks + 1 entries), all zeroed by the caller.
 */
eq_status eq_huff_sym_plan_host(const uint8_t *sym, uint64_t n, const uint32_t *lengths,
                                uint64_t *total_bits);
eq_status eq_huff_sym_encode_host(const uint8_t *sym, uint64_t n, const uint32_t *lengths,
                                  uint32_t threads_per_block, uint64_t total_bits, uint8_t *enc,
                                  uint8_t *gaps, uint64_t *block_out);

/* Optimal Huffman code lengths (no length above max_len) for 256 symbol counts. */
eq_status eq_huff_lengths_host(const uint64_t *counts, uint32_t max_len, uint32_t *lengths);

/*
 * DFloat11 coding of n bf16 weights (eq_huff_tensor format) with the given code lengths.
 * First call eq_huff_plan_host to learn total_bits; the caller then allocates
 *   enc_exp   threads * 8 + 16 bytes,   sign_mant n bytes,
 *   gaps      ceil(5 * threads / 8) + 8 bytes,   block_out blocks + 1 entries,
 * with threads = ceil(total_bits / 64) and blocks = ceil(threads / threads_per_block), zeroed.
 */
eq_status eq_huff_plan_host(const uint16_t *w, uint64_t n, const uint32_t *lengths,
                            uint64_t *total_bits);
eq_status eq_huff_encode_host(const uint16_t *w, uint64_t n, const uint32_t *lengths,
                              uint32_t threads_per_block, uint64_t total_bits, uint8_t *enc_exp,
                              uint8_t *sign_mant, uint8_t *gaps, uint64_t *block_out);

/* Release a buffer returned by eq_rans_encode_host. */
void eq_free_host(void *p);

/*
 * The same compressor on the GPU: every pointer below is device memory owned by the caller,
 * every call is asynchronous on `stream` and allocates nothing.  The results are bit-identical
 * to the host calls above.
 *
 * eq_quantize_device: as eq_quantize_host (one CTA per row).
 * eq_histogram_device: d_counts[256] += the number of each byte value among d_sym[0 .. n)
 *   (zero d_counts first).
 * eq_rans_plan_device: encodes every chunk once to learn the final states (d_states,
 *   [num_chunks * streams]) and each substream's word count, then turns the counts into the
 *   offsets d_word_off ([num_chunks * streams / 32 + 1]; d_word_off[last] = total words).
 * eq_rans_encode_device: encodes again and writes the words at those offsets into d_words (room
 *   for d_word_off[last] words, rounded up to a multiple of 8 and zero-filled by the caller).
 * host_freqs: the frequency table (host memory, 256 entries summing to 4096, or to 256 / 128 for
 * an 8- / 7-bit table, which needs run == 8 and cols % 8 == 0, else EQ_ERR_UNSUPPORTED).  A symbol without
 * frequency sets EQ_DEV_BAD_CODE in *d_status; a word count that does not match the plan sets
 * EQ_DEV_COUNT_MISMATCH.
 */
eq_status eq_quantize_device(const float *d_w, uint32_t rows, uint32_t cols, uint32_t symfmt,
                             float int8_div, uint8_t *d_sym, uint16_t *d_scales, void *stream);
eq_status eq_histogram_device(const uint8_t *d_sym, uint64_t n, uint32_t *d_counts, void *stream);
eq_status eq_rans_plan_device(const uint8_t *d_sym, uint32_t rows, uint32_t cols,
                              const uint32_t *host_freqs, uint32_t chunk_symbols, uint32_t streams,
                              uint32_t run, uint32_t *d_states, uint64_t *d_word_off,
                              uint32_t *d_status, void *stream);
eq_status eq_rans_encode_device(const uint8_t *d_sym, uint32_t rows, uint32_t cols,
                                const uint32_t *host_freqs, uint32_t chunk_symbols,
                                uint32_t streams, uint32_t run, const uint64_t *d_word_off,
                                uint16_t *d_words, uint32_t *d_status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* EQ_ENCODE_H */
