// eq_decode_from_host: eq_decode of a tensor whose coded arrays live in host memory.
//
// The pages keep the coded weights in GPU memory and decode them there ("Float8@2bits" summary,
// "Decodificacion en Tiempo de Inferencia"); when the weights are offloaded to the host (the case
// the DFloat11 page compares against), the coded arrays must cross the bus every time.  Here they
// cross in pieces of whole chunks that end on a row boundary, each piece decoding on the GPU as
// soon as its copy has landed while the next piece is still being copied, so the decode hides
// behind the transfer.  Copies are plain cudaMemcpyAsync calls on the caller's copy stream;
// ordering between the streams uses events created and released inside the call.
#include <algorithm>
#include <numeric>
#include <vector>

#include "eq_internal.cuh"

namespace eq {
eq_status validate_rans_tensor(const eq_rans_tensor &t);  // eq_rans_decode.cu
}  // namespace eq

using namespace eq;

extern "C" eq_status eq_decode_from_host(const eq_rans_tensor *t, const uint32_t *h_states,
                                         const uint64_t *h_word_off, const uint16_t *h_words,
                                         uint64_t n_words, const uint16_t *h_scales,
                                         uint32_t pieces, uint16_t *d_out, uint32_t *d_status,
                                         void *stream, void *copy_stream) {
  if (!t || !d_status) return EQ_ERR_ARG;
  eq_status s = validate_rans_tensor(*t);
  if (s != EQ_OK) return s;
  if (t->num_chunks == 0) return EQ_OK;
  if (!h_states || !h_word_off || !h_words || !h_scales || !d_out) return EQ_ERR_ARG;
  if (!aligned(d_out, t->run == 8 ? 16 : 2)) return EQ_ERR_ARG;
  const uint64_t S = t->streams, g = S / 32, units = t->num_chunks * g;
  if (h_word_off[units] > n_words) return EQ_ERR_ARG;
  const uint64_t chunk = t->chunk_symbols, cols = t->cols;
  // chunks per piece: a multiple of the smallest run of chunks that ends on a row boundary
  const uint64_t k0 = cols / std::gcd(chunk, cols);
  const uint64_t want = (t->num_chunks + std::max(1u, pieces) - 1) / std::max(1u, pieces);
  const uint64_t per = std::max(k0, want / k0 * k0);
  std::vector<uint64_t> bounds{0};
  if (pieces > 1 && t->n_patch == 0 && per < t->num_chunks)
    for (uint64_t c = per; c < t->num_chunks; c += per) bounds.push_back(c);
  bounds.push_back(t->num_chunks);

  cudaStream_t st = static_cast<cudaStream_t>(stream), cs = static_cast<cudaStream_t>(copy_stream);
  std::vector<cudaEvent_t> ev(bounds.size());
  for (auto &e : ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return EQ_ERR_CUDA;
  eq_status rc = EQ_OK;
  // the copies overwrite t's device arrays: first let the stream's earlier work finish with them
  if (cudaEventRecord(ev[0], st) != cudaSuccess || cudaStreamWaitEvent(cs, ev[0], 0) != cudaSuccess)
    rc = EQ_ERR_CUDA;
  auto *d_states = const_cast<uint32_t *>(t->states);
  auto *d_word_off = const_cast<uint64_t *>(t->word_off);
  auto *d_words = const_cast<uint16_t *>(t->words);
  auto *d_scales = const_cast<uint16_t *>(t->scales);
  for (size_t p = 0; p + 1 < bounds.size() && rc == EQ_OK; ++p) {
    const uint64_t c0 = bounds[p], c1 = bounds[p + 1];
    const bool last = c1 == t->num_chunks;
    const uint64_t r0 = c0 * chunk / cols, r1 = last ? t->rows : c1 * chunk / cols;
    // whole 16-byte lines of words, as the decoder's bulk copies read them
    const uint64_t w0 = h_word_off[c0 * g] & ~uint64_t(7);
    const uint64_t w1 = last ? n_words : std::min(n_words, (h_word_off[c1 * g] + 7) & ~uint64_t(7));
    bool ok = cudaMemcpyAsync(d_states + c0 * S, h_states + c0 * S, (c1 - c0) * S * 4,
                              cudaMemcpyHostToDevice, cs) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(d_word_off + c0 * g, h_word_off + c0 * g, ((c1 - c0) * g + 1) * 8,
                               cudaMemcpyHostToDevice, cs) == cudaSuccess;
    ok = ok && (w1 <= w0 || cudaMemcpyAsync(d_words + w0, h_words + w0, (w1 - w0) * 2,
                                            cudaMemcpyHostToDevice, cs) == cudaSuccess);
    ok = ok && cudaMemcpyAsync(d_scales + r0, h_scales + r0, (r1 - r0) * 2, cudaMemcpyHostToDevice,
                               cs) == cudaSuccess;
    ok = ok && cudaEventRecord(ev[p + 1], cs) == cudaSuccess;
    ok = ok && cudaStreamWaitEvent(st, ev[p + 1], 0) == cudaSuccess;
    if (!ok) {
      rc = EQ_ERR_CUDA;
      break;
    }
    eq_rans_tensor part = *t;  // the piece's chunks: its rows, states, offsets and scales
    part.rows = uint32_t(r1 - r0);
    part.num_chunks = c1 - c0;
    part.states = d_states + c0 * S;
    part.word_off = d_word_off + c0 * g;
    part.scales = d_scales + r0;
    uint16_t *out = d_out + r0 * cols;
    rc = eq_decode(&part, 1, &out, d_status, stream);
  }
  for (auto &e : ev) cudaEventDestroy(e);  // released once the work recorded on it completes
  return rc;
}
