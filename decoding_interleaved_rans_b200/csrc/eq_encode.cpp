// Host-side compressor: quantisation, rANS tables and encoding, DFloat11 Huffman encoding.
// Produces exactly the formats the decoders of eq.h read.  Runs on CPU threads; no CUDA calls.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <queue>
#include <thread>
#include <vector>

#include "eq_encode.h"

namespace {

unsigned worker_count(uint32_t threads) {
  unsigned hw = std::thread::hardware_concurrency();
  if (hw == 0) hw = 1;
  return threads ? threads : hw;
}

template <class F>
void parallel_for(uint64_t n, uint32_t threads, F &&f) {
  const unsigned nt = std::max<unsigned>(1, std::min<uint64_t>(worker_count(threads), n));
  if (nt <= 1) {
    for (uint64_t i = 0; i < n; ++i) f(i);
    return;
  }
  std::atomic<uint64_t> next{0};
  std::vector<std::thread> pool;
  for (unsigned t = 0; t < nt; ++t)
    pool.emplace_back([&] {
      for (uint64_t i = next++; i < n; i = next++) f(i);
    });
  for (auto &th : pool) th.join();
}

uint32_t f32_bits(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return u;
}

float bits_f32(uint32_t u) {
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// binary32 -> bf16, round to nearest even (finite inputs)
uint16_t to_bf16(float f) {
  uint32_t u = f32_bits(f);
  return uint16_t((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

// binary32 -> E4M3 (bias 7, 3 fraction bits), round to nearest even, saturate at 448
uint8_t to_e4m3(float f) {
  const uint32_t u = f32_bits(f);
  const uint8_t sign = uint8_t((u >> 24) & 0x80u);
  const uint32_t mag = u & 0x7FFFFFFFu;
  if (mag > 0x7F800000u) return 0x7F;                       // NaN
  if (mag >= f32_bits(0.015625f)) {                         // normal E4M3 range: 2^-6 and up
    uint32_t r = (mag + 0x7FFFFu + ((mag >> 20) & 1u)) >> 20;  // keep 3 fraction bits
    int32_t e = int32_t(r >> 3) - 127 + 7;
    if (e > 15 || (e == 15 && (r & 7u) > 6u)) return uint8_t(sign | 0x7E);
    return uint8_t(sign | (uint32_t(e) << 3) | (r & 7u));
  }
  // subnormal range: multiples of 2^-9
  const float k = std::nearbyintf(bits_f32(mag) * 512.0f);
  return uint8_t(sign | uint32_t(k));
}

}  // namespace

extern "C" eq_status eq_quantize_host(const float *w, uint32_t rows, uint32_t cols, uint32_t symfmt,
                                      float int8_div, uint8_t *sym, uint16_t *scales,
                                      uint32_t threads) {
  if ((!w || !sym || !scales) && uint64_t(rows) * cols) return EQ_ERR_ARG;
  if (symfmt != EQ_SYM_E4M3 && symfmt != EQ_SYM_INT8) return EQ_ERR_ARG;
  if (symfmt == EQ_SYM_INT8 && !(int8_div > 0.0f)) return EQ_ERR_ARG;
  const float div = symfmt == EQ_SYM_E4M3 ? 448.0f : int8_div;
  parallel_for(rows, threads, [&](uint64_t r) {
    const float *wr = w + r * cols;
    float amax = 0.0f;
    for (uint32_t c = 0; c < cols; ++c) amax = std::max(amax, std::fabs(wr[c]));
    uint16_t sb = to_bf16(amax / div);
    if (amax == 0.0f || (sb & 0x7FFFu) == 0) sb = 0x3F80u;
    scales[r] = sb;
    const float s = bits_f32(uint32_t(sb) << 16);
    uint8_t *out = sym + r * cols;
    if (symfmt == EQ_SYM_E4M3) {
      for (uint32_t c = 0; c < cols; ++c) out[c] = to_e4m3(wr[c] / s);
    } else {
      for (uint32_t c = 0; c < cols; ++c) {
        float q = std::nearbyintf(wr[c] / s);
        q = std::min(127.0f, std::max(-127.0f, q));
        out[c] = uint8_t(int8_t(q));
      }
    }
  });
  return EQ_OK;
}

extern "C" eq_status eq_super_weights_host(const float *w, uint32_t rows, uint32_t cols,
                                           double tau, uint64_t max_out, uint64_t *idx,
                                           uint16_t *val, uint64_t *n_out) {
  const uint64_t n = uint64_t(rows) * cols;
  if (!n_out || (n && !w) || !(tau > 0.0) || (max_out && (!idx || !val))) return EQ_ERR_ARG;
  std::vector<double> part(rows, 0.0);
  parallel_for(rows, 0, [&](uint64_t r) {
    double ss = 0.0;
    for (uint32_t c = 0; c < cols; ++c) ss += double(w[r * cols + c]) * double(w[r * cols + c]);
    part[r] = ss;
  });
  double ss = 0.0;
  for (double v : part) ss += v;
  const double limit = n ? tau * std::sqrt(ss / double(n)) : 0.0;
  uint64_t k = 0;
  for (uint64_t j = 0; j < n; ++j)
    if (std::fabs(double(w[j])) > limit) {
      if (k < max_out) {
        idx[k] = j;
        val[k] = to_bf16(w[j]);
      }
      ++k;
    }
  *n_out = k;
  return EQ_OK;
}

extern "C" eq_status eq_quantize_excluding_host(const float *w, uint32_t rows, uint32_t cols,
                                                uint32_t symfmt, float int8_div,
                                                const uint64_t *idx, uint64_t n_idx, uint8_t *sym,
                                                uint16_t *scales, uint32_t threads) {
  if (n_idx && !idx) return EQ_ERR_ARG;
  for (uint64_t i = 0; i < n_idx; ++i)
    if (idx[i] >= uint64_t(rows) * cols || (i && idx[i] <= idx[i - 1])) return EQ_ERR_ARG;
  if (n_idx == 0) return eq_quantize_host(w, rows, cols, symfmt, int8_div, sym, scales, threads);
  if ((!w || !sym || !scales) && uint64_t(rows) * cols) return EQ_ERR_ARG;
  if (symfmt != EQ_SYM_E4M3 && symfmt != EQ_SYM_INT8) return EQ_ERR_ARG;
  if (symfmt == EQ_SYM_INT8 && !(int8_div > 0.0f)) return EQ_ERR_ARG;
  const uint64_t *end = idx + n_idx;
  std::atomic<int> bad{0};
  parallel_for(rows, threads, [&](uint64_t r) {
    // this row's excluded entries, zeroed in a copy of the row, then the ordinary quantiser
    const uint64_t *lo = std::lower_bound(idx, end, r * cols);
    const uint64_t *hi = std::lower_bound(lo, end, (r + 1) * cols);
    std::vector<float> row(w + r * cols, w + (r + 1) * cols);
    for (const uint64_t *p = lo; p < hi; ++p) row[*p - r * cols] = 0.0f;
    if (eq_quantize_host(row.data(), 1, cols, symfmt, int8_div, sym + r * cols, scales + r, 1) !=
        EQ_OK)
      bad = 1;
  });
  return bad ? EQ_ERR_ARG : EQ_OK;
}

extern "C" eq_status eq_rans_normalize_host(const uint64_t *counts, uint32_t prob_bits,
                                            uint32_t *freqs) {
  if (!counts || !freqs || prob_bits < 7 || prob_bits > 15) return EQ_ERR_ARG;
  const uint64_t M = 1ull << prob_bits;
  uint64_t n = 0;
  for (int s = 0; s < 256; ++s) n += counts[s];
  std::fill(freqs, freqs + 256, 0u);
  if (n == 0) {
    freqs[0] = uint32_t(M);
    return EQ_OK;
  }
  int top = 0;
  uint64_t total = 0;
  for (int s = 0; s < 256; ++s) {
    if (counts[s] > counts[top]) top = s;
    if (!counts[s]) continue;
    const uint64_t f = std::max<uint64_t>(1, uint64_t((static_cast<unsigned __int128>(counts[s]) * M) / n));
    freqs[s] = uint32_t(f);
    total += f;
  }
  if (total < M) freqs[top] += uint32_t(M - total);
  for (; total > M; --total) {
    int big = -1;
    for (int s = 0; s < 256; ++s)
      if (freqs[s] > 1 && (big < 0 || freqs[s] > freqs[big])) big = s;
    --freqs[big];
  }
  return EQ_OK;
}

extern "C" eq_status eq_rans_freqs_host(const uint8_t *sym, uint64_t n, uint32_t prob_bits,
                                        uint32_t *freqs) {
  if (!freqs || (n && !sym)) return EQ_ERR_ARG;
  uint64_t cnt[256] = {0};
  for (uint64_t i = 0; i < n; ++i) ++cnt[sym[i]];
  return eq_rans_normalize_host(cnt, prob_bits, freqs);
}

extern "C" eq_status eq_rans_encode_host(const uint8_t *sym, uint32_t rows, uint32_t cols,
                                         const uint32_t *freqs, uint32_t chunk_symbols,
                                         uint32_t streams, uint32_t run, uint32_t threads,
                                         uint32_t *states, uint64_t *word_off, uint16_t **words,
                                         uint64_t *n_words) {
  const uint64_t N = uint64_t(rows) * cols;
  const uint64_t chunk = chunk_symbols ? chunk_symbols : cols;
  if (!freqs || !word_off || !words || !n_words || (N && (!sym || !states)) || streams == 0 ||
      run == 0 || chunk == 0)
    return EQ_ERR_ARG;
  uint32_t cum[257];
  cum[0] = 0;
  for (int s = 0; s < 256; ++s) cum[s + 1] = cum[s] + freqs[s];
  if (cum[256] != 128u && cum[256] != 256u && cum[256] != 4096u) return EQ_ERR_FORMAT;
  // 7- and 8-bit tables renormalise after every second step of a stream, 12-bit ones after
  // every step
  const uint32_t pb = cum[256] == 128u ? 7u : cum[256] == 256u ? 8u : 12u, k = 16u / pb;
  const uint64_t nchunks = (N + chunk - 1) / chunk;
  const uint32_t groups = (streams + 31) / 32;  // 32 streams share one word substream
  std::vector<std::vector<uint16_t>> pieces(nchunks * groups);
  std::atomic<int> bad{0};
  parallel_for(nchunks, threads, [&](uint64_t c) {
    const uint64_t j0 = c * chunk;
    const uint64_t n = std::min(chunk, N - j0);
    const uint8_t *s = sym + j0;
    std::vector<uint32_t> x(streams, 1u << 16);
    std::vector<uint16_t> *out = &pieces[c * groups];  // encoder order, reversed at the end
    const uint64_t nruns = (n + run - 1) / run;
    const uint64_t nrounds = (nruns + streams - 1) / streams;
    // steps of stream st: its runs st, st + S, ... are full except the chunk's last run
    auto steps_of = [&](uint32_t st) -> uint64_t {
      if (st >= nruns) return 0;
      uint64_t t = ((nruns - 1 - st) / streams + 1) * run;
      if ((nruns - 1) % streams == st) t -= nruns * run - n;
      return t;
    };
    auto sym_of_step = [&](uint64_t t, uint32_t st) {
      return s[((t / run) * streams + st) * run + t % run];
    };
    for (uint64_t rr = nrounds; rr-- > 0;)
      for (uint32_t p = run; p-- > 0;)
        for (uint32_t st = streams; st-- > 0;) {
          const uint64_t j = (rr * streams + st) * run + p;
          if (j >= n) continue;
          const uint32_t q = s[j], f = freqs[q];
          if (!f) {
            bad = 1;
            return;
          }
          uint32_t v = x[st];
          // flush on the last step of a renormalisation group, before its coding steps
          const uint64_t t = rr * run + p, g0 = t / k * k;
          const uint64_t g1 = k == 1 ? t + 1 : std::min<uint64_t>(g0 + k, steps_of(st));
          if (t + 1 == g1) {
            uint64_t xmax = 1ull << (32 - (g1 - g0) * pb);
            for (uint64_t u = g0; u < g1; ++u) xmax *= freqs[sym_of_step(u, st)];
            if (uint64_t(v) >= xmax) {
              out[st / 32].push_back(uint16_t(v));
              v >>= 16;
            }
          }
          x[st] = ((v / f) << pb) + v % f + cum[q];
        }
    for (uint32_t g = 0; g < groups; ++g) std::reverse(out[g].begin(), out[g].end());
    std::memcpy(states + c * streams, x.data(), streams * sizeof(uint32_t));
  });
  if (bad) return EQ_ERR_FORMAT;
  const uint64_t units = nchunks * groups;
  word_off[0] = 0;
  for (uint64_t u = 0; u < units; ++u) word_off[u + 1] = word_off[u] + pieces[u].size();
  const uint64_t total = word_off[units];
  const uint64_t padded = std::max<uint64_t>(8, (total + 7) / 8 * 8);
  uint16_t *buf = static_cast<uint16_t *>(std::calloc(padded, sizeof(uint16_t)));
  if (!buf) return EQ_ERR_ARG;
  parallel_for(units, threads, [&](uint64_t u) {
    if (!pieces[u].empty())
      std::memcpy(buf + word_off[u], pieces[u].data(), pieces[u].size() * sizeof(uint16_t));
  });
  *words = buf;
  *n_words = padded;
  return EQ_OK;
}

extern "C" void eq_free_host(void *p) { std::free(p); }

// ------------------------------------------------------------------------------------------------
// Huffman code lengths: heap-built tree, ties broken by (weight, key), leaf key = byte value,
// inner node key = 256 + creation order; depths above max_len fall back to package-merge.
// ------------------------------------------------------------------------------------------------
namespace {

bool tree_lengths(const uint64_t *counts, uint32_t *len, uint32_t &maxd) {
  struct Node {
    uint64_t w;
    uint32_t key;
  };
  auto cmp = [](const Node &a, const Node &b) { return a.w != b.w ? a.w > b.w : a.key > b.key; };
  std::priority_queue<Node, std::vector<Node>, decltype(cmp)> heap(cmp);
  std::vector<int> parent(512, -1);
  for (uint32_t s = 0; s < 256; ++s)
    if (counts[s]) heap.push({counts[s], s});
  uint32_t inner = 0;
  while (heap.size() > 1) {
    Node a = heap.top();
    heap.pop();
    Node b = heap.top();
    heap.pop();
    const uint32_t id = 256 + inner++;
    parent[a.key] = int(id);
    parent[b.key] = int(id);
    heap.push({a.w + b.w, id});
  }
  maxd = 0;
  for (uint32_t s = 0; s < 256; ++s) {
    len[s] = 0;
    if (!counts[s]) continue;
    uint32_t d = 0;
    for (int v = int(s); parent[v] >= 0; v = parent[v]) ++d;
    len[s] = d;
    maxd = std::max(maxd, d);
  }
  return true;
}

// package-merge over (weight, multiset of symbols) items kept as count vectors
void package_merge(const uint64_t *counts, uint32_t max_len, uint32_t *len) {
  struct Item {
    uint64_t w;
    std::vector<uint16_t> cnt;
  };
  std::vector<std::pair<uint64_t, uint32_t>> leaves;
  for (uint32_t s = 0; s < 256; ++s)
    if (counts[s]) leaves.push_back({counts[s], s});
  std::sort(leaves.begin(), leaves.end());
  const size_t n = leaves.size();
  auto leaf_item = [&](size_t i) {
    Item it{leaves[i].first, std::vector<uint16_t>(256, 0)};
    it.cnt[leaves[i].second] = 1;
    return it;
  };
  std::vector<Item> list;
  for (size_t i = 0; i < n; ++i) list.push_back(leaf_item(i));
  for (uint32_t level = 1; level < max_len; ++level) {
    std::vector<Item> packs;
    for (size_t i = 0; i + 1 < list.size(); i += 2) {
      Item p{list[i].w + list[i + 1].w, list[i].cnt};
      for (int s = 0; s < 256; ++s) p.cnt[s] += list[i + 1].cnt[s];
      packs.push_back(std::move(p));
    }
    std::vector<Item> merged;
    size_t a = 0, b = 0;
    while (a < n || b < packs.size()) {
      if (b >= packs.size() || (a < n && leaves[a].first <= packs[b].w)) merged.push_back(leaf_item(a++));
      else merged.push_back(std::move(packs[b++]));
    }
    list.swap(merged);
  }
  std::fill(len, len + 256, 0u);
  for (size_t i = 0; i < 2 * n - 2 && i < list.size(); ++i)
    for (int s = 0; s < 256; ++s) len[s] += list[i].cnt[s];
}

}  // namespace

extern "C" eq_status eq_huff_lengths_host(const uint64_t *counts, uint32_t max_len, uint32_t *lengths) {
  if (!counts || !lengths || max_len < 1 || max_len > 32) return EQ_ERR_ARG;
  uint32_t used = 0;
  for (int s = 0; s < 256; ++s) used += counts[s] != 0;
  std::fill(lengths, lengths + 256, 0u);
  if (used == 0) return EQ_OK;
  if (used == 1) {
    for (int s = 0; s < 256; ++s)
      if (counts[s]) lengths[s] = 1;
    return EQ_OK;
  }
  if (used > (1ull << max_len)) return EQ_ERR_ARG;
  uint32_t maxd = 0;
  tree_lengths(counts, lengths, maxd);
  if (maxd > max_len) package_merge(counts, max_len, lengths);
  return EQ_OK;
}

namespace {

// Total code bits of n symbols; EQ_ERR_FORMAT if one has no code.
template <class SymOf>
eq_status huff_plan(uint64_t n, SymOf sym_of, const uint32_t *lengths, uint64_t *total_bits) {
  uint64_t bits = 0;
  for (uint64_t i = 0; i < n; ++i) {
    const uint32_t l = lengths[sym_of(i)];
    if (!l) return EQ_ERR_FORMAT;
    bits += l;
  }
  *total_bits = bits;
  return EQ_OK;
}

// The DFloat11 layout for any byte-symbol stream: canonical codes MSB-first into enc, a 5-bit Gap
// per 64-bit thread segment and the first output index of every block of threads.  side(i) runs
// once per symbol (DFloat11 stores the sign and mantissa there).
template <class SymOf, class Side>
eq_status huff_encode(uint64_t n, SymOf sym_of, Side side, const uint32_t *lengths,
                      uint32_t threads_per_block, uint64_t total_bits, uint8_t *enc,
                      uint8_t *gaps, uint64_t *block_out) {
  // canonical codes from the lengths
  uint32_t code[256] = {0};
  {
    uint64_t c = 0;
    uint32_t prev = 0;
    for (uint32_t l = 1; l <= 32; ++l)
      for (int s = 0; s < 256; ++s)
        if (lengths[s] == l) {
          if (prev) c <<= (l - prev);
          prev = l;
          code[s] = uint32_t(c++);
        }
  }
  const uint64_t threads = (total_bits + 63) / 64;
  uint64_t pos = 0, t = 0, blk = 0;
  uint64_t acc = 0;  // pending bits, left-aligned
  uint32_t nacc = 0;
  uint64_t byte = 0;
  auto set_gap = [&](uint64_t th, uint64_t g) {
    const uint64_t bit = 5 * th;
    const uint32_t v = uint32_t(g) << (bit & 7);
    gaps[bit >> 3] |= uint8_t(v);
    gaps[(bit >> 3) + 1] |= uint8_t(v >> 8);
  };
  for (uint64_t i = 0; i < n; ++i) {
    const uint32_t e = sym_of(i), l = lengths[e];
    if (!l) return EQ_ERR_FORMAT;
    for (; t < threads && 64 * t <= pos; ++t) {  // threads whose first code starts here
      if (pos - 64 * t > 31) return EQ_ERR_FORMAT;
      set_gap(t, pos - 64 * t);
      if (t % threads_per_block == 0) block_out[blk++] = i;
    }
    acc |= uint64_t(code[e]) << (64 - nacc - l);
    nacc += l;
    while (nacc >= 8) {
      enc[byte++] = uint8_t(acc >> 56);
      acc <<= 8;
      nacc -= 8;
    }
    pos += l;
    side(i);
  }
  if (nacc) enc[byte++] = uint8_t(acc >> 56);
  if (pos != total_bits) return EQ_ERR_ARG;
  for (; t < threads; ++t) {
    if (pos < 64 * t || pos - 64 * t > 31) return EQ_ERR_FORMAT;
    set_gap(t, pos - 64 * t);
    if (t % threads_per_block == 0) block_out[blk++] = n;
  }
  block_out[blk] = n;
  return EQ_OK;
}

}  // namespace

extern "C" eq_status eq_huff_plan_host(const uint16_t *w, uint64_t n, const uint32_t *lengths,
                                       uint64_t *total_bits) {
  if ((n && !w) || !lengths || !total_bits) return EQ_ERR_ARG;
  return huff_plan(n, [&](uint64_t i) { return (w[i] >> 7) & 0xFFu; }, lengths, total_bits);
}

extern "C" eq_status eq_huff_encode_host(const uint16_t *w, uint64_t n, const uint32_t *lengths,
                                         uint32_t threads_per_block, uint64_t total_bits,
                                         uint8_t *enc_exp, uint8_t *sign_mant, uint8_t *gaps,
                                         uint64_t *block_out) {
  if ((n && (!w || !sign_mant)) || !lengths || !enc_exp || !gaps || !block_out ||
      threads_per_block == 0)
    return EQ_ERR_ARG;
  return huff_encode(
      n, [&](uint64_t i) { return (w[i] >> 7) & 0xFFu; },
      [&](uint64_t i) { sign_mant[i] = uint8_t(((w[i] >> 8) & 0x80u) | (w[i] & 0x7Fu)); },
      lengths, threads_per_block, total_bits, enc_exp, gaps, block_out);
}

extern "C" eq_status eq_huff_sym_plan_host(const uint8_t *sym, uint64_t n,
                                           const uint32_t *lengths, uint64_t *total_bits) {
  if ((n && !sym) || !lengths || !total_bits) return EQ_ERR_ARG;
  return huff_plan(n, [&](uint64_t i) { return uint32_t(sym[i]); }, lengths, total_bits);
}

extern "C" eq_status eq_huff_sym_encode_host(const uint8_t *sym, uint64_t n,
                                             const uint32_t *lengths, uint32_t threads_per_block,
                                             uint64_t total_bits, uint8_t *enc, uint8_t *gaps,
                                             uint64_t *block_out) {
  if ((n && !sym) || !lengths || !enc || !gaps || !block_out || threads_per_block == 0)
    return EQ_ERR_ARG;
  return huff_encode(
      n, [&](uint64_t i) { return uint32_t(sym[i]); }, [](uint64_t) {}, lengths,
      threads_per_block, total_bits, enc, gaps, block_out);
}

extern "C" eq_status eq_intq_quantize_host(const float *w, uint64_t n, uint32_t bits,
                                           uint32_t scheme, uint8_t *sym, uint16_t *scale,
                                           int32_t *zero) {
  if ((n && (!w || !sym)) || !scale || !zero || (bits != 8 && bits != 4) ||
      (scheme != EQ_INTQ_ASYM && scheme != EQ_INTQ_UNSIGNED))
    return EQ_ERR_ARG;
  const int32_t L = 1 << bits;
  float lo = 0.0f, hi = 0.0f, amax = 0.0f;
  for (uint64_t i = 0; i < n; ++i) {
    if (i == 0 || w[i] < lo) lo = w[i];
    if (i == 0 || w[i] > hi) hi = w[i];
    amax = std::max(amax, std::fabs(w[i]));
  }
  uint16_t sb;
  int32_t z;
  if (scheme == EQ_INTQ_ASYM) {
    sb = to_bf16((hi - lo) / float(L - 1));
    if ((sb & 0x7FFFu) == 0) sb = 0x3F80u;
    const float zf = std::nearbyintf(-lo / bits_f32(uint32_t(sb) << 16));
    z = int32_t(std::min(float(L - 1), std::max(0.0f, zf)));
  } else {
    sb = to_bf16(amax / float(L / 2 - 1));
    if ((sb & 0x7FFFu) == 0) sb = 0x3F80u;
    z = L / 2;
  }
  const float s = bits_f32(uint32_t(sb) << 16);
  parallel_for((n + 65535) / 65536, 0, [&](uint64_t b) {
    for (uint64_t i = b * 65536; i < std::min(n, (b + 1) * 65536); ++i) {
      const float q = std::nearbyintf(w[i] / s) + float(z);
      sym[i] = uint8_t(std::min(float(L - 1), std::max(0.0f, q)));
    }
  });
  *scale = sb;
  *zero = z;
  return EQ_OK;
}
