/*
 * eq_oracle.c -- plain, slow CPU oracle for entropy-coded LLM weights.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library links or calls this file; only the tests,
 * the package's smoke entry and the bench's CPU-baseline leg load it (through oracle/__init__.py).
 * It shares no code, header, table or constant generator with the CUDA path.
 *
 * What it computes, and the passage each part follows:
 *   - bf16 and Float8-E4M3 conversions, written from the bit-layout definitions
 *     (1-8-7 and 1-4-3 with bias 7, no infinities, 0x7F/0xFF = NaN), round-to-nearest-even.
 *   - Per-output-channel AbsMax scales and the Float8/Int8 base alphabets
 *     ("Float8@2bits" summary, section "Optimizacion con Restriccion de Entropia": per-channel
 *     scales S initialised by AbsMax; Float8 or Int8 keeps the full dynamic range).
 *   - Interleaved rANS encode/decode of the flattened symbol stream ("Float8@2bits" summary,
 *     section "Codificacion de Pesos": the weights are flattened into a symbol stream and
 *     ANS-coded; section "Decodificacion en Tiempo de Inferencia": a parallel ANS decoder).
 *     The pages fix no rANS variant; the reading used here is: 12-bit probabilities, 32-bit
 *     state in [2^16, 2^32), 16-bit renormalisation words, S interleaved streams per chunk,
 *     a stream decoding G consecutive symbols before the next stream takes over.
 *   - Dequantisation value(q) * scale[row], one rounding to bf16.
 *   - DFloat11: Huffman code lengths of the bf16 exponent, canonical codes, MSB-first
 *     EncodedExponent, raw PackedSignMantissa, per-thread 5-bit Gaps and per-block output
 *     positions (DFloat11 page, sections "Formato DFloat11" and "Kernels GPU de 2 etapas y
 *     metadatos auxiliares").
 *   - GEMV y = W x in fp64 over the decoded bf16 weights.
 *
 * Parity pins live in tests/test_oracle_*.py: exact rationals, brute force on tiny inputs,
 * closed forms, Shannon-entropy bounds and the Kraft equality.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG (-1)
#define ORC_ERR_SYMBOL (-2)  /* symbol with zero frequency */
#define ORC_ERR_CORRUPT (-3) /* final states / word count do not match */
#define ORC_ERR_OVERRUN (-4) /* a stream asked for more words than the chunk holds */
#define ORC_ERR_CODE (-5)    /* no Huffman code matches */

/* ============================================================================================
 * bf16 (1 sign, 8 exponent, 7 fraction bits: the top half of an IEEE binary32)
 * ========================================================================================== */

float orc_bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* binary32 -> bf16, round to nearest, ties to even, on the 16 dropped bits. NaN -> quiet NaN. */
uint16_t orc_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu))
    return (uint16_t)(((u >> 16) & 0x8000u) | 0x7FC0u);
  uint32_t hi = u >> 16, lo = u & 0xFFFFu;
  if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u))) hi += 1u;
  return (uint16_t)hi;
}

/* Any double -> bf16 with one round-to-nearest-even step (exponent range of binary32,
 * subnormal quantum 2^-133, overflow to infinity). */
uint16_t orc_f64_to_bf16(double v) {
  if (isnan(v)) return signbit(v) ? 0xFFC0u : 0x7FC0u;
  uint16_t sign = signbit(v) ? 0x8000u : 0u;
  double a = fabs(v);
  if (a == 0.0) return sign;
  if (isinf(a)) return (uint16_t)(sign | 0x7F80u);
  int e;
  frexp(a, &e); /* a = m 2^e, m in [0.5, 1): floor(log2 a) = e - 1 */
  int E = e - 1;
  if (E < -126) E = -126;
  double q = ldexp(1.0, E - 7); /* spacing of bf16 values in this binade */
  double r = nearbyint(a / q) * q;
  if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80u);
  float rf = (float)r; /* exact: at most 9 significant bits */
  uint32_t u;
  memcpy(&u, &rf, 4);
  return (uint16_t)(sign | (u >> 16));
}

/* ============================================================================================
 * Float8 E4M3 ("FN" flavour: bias 7, no infinities, S.1111.111 is NaN, max 448)
 * ========================================================================================== */

double orc_e4m3_value(uint8_t b) {
  int s = b >> 7, e = (b >> 3) & 15, m = b & 7;
  if (e == 15 && m == 7) return s ? -NAN : NAN;
  double v = (e == 0) ? ldexp((double)m, -9) : ldexp(8.0 + (double)m, e - 10);
  return s ? -v : v;
}

/* binary32 -> E4M3, round to nearest even on the E4M3 grid, magnitudes above 448 saturate. */
uint8_t orc_f32_to_e4m3(float f) {
  if (isnan(f)) return 0x7Fu;
  uint8_t sign = signbit(f) ? 0x80u : 0u;
  double a = fabs((double)f);
  if (a == 0.0) return sign;
  int e;
  frexp(a, &e);
  int E = e - 1;
  if (E < -6) E = -6;                    /* below the smallest normal the spacing is 2^-9 */
  double q = ldexp(1.0, E - 3);          /* 3 fraction bits */
  double r = nearbyint(a / q) * q;
  if (r > 448.0) r = 448.0;
  if (r == 0.0) return sign;
  if (r < ldexp(1.0, -6)) return (uint8_t)(sign | (uint8_t)(r / ldexp(1.0, -9)));
  frexp(r, &e);
  E = e - 1;
  int m = (int)(r / ldexp(1.0, E) * 8.0) - 8;
  return (uint8_t)(sign | ((E + 7) << 3) | m);
}

/* value of an Int8 symbol: the byte read as two's complement */
static double int8_value(uint8_t b) { return (double)(int8_t)b; }

/* ============================================================================================
 * AbsMax quantisation to the base alphabets (one scale per output channel = row)
 * ========================================================================================== */

static uint16_t absmax_scale(const float *w, int64_t cols, float div) {
  float amax = 0.0f;
  for (int64_t c = 0; c < cols; ++c) {
    float a = fabsf(w[c]);
    if (a > amax) amax = a;
  }
  uint16_t sb = orc_f32_to_bf16(amax / div);
  if (amax == 0.0f || orc_bf16_to_f32(sb) == 0.0f) sb = 0x3F80u; /* 1.0 */
  return sb;
}

/* symbol = E4M3(w / s_r) with s_r = bf16(max_c |w[r][c]| / 448); the division is binary32. */
void orc_quantize_e4m3(const float *w, int64_t rows, int64_t cols, uint8_t *sym, uint16_t *scale) {
  for (int64_t r = 0; r < rows; ++r) {
    const float *wr = w + r * cols;
    uint16_t sb = absmax_scale(wr, cols, 448.0f);
    float s = orc_bf16_to_f32(sb);
    scale[r] = sb;
    for (int64_t c = 0; c < cols; ++c) sym[r * cols + c] = orc_f32_to_e4m3(wr[c] / s);
  }
}

/* symbol = clamp(rne(w / s_r), -127, 127) with s_r = bf16(max_c |w[r][c]| / div). */
void orc_quantize_int8(const float *w, int64_t rows, int64_t cols, float div, uint8_t *sym,
                       uint16_t *scale) {
  for (int64_t r = 0; r < rows; ++r) {
    const float *wr = w + r * cols;
    uint16_t sb = absmax_scale(wr, cols, div);
    float s = orc_bf16_to_f32(sb);
    scale[r] = sb;
    for (int64_t c = 0; c < cols; ++c) {
      float q = nearbyintf(wr[c] / s);
      if (q > 127.0f) q = 127.0f;
      if (q < -127.0f) q = -127.0f;
      sym[r * cols + c] = (uint8_t)(int8_t)q;
    }
  }
}

/* ============================================================================================
 * Super-weight exclusion ("Float8@2bits" summary, section "Manejo de Pesos Superiores": for Int8
 * bases, extreme outliers are detected and kept out of the entropy optimisation, so they do not
 * crush the rest of their channel).  Reading: a weight is a super weight when
 * |w| > tau * rms(w), rms over the whole tensor in binary64; super weights are stored exactly as
 * bf16(w) in a list sorted by flat row-major index, their symbol is 0 and they take no part in
 * their row's AbsMax scale; decoding writes them back over the decoded value.
 * ========================================================================================== */

/* Returns the number of super weights (writing at most max_out of them), or -1 on bad input. */
int64_t orc_super_weights(const float *w, int64_t rows, int64_t cols, double tau, int64_t max_out,
                          uint64_t *idx, uint16_t *val) {
  if (rows < 0 || cols < 0 || tau <= 0.0) return -1;
  const int64_t n = rows * cols;
  double ss = 0.0;
  for (int64_t j = 0; j < n; ++j) ss += (double)w[j] * (double)w[j];
  const double limit = n ? tau * sqrt(ss / (double)n) : 0.0;
  int64_t k = 0;
  for (int64_t j = 0; j < n; ++j)
    if (fabs((double)w[j]) > limit) {
      if (k < max_out) {
        idx[k] = (uint64_t)j;
        val[k] = orc_f32_to_bf16(w[j]);
      }
      ++k;
    }
  return k;
}

/* AbsMax quantisation (symfmt 1 = E4M3, 2 = Int8) of w with the listed positions excluded: they
 * take no part in their row's scale and get symbol 0.  idx sorted ascending, n entries. */
void orc_quantize_excluding(const float *w, int64_t rows, int64_t cols, int symfmt, float div,
                            const uint64_t *idx, int64_t n, uint8_t *sym, uint16_t *scale) {
  uint8_t *skip = (uint8_t *)calloc((size_t)(rows * cols > 0 ? rows * cols : 1), 1);
  for (int64_t i = 0; i < n; ++i) skip[idx[i]] = 1;
  float *row = (float *)malloc((size_t)(cols > 0 ? cols : 1) * sizeof(float));
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c = 0; c < cols; ++c) row[c] = skip[r * cols + c] ? 0.0f : w[r * cols + c];
    if (symfmt == 1)
      orc_quantize_e4m3(row, 1, cols, sym + r * cols, scale + r);
    else
      orc_quantize_int8(row, 1, cols, div, sym + r * cols, scale + r);
  }
  free(row);
  free(skip);
}

/* ============================================================================================
 * Dequantisation: bf16( value(q) * scale[row] ); the product is exact in binary64
 * (at most 7 x 8 significant bits), so there is exactly one rounding.
 * symfmt: 1 = E4M3, 2 = Int8.
 * ========================================================================================== */

uint16_t orc_dequant_one(uint8_t q, uint16_t scale, int symfmt) {
  double v = (symfmt == 1) ? orc_e4m3_value(q) : int8_value(q);
  if (isnan(v)) return signbit(v) ? 0xFFC0u : 0x7FC0u;
  return orc_f64_to_bf16(v * (double)orc_bf16_to_f32(scale));
}

void orc_dequant(const uint8_t *sym, const uint16_t *scale, int64_t rows, int64_t cols,
                 int symfmt, uint16_t *out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c)
      out[r * cols + c] = orc_dequant_one(sym[r * cols + c], scale[r], symfmt);
}

/* ============================================================================================
 * rANS: frequency normalisation to M = 2^prob_bits
 *   f_s = 0 if c_s = 0, else max(1, floor(c_s M / N)); the remainder M - sum f goes to the most
 *   frequent symbol (lowest byte on ties); a negative remainder is paid back one unit at a time
 *   by the largest f_s > 1 (lowest byte on ties).  N = 0 or one symbol: that symbol gets M.
 * ========================================================================================== */

int orc_rans_normalize(const uint64_t *counts, uint32_t prob_bits, uint32_t *freqs) {
  if (prob_bits < 1 || prob_bits > 15) return ORC_ERR_ARG;
  const int64_t M = (int64_t)1 << prob_bits;
  uint64_t N = 0;
  int nz = 0, top = 0;
  for (int s = 0; s < 256; ++s) {
    N += counts[s];
    nz += counts[s] != 0;
    if (counts[s] > counts[top]) top = s;
  }
  if (nz > M) return ORC_ERR_ARG;
  memset(freqs, 0, 256 * sizeof(uint32_t));
  if (N == 0) {
    freqs[0] = (uint32_t)M;
    return ORC_OK;
  }
  int64_t sum = 0;
  for (int s = 0; s < 256; ++s) {
    if (!counts[s]) continue;
    uint64_t f = (uint64_t)(((unsigned __int128)counts[s] * (uint64_t)M) / N);
    if (f < 1) f = 1;
    freqs[s] = (uint32_t)f;
    sum += (int64_t)f;
  }
  if (sum < M) freqs[top] += (uint32_t)(M - sum);
  while (sum > M) {
    int big = -1;
    for (int s = 0; s < 256; ++s)
      if (freqs[s] > 1 && (big < 0 || freqs[s] > freqs[big])) big = s;
    freqs[big] -= 1;
    sum -= 1;
  }
  return ORC_OK;
}

/* ============================================================================================
 * rANS chunk coder.
 *
 * Layout of one chunk of n symbols (j = 0..n-1, in row-major order of the weight):
 *   run r = j / G, stream = r mod S, round = r / S, position p = j mod G;
 *   decode steps go in order (round, p, stream); a stream with no symbol at a step is skipped.
 * Streams form groups of 32 (group g = streams 32g .. 32g+31, the last group may be smaller);
 *   every group has its own word substream, holding the words its streams read, in the order
 *   they read them.  Groups never share words, so a chunk's groups decode independently.
 * Renormalisation interval: with M = 2^prob_bits, a stream renormalises after every k-th of its
 *   own steps and after its last step, k = floor(16 / prob_bits) (k = 1 for 12-bit tables, k = 2
 *   for 8-bit ones).  M^k <= 2^16 = L makes one 16-bit word always enough: k steps shrink a state
 *   >= L by at most a factor M^k, so it stays >= 1.  A stream's steps are counted t = 0, 1, ...
 *   in decode order (step t is position t mod G of its (t div G)-th run); the steps between two
 *   renormalisation points form a group of m <= k steps.
 * Encoder: all S states start at L = 2^16; steps are taken in exactly the reverse order.  On the
 *   last step of a group (the first the encoder meets), if x >= 2^(32 - m * prob_bits) times the
 *   product of the group's m frequencies, the low 16 bits of x are emitted onto its group's stack
 *   and x >>= 16 (that bound is the largest x from which the m coding steps stay below 2^32);
 *   then, on every step, coding s with frequency f and cumulative frequency c is
 *   x = floor(x / f) * M + (x mod f) + c.  Each group's stack, reversed, is its substream in
 *   decoder-forward order; the chunk's words are the substreams of groups 0, 1, ... in turn.
 * Decoder: slot = x mod M; s is the symbol with c_s <= slot < c_s + f_s;
 *   x = f_s * floor(x / M) + slot - c_s; at a renormalisation point, if x < L then
 *   x = x * 2^16 + next word of its group.  At the end every x is L again and every group has
 *   read all of its words.
 * ========================================================================================== */

#define RANS_L 65536u
#define RANS_GROUP 32

static void cum_of(const uint32_t *freqs, uint32_t *cum) {
  uint32_t c = 0;
  for (int s = 0; s < 256; ++s) {
    cum[s] = c;
    c += freqs[s];
  }
}

int64_t orc_rans_groups(uint32_t S) { return ((int64_t)S + RANS_GROUP - 1) / RANS_GROUP; }

/* Steps of stream s in a chunk of n symbols: its runs are s, s + S, s + 2S, ... below the run
 * count, all G long except the chunk's last run, which may be short. */
static int64_t stream_steps(int64_t n, uint32_t S, uint32_t G, uint32_t s) {
  const int64_t runs = (n + G - 1) / G;
  if ((int64_t)s >= runs) return 0;
  int64_t T = ((runs - 1 - (int64_t)s) / S + 1) * G;
  if ((runs - 1) % S == (int64_t)s) T -= runs * (int64_t)G - n;
  return T;
}

/* index in the chunk of step t of stream s */
static int64_t step_symbol(int64_t t, uint32_t S, uint32_t G, uint32_t s) {
  return ((t / G) * S + s) * G + t % G;
}

static uint32_t renorm_interval(uint32_t prob_bits) { return 16u / prob_bits; }

/* Returns the number of words written to words_out (capacity must be >= n), or < 0.
 * group_count[g] receives the length of group g's substream (ceil(S / 32) entries). */
int64_t orc_rans_encode_chunk(const uint8_t *sym, int64_t n, const uint32_t *freqs,
                              uint32_t prob_bits, uint32_t S, uint32_t G, uint32_t *states_out,
                              uint16_t *words_out, int64_t *group_count) {
  if (S < 1 || G < 1 || n < 0 || prob_bits < 1 || prob_bits > 16) return ORC_ERR_ARG;
  uint32_t cum[256];
  cum_of(freqs, cum);
  const int64_t ng = orc_rans_groups(S);
  const int64_t k = renorm_interval(prob_bits);
  uint32_t *x = (uint32_t *)malloc(S * sizeof(uint32_t));
  int64_t *T = (int64_t *)malloc(S * sizeof(int64_t));
  /* one stack per group, each with room for every symbol of the chunk */
  uint16_t *stack = (uint16_t *)malloc((size_t)(ng * (n > 0 ? n : 1)) * sizeof(uint16_t));
  int64_t *depth = (int64_t *)calloc((size_t)ng, sizeof(int64_t));
  for (uint32_t s = 0; s < S; ++s) {
    x[s] = RANS_L;
    T[s] = stream_steps(n, S, G, s);
  }
  for (int64_t j = 0; j < n; ++j)
    if (freqs[sym[j]] == 0) {
      free(x);
      free(T);
      free(stack);
      free(depth);
      return ORC_ERR_SYMBOL;
    }
  int64_t runs = (n + G - 1) / G, rounds = (runs + S - 1) / S;
  for (int64_t round = rounds - 1; round >= 0; --round)
    for (int64_t p = (int64_t)G - 1; p >= 0; --p)
      for (int64_t s = (int64_t)S - 1; s >= 0; --s) {
        int64_t j = (round * S + s) * G + p;
        if (j >= n) continue;
        const int64_t t = round * G + p;
        const int64_t g0 = t / k * k;
        const int64_t g1 = g0 + k < T[s] ? g0 + k : T[s];
        uint32_t xs = x[s];
        if (t == g1 - 1) { /* the group's last step: flush before its m coding steps */
          uint64_t xmax = (uint64_t)1 << (32 - (g1 - g0) * prob_bits);
          for (int64_t u = g0; u < g1; ++u) xmax *= freqs[sym[step_symbol(u, S, G, (uint32_t)s)]];
          if ((uint64_t)xs >= xmax) {
            int64_t g = s / RANS_GROUP;
            stack[g * n + depth[g]++] = (uint16_t)(xs & 0xFFFFu);
            xs >>= 16;
          }
        }
        uint32_t f = freqs[sym[j]];
        x[s] = ((xs / f) << prob_bits) + (xs % f) + cum[sym[j]];
      }
  int64_t nw = 0;
  for (int64_t g = 0; g < ng; ++g) {
    for (int64_t i = depth[g] - 1; i >= 0; --i) words_out[nw++] = stack[g * n + i];
    group_count[g] = depth[g];
  }
  memcpy(states_out, x, S * sizeof(uint32_t));
  free(x);
  free(T);
  free(stack);
  free(depth);
  return nw;
}

/* group_off[g] .. group_off[g + 1]: group g's words inside `words` (ceil(S / 32) + 1 entries). */
int orc_rans_decode_chunk(const uint16_t *words, const int64_t *group_off, const uint32_t *states,
                          int64_t n, const uint32_t *freqs, uint32_t prob_bits, uint32_t S,
                          uint32_t G, uint8_t *sym_out) {
  if (S < 1 || G < 1 || n < 0 || prob_bits < 1 || prob_bits > 16) return ORC_ERR_ARG;
  const uint32_t M = 1u << prob_bits;
  const int64_t ng = orc_rans_groups(S);
  const int64_t k = renorm_interval(prob_bits);
  uint32_t cum[256];
  cum_of(freqs, cum);
  uint8_t *slot_sym = (uint8_t *)malloc(M);
  for (int s = 0; s < 256; ++s)
    for (uint32_t k = 0; k < freqs[s]; ++k) slot_sym[cum[s] + k] = (uint8_t)s;
  uint32_t *x = (uint32_t *)malloc(S * sizeof(uint32_t));
  int64_t *ptr = (int64_t *)malloc((size_t)ng * sizeof(int64_t));
  int rc = ORC_OK;
  for (int64_t g = 0; g < ng; ++g) {
    ptr[g] = group_off[g];
    if (group_off[g + 1] < group_off[g]) rc = ORC_ERR_ARG;
  }
  for (uint32_t s = 0; s < S; ++s) {
    x[s] = states[s];
    if (x[s] < RANS_L) rc = ORC_ERR_CORRUPT;
  }
  int64_t runs = (n + G - 1) / G, rounds = (runs + S - 1) / S;
  for (int64_t round = 0; round < rounds && rc == ORC_OK; ++round)
    for (int64_t p = 0; p < (int64_t)G && rc == ORC_OK; ++p)
      for (int64_t s = 0; s < (int64_t)S; ++s) {
        int64_t j = (round * S + s) * G + p;
        if (j >= n) continue;
        uint32_t slot = x[s] & (M - 1);
        uint8_t q = slot_sym[slot];
        x[s] = freqs[q] * (x[s] >> prob_bits) + slot - cum[q];
        const int64_t t = round * G + p;
        const int renorm_point = (t + 1) % k == 0 || t + 1 == stream_steps(n, S, G, (uint32_t)s);
        if (renorm_point && x[s] < RANS_L) {
          int64_t g = s / RANS_GROUP;
          if (ptr[g] >= group_off[g + 1]) {
            rc = ORC_ERR_OVERRUN;
            break;
          }
          x[s] = (x[s] << 16) | words[ptr[g]++];
        }
        sym_out[j] = q;
      }
  if (rc == ORC_OK) {
    for (uint32_t s = 0; s < S; ++s)
      if (x[s] != RANS_L) rc = ORC_ERR_CORRUPT;
    for (int64_t g = 0; g < ng; ++g)
      if (ptr[g] != group_off[g + 1]) rc = ORC_ERR_CORRUPT;
  }
  free(x);
  free(ptr);
  free(slot_sym);
  return rc;
}

/* Decode chunks [c0, c1) of a tensor container and dequantise them to bf16 (the whole job of the
 * GPU decode, done plainly).  Chunk c holds symbols [c*chunk, min(N, (c+1)*chunk)); its group g
 * substream is words[word_off[c * groups + g] .. word_off[c * groups + g + 1]). */
int orc_rans_decode_bf16(const uint16_t *words, const uint64_t *word_off, const uint32_t *states,
                         const uint32_t *freqs, const uint16_t *scales, int64_t rows, int64_t cols,
                         int symfmt, uint32_t prob_bits, int64_t chunk, uint32_t S, uint32_t G,
                         int64_t c0, int64_t c1, uint16_t *out) {
  int64_t N = rows * cols;
  const int64_t ng = orc_rans_groups(S);
  uint8_t *tmp = (uint8_t *)malloc((size_t)(chunk > 0 ? chunk : 1));
  int64_t *goff = (int64_t *)malloc((size_t)(ng + 1) * sizeof(int64_t));
  int rc = ORC_OK;
  for (int64_t c = c0; c < c1 && rc == ORC_OK; ++c) {
    int64_t j0 = c * chunk, n = (N - j0 < chunk) ? N - j0 : chunk;
    for (int64_t g = 0; g <= ng; ++g) goff[g] = (int64_t)(word_off[c * ng + g] - word_off[c * ng]);
    rc = orc_rans_decode_chunk(words + word_off[c * ng], goff, states + (size_t)c * S, n, freqs,
                               prob_bits, S, G, tmp);
    for (int64_t i = 0; i < n && rc == ORC_OK; ++i) {
      int64_t j = j0 + i;
      out[j] = orc_dequant_one(tmp[i], scales[j / cols], symfmt);
    }
  }
  free(goff);
  free(tmp);
  return rc;
}

/* ============================================================================================
 * EntroLLM-style integer weights (EntroLLM page, "Metodologia": per-tensor unsigned or
 * asymmetric integer quantisation, the codes Huffman-coded and decoded in parallel).
 * Reading: b-bit codes (b = 8 or 4, L = 2^b levels), one bf16 scale s and one integer zero point z
 * per tensor, value = (q - z) * s rounded once to bf16.
 *   scheme 0, asymmetric: s = bf16((max - min) / (L - 1)), z = clamp(rne(-min / s), 0, L - 1);
 *   scheme 1, unsigned:   s = bf16(max|w| / (L/2 - 1)), z = L/2 (the symmetric grid, offset);
 *   q = clamp(rne(w / s) + z, 0, L - 1), divisions in binary32.  s = 0 becomes 1.
 * The codes are Huffman-coded in the DFloat11 layout (MSB-first stream, thread t owns bits
 * [64t, 64t + 64), 5-bit Gaps, one output position per block of threads), with the code bytes
 * in place of the exponents and no sign/mantissa stream.
 * ========================================================================================== */

int orc_intq_quantize(const float *w, int64_t n, int bits, int scheme, uint8_t *sym,
                      uint16_t *scale_out, int32_t *zero_out) {
  if ((bits != 8 && bits != 4) || (scheme != 0 && scheme != 1) || n < 0) return ORC_ERR_ARG;
  const int L = 1 << bits;
  float lo = 0.0f, hi = 0.0f, amax = 0.0f;
  for (int64_t i = 0; i < n; ++i) {
    if (i == 0 || w[i] < lo) lo = w[i];
    if (i == 0 || w[i] > hi) hi = w[i];
    if (fabsf(w[i]) > amax) amax = fabsf(w[i]);
  }
  uint16_t sb;
  int32_t z;
  if (scheme == 0) {
    sb = orc_f32_to_bf16((hi - lo) / (float)(L - 1));
    if (orc_bf16_to_f32(sb) == 0.0f) sb = 0x3F80u;
    float zf = nearbyintf(-lo / orc_bf16_to_f32(sb));
    if (zf < 0.0f) zf = 0.0f;
    if (zf > (float)(L - 1)) zf = (float)(L - 1);
    z = (int32_t)zf;
  } else {
    sb = orc_f32_to_bf16(amax / (float)(L / 2 - 1));
    if (orc_bf16_to_f32(sb) == 0.0f) sb = 0x3F80u;
    z = L / 2;
  }
  const float s = orc_bf16_to_f32(sb);
  for (int64_t i = 0; i < n; ++i) {
    float q = nearbyintf(w[i] / s) + (float)z;
    if (q < 0.0f) q = 0.0f;
    if (q > (float)(L - 1)) q = (float)(L - 1);
    sym[i] = (uint8_t)q;
  }
  *scale_out = sb;
  *zero_out = z;
  return ORC_OK;
}

/* bf16( (q - z) * s ): |q - z| < 512 and s has 8 significant bits, so the binary64 product is
 * exact and rounding it is the only rounding. */
void orc_intq_dequant(const uint8_t *sym, int64_t n, uint16_t scale, int32_t zero, uint16_t *out) {
  const double s = (double)orc_bf16_to_f32(scale);
  for (int64_t i = 0; i < n; ++i) out[i] = orc_f64_to_bf16((double)((int32_t)sym[i] - zero) * s);
}

uint64_t orc_huff_total_bits_sym(const uint8_t *sym, int64_t n, const uint8_t *len) {
  uint64_t bits = 0;
  for (int64_t i = 0; i < n; ++i) bits += len[sym[i]];
  return bits;
}

/* The DFloat11 layout for byte symbols; buffers as for orc_huff_encode. */
int orc_huff_encode_sym(const uint8_t *sym, int64_t n, const uint8_t *len, const uint32_t *codes,
                        uint32_t threads_per_block, uint8_t *enc, uint8_t *gaps,
                        uint64_t *block_out, uint64_t threads) {
  uint64_t pos = 0, next_thread = 0, next_block = 0;
  for (int64_t i = 0; i <= n; ++i) {
    /* every thread whose segment starts at or before this code's start takes its Gap from it;
     * after the last code (i == n) the remaining threads point at the end of the stream */
    while (next_thread < threads && (i == n || 64 * next_thread <= pos)) {
      if (pos < 64 * next_thread || pos - 64 * next_thread > 31) return ORC_ERR_ARG;
      uint64_t g = pos - 64 * next_thread, bit = 5 * next_thread;
      for (int k = 0; k < 5; ++k)
        if ((g >> k) & 1) gaps[(bit + k) >> 3] |= (uint8_t)(1u << ((bit + k) & 7));
      if (next_thread % threads_per_block == 0) block_out[next_block++] = (uint64_t)i;
      ++next_thread;
    }
    if (i == n) break;
    int l = len[sym[i]];
    if (l == 0) return ORC_ERR_SYMBOL;
    for (int k = l - 1; k >= 0; --k) {
      if ((codes[sym[i]] >> k) & 1) enc[pos >> 3] |= (uint8_t)(0x80u >> (pos & 7));
      ++pos;
    }
  }
  block_out[next_block] = (uint64_t)n;
  return ORC_OK;
}

/* Sequential canonical decode of n byte symbols, one bit at a time. */
int orc_huff_decode_sym(const uint8_t *enc, uint64_t total_bits, int64_t n, const uint8_t *len,
                        uint8_t *out) {
  uint32_t count[33] = {0};
  uint8_t sorted[256];
  int ns = 0;
  for (int l = 1; l <= 32; ++l)
    for (int s = 0; s < 256; ++s)
      if (len[s] == l) {
        sorted[ns++] = (uint8_t)s;
        count[l]++;
      }
  uint64_t first[33], index[33], code = 0;
  int idx = 0;
  for (int l = 1; l <= 32; ++l) {
    first[l] = code;
    index[l] = (uint64_t)idx;
    code = (code + count[l]) << 1;
    idx += (int)count[l];
  }
  uint64_t pos = 0;
  for (int64_t i = 0; i < n; ++i) {
    uint64_t c = 0;
    int found = -1;
    for (int l = 1; l <= 32; ++l) {
      if (pos >= total_bits) return ORC_ERR_OVERRUN;
      c = (c << 1) | ((enc[pos >> 3] >> (7 - (pos & 7))) & 1u);
      ++pos;
      if (count[l] && c >= first[l] && c - first[l] < count[l]) {
        found = sorted[index[l] + (c - first[l])];
        break;
      }
    }
    if (found < 0) return ORC_ERR_CODE;
    out[i] = (uint8_t)found;
  }
  return pos == total_bits ? ORC_OK : ORC_ERR_CORRUPT;
}

/* ============================================================================================
 * GEMV in binary64 over bf16 operands: y[b][r] = sum_c W[r][c] * x[b][c], summed in column order.
 * ========================================================================================== */

void orc_gemv_f64(const uint16_t *w, const uint16_t *x, int64_t rows, int64_t cols, int64_t batch,
                  double *y) {
  for (int64_t b = 0; b < batch; ++b)
    for (int64_t r = 0; r < rows; ++r) {
      double acc = 0.0;
      for (int64_t c = 0; c < cols; ++c)
        acc += (double)orc_bf16_to_f32(w[r * cols + c]) * (double)orc_bf16_to_f32(x[b * cols + c]);
      y[b * rows + r] = acc;
    }
}

/* ============================================================================================
 * Huffman code lengths (DFloat11 page, "Formato DFloat11": a Huffman tree built from the
 * exponent histogram, frequent values get short codes).
 *
 * Tree build: repeatedly join the two lightest nodes; ties go to the node with the smaller key
 * (a leaf's key is its byte, an internal node's key is 256 + its creation index).  A symbol's
 * length is its leaf depth.  If the deepest leaf exceeds max_len, the lengths are recomputed
 * with package-merge (optimal lengths under the cap).  One used symbol gets length 1.
 * ========================================================================================== */

static int huff_tree_lengths(const uint64_t *counts, uint8_t *len) {
  uint64_t w[512];
  int key[512], parent[512], alive[512];
  int nn = 0;
  int leaf_node[256];
  for (int s = 0; s < 256; ++s) {
    leaf_node[s] = -1;
    if (counts[s]) {
      w[nn] = counts[s];
      key[nn] = s;
      parent[nn] = -1;
      alive[nn] = 1;
      leaf_node[s] = nn++;
    }
  }
  int nleaves = nn, nint = 0;
  for (int k = 0; k < nleaves - 1; ++k) {
    int a = -1, b = -1;
    for (int i = 0; i < nn; ++i) {
      if (!alive[i]) continue;
      if (a < 0 || w[i] < w[a] || (w[i] == w[a] && key[i] < key[a])) {
        b = a;
        a = i;
      } else if (b < 0 || w[i] < w[b] || (w[i] == w[b] && key[i] < key[b])) {
        b = i;
      }
    }
    alive[a] = alive[b] = 0;
    w[nn] = w[a] + w[b];
    key[nn] = 256 + nint++;
    parent[nn] = -1;
    alive[nn] = 1;
    parent[a] = parent[b] = nn;
    ++nn;
  }
  int maxd = 0;
  for (int s = 0; s < 256; ++s) {
    len[s] = 0;
    if (leaf_node[s] < 0) continue;
    int d = 0;
    for (int i = leaf_node[s]; parent[i] >= 0; i = parent[i]) ++d;
    len[s] = (uint8_t)d;
    if (d > maxd) maxd = d;
  }
  return maxd;
}

typedef struct {
  uint64_t w;
  uint16_t cnt[256]; /* how many times each symbol sits inside this item */
} pm_item;

static int pm_cmp_leaf(const void *pa, const void *pb) {
  const uint64_t *a = (const uint64_t *)pa, *b = (const uint64_t *)pb;
  if (a[0] != b[0]) return a[0] < b[0] ? -1 : 1;
  return a[1] < b[1] ? -1 : (a[1] > b[1]);
}

/* package-merge: lengths of an optimal prefix code with no length above max_len */
static int huff_package_merge(const uint64_t *counts, int max_len, uint8_t *len) {
  uint64_t leaves[256][2];
  int n = 0;
  for (int s = 0; s < 256; ++s)
    if (counts[s]) {
      leaves[n][0] = counts[s];
      leaves[n][1] = (uint64_t)s;
      ++n;
    }
  if (n < 2 || max_len >= 63 || ((uint64_t)1 << max_len) < (uint64_t)n) return -1;
  qsort(leaves, (size_t)n, sizeof(leaves[0]), pm_cmp_leaf);
  size_t cap = 2 * (size_t)(unsigned)n;
  pm_item *cur = (pm_item *)calloc(cap, sizeof(pm_item));
  pm_item *nxt = (pm_item *)calloc(cap, sizeof(pm_item));
  pm_item *pkg = (pm_item *)calloc(cap, sizeof(pm_item));
  int ncur = n;
  for (int i = 0; i < n; ++i) {
    memset(&cur[i], 0, sizeof(pm_item));
    cur[i].w = leaves[i][0];
    cur[i].cnt[leaves[i][1]] = 1;
  }
  for (int level = 1; level < max_len; ++level) {
    int np = ncur / 2;
    for (int i = 0; i < np; ++i) {
      pkg[i].w = cur[2 * i].w + cur[2 * i + 1].w;
      for (int s = 0; s < 256; ++s) pkg[i].cnt[s] = cur[2 * i].cnt[s] + cur[2 * i + 1].cnt[s];
    }
    /* merge the leaves with the packages, by weight (a leaf goes first on equal weight) */
    int a = 0, b = 0, k = 0;
    while (a < n || b < np) {
      if (b >= np || (a < n && leaves[a][0] <= pkg[b].w)) {
        memset(&nxt[k], 0, sizeof(pm_item));
        nxt[k].w = leaves[a][0];
        nxt[k].cnt[leaves[a][1]] = 1;
        ++a;
      } else {
        nxt[k] = pkg[b++];
      }
      ++k;
    }
    pm_item *t = cur;
    cur = nxt;
    nxt = t;
    ncur = k;
  }
  for (int s = 0; s < 256; ++s) len[s] = 0;
  for (int i = 0; i < 2 * n - 2 && i < ncur; ++i)
    for (int s = 0; s < 256; ++s) len[s] = (uint8_t)(len[s] + cur[i].cnt[s]);
  free(cur);
  free(nxt);
  free(pkg);
  return 0;
}

int orc_huff_lengths(const uint64_t *counts, int max_len, uint8_t *len) {
  int used = 0;
  for (int s = 0; s < 256; ++s) used += counts[s] != 0;
  memset(len, 0, 256);
  if (used == 0) return ORC_OK;
  if (used == 1) {
    for (int s = 0; s < 256; ++s)
      if (counts[s]) len[s] = 1;
    return ORC_OK;
  }
  int maxd = huff_tree_lengths(counts, len);
  if (maxd > max_len) return huff_package_merge(counts, max_len, len) ? ORC_ERR_ARG : ORC_OK;
  return ORC_OK;
}

/* Canonical codes: symbols in (length, byte) order get consecutive code values, each code
 * shifted left when the length grows.  codes[s] holds the code in its low len[s] bits. */
void orc_huff_canonical(const uint8_t *len, uint32_t *codes) {
  uint64_t code = 0;
  int prev = 0;
  for (int l = 1; l <= 32; ++l)
    for (int s = 0; s < 256; ++s) {
      if (len[s] != l) continue;
      if (prev) code <<= (l - prev);
      prev = l;
      codes[s] = (uint32_t)code;
      code += 1;
    }
  for (int s = 0; s < 256; ++s)
    if (!len[s]) codes[s] = 0;
}

/* ============================================================================================
 * DFloat11 encoding of bf16 weights.
 *   exponent e = bits 14..7; PackedSignMantissa byte = sign << 7 | 7 fraction bits;
 *   EncodedExponent = the exponents' codes, concatenated MSB-first from bit 0 of byte 0;
 *   thread t owns bits [64 t, 64 t + 64) (8 bytes, as on the page);
 *   Gap[t] = (first code start >= 64 t) - 64 t, in [0, 31], packed 5 bits per thread, LSB-first;
 *   block_out[b] = number of codes starting before bit 64 * T * b; block_out[nblocks] = n.
 * Sizes (all computed by the caller from total_bits): threads = ceil(total_bits / 64).
 * ========================================================================================== */

/* Pass 1: total number of code bits. */
uint64_t orc_huff_total_bits(const uint16_t *w, int64_t n, const uint8_t *len) {
  uint64_t bits = 0;
  for (int64_t i = 0; i < n; ++i) bits += len[(w[i] >> 7) & 0xFF];
  return bits;
}

/* Pass 2: fill the arrays.  enc must be zeroed, with room for threads * 8 bytes; gaps zeroed with
 * room for ceil(5 * threads / 8) bytes; block_out has nblocks + 1 entries. */
int orc_huff_encode(const uint16_t *w, int64_t n, const uint8_t *len, const uint32_t *codes,
                    uint32_t threads_per_block, uint8_t *enc, uint8_t *sign_mant, uint8_t *gaps,
                    uint64_t *block_out, uint64_t threads) {
  uint64_t pos = 0;
  uint64_t next_thread = 0; /* first thread whose gap is still unknown */
  uint64_t next_block = 0;
  for (int64_t i = 0; i < n; ++i) {
    uint16_t b = w[i];
    int e = (b >> 7) & 0xFF;
    int l = len[e];
    if (l == 0) return ORC_ERR_SYMBOL;
    /* this code starts at pos: every thread whose segment starts in (prev code start, pos] gets
     * its gap from here, and so does every block */
    while (next_thread < threads && 64 * next_thread <= pos) {
      uint64_t g = pos - 64 * next_thread;
      if (g > 31) return ORC_ERR_ARG;
      uint64_t bit = 5 * next_thread;
      for (int k = 0; k < 5; ++k)
        if ((g >> k) & 1) gaps[(bit + k) >> 3] |= (uint8_t)(1u << ((bit + k) & 7));
      if (next_thread % threads_per_block == 0) block_out[next_block++] = (uint64_t)i;
      ++next_thread;
    }
    uint32_t code = codes[e];
    for (int k = l - 1; k >= 0; --k) {
      if ((code >> k) & 1) enc[pos >> 3] |= (uint8_t)(0x80u >> (pos & 7));
      ++pos;
    }
    sign_mant[i] = (uint8_t)(((b >> 8) & 0x80) | (b & 0x7F));
  }
  /* threads whose segment holds no code start (only the tail can) */
  while (next_thread < threads) {
    uint64_t g = pos - 64 * next_thread;
    if (pos < 64 * next_thread || g > 31) return ORC_ERR_ARG;
    uint64_t bit = 5 * next_thread;
    for (int k = 0; k < 5; ++k)
      if ((g >> k) & 1) gaps[(bit + k) >> 3] |= (uint8_t)(1u << ((bit + k) & 7));
    if (next_thread % threads_per_block == 0) block_out[next_block++] = (uint64_t)n;
    ++next_thread;
  }
  block_out[next_block] = (uint64_t)n;
  return ORC_OK;
}

/* Plain sequential decode of the whole EncodedExponent (canonical decoding, one bit at a time),
 * merged with PackedSignMantissa back into bf16. */
int orc_huff_decode(const uint8_t *enc, uint64_t total_bits, const uint8_t *sign_mant, int64_t n,
                    const uint8_t *len, uint16_t *out) {
  /* canonical decoding tables: first code and first index of each length */
  uint32_t count[33] = {0};
  uint8_t sorted[256];
  int ns = 0;
  for (int l = 1; l <= 32; ++l)
    for (int s = 0; s < 256; ++s)
      if (len[s] == l) {
        sorted[ns++] = (uint8_t)s;
        count[l]++;
      }
  uint64_t first[33], index[33];
  uint64_t code = 0;
  int idx = 0;
  for (int l = 1; l <= 32; ++l) {
    first[l] = code;
    index[l] = (uint64_t)idx;
    code = (code + count[l]) << 1;
    idx += (int)count[l];
  }
  uint64_t pos = 0;
  for (int64_t i = 0; i < n; ++i) {
    uint64_t c = 0;
    int found = -1;
    for (int l = 1; l <= 32; ++l) {
      if (pos >= total_bits) return ORC_ERR_OVERRUN;
      c = (c << 1) | ((enc[pos >> 3] >> (7 - (pos & 7))) & 1u);
      ++pos;
      if (count[l] && c >= first[l] && c - first[l] < count[l]) {
        found = sorted[index[l] + (c - first[l])];
        break;
      }
    }
    if (found < 0) return ORC_ERR_CODE;
    uint8_t sm = sign_mant[i];
    out[i] = (uint16_t)(((uint16_t)(sm & 0x80) << 8) | ((uint16_t)found << 7) | (sm & 0x7F));
  }
  return pos == total_bits ? ORC_OK : ORC_ERR_CORRUPT;
}
