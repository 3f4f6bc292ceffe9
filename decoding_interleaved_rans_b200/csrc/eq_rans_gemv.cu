// eq_decode_gemv: y = W x with W decoded from its interleaved-rANS stream on chip (sm_100a).
//
// The pages name fused decompression + compute kernels as the next step after block-wise
// decompression ("Float8@2bits" summary, closing section; DFloat11 page, forum section: a GEMM that
// decompresses each tile before the arithmetic).  Here the decoded weights never reach memory:
//   * one warp decodes one chunk of whole rows with the same core as eq_decode (slot table in
//     shared memory, word ring fed by bulk copies, ballot/popcount renormalisation);
//   * each run of 8 symbols is dequantised exactly as eq_decode would write it (bf16 of
//     value * row scale), so y is the product of the very weights eq_decode returns;
//   * the lane multiplies its 8 weights by the matching 8 activations of every batch row
//     (16-byte loads of x, which stays in L1/L2) and accumulates in fp32;
//   * at the end of each weight row the warp reduces its partial sums with shuffles and writes
//     y[b][row] once.  The reduction order is fixed, so results are reproducible.
// The chunk has one group of 32 streams (streams == 32), so its partial sums never leave the warp.
// With chunks of several rows, a round (32 * 8 symbols) must not straddle a row, so cols must be a
// multiple of 256.  12-, 8- and 7-bit tables take the decode kernel's steps (7-bit: the 128 KiB
// pair table, one CTA per SM whose warps take chunk after chunk).
#include <algorithm>

#include "eq_dequant.cuh"
#include "eq_rans_core.cuh"

namespace eq {

eq_status validate_rans_tensor(const eq_rans_tensor &t);  // eq_rans_decode.cu

struct GemvParams {
  const uint32_t *states;
  const uint64_t *word_off;
  const uint16_t *words;
  const uint16_t *scales;
  const uint32_t *table;
  const uint16_t *x;
  float *y;
  uint32_t *status;
  const uint64_t *patch_idx;  // super weights (sorted flat indices, bf16 values)
  const uint16_t *patch_val;
  uint64_t n_patch;
  uint64_t numel;
  uint64_t num_chunks;
  uint32_t rows, cols, chunk_symbols, rows_per_chunk, rounds_per_row, batch, warps;
};

// a.x += lo(w) * lo(x), a.y += hi(w) * hi(x): fp32 FMAs that take their factors as bf16 halves
// of a register (no conversion; the product of two bf16 is exact, so each is the same single
// rounding as an fp32 FMA of the converted factors)
__device__ __forceinline__ void fma_bf16x2(float2 &a, uint32_t w, uint32_t x) {
  asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\t"
      "mov.b32 {wl, wh}, %2;\n\t"
      "mov.b32 {xl, xh}, %3;\n\t"
      "fma.rn.f32.bf16 %0, wl, xl, %0;\n\t"
      "fma.rn.f32.bf16 %1, wh, xh, %1;\n\t}"
      : "+f"(a.x), "+f"(a.y)
      : "r"(w), "r"(x));
}

// acc[b] += w[i] * x[b][col + i] over one run of 8 weights (packed bf16 pairs), the even columns
// in acc[b].x and the odd ones in acc[b].y (two independent sums: half the dependency chain)
template <int BMAX>
__device__ __forceinline__ void fma_run(float2 (&acc)[BMAX], uint2 wa, uint2 wb, const uint16_t *x,
                                        uint32_t cols, uint32_t col, uint32_t batch) {
#pragma unroll
  for (int b = 0; b < BMAX; ++b) {
    if (b < int(batch)) {
      const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(x + size_t(b) * cols + col));
      float2 a = acc[b];
      fma_bf16x2(a, wa.x, xv.x);
      fma_bf16x2(a, wa.y, xv.y);
      fma_bf16x2(a, wb.x, xv.z);
      fma_bf16x2(a, wb.y, xv.w);
      acc[b] = a;
    }
  }
}

// One round (8 steps) of the lane's stream -> its 8 symbols as 4 pairs, the first of each in the
// low byte (8- and 7-bit tables: the symbols' values, bf16x2).  12-bit tables renormalise after every
// step, 8-bit ones after every second, 7-bit ones look up two steps at once in the pair table (the
// steps of the decode kernel).
template <uint32_t PB>
__device__ __forceinline__ void round_pairs(uint32_t (&pr)[4], uint32_t &x, bool act,
                                            const uint32_t *lut, const unsigned char *smem,
                                            const WordRing &R, uint32_t &q, uint32_t lt) {
  if constexpr (PB == kRansPairBits) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      pr[k] = rans_pair_step<false>(x, act, lut);
      rans_renorm<false>(x, act, smem, R.ring_off, q, lt);
    }
  } else if constexpr (PB == 12) {  // the table rearranged to [symbol | f | slot - cum]
    const uint32_t tb = smem_addr(lut);
    uint32_t e[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      e[p] = rans_sym_step<false>(x, act, tb);
      rans_renorm<false>(x, act, smem, R.ring_off, q, lt);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) pr[k] = __byte_perm(e[2 * k], e[2 * k + 1], 0x0073u);
  } else {
    uint32_t e[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      e[p] = rans_decode_step<false, PB>(x, act, lut);
      if (p & 1) rans_renorm<false>(x, act, smem, R.ring_off, q, lt);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) pr[k] = value_pair8(e[2 * k], e[2 * k + 1]);
  }
}

// Two weights, exactly as eq_decode writes them, from a pair: of symbols (12-bit tables) or of
// the symbols' values (8-bit slot and 7-bit pair tables).
template <int FMT, uint32_t PB>
__device__ __forceinline__ uint32_t weights2(uint32_t pair, float sc, bool nan_codes) {
  if constexpr (PB != 12) return pair_dequant(pair, scale_bf16x2(sc), nan_codes);
  else return dequant2<FMT>(pair, sc, nan_codes);
}

// the pair a one-symbol table decodes to, in the form weights2 takes
template <int FMT, uint32_t PB>
__device__ __forceinline__ uint32_t single_pair(uint32_t sym) {
  if constexpr (PB != 12) return symbol_bf16(sym, FMT) * 0x10001u;
  else return sym * 0x0101u;
}

// Copy the PB-bit slot table (7 bits: the pair table) behind the header into shared memory, only
// when the header names a table of that size; false otherwise (a table of another size is never
// read past its end).
template <int FMT, uint32_t PB>
__device__ __forceinline__ bool load_table(uint32_t *lut, const uint32_t *table,
                                           const RansTableHeader &hdr) {
  const bool ok = hdr.magic == rans_table_magic<FMT, PB>() && hdr.prob_bits == PB;
  constexpr uint32_t kVec = PB == kRansPairBits ? kRansPairEntries / 2 : (1u << PB) / 4;
  const uint4 *src = reinterpret_cast<const uint4 *>(table + sizeof(RansTableHeader) / 4);
  if (ok) {
    for (uint32_t i = threadIdx.x; i < kVec; i += blockDim.x) {
      uint4 e = __ldg(src + i);
      if constexpr (PB == 12)  // [symbol | f | slot - cum], as the decode kernel holds it
        e = make_uint4(sym_first_entry(e.x), sym_first_entry(e.y), sym_first_entry(e.z),
                       sym_first_entry(e.w));
      reinterpret_cast<uint4 *>(lut)[i] = e;
    }
  }
  return ok;
}

// One warp = one chunk of whole rows, 32 streams (one per lane), run length 8.
// SUMS: the chunk is one row, and its sums go to sums[b] (in every lane) instead of y.
template <int FMT, int BMAX, uint32_t PB, bool SUMS = false>
__device__ __forceinline__ uint32_t gemv_chunk(const GemvParams &P, uint64_t chunk,
                                               const RansTableHeader &hdr, const uint32_t *lut,
                                               const unsigned char *smem, WordRing &R,
                                               uint32_t lane, float *sums = nullptr) {
  constexpr uint32_t S = 32;
  uint32_t status = 0;
  const bool single = hdr.flags & kRansFlagSingle;
  const bool nan_codes = (FMT == EQ_SYM_E4M3) && (hdr.flags & (kRansFlagNaN7F | kRansFlagNaNFF));
  const uint64_t j0 = chunk * uint64_t(P.chunk_symbols);
  const uint32_t n = uint32_t(P.numel - j0 < P.chunk_symbols ? P.numel - j0 : P.chunk_symbols);
  const uint64_t w0 = P.word_off[chunk], w1 = P.word_off[chunk + 1];
  if (w1 < w0 || w1 - w0 >= (1ull << 30)) return EQ_DEV_OVERRUN;
  uint32_t x = P.states[chunk * S + lane];
  const uint32_t nwords = uint32_t(w1 - w0);
  if (!single) R.start(P.words, w0, nwords, lane);

  const uint32_t lt = lanemask_lt();
  const uint32_t runs = n / 8;
  const uint32_t rounds = (runs + S - 1) / S;
  const uint32_t row0 = uint32_t(chunk * P.rows_per_chunk);
  const uint32_t batch = P.batch;
  float2 acc[BMAX];
#pragma unroll
  for (int b = 0; b < BMAX; ++b) acc[b] = make_float2(0.0f, 0.0f);
  uint32_t row_local = 0;
  float sc = bf16_bits_to_float(P.scales[row0]);
  uint32_t q = R.off0;
  // At batch 1 the ring work (overrun check, refill, wait) runs only once q reaches q_next; with
  // more accumulators the registers go to them (this bookkeeping spilled) and the checks run
  // every round.
  constexpr bool kQuiet = BMAX == 1;
  const uint32_t q_end = R.off0 + 2 * nwords;
  uint32_t q_next = 0;

  // 12-bit tables of E4M3 symbols without NaN codes: rounds in which every lane holds a run go
  // through the decode kernel's E4M3 round block (the weights come out dequantised), while the
  // row's scale is below 2^8 in magnitude
  const uint32_t tb = smem_addr(lut), ring_abs = R.buf_s;
  auto e4_row = [&](uint32_t row) {
    return PB == 12 && FMT == EQ_SYM_E4M3 && !nan_codes && !single &&
           (P.scales[row] & 0x7FFFu) < 0x4380u;
  };
  bool e4 = e4_row(row0);

  // One row per chunk in whole rounds with the E4M3 round block (no super weights): a loop with
  // nothing in it but the ring work, the round and its products, then the row's sum.
  if constexpr (PB == 12 && FMT == EQ_SYM_E4M3) {
    if (e4 && P.rows_per_chunk == 1 && runs % S == 0 && P.n_patch == 0) {
      const uint32_t sc2e = scale_e4m3_offset(sc);
      for (uint32_t r = 0; r < rounds; ++r) {
        if (q >= q_next) {
          if (q > q_end) {
            status |= EQ_DEV_OVERRUN;
            break;
          }
          R.round_refill(q, lane);
          if (!R.round_wait(q)) {
            status |= EQ_DEV_TIMEOUT;
            break;
          }
          q_next = R.quiet_until(q_end);
        }
        const uint4 o = rans_round12_e4m3<kRingBytes, false>(x, q, tb, ring_abs, lt, sc2e);
        fma_run<BMAX>(acc, make_uint2(o.x, o.y), make_uint2(o.z, o.w), P.x, P.cols,
                      (r * S + lane) * 8, batch);
      }
      if (!status && !__all_sync(0xFFFFFFFFu, q - R.off0 == 2 * nwords && x == kRansL))
        status |= EQ_DEV_CORRUPT_STATE;
      if (!status) {
#pragma unroll
        for (int b = 0; b < BMAX; ++b) {
          float v = acc[b].x + acc[b].y;
#pragma unroll
          for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, d);
          if constexpr (SUMS) sums[b] = v;
          else if (lane == 0 && b < int(batch)) P.y[size_t(b) * P.rows + row0] = v;
        }
      }
      status |= R.drain();
      return status;
    }
  }

  for (uint32_t r = 0; r < rounds; ++r) {
    const bool act = r * S + lane < runs;
    if constexpr (PB == 12 && FMT == EQ_SYM_E4M3) {
      if (e4 && (r + 1) * S <= runs) {  // every lane holds a run
        if constexpr (kQuiet) {
          if (q >= q_next) {
            if (q > q_end) {
              status |= EQ_DEV_OVERRUN;
              break;
            }
            R.round_refill(q, lane);
            if (!R.round_wait(q)) {
              status |= EQ_DEV_TIMEOUT;
              break;
            }
            q_next = R.quiet_until(q_end);
          }
        } else if (!R.round_wait(q)) {
          status |= EQ_DEV_TIMEOUT;
          break;
        }
        const uint4 o = rans_round12_e4m3<kRingBytes, false>(x, q, tb, ring_abs, lt,
                                                             scale_e4m3_offset(sc));
        if constexpr (!kQuiet) {
          if (q - R.off0 > 2 * nwords) {
            status |= EQ_DEV_OVERRUN;
            break;
          }
          R.round_refill(q, lane);
        }
        const uint32_t col = (r * S + lane) * 8 - row_local * P.cols;
        fma_run<BMAX>(acc, make_uint2(o.x, o.y), make_uint2(o.z, o.w), P.x, P.cols, col, batch);
        goto row_end_check;
      }
    }
    {
    uint32_t pr[4];  // the round's 8 symbols as 4 pairs (8/7-bit tables: their values, bf16x2)
    if (single) {
      pr[0] = pr[1] = pr[2] = pr[3] = single_pair<FMT, PB>(hdr.single_sym);
    } else if constexpr (kQuiet) {
      if (q >= q_next) {
        if (q > q_end) {
          status |= EQ_DEV_OVERRUN;
          break;
        }
        R.round_refill(q, lane);
        if (!R.round_wait(q)) {
          status |= EQ_DEV_TIMEOUT;
          break;
        }
        q_next = R.quiet_until(q_end);
      }
      round_pairs<PB>(pr, x, act, lut, smem, R, q, lt);
    } else {
      if (!R.round_wait(q)) {
        status |= EQ_DEV_TIMEOUT;
        break;
      }
      round_pairs<PB>(pr, x, act, lut, smem, R, q, lt);
      if (q - R.off0 > 2 * nwords) {
        status |= EQ_DEV_OVERRUN;
        break;
      }
      R.round_refill(q, lane);
    }
    if (act) {  // the weights exactly as eq_decode writes them, times the activations
      const uint32_t col = (r * S + lane) * 8 - row_local * P.cols;
      const uint2 wa = make_uint2(weights2<FMT, PB>(pr[0], sc, nan_codes), weights2<FMT, PB>(pr[1], sc, nan_codes));
      const uint2 wb = make_uint2(weights2<FMT, PB>(pr[2], sc, nan_codes), weights2<FMT, PB>(pr[3], sc, nan_codes));
      fma_run<BMAX>(acc, wa, wb, P.x, P.cols, col, batch);
    }
    }
  row_end_check:
    // end of a weight row: add its super weights' products, reduce across the warp, write y
    const bool row_end = (r + 1 == rounds) || (P.rows_per_chunk > 1 && (r + 1) % P.rounds_per_row == 0);
    if (row_end) {
      if (P.n_patch) {
        const uint64_t rs = uint64_t(row0 + row_local) * P.cols;
        const uint64_t lo = patch_lower_bound(P.patch_idx, P.n_patch, rs);
        const uint64_t hi = patch_lower_bound(P.patch_idx, P.n_patch, rs + P.cols);
        for (uint64_t i = lo + lane; i < hi; i += 32) {
          const uint32_t col = uint32_t(__ldg(P.patch_idx + i) - rs);
          const float v = bf16_bits_to_float(__ldg(P.patch_val + i));
#pragma unroll
          for (int b = 0; b < BMAX; ++b)
            if (b < int(batch)) acc[b].x = fmaf(v, bf16_bits_to_float(P.x[size_t(b) * P.cols + col]), acc[b].x);
        }
      }
#pragma unroll
      for (int b = 0; b < BMAX; ++b) {
        float v = acc[b].x + acc[b].y;
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, d);
        if constexpr (SUMS) sums[b] = v;
        else if (lane == 0 && b < int(batch)) P.y[size_t(b) * P.rows + row0 + row_local] = v;
        acc[b] = make_float2(0.0f, 0.0f);
      }
      ++row_local;
      if (row_local < P.rows_per_chunk && r + 1 < rounds) {
        sc = bf16_bits_to_float(P.scales[row0 + row_local]);
        e4 = e4_row(row0 + row_local);
      }
    }
  }
  if (!status) {
    const bool ok = single ? (nwords == 0 && x == kRansL) : (q - R.off0 == 2 * nwords && x == kRansL);
    if (!__all_sync(0xFFFFFFFFu, ok)) status |= EQ_DEV_CORRUPT_STATE;
  }
  // every copy handed to the engine lands before the ring takes the warp's next chunk
  if (!single) status |= R.drain();
  return status;
}

// CTA shapes.  7-bit tables: one CTA of up to 32 warps per SM (the pair table fills most of its
// shared memory) while the accumulators are few, else 16.  Other tables with few accumulators:
// CTAs of 4 warps, 9 per SM (at most 56 registers a thread), so that 36 warps share an SM and a
// tensor of long rows (5120 chunks of 13824 weights) runs in one wave instead of a full wave and a
// tail; else up to 16 warps.
__host__ __device__ constexpr uint32_t gemv_max_warps(uint32_t pb, int bmax) {
  return pb == kRansPairBits ? (bmax <= 4 ? 32u : 16u) : (bmax <= 4 ? 4u : 16u);
}
__host__ __device__ constexpr uint32_t gemv_min_ctas(uint32_t pb, int bmax) {
  return pb != kRansPairBits && bmax <= 4 ? 9u : 1u;
}

template <int FMT, int BMAX, uint32_t PB>
__global__ void __launch_bounds__(32 * gemv_max_warps(PB, BMAX), gemv_min_ctas(PB, BMAX))
    rans_gemv_kernel(const __grid_constant__ GemvParams P) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint32_t *lut = reinterpret_cast<uint32_t *>(smem);
  unsigned char *rings = smem + rans_lut_bytes(PB);
  uint64_t *bars = reinterpret_cast<uint64_t *>(rings + P.warps * kRingBytes);
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const RansTableHeader hdr = *reinterpret_cast<const RansTableHeader *>(P.table);
  const bool table_ok = load_table<FMT, PB>(lut, P.table, hdr);
  WordRing R;
  ring_init(R, smem, rings, bars, warp, lane);
  __syncthreads();

  uint64_t chunk = uint64_t(blockIdx.x) * P.warps + warp;
  if (chunk >= P.num_chunks) return;
  const uint64_t stride = uint64_t(gridDim.x) * P.warps;
  uint32_t status = table_ok ? 0u : EQ_DEV_CORRUPT_STATE;
  for (; chunk < P.num_chunks && !status; chunk += stride)
    status = gemv_chunk<FMT, BMAX, PB>(P, chunk, hdr, lut, smem, R, lane);
  if (lane == 0) report(P.status, status);
}

// ------------------------------------------------------------------------------------------------
// The gate and up products of a LLaMA-style MLP block and its SiLU gate in one kernel: a warp
// takes row r of gate and then row r of up (one row per chunk; the CTA holds both tables and
// the warp's ring takes one substream after the other), and writes h[b][r] = bf16(silu(g) * u)
// with silu(v) = v / (1 + e^-v).  The gate's and up's products never leave the warp.
// ------------------------------------------------------------------------------------------------
struct GateUpParams {
  GemvParams g, u;  // gate and up (their y is not used)
  uint16_t *h;      // bf16 [batch][rows]
};

constexpr uint32_t kGateUpWarps = 8;

template <int FMT, int BMAX, uint32_t PB>
__global__ void __launch_bounds__(32 * kGateUpWarps, 4)
    rans_gate_up_kernel(const __grid_constant__ GateUpParams P) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint32_t *lut_g = reinterpret_cast<uint32_t *>(smem);
  uint32_t *lut_u = reinterpret_cast<uint32_t *>(smem + rans_lut_bytes(PB));
  unsigned char *rings = smem + 2 * rans_lut_bytes(PB);
  uint64_t *bars = reinterpret_cast<uint64_t *>(rings + kGateUpWarps * kRingBytes);
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const RansTableHeader hg = *reinterpret_cast<const RansTableHeader *>(P.g.table);
  const RansTableHeader hu = *reinterpret_cast<const RansTableHeader *>(P.u.table);
  const bool ok_g = load_table<FMT, PB>(lut_g, P.g.table, hg);
  const bool ok_u = load_table<FMT, PB>(lut_u, P.u.table, hu);
  WordRing R;
  ring_init(R, smem, rings, bars, warp, lane);
  __syncthreads();

  uint32_t status = ok_g && ok_u ? 0u : EQ_DEV_CORRUPT_STATE;
  for (uint64_t row = uint64_t(blockIdx.x) * kGateUpWarps + warp; row < P.g.num_chunks && !status;
       row += uint64_t(gridDim.x) * kGateUpWarps) {
    float sg[BMAX], su[BMAX];
    status = gemv_chunk<FMT, BMAX, PB, true>(P.g, row, hg, lut_g, smem, R, lane, sg);
    if (!status) status = gemv_chunk<FMT, BMAX, PB, true>(P.u, row, hu, lut_u, smem, R, lane, su);
    if (!status && lane == 0) {
#pragma unroll
      for (int b = 0; b < BMAX; ++b) {
        if (b < int(P.g.batch)) {
          const float v = sg[b];
          const __nv_bfloat16 hb = __float2bfloat16_rn(v / (1.0f + expf(-v)) * su[b]);
          P.h[size_t(b) * P.g.rows + row] = *reinterpret_cast<const uint16_t *>(&hb);
        }
      }
    }
  }
  if (lane == 0) report(P.g.status, status);
}

__host__ __device__ constexpr size_t gate_up_smem_bytes(uint32_t pb) {
  return 2 * rans_lut_bytes(pb) + kGateUpWarps * (kRingBytes + kNumSeg * 8);
}

// ------------------------------------------------------------------------------------------------
// Batch >= 8: the product goes to the tensor cores.  A CTA of 16 warps decodes 16 chunks in
// lock-step, one round (256 weights of one row per warp) at a time; each warp writes its
// dequantised bf16 weights into a shared 16 x 256 tile, and after a barrier the 16 warps multiply
// the tile by the matching 256 x batch slice of x with mma.m16n8k16 (bf16 in, fp32 accumulate),
// one 16-column k-step each.  At the end of a weight row the 16 warps' partial products are
// summed in a fixed order through shared memory and written to y.  The weights are the ones
// eq_decode returns and every product is exact in fp32, as in the CUDA-core path.
// ------------------------------------------------------------------------------------------------
constexpr uint32_t kTcWarps = 16;
constexpr uint32_t kTcRowBytes = 256 * 2 + 16;  // one tile row, padded against bank conflicts
constexpr uint32_t kTcTileBytes = kTcWarps * kTcRowBytes;
constexpr uint32_t kTcRedBytes = kTcWarps * 16 * 16 * 4;  // [16 warps][16 rows][16 b] fp32
static_assert(2 * kTcTileBytes >= kTcRedBytes, "the reduction buffer fits over the two tiles");

// A CTA is HALVES independent groups of 16 warps.  With two (7-bit tables, one CTA per SM beside
// the pair table), each half's reduction buffer lies over its own two tiles, so both fit.
__host__ __device__ constexpr uint32_t gemv_tc_half_bytes(int halves) {
  return halves > 1 ? 2 * kTcTileBytes : 2 * kTcTileBytes + kTcRedBytes;
}
__host__ __device__ constexpr size_t gemv_tc_smem_bytes(uint32_t pb, int halves) {
  return rans_smem_bytes(halves * kTcWarps, pb) + halves * gemv_tc_half_bytes(halves);
}
static_assert(gemv_tc_smem_bytes(kRansPairBits, 2) <= 227 * 1024, "two halves beside the pair table");

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&a)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(addr));
}

// Each half of the CTA takes group after group of 16 chunks; every warp of a half runs the same
// rounds, so its barriers line up.
template <int FMT, uint32_t PB, int HALVES>
__global__ void __launch_bounds__(HALVES * kTcWarps * 32, HALVES == 1 ? 2 : 1)
    rans_gemv_tc_kernel(const __grid_constant__ GemvParams P) {
  constexpr uint32_t S = 32;
  constexpr bool kAlias = HALVES > 1;  // the reduction buffer lies over the half's tiles
  extern __shared__ __align__(128) unsigned char smem[];
  uint32_t *lut = reinterpret_cast<uint32_t *>(smem);
  unsigned char *rings = smem + rans_lut_bytes(PB);
  uint64_t *bars = reinterpret_cast<uint64_t *>(rings + HALVES * kTcWarps * kRingBytes);
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t half = warp / kTcWarps, hw = warp % kTcWarps;  // hw: this warp's tile row
  const uint32_t grp = lane >> 2, tig = lane & 3;
  unsigned char *tiles = smem + rans_smem_bytes(HALVES * kTcWarps, PB) +
                         half * gemv_tc_half_bytes(HALVES);  // 2 x [16][264] bf16
  float *red = reinterpret_cast<float *>(kAlias ? tiles : tiles + 2 * kTcTileBytes);
  // the half's own barrier (named barrier 1 + half; barrier 0 is the CTA's)
  auto half_sync = [&]() {
    if constexpr (HALVES == 1) __syncthreads();
    else asm volatile("bar.sync %0, %1;" ::"r"(1u + half), "n"(kTcWarps * 32) : "memory");
  };

  const RansTableHeader hdr = *reinterpret_cast<const RansTableHeader *>(P.table);
  const bool table_ok = load_table<FMT, PB>(lut, P.table, hdr);
  WordRing R;
  ring_init(R, smem, rings, bars, warp, lane);
  __syncthreads();

  const bool single = hdr.flags & kRansFlagSingle;
  const bool nan_codes = (FMT == EQ_SYM_E4M3) && (hdr.flags & (kRansFlagNaN7F | kRansFlagNaNFF));
  const uint32_t lt = lanemask_lt();
  const uint32_t rounds = P.chunk_symbols / 256;  // the same for every warp of the launch
  const uint32_t rpr = P.rows_per_chunk > 1 ? P.rounds_per_row : rounds;
  const uint32_t ntiles = (P.batch + 7) / 8;
  const uint32_t tiles_addr = smem_addr(tiles);
  const uint32_t tb = smem_addr(lut), ring_abs = R.buf_s;
  const uint64_t ngroups = (P.num_chunks + kTcWarps - 1) / kTcWarps;
  // sticky: a warp whose chunk failed feeds zeros from then on (the launch reports the failure)
  uint32_t status = 0;

  for (uint64_t cg = uint64_t(blockIdx.x) * HALVES + half; cg < ngroups; cg += uint64_t(gridDim.x) * HALVES) {
    // a warp without a chunk, or whose chunk failed, feeds zeros
    const uint64_t chunk = cg * kTcWarps + hw;
    const bool have = chunk < P.num_chunks;
    if (have && !table_ok) status |= EQ_DEV_CORRUPT_STATE;
    uint32_t x = kRansL, nwords = 0, q = 0, n = 0;
    bool started = false;
    if (have && !status) {
      const uint64_t j0 = chunk * uint64_t(P.chunk_symbols);
      n = uint32_t(P.numel - j0 < P.chunk_symbols ? P.numel - j0 : P.chunk_symbols);
      const uint64_t w0 = P.word_off[chunk], w1 = P.word_off[chunk + 1];
      if (w1 < w0 || w1 - w0 >= (1ull << 30)) status |= EQ_DEV_OVERRUN;
      nwords = status ? 0u : uint32_t(w1 - w0);
      x = P.states[chunk * S + lane];
      if (!status && !single) {
        R.start(P.words, w0, nwords, lane);
        q = R.off0;
        started = true;
      }
    }
    const bool valid = have && !status;  // this chunk decodes (status may still turn nonzero)
    bool live = valid && !single;        // decoding from the stream
    const uint32_t runs = n / 8;
    const uint32_t row0 = uint32_t(chunk * P.rows_per_chunk);
    float c[2][4] = {};
    uint32_t row_local = 0;
    float sc = valid ? bf16_bits_to_float(P.scales[row0]) : 0.0f;
    auto e4_row = [&](uint32_t row) {
      return PB == 12 && FMT == EQ_SYM_E4M3 && !nan_codes && !single &&
             (P.scales[row] & 0x7FFFu) < 0x4380u;
    };
    bool e4 = valid && e4_row(row0);

    for (uint32_t r = 0; r < rounds; ++r) {
      const bool act = valid && !status && r * S + lane < runs;
      // this warp's slice of x for the round's product, loaded before the decode so that the
      // loads' latency passes while the round decodes: columns col0, col0 + 8 of batch rows
      // nt * 8 + grp (a 16-column k-step per warp)
      uint32_t xb[2][2] = {{0u, 0u}, {0u, 0u}};
      {
        const uint32_t col0 = (r % rpr) * 256 + hw * 16 + 2 * tig;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const uint32_t b = nt * 8 + grp;
          if (uint32_t(nt) < ntiles && b < P.batch) {
            const uint16_t *xr = P.x + size_t(b) * P.cols + col0;
            xb[nt][0] = __ldg(reinterpret_cast<const uint32_t *>(xr));
            xb[nt][1] = __ldg(reinterpret_cast<const uint32_t *>(xr + 8));
          }
        }
      }
      uint32_t pr[4] = {0u, 0u, 0u, 0u};
      // E4M3 rounds in which every lane holds a run (no NaN codes, row scale below 2^8): the
      // decode kernel's round block, whose weights come out dequantised
      bool done = false;
      uint4 wv = make_uint4(0u, 0u, 0u, 0u);
      if (live) {
        if (!R.round_wait(q)) {
          status |= EQ_DEV_TIMEOUT;
          live = false;
        } else {
          if constexpr (PB == 12 && FMT == EQ_SYM_E4M3) {
            if (e4 && (r + 1) * S <= runs) {
              wv = rans_round12_e4m3<kRingBytes, false>(x, q, tb, ring_abs, lt, scale_e4m3_offset(sc));
              done = true;
            }
          }
          if (!done) round_pairs<PB>(pr, x, act, lut, smem, R, q, lt);
          if (q - R.off0 > 2 * nwords) {
            status |= EQ_DEV_OVERRUN;
            live = false;
            wv = make_uint4(0u, 0u, 0u, 0u);
          } else {
            R.round_refill(q, lane);
          }
        }
      } else if (single) {
        pr[0] = pr[1] = pr[2] = pr[3] = single_pair<FMT, PB>(hdr.single_sym);
      }
      // this warp's 256 weights of the round -> tile row hw
      if (act && !status && !done) {
        wv.x = weights2<FMT, PB>(pr[0], sc, nan_codes);
        wv.y = weights2<FMT, PB>(pr[1], sc, nan_codes);
        wv.z = weights2<FMT, PB>(pr[2], sc, nan_codes);
        wv.w = weights2<FMT, PB>(pr[3], sc, nan_codes);
      }
      unsigned char *tile = tiles + (r & 1) * kTcTileBytes;
      *reinterpret_cast<uint4 *>(tile + hw * kTcRowBytes + lane * 16) = wv;
      half_sync();
      // warp w multiplies tile columns [16 w, 16 w + 16) by x[:, col0 + 16 w ...]
      {
        uint32_t a[4];
        const uint32_t arow = lane & 15, acol = (lane >> 4) * 8 + hw * 16;
        ldmatrix_x4(a, tiles_addr + (r & 1) * kTcTileBytes + arow * kTcRowBytes + acol * 2);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
          if (uint32_t(nt) < ntiles) mma_bf16_16816(c[nt], a, xb[nt][0], xb[nt][1]);
      }
      // end of a weight row: sum the 16 warps' partial products in a fixed order
      if ((r + 1) % rpr == 0) {
        if constexpr (kAlias) half_sync();  // every warp is done with the tiles
        float *mine = red + hw * 256;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          mine[grp * 16 + nt * 8 + 2 * tig] = c[nt][0];
          mine[grp * 16 + nt * 8 + 2 * tig + 1] = c[nt][1];
          mine[(grp + 8) * 16 + nt * 8 + 2 * tig] = c[nt][2];
          mine[(grp + 8) * 16 + nt * 8 + 2 * tig + 1] = c[nt][3];
          c[nt][0] = c[nt][1] = c[nt][2] = c[nt][3] = 0.0f;
        }
        half_sync();
        const uint32_t th = threadIdx.x - half * kTcWarps * 32;
        if (th < 256) {
          const uint32_t wr = th >> 4, b = th & 15;  // tile row wr
          float v = 0.0f;
          for (uint32_t w = 0; w < kTcWarps; ++w) v += red[w * 256 + wr * 16 + b];
          const uint64_t ch = cg * kTcWarps + wr;
          const uint64_t row = ch * P.rows_per_chunk + (r / rpr);
          if (P.n_patch && ch < P.num_chunks && b < P.batch && row < P.rows) {  // super weights
            const uint64_t rs = row * P.cols;
            const uint64_t hi = patch_lower_bound(P.patch_idx, P.n_patch, rs + P.cols);
            for (uint64_t i = patch_lower_bound(P.patch_idx, P.n_patch, rs); i < hi; ++i)
              v = fmaf(bf16_bits_to_float(__ldg(P.patch_val + i)),
                       bf16_bits_to_float(P.x[size_t(b) * P.cols + (__ldg(P.patch_idx + i) - rs)]), v);
          }
          if (ch < P.num_chunks && b < P.batch && row < P.rows) P.y[size_t(b) * P.rows + row] = v;
        }
        if constexpr (kAlias) half_sync();  // the sums are read before the tiles are rewritten
        ++row_local;
        if (valid && !status && row_local < P.rows_per_chunk) {
          sc = bf16_bits_to_float(P.scales[row0 + row_local]);
          e4 = e4_row(row0 + row_local);
        }
      }
    }
    if (valid && !status) {
      const bool ok = single ? (nwords == 0 && x == kRansL) : (q - R.off0 == 2 * nwords && x == kRansL);
      if (!__all_sync(0xFFFFFFFFu, ok)) status |= EQ_DEV_CORRUPT_STATE;
    }
    // every copy handed to the engine lands before the ring takes the next chunk
    if (started) status |= R.drain();
  }
  if (lane == 0) report(P.status, status);
}

using GemvFn = void (*)(GemvParams);

template <int FMT, uint32_t PB>
static GemvFn pick_b(uint32_t batch, bool tc) {
  if (tc) return rans_gemv_tc_kernel<FMT, PB, PB == kRansPairBits ? 2 : 1>;
  if (batch <= 1) return rans_gemv_kernel<FMT, 1, PB>;
  if (batch <= 2) return rans_gemv_kernel<FMT, 2, PB>;
  if (batch <= 4) return rans_gemv_kernel<FMT, 4, PB>;
  if (batch <= 8) return rans_gemv_kernel<FMT, 8, PB>;
  return rans_gemv_kernel<FMT, 16, PB>;
}

template <int FMT>
static GemvFn pick_pb(uint32_t pb, uint32_t batch, bool tc) {
  return pb == 12 ? pick_b<FMT, 12>(batch, tc) : pb == 8 ? pick_b<FMT, 8>(batch, tc)
                                                         : pick_b<FMT, kRansPairBits>(batch, tc);
}

static std::atomic<bool> g_gemv_attr[64][2][3][6];
static std::atomic<bool> g_gate_up_attr[64][2][2][3];  // device, symfmt, table (12 / 8), batch kind

// the kernel parameters of one tensor's product
static GemvParams gemv_params(const eq_rans_tensor *t, const uint16_t *d_x, uint32_t batch,
                              float *d_y, uint32_t *d_status, uint32_t warps) {
  const uint32_t rpc = t->chunk_symbols / t->cols;
  GemvParams P;
  P.states = t->states;
  P.word_off = t->word_off;
  P.words = t->words;
  P.scales = t->scales;
  P.table = static_cast<const uint32_t *>(t->tables);
  P.x = d_x;
  P.y = d_y;
  P.status = d_status;
  P.patch_idx = t->patch_idx;
  P.patch_val = t->patch_val;
  P.n_patch = t->n_patch;
  P.numel = uint64_t(t->rows) * t->cols;
  P.num_chunks = t->num_chunks;
  P.rows = t->rows;
  P.cols = t->cols;
  P.chunk_symbols = t->chunk_symbols;
  P.rows_per_chunk = rpc;
  P.rounds_per_row = rpc > 1 ? t->cols / (t->streams * 8) : 0;
  P.batch = batch;
  P.warps = warps;
  return P;
}

template <int FMT, uint32_t PB>
static void (*pick_gate_up(uint32_t batch))(GateUpParams) {
  if (batch <= 1) return rans_gate_up_kernel<FMT, 1, PB>;
  if (batch <= 2) return rans_gate_up_kernel<FMT, 2, PB>;
  return rans_gate_up_kernel<FMT, 4, PB>;
}

// The gate and up products and the SiLU gate of an MLP block in one launch, h = bf16(silu(W_gate
// x) * (W_up x)), when both tensors take the fused kernel: batch <= 4, 12- or 8-bit tables of one
// symbol format, one row per chunk (chunk_symbols == cols), 32 streams, run 8.  EQ_ERR_UNSUPPORTED
// (nothing launched) otherwise.  Both descriptors were validated by the caller.
eq_status gate_up_launch(const eq_rans_tensor *g, const eq_rans_tensor *u, const uint16_t *d_x,
                         uint32_t batch, uint16_t *d_h, uint32_t *d_status, cudaStream_t st) {
  if (batch > 4 || g->symfmt != u->symfmt || g->prob_bits != u->prob_bits) return EQ_ERR_UNSUPPORTED;
  if (g->prob_bits != 12 && g->prob_bits != 8) return EQ_ERR_UNSUPPORTED;
  for (const eq_rans_tensor *t : {g, u})
    if (t->run != 8 || t->streams != 32 || t->chunk_symbols != t->cols || t->rows != g->rows ||
        t->cols != g->cols)
      return EQ_ERR_UNSUPPORTED;
  if (!d_x || !d_h || !aligned(d_x, 16)) return EQ_ERR_ARG;
  const uint32_t pb = g->prob_bits;
  auto fn = g->symfmt == EQ_SYM_E4M3
                ? (pb == 12 ? pick_gate_up<EQ_SYM_E4M3, 12>(batch) : pick_gate_up<EQ_SYM_E4M3, 8>(batch))
                : (pb == 12 ? pick_gate_up<EQ_SYM_INT8, 12>(batch) : pick_gate_up<EQ_SYM_INT8, 8>(batch));
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return EQ_ERR_CUDA;
  const int bi = batch <= 1 ? 0 : batch <= 2 ? 1 : 2;
  if (smem_optin_once(g_gate_up_attr[dev][g->symfmt - 1][pb == 12 ? 0 : 1][bi],
                      reinterpret_cast<const void *>(fn), gate_up_smem_bytes(pb)) != EQ_OK)
    return EQ_ERR_CUDA;
  GateUpParams P;
  P.g = gemv_params(g, d_x, batch, nullptr, d_status, kGateUpWarps);
  P.u = gemv_params(u, d_x, batch, nullptr, d_status, kGateUpWarps);
  P.h = d_h;
  const uint64_t ctas = (uint64_t(g->rows) + kGateUpWarps - 1) / kGateUpWarps;
  if (ctas >= (1ull << 31)) return EQ_ERR_UNSUPPORTED;
  fn<<<uint32_t(ctas), 32 * kGateUpWarps, gate_up_smem_bytes(pb), st>>>(P);
  return cuda_status(cudaGetLastError());
}  // device, symfmt, table (12 / 8 / 7 bits), kernel instance

}  // namespace eq

using namespace eq;

extern "C" eq_status eq_decode_gemv(const eq_rans_tensor *t, const uint16_t *d_x, uint32_t batch,
                                    float *d_y, uint32_t *d_status, void *stream) {
  if (!t || !d_status) return EQ_ERR_ARG;
  eq_status s = validate_rans_tensor(*t);
  if (s != EQ_OK) return s;
  if (batch < 1 || batch > 16) return EQ_ERR_ARG;
  if (t->rows == 0 || t->cols == 0) return EQ_OK;
  if (!d_x || !d_y || !aligned(d_x, 16) || !aligned(d_y, 4)) return EQ_ERR_ARG;
  if (t->run != 8 || t->streams != 32 || t->chunk_symbols % t->cols) return EQ_ERR_UNSUPPORTED;
  const uint32_t rpc = t->chunk_symbols / t->cols;
  if (rpc > 1 && t->cols % (t->streams * 8)) return EQ_ERR_UNSUPPORTED;
  // batch >= 8 on the tensor cores when a round never straddles a chunk's 256-column tiles
  const bool tc = batch >= 8 && t->chunk_symbols % 256 == 0;
  const uint32_t pb = t->prob_bits;
  const bool pair = pb == kRansPairBits;
  GemvFn fn = t->symfmt == EQ_SYM_E4M3 ? pick_pb<EQ_SYM_E4M3>(pb, batch, tc) : pick_pb<EQ_SYM_INT8>(pb, batch, tc);
  const uint64_t sms = uint64_t(device_sm_count());
  const int bmax = batch <= 1 ? 1 : batch <= 2 ? 2 : batch <= 4 ? 4 : batch <= 8 ? 8 : 16;
  uint32_t warps, max_warps;
  uint64_t ctas;
  if (tc) {
    // 7-bit tables: one CTA per SM, two halves of 16 warps, each taking group after group
    warps = max_warps = pair ? 2 * kTcWarps : kTcWarps;
    ctas = (t->num_chunks + warps - 1) / warps;
    if (pair) ctas = std::min<uint64_t>(ctas, sms);
  } else if (pair) {
    // one CTA per SM holds the pair table; enough warps that the SMs' CTAs take every chunk
    // about once (more chunks: the warps loop)
    max_warps = gemv_max_warps(pb, bmax);
    warps = uint32_t(std::min<uint64_t>(max_warps, std::max<uint64_t>(1, (t->num_chunks + sms - 1) / sms)));
    ctas = std::min<uint64_t>(sms, (t->num_chunks + warps - 1) / warps);
  } else {
    warps = max_warps = gemv_max_warps(pb, bmax);
    while (warps > 1 && (t->num_chunks + warps - 1) / warps < 4 * sms) warps >>= 1;
    ctas = (t->num_chunks + warps - 1) / warps;
  }
  if (ctas >= (1ull << 31)) return EQ_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return EQ_ERR_CUDA;
  // one flag per kernel instance that pick_pb can return
  const int bi = tc ? 5 : bmax == 1 ? 0 : bmax == 2 ? 1 : bmax == 4 ? 2 : bmax == 8 ? 3 : 4;
  if (smem_optin_once(g_gemv_attr[dev][t->symfmt - 1][pb == 12 ? 0 : pb == 8 ? 1 : 2][bi],
                      reinterpret_cast<const void *>(fn),
                      tc ? gemv_tc_smem_bytes(pb, pair ? 2 : 1) : rans_smem_bytes(max_warps, pb)) != EQ_OK)
    return EQ_ERR_CUDA;
  const GemvParams P = gemv_params(t, d_x, batch, d_y, d_status, warps);
  fn<<<uint32_t(ctas), 32 * warps, tc ? gemv_tc_smem_bytes(pb, pair ? 2 : 1) : rans_smem_bytes(warps, pb),
       static_cast<cudaStream_t>(stream)>>>(P);
  return cuda_status(cudaGetLastError());
}
