// eq_decode: interleaved-rANS decode + dequantisation to bf16 on sm_100a.
//
// What it computes is fixed by the format in eq.h ("Float8@2bits" summary: Float8-E4M3 / Int8
// symbols with per-channel scales, flattened and ANS-coded, decoded on the GPU into a buffer before
// the layer runs).  How, on B200:
//   * one warp decodes one group of 32 streams of a chunk, one rANS state per lane; the groups of a
//     chunk read separate word substreams, so a 64 KiB chunk keeps several warps busy and an SM
//     holds dozens of independent decoders to hide the shared-memory latency of each step;
//   * the 4096-entry slot table (16 KiB) sits in shared memory, one 32-bit load per symbol;
//   * the group's 16-bit words stream through a per-warp shared-memory ring fed by 1-D bulk copies
//     (TMA engine, completion on an mbarrier), checked and refilled once per round of 8 steps;
//   * renormalisation is warp-cooperative: a ballot of the lanes whose state fell below 2^16, a
//     popcount rank hands each its word, in stream order;
//   * with run = 8 a lane emits eight consecutive bf16 per round: one 16-byte store, the warp
//     writes 512 contiguous bytes;
//   * dequantisation (value * row scale, one rounding) happens in registers before the store.
// Many tensors go in one launch (the pages decode all weights of a transformer block together).
#include <algorithm>
#include <mutex>
#include <type_traits>
#include <vector>

#include "eq_dequant.cuh"
#include "eq_rans_core.cuh"

namespace eq {

// descriptors one launch carries as kernel parameters (128 bytes each, within the 32764-byte
// parameter limit); a larger group goes in several launches of nearly equal size
constexpr int kMaxDecodeTensors = 255;

struct RansDesc {
  const uint32_t *states;
  const uint64_t *word_off;
  const uint16_t *words;
  const uint16_t *scales;
  const uint32_t *table;  // RansTableHeader followed by the slot table
  uint16_t *out;
  const uint64_t *patch_idx;  // super weights: sorted flat indices and bf16 values
  const uint16_t *patch_val;
  uint64_t n_patch;
  uint64_t numel;
  uint64_t units;         // num_chunks * groups: one warp each
  uint64_t row_magic;     // floor(j / cols) = __umul64hi(j, row_magic) (0: cols == 1)
  uint64_t group_magic;   // the same for floor(unit / groups)
  uint32_t rows, cols;
  uint32_t chunk_symbols;
  uint32_t groups;        // streams / 32
  uint32_t cta_begin;     // first CTA of this tensor in the launch
  uint32_t ctas;          // CTAs of this tensor: its warps take units cta_warp, + ctas * warps, ...
};

struct RansDecodeParams {
  uint32_t *status;
  uint32_t n;
  uint32_t warps;  // warps (= groups decoded) per CTA
  uint32_t spread; // units dealt out round-robin over a tensor's CTAs (see the kernel)
  RansDesc d[kMaxDecodeTensors];
};
static_assert(sizeof(RansDecodeParams) <= 32764, "kernel parameters above the launch limit");

// ------------------------------------------------------------------------------------------------
// one round (G steps) of one group; FULL: every lane holds a run this round.  A 12-bit stream
// renormalises after every step; an 8-bit one (G = 8) after positions 1, 3, 5 and 7, i.e. after
// every second of its own steps, since each round gives it one whole run.
// ------------------------------------------------------------------------------------------------
template <bool FULL, int G, int FMT, uint32_t PB, bool MAYBE_NAN = true, class Ring>
__device__ __forceinline__ void decode_round(const RansDesc &D, uint32_t &x, bool act,
                                             const uint32_t *lut, const unsigned char *smem,
                                             const Ring &R, uint32_t &q, uint32_t lt,
                                             uint16_t *out, float sc, bool nan_codes_,
                                             uint32_t tb = 0, uint32_t ring = 0) {
  static_assert(PB == 12 || G == 8, "7- and 8-bit tables need whole runs of 8");
  // MAYBE_NAN false: the table has no NaN code, and the checks compile away
  const bool nan_codes = MAYBE_NAN && nan_codes_;
  if constexpr (PB == kRansPairBits) {  // one lookup per pair of steps
    uint32_t pv[4];  // the pairs' values (bf16x2)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      pv[k] = rans_pair_step<FULL>(x, act, lut);
      rans_renorm<FULL>(x, act, smem, R.ring_off, q, lt);
    }
    if (FULL || act) {
      const uint32_t sc2 = scale_bf16x2(sc);
      *reinterpret_cast<uint4 *>(out) =
          make_uint4(pair_dequant(pv[0], sc2, nan_codes), pair_dequant(pv[1], sc2, nan_codes),
                     pair_dequant(pv[2], sc2, nan_codes), pair_dequant(pv[3], sc2, nan_codes));
    }
  } else if constexpr (PB == 12) {  // entries [symbol | f | slot - cum]
    // tb, ring: shared addresses of the table (the start of the shared memory) and of this
    // warp's ring, converted once per unit by the caller.  (The caller runs the E4M3 round block
    // itself where it applies.)
    if constexpr (G == 8) {
      uint32_t e[8];
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        e[p] = rans_sym_step<FULL>(x, act, tb);
        rans_renorm_abs<FULL, Ring::kBytes>(x, act, ring, q, lt);
      }
      if (FULL || act) {
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
          o[k] = dequant2<FMT>(__byte_perm(e[2 * k], e[2 * k + 1], 0x0073u), sc, nan_codes);
        *reinterpret_cast<uint4 *>(out) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    } else {
      const uint32_t e = rans_sym_step<FULL>(x, act, tb);
      rans_renorm_abs<FULL, Ring::kBytes>(x, act, ring, q, lt);
      if (FULL || act) *out = dequant1<FMT>(e >> 24, sc);
    }
  } else {
    uint32_t e[G];
#pragma unroll
    for (int p = 0; p < G; ++p) {
      e[p] = rans_decode_step<FULL, PB>(x, act, lut);
      if (p & 1) rans_renorm<FULL>(x, act, smem, R.ring_off, q, lt);
    }
    if (FULL || act) *reinterpret_cast<uint4 *>(out) = dequant8<FMT, PB>(e, sc, nan_codes);
  }
}

// Write the chunk's super weights that fall in this warp's group back over the decoded values
// (after a warp barrier, so the lanes' own stores are ordered before).  A listed position must
// have decoded to zero, and the list must increase; otherwise EQ_DEV_CORRUPT_STATE.
template <int G>
__device__ __forceinline__ uint32_t apply_patches(const RansDesc &D, uint64_t j0, uint32_t n,
                                                  uint32_t g, uint32_t S, uint32_t lane) {
  const uint64_t lo = patch_lower_bound(D.patch_idx, D.n_patch, j0);
  const uint64_t hi = patch_lower_bound(D.patch_idx, D.n_patch, j0 + n);
  uint32_t bad = 0;
  __syncwarp();
  for (uint64_t i = lo + lane; i < hi; i += 32) {
    const uint64_t j = __ldg(D.patch_idx + i);
    if (i + 1 < D.n_patch && __ldg(D.patch_idx + i + 1) <= j) bad = EQ_DEV_CORRUPT_STATE;
    if (((uint32_t(j - j0) / G) % S) / 32 != g) continue;  // another group's run
    if (D.out[j] & 0x7FFFu) bad = EQ_DEV_CORRUPT_STATE;
    D.out[j] = __ldg(D.patch_val + i);
  }
  return __reduce_or_sync(0xFFFFFFFFu, bad);  // lane 0 reports the warp's status
}

template <int G, int FMT, uint32_t PB, class Ring>
__device__ __forceinline__ uint32_t decode_group(const RansDesc &D, const uint32_t *lut,
                                                 const unsigned char *smem, uint32_t flags,
                                                 uint32_t single_sym, Ring &R, uint64_t unit,
                                                 uint32_t lane) {
  const uint64_t chunk = div_by_magic(unit, D.group_magic);
  const uint32_t g = uint32_t(unit - chunk * D.groups);
  const uint32_t S = 32 * D.groups, s = 32 * g + lane;
  const uint64_t j0 = chunk * uint64_t(D.chunk_symbols);
  const uint32_t n = uint32_t(D.numel - j0 < D.chunk_symbols ? D.numel - j0 : D.chunk_symbols);
  const uint64_t w0 = D.word_off[unit], w1 = D.word_off[unit + 1];
  if (w1 < w0 || w1 - w0 >= (1ull << 30)) return EQ_DEV_OVERRUN;
  const uint32_t nwords = uint32_t(w1 - w0);
  const uint32_t runs = (n + G - 1) / G;
  const uint32_t rounds = (runs + S - 1) / S;
  uint32_t x = D.states[chunk * S + s];
  uint32_t status = 0;

  if (flags & kRansFlagSingle) {  // one symbol owns every slot: states never move, no words
    if (!__all_sync(0xFFFFFFFFu, nwords == 0 && x == kRansL)) status |= EQ_DEV_CORRUPT_STATE;
    for (uint32_t r = 0; r < rounds; ++r) {
      const uint32_t run = r * S + s;
      if (run >= runs) continue;
      for (uint32_t i = 0; i < uint32_t(G); ++i) {
        const uint64_t j = j0 + uint64_t(run) * G + i;
        if (j >= j0 + n) break;
        D.out[j] = dequant1<FMT>(single_sym, bf16_bits_to_float(D.scales[div_by_magic(j, D.row_magic)]));
      }
    }
    if (D.n_patch && !status) status |= apply_patches<G>(D, j0, n, g, S, lane);
    return status;
  }

  R.start(D.words, w0, nwords, lane);
  const bool nan_codes = (FMT == EQ_SYM_E4M3) && (flags & (kRansFlagNaN7F | kRansFlagNaNFF));
  const uint32_t lt = lanemask_lt_once();
  const uint32_t tb = smem_addr(smem), ring = R.buf_s;
  // rounds in which all 32 lanes of this group hold a run
  const uint32_t full = runs >= 32 * g + 32 ? (runs - 32 * g - 32) / S + 1 : 0;
  uint32_t q = R.off0;
  // the lane's first output and its row; both advance by S runs per round
  uint64_t jrun = j0 + uint64_t(s) * G;
  const uint32_t step = S * G, cols = D.cols;
  uint32_t row = uint32_t(div_by_magic(jrun, D.row_magic));
  uint32_t col = uint32_t(jrun - uint64_t(row) * cols);
  float sc = bf16_bits_to_float(D.scales[row < D.rows ? row : 0]);
  uint16_t *out = D.out + jrun;
  // ring checks once per round (12-bit: up to 256 words a round), or once per two rounds
  // (8-bit: up to 128 words a round); round_wait covers 256 words and one more
  constexpr uint32_t kRoundsPerCheck = PB == 12 ? 1 : 2;
  const uint32_t q_end = R.off0 + 2 * nwords;
  uint32_t r0 = 0;

  // One round's advance of the lane's output position, row and scale.  ONE_WRAP (rows of at
  // least S * G symbols): a round crosses at most one row end, so a compare and a conditional
  // update, no loop.
  auto advance = [&](auto one_wrap) {
    out += step;
    col += step;
    if constexpr (decltype(one_wrap)::value) {
      if (col >= cols) {
        col -= cols;
        ++row;
        sc = bf16_bits_to_float(D.scales[row < D.rows ? row : 0]);
      }
    } else if (col >= cols) {
      do {
        col -= cols;
        ++row;
      } while (col >= cols);
      if (row < D.rows) sc = bf16_bits_to_float(D.scales[row]);
    }
  };
  // 8- and 7-bit tables: the rounds in which every lane of the group holds a run, the ring work
  // (overrun check, refill, wait) every second round and only once q reaches q_next; refill comes
  // before the wait, so every segment a wait needs has been handed to the copy engine.
  // Instantiated for tables with and without NaN codes and for one or several row ends per
  // round, so that none of those tests is left in the loop.
  uint32_t q_next = 0;
  auto run_full = [&](auto maybe_nan, auto one_wrap) -> uint32_t {
    for (; r0 + kRoundsPerCheck <= full; r0 += kRoundsPerCheck) {
      if (q >= q_next) {
        if (q > q_end) return EQ_DEV_OVERRUN;
        R.round_refill(q, lane);
        if (!R.round_wait(q)) return EQ_DEV_TIMEOUT;
        q_next = R.quiet_until(q_end);
      }
#pragma unroll
      for (uint32_t k = 0; k < kRoundsPerCheck; ++k) {
        decode_round<true, G, FMT, PB, decltype(maybe_nan)::value>(D, x, true, lut, smem, R, q,
                                                                   lt, out, sc, true, tb, ring);
        advance(one_wrap);
      }
    }
    return 0u;
  };
  // 12-bit tables: the full rounds in batches (the ring's batch protocol), each batch a loop with
  // nothing in it but the round, its store and the row tracking; the edges after it.  FAST: the
  // E4M3 round block (Float8-E4M3 symbols, no NaN code in the table, every row scale of the unit
  // below 2^8 in magnitude), with the row scale as its factor scale * 2^120.  MODE 0: rounds
  // never straddle a row (cols and the chunk length multiples of S * G), so the row and its
  // scale are the warp's and change every cols / step rounds (with the E4M3 block the unit's
  // row factors are held one row per lane, 32 rows at a time, and a row change is a shuffle),
  // and each lane's row, column and scale are recomputed afterwards for the general loop;
  // MODE 1: a round crosses at most one row end (a compare and a conditional update); MODE 2:
  // rows shorter than a round.
  auto run_batches = [&](auto fast, auto maybe_nan, auto mode) -> uint32_t {
    constexpr bool FAST = decltype(fast)::value;
    constexpr int MODE = decltype(mode)::value;
    uint32_t per_row = 0, left = 0;
    if constexpr (MODE == 0) {
      per_row = cols / step;
      row = uint32_t(div_by_magic(j0, D.row_magic));
      left = per_row - uint32_t(j0 - uint64_t(row) * cols) / step;
      sc = bf16_bits_to_float(D.scales[row]);
    }
    uint32_t sc2e = FAST ? scale_e4m3_offset(sc) : 0u;
    uint32_t tab_base = row, tab = 0;  // MODE 0 with FAST: row tab_base + lane's factor
    auto load_tab = [&]() {
      const uint32_t r = tab_base + lane;
      tab = scale_e4m3_offset(bf16_bits_to_float(D.scales[r < D.rows ? r : 0]));
    };
    if constexpr (MODE == 0 && FAST) load_tab();
    uint32_t st = 0;
    while (r0 < full) {
      uint32_t nb = min(R.template batch_rounds<G>(q), full - r0);
      r0 += nb;
      auto one_round = [&]() {
        if constexpr (FAST)
          *reinterpret_cast<uint4 *>(out) = rans_round12_e4m3<Ring::kBytes>(x, q, tb, ring, lt, sc2e);
        else
          decode_round<true, G, FMT, PB, decltype(maybe_nan)::value>(D, x, true, lut, smem, R, q,
                                                                     lt, out, sc, true, tb, ring);
        out += step;
      };
      if constexpr (MODE == 0) {
        do {
          one_round();
          if (--left == 0) {
            left = per_row;
            ++row;
            if constexpr (FAST) {
              if (row - tab_base == 32) {
                tab_base = row;
                load_tab();
              }
              sc2e = __shfl_sync(0xFFFFFFFFu, tab, row - tab_base);
            } else {
              sc = bf16_bits_to_float(D.scales[row < D.rows ? row : 0]);
            }
          }
        } while (--nb);
      } else {
        do {
          one_round();
          col += step;
          if (col >= cols) {
            do {
              col -= cols;
              ++row;
            } while (MODE == 2 && col >= cols);
            sc = bf16_bits_to_float(D.scales[row < D.rows ? row : 0]);
            if constexpr (FAST) sc2e = scale_e4m3_offset(sc);
          }
        } while (--nb);
      }
      while (q >= R.edge_next) {
        if (q > q_end) {
          st = EQ_DEV_OVERRUN;
          break;
        }
        if (!R.batch_edge(lane)) {
          st = EQ_DEV_TIMEOUT;
          break;
        }
      }
      if (st) break;
    }
    if constexpr (MODE == 0) {
      const uint64_t j = j0 + (uint64_t(r0) * S + s) * G;
      row = uint32_t(div_by_magic(j, D.row_magic));
      col = uint32_t(j - uint64_t(row) * cols);
      sc = bf16_bits_to_float(D.scales[row < D.rows ? row : 0]);
    }
    return st;
  };
  using T = std::true_type;
  using F = std::false_type;
  using M0 = std::integral_constant<int, 0>;
  using M1 = std::integral_constant<int, 1>;
  using M2 = std::integral_constant<int, 2>;
  // The full rounds go without NaN checks when the table has no NaN code; for 12-bit tables that
  // also selects the E4M3 round block, which needs Float8-E4M3 symbols and every row scale of the
  // unit below 2^8 in magnitude (checked here, one scale per lane).
  if constexpr (PB == 12)
    if (!R.batch_begin(q, lane)) status = EQ_DEV_TIMEOUT;
  bool plain = !nan_codes;
  if constexpr (PB == 12) {
    if (FMT != EQ_SYM_E4M3) plain = false;
    const uint32_t r_first = uint32_t(div_by_magic(j0, D.row_magic));
    const uint32_t r_last = uint32_t(div_by_magic(j0 + n - 1, D.row_magic));
    bool ok = true;
    for (uint32_t r = r_first + lane; r <= r_last; r += 32) ok &= (D.scales[r] & 0x7FFFu) < 0x4380u;
    plain = __all_sync(0xFFFFFFFFu, ok) && plain;
  }
  if constexpr (PB == 12) {
    const bool row_rounds = G == 8 && cols % step == 0 && D.chunk_symbols % step == 0;
    auto dispatch = [&](auto fast, auto maybe_nan) -> uint32_t {
      if constexpr (G == 8)
        if (row_rounds) return run_batches(fast, maybe_nan, M0{});
      return step <= cols ? run_batches(fast, maybe_nan, M1{}) : run_batches(fast, maybe_nan, M2{});
    };
    if (!status) {
      if constexpr (G == 8 && FMT == EQ_SYM_E4M3) status = plain ? dispatch(T{}, F{}) : dispatch(F{}, T{});
      else status = dispatch(F{}, T{});
    }
    R.batch_end();
  } else if (!status) {
    if (!plain) status = step <= cols ? run_full(T{}, T{}) : run_full(T{}, F{});
    else status = step <= cols ? run_full(F{}, T{}) : run_full(F{}, F{});
  }
  if (!status) {  // the general loop below waits first: hand out the used-up slots
    if (q > q_end) status |= EQ_DEV_OVERRUN;
    else R.round_refill(q, lane);
  }
  // the rest (lanes without a run from some round on)
  for (uint32_t r = r0; r < rounds && !status; r += kRoundsPerCheck) {
    if (!R.round_wait(q)) {
      status |= EQ_DEV_TIMEOUT;
      break;
    }
#pragma unroll
    for (uint32_t k = 0; k < kRoundsPerCheck; ++k) {
      const uint32_t rk = r + k;
      if (kRoundsPerCheck > 1 && rk >= rounds) break;
      if (rk < full) decode_round<true, G, FMT, PB>(D, x, true, lut, smem, R, q, lt, out, sc, nan_codes, tb, ring);
      else decode_round<false, G, FMT, PB>(D, x, rk * S + s < runs, lut, smem, R, q, lt, out, sc, nan_codes, tb, ring);
      advance(F{});
    }
    if (q - R.off0 > 2 * nwords) {
      status |= EQ_DEV_OVERRUN;
      break;
    }
    R.round_refill(q, lane);
  }
  if (!status && !__all_sync(0xFFFFFFFFu, q - R.off0 == 2 * nwords && x == kRansL))
    status |= EQ_DEV_CORRUPT_STATE;
  if (D.n_patch && !status) status |= apply_patches<G>(D, j0, n, g, S, lane);
  // every copy handed to the engine must land before the ring is reused or the CTA exits
  status |= R.drain();
  return status;
}

// 7-bit tables: one CTA of up to 32 warps per SM shares the 128 KiB pair table, each warp
// decoding unit after unit; otherwise CTAs of 12 warps (12-bit tables, three per SM) or 16 warps
// (8-bit tables, two per SM), one unit each.  The launch bounds give the register allocator the
// budget of that occupancy.
constexpr uint32_t decode_max_threads(uint32_t pb) {
  return pb == kRansPairBits ? 1024 : pb == 12 ? 384 : 512;
}
constexpr uint32_t decode_min_ctas(uint32_t pb) { return pb == kRansPairBits ? 1 : pb == 12 ? 3 : 2; }

template <int G, int FMT, uint32_t PB>
__global__ void __launch_bounds__(decode_max_threads(PB), decode_min_ctas(PB))
    rans_decode_kernel(const __grid_constant__ RansDecodeParams P) {
  extern __shared__ __align__(128) unsigned char smem[];
  using Ring = WordRingT<PB == 12 ? kSegBytesWide : kSegBytes>;
  uint32_t *lut = reinterpret_cast<uint32_t *>(smem);
  // 12-bit tables: rings at a shared address that is a multiple of their size (the word address
  // is then one mask-and-or); the others right after the table (a multiple of the ring size from
  // the base, which the renormalisation ORs in)
  uint32_t ring_start = decode_lut_bytes(PB);
  if constexpr (PB == 12) {
    const uint32_t base = smem_addr(smem);
    ring_start = ((base + ring_start + Ring::kBytes - 1) & ~(Ring::kBytes - 1)) - base;
  }
  unsigned char *rings = smem + ring_start;
  uint64_t *bars = reinterpret_cast<uint64_t *>(rings + P.warps * Ring::kBytes);

  // tensor of this CTA: the last one whose first CTA is <= blockIdx.x
  uint32_t lo = 0, hi = P.n - 1;
  while (lo < hi) {
    const uint32_t mid = (lo + hi + 1) >> 1;
    if (P.d[mid].cta_begin <= blockIdx.x) lo = mid; else hi = mid - 1;
  }
  const RansDesc D = P.d[lo];
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const RansTableHeader hdr = *reinterpret_cast<const RansTableHeader *>(D.table);
  // the table is only read as far as its header says it reaches: a descriptor whose table is of
  // another size is reported below, never read past its end
  const bool table_ok = hdr.magic == rans_table_magic<FMT, PB>() && hdr.prob_bits == PB;
  const uint4 *src = reinterpret_cast<const uint4 *>(D.table + sizeof(RansTableHeader) / 4);
  constexpr uint32_t kLutVec = PB == kRansPairBits ? kRansPairEntries / 2 : (1u << PB) / 4;
  if (table_ok) {
    if constexpr (PB == 12) {
      // [f:12 | symbol:8 | slot - cum:12] -> [symbol:8 | f:12 | slot - cum:12]
      for (uint32_t i = threadIdx.x; i < kLutVec; i += blockDim.x) {
        const uint4 e = __ldg(src + i);
        reinterpret_cast<uint4 *>(lut)[i] = make_uint4(sym_first_entry(e.x), sym_first_entry(e.y),
                                                       sym_first_entry(e.z), sym_first_entry(e.w));
      }
    } else {
      for (uint32_t i = threadIdx.x; i < kLutVec; i += blockDim.x)
        reinterpret_cast<uint4 *>(lut)[i] = __ldg(src + i);
    }
  }
  Ring R;
  ring_init(R, smem, rings, bars, warp, lane);
  __syncthreads();

  // A CTA's warps take consecutive units (CTA c, warp w: unit c * warps + w, then every
  // ctas * warps), so that an SM writes a few contiguous stretches of the output.  A launch of
  // fewer units than warp slots (P.spread) deals them out round-robin instead (unit w * ctas + c),
  // so that every CTA, and so every SM, gets about the same number.
  const uint64_t cta = blockIdx.x - D.cta_begin;
  uint64_t unit = P.spread ? uint64_t(warp) * D.ctas + cta : cta * P.warps + warp;
  if (unit >= D.units) return;
  const uint64_t stride = uint64_t(D.ctas) * P.warps;
  uint32_t status = table_ok ? 0u : EQ_DEV_CORRUPT_STATE;
  for (; unit < D.units && !status; unit += stride)
    status = decode_group<G, FMT, PB>(D, lut, smem, hdr.flags, hdr.single_sym, R, unit, lane);
  if (lane == 0) report(P.status, status);
}

// ------------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------------
using KernelFn = void (*)(RansDecodeParams);

static KernelFn pick_kernel(uint32_t symfmt, uint32_t run, uint32_t pb) {
  const bool e4 = symfmt == EQ_SYM_E4M3;
  if (run == 8 && pb == 12)
    return e4 ? rans_decode_kernel<8, EQ_SYM_E4M3, 12> : rans_decode_kernel<8, EQ_SYM_INT8, 12>;
  if (run == 8 && pb == 8)
    return e4 ? rans_decode_kernel<8, EQ_SYM_E4M3, 8> : rans_decode_kernel<8, EQ_SYM_INT8, 8>;
  if (run == 8 && pb == kRansPairBits)
    return e4 ? rans_decode_kernel<8, EQ_SYM_E4M3, kRansPairBits>
              : rans_decode_kernel<8, EQ_SYM_INT8, kRansPairBits>;
  if (run == 1 && pb == 12)
    return e4 ? rans_decode_kernel<1, EQ_SYM_E4M3, 12> : rans_decode_kernel<1, EQ_SYM_INT8, 12>;
  return nullptr;
}

// Host-side checks of one descriptor (shared with the fused GEMV).
eq_status validate_rans_tensor(const eq_rans_tensor &t) {
  if (t.version != EQ_ABI_VERSION) return EQ_ERR_ARG;
  if (t.symfmt != EQ_SYM_E4M3 && t.symfmt != EQ_SYM_INT8) return EQ_ERR_ARG;
  if (t.prob_bits != 12 && t.prob_bits != 8 && t.prob_bits != kRansPairBits) return EQ_ERR_UNSUPPORTED;
  if (t.run != 1 && t.run != 8) return EQ_ERR_UNSUPPORTED;
  if (t.prob_bits != 12 && t.run != 8) return EQ_ERR_UNSUPPORTED;  // pairs of steps inside runs
  if (t.streams == 0 || t.streams % 32 || t.streams > 1024) return EQ_ERR_UNSUPPORTED;
  const uint64_t numel = uint64_t(t.rows) * t.cols;
  if (numel >= (1ull << 40)) return EQ_ERR_UNSUPPORTED;
  if (numel == 0) return t.num_chunks == 0 ? EQ_OK : EQ_ERR_ARG;
  if (t.chunk_symbols == 0 || t.chunk_symbols % t.run) return EQ_ERR_ARG;
  if (t.run == 8 && t.cols % 8) return EQ_ERR_UNSUPPORTED;
  if (t.num_chunks != (numel + t.chunk_symbols - 1) / t.chunk_symbols) return EQ_ERR_ARG;
  if (!t.states || !t.word_off || !t.words || !t.scales || !t.tables) return EQ_ERR_ARG;
  if (t.n_patch && (!t.patch_idx || !t.patch_val || !aligned(t.patch_idx, 8) ||
                    t.n_patch > numel))
    return EQ_ERR_ARG;
  if (!aligned(t.words, 16) || !aligned(t.tables, 16) || !aligned(t.states, 4) ||
      !aligned(t.word_off, 8) || !aligned(t.scales, 2))
    return EQ_ERR_ARG;
  return EQ_OK;
}

static std::atomic<bool> g_attr_set[64][2][2][3];  // device, symfmt, run == 8, table (12 / 8 / 7 bits)

// CTAs of `fn` that fit on one SM with `threads` threads and `smem` bytes of dynamic shared
// memory (the occupancy query, cached per device, kernel and block size; at least 1).  Lookups
// take no lock; an entry is filled under a mutex and published by its kernel pointer.
static int ctas_per_sm(KernelFn fn, uint32_t threads, size_t smem) {
  struct Entry {
    std::atomic<const void *> fn{nullptr};
    uint32_t threads = 0;
    int n = 0;
  };
  static Entry cache[64][16];
  static std::mutex fill;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  const void *key = reinterpret_cast<const void *>(fn);
  for (auto &c : cache[dev])
    if (c.fn.load(std::memory_order_acquire) == key && c.threads == threads) return c.n;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, int(threads), smem) != cudaSuccess || n < 1)
    n = 1;
  std::lock_guard<std::mutex> lock(fill);
  for (auto &c : cache[dev]) {
    const void *f = c.fn.load(std::memory_order_relaxed);
    if (f == key && c.threads == threads) break;  // another thread filled it
    if (f == nullptr) {
      c.threads = threads;
      c.n = n;
      c.fn.store(key, std::memory_order_release);
      break;
    }
  }
  return n;
}

// One launch over tensors idx[b, e) of one kernel variant.  Every size that shapes the launch
// (warps per CTA, each tensor's share of the CTAs) comes from the units of these tensors alone.
static eq_status launch_part(KernelFn fn, const eq_rans_tensor *ts, const std::vector<uint32_t> &idx,
                             size_t b, size_t e, uint16_t *const *d_out, uint32_t *d_status,
                             cudaStream_t st) {
  const eq_rans_tensor &t0 = ts[idx[b]];
  uint64_t total_units = 0;
  for (size_t q = b; q < e; ++q) total_units += ts[idx[q]].num_chunks * (ts[idx[q]].streams / 32);
  if (total_units == 0) return EQ_OK;
  const uint64_t sms = uint64_t(device_sm_count());
  const bool pair = t0.prob_bits == kRansPairBits;
  uint32_t warps;
  if (pair) {
    // one CTA per SM holds the 128 KiB pair table; enough warps that the SMs' CTAs take every
    // unit about once (larger tensors: the warps loop)
    warps = uint32_t(std::min<uint64_t>(32, std::max<uint64_t>(1, (total_units + sms - 1) / sms)));
  } else {
    // warps (= groups) per CTA sharing one copy of the table: 12 with 12-bit tables (three such
    // CTAs fit an SM beside their 4 KiB rings: 36 warps; 16-warp CTAs fit two), else 16
    warps = t0.prob_bits == 12 ? 12 : 16;
  }
  // CTAs of this kernel one wave holds (occupancy: registers and shared memory)
  const uint64_t wave = sms * uint64_t(ctas_per_sm(fn, 32 * warps, decode_smem_bytes(warps, t0.prob_bits)));
  uint64_t natural = 0;  // one CTA per `warps` units of each tensor
  for (size_t q = b; q < e; ++q)
    natural += (ts[idx[q]].num_chunks * (ts[idx[q]].streams / 32) + warps - 1) / warps;
  // A launch of under two waves: at most one wave of CTAs, each tensor's share of them in
  // proportion to its units (the kernel spreads a tensor's units over its CTAs round-robin), so
  // every SM gets about the same work instead of some holding one CTA more.
  const bool spread = !pair && natural < 2 * wave;
  static thread_local RansDecodeParams P;
  P.status = d_status;
  P.warps = warps;
  P.spread = spread ? 1u : 0u;
  P.n = 0;
  uint64_t ctas = 0;
  for (size_t q = b; q < e; ++q) {
    const eq_rans_tensor &t = ts[idx[q]];
    if (t.num_chunks == 0) continue;
    RansDesc &D = P.d[P.n++];
    D.states = t.states;
    D.word_off = t.word_off;
    D.words = t.words;
    D.scales = t.scales;
    D.table = static_cast<const uint32_t *>(t.tables);
    D.out = d_out[idx[q]];
    D.patch_idx = t.patch_idx;
    D.patch_val = t.patch_val;
    D.n_patch = t.n_patch;
    D.numel = uint64_t(t.rows) * t.cols;
    D.groups = t.streams / 32;
    D.units = t.num_chunks * D.groups;
    D.row_magic = div_magic(t.cols);
    D.group_magic = div_magic(D.groups);
    D.rows = t.rows;
    D.cols = t.cols;
    D.chunk_symbols = t.chunk_symbols;
    uint64_t n_ctas = (D.units + warps - 1) / warps;
    if (pair)  // at most the tensor's share of the SMs, at least one CTA
      n_ctas = std::min<uint64_t>(n_ctas, std::max<uint64_t>(1, D.units * sms / total_units));
    else if (spread)  // the tensor's share of one wave (some of its warps may have no unit)
      n_ctas = std::max<uint64_t>(1, (D.units * wave + total_units / 2) / total_units);
    D.cta_begin = uint32_t(ctas);
    D.ctas = uint32_t(n_ctas);
    ctas += n_ctas;
  }
  if (ctas >= (1ull << 31)) return EQ_ERR_UNSUPPORTED;
  fn<<<uint32_t(ctas), 32 * warps, decode_smem_bytes(warps, t0.prob_bits), st>>>(P);
  return cuda_status(cudaGetLastError());
}

static eq_status launch_group(const eq_rans_tensor *ts, const std::vector<uint32_t> &idx,
                              uint16_t *const *d_out, uint32_t *d_status, cudaStream_t st) {
  const eq_rans_tensor &t0 = ts[idx[0]];
  KernelFn fn = pick_kernel(t0.symfmt, t0.run, t0.prob_bits);
  if (!fn) return EQ_ERR_UNSUPPORTED;
  const bool pair = t0.prob_bits == kRansPairBits;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return EQ_ERR_CUDA;
  if (smem_optin_once(g_attr_set[dev][t0.symfmt - 1][t0.run == 8][pair ? 2 : t0.prob_bits == 8],
                      reinterpret_cast<const void *>(fn),
                      decode_smem_bytes(pair ? 32 : t0.prob_bits == 12 ? 12 : 16, t0.prob_bits)) != EQ_OK)
    return EQ_ERR_CUDA;
  // launches of nearly equal tensor counts, so that none is a small tail
  const size_t n = idx.size();
  const size_t parts = (n + kMaxDecodeTensors - 1) / kMaxDecodeTensors;
  for (size_t p = 0; p < parts; ++p) {
    const eq_status s = launch_part(fn, ts, idx, n * p / parts, n * (p + 1) / parts, d_out,
                                    d_status, st);
    if (s != EQ_OK) return s;
  }
  return EQ_OK;
}

}  // namespace eq

using namespace eq;

extern "C" eq_status eq_decode(const eq_rans_tensor *ts, uint32_t n_tensors, uint16_t *const *d_out,
                               uint32_t *d_status, void *stream) {
  if (n_tensors == 0) return EQ_OK;
  if (!ts || !d_out || !d_status) return EQ_ERR_ARG;
  // validate everything before launching anything
  for (uint32_t i = 0; i < n_tensors; ++i) {
    eq_status s = validate_rans_tensor(ts[i]);
    if (s != EQ_OK) return s;
    if (ts[i].num_chunks && (!d_out[i] || !aligned(d_out[i], ts[i].run == 8 ? 16 : 2)))
      return EQ_ERR_ARG;
  }
  // one launch per kernel variant (symbol format x run length x table size)
  std::vector<std::vector<uint32_t>> groups(12);
  for (uint32_t i = 0; i < n_tensors; ++i) {
    const uint32_t table = ts[i].prob_bits == 12 ? 0 : ts[i].prob_bits == 8 ? 1 : 2;
    groups[(ts[i].symfmt - 1) * 6 + (ts[i].run == 8) * 3 + table].push_back(i);
  }
  for (auto &g : groups) {
    if (g.empty()) continue;
    eq_status s = launch_group(ts, g, d_out, d_status, static_cast<cudaStream_t>(stream));
    if (s != EQ_OK) return s;
  }
  return EQ_OK;
}
