// eq_huff_bf16_decode: DFloat11 reconstruction of bf16 weights on sm_100a.
//
// Format and parallel decomposition follow the DFloat11 page ("Kernels GPU de 2 etapas y
// metadatos auxiliares"): thread t owns bytes [8t, 8t + 8) of EncodedExponent and decodes the
// codes that start there, beginning at its 5-bit Gap; one output position is stored per block of
// threads; on the page, stage 1 decodes and only counts, a block-wide prefix sum of the counts
// gives every thread its output offset, and stage 2 decodes again and writes the exponents into a
// shared-memory buffer; the block then merges them with PackedSignMantissa and writes its span
// once, coalesced.
//
// Different from the page's kernel, for B200:
//   * codes are read through an 11-bit window table (16 KiB in shared memory) that returns up to
//     four whole codes per lookup (the common exponent codes are 2-3 bits long); the rare codes
//     longer than 11 bits fall back to the page's hierarchical 8-bit tables ("Decodificacion
//     basada en LUT jerarquicas"), read through L1, with 16-bit entries so no exponent value has
//     to be given up as a pointer;
//   * blocks are persistent: each CTA loads the window table once and walks over many blocks of
//     the stream, fetching the next block's bits while it merges the current one;
//   * the block scan is a warp-shuffle scan rather than Blelloch's tree;
//   * codes are decoded once: stage 1 packs each thread's values into its own column of the
//     shared buffer, and stage 2 only moves them to their offsets (a second decode cost more
//     than a third of the kernel).
#include <algorithm>

#include <cstring>

#include "eq_dequant.cuh"

namespace eq {

// What the decoded byte stream becomes: DFloat11 exponents merged with PackedSignMantissa, or
// integer codes q turned into bf16((q - zero) * scale).
constexpr int kHuffDf11 = 0, kHuffInt = 1;

struct HuffParams {
  const uint8_t *enc;
  const uint8_t *sign_mant;  // DFloat11 only
  float scale;               // integer codes only
  int32_t zero;
  uint32_t code_limit;       // largest valid integer code
  const uint8_t *gaps;
  const uint64_t *block_out;
  const unsigned char *table;
  uint16_t *out;
  uint32_t *status;
  uint64_t n;
  uint64_t total_bits;
  uint64_t threads;
  uint64_t blocks;
};

__host__ __device__ constexpr size_t huff_smem_bytes(uint32_t tpb) {
  return kHuffWindow * 8 + size_t(tpb) * 64 + 16 + 66 * 4;
}

__device__ __forceinline__ uint32_t bswap32(uint32_t v) { return __byte_perm(v, 0, 0x0123); }

__device__ __forceinline__ uint32_t tree_decode(const uint16_t *tree, uint32_t ntab, uint32_t w,
                                                uint32_t *sym) {
  uint32_t e = __ldg(tree + (w >> 24)), used = 0;
  while ((e & 0x8000u) && e != kHuffInvalid) {
    const uint32_t tab = e & 0xFFu;
    used += 8;
    if (tab >= ntab || used > 24) return 0;
    e = __ldg(tree + tab * 256 + ((w >> (24 - used)) & 0xFFu));
  }
  const uint32_t rem = (e >> 8) & 0xFu;
  if (e == kHuffInvalid || rem == 0 || rem > 8) return 0;
  *sym = e & 0xFFu;
  return used + rem;
}

// A thread's decoded values, packed as bytes (value i = byte i, little-endian) into its private
// column of 32-bit words: word i at col[i * T], so the 32 lanes of a warp touch 32 banks.
struct BytePacker {
  uint32_t *col;
  uint32_t T;
  uint64_t acc = 0;  // pending bytes, the oldest in the low bits
  uint32_t nb = 0, wp = 0;

  // append the low k (1..4) bytes of v, whose higher bytes are zero (window-table entries hold
  // zeros past their k values; single values are below 256)
  __device__ __forceinline__ void put(uint32_t v, uint32_t k) {
    acc |= uint64_t(v) << (8 * nb);
    nb += k;
    if (nb >= 4) {
      col[wp * T] = uint32_t(acc);
      ++wp;
      acc >>= 32;
      nb -= 4;
    }
  }
  __device__ __forceinline__ void flush() {
    if (nb) col[wp * T] = uint32_t(acc);
  }
};

// Decode the codes starting in bits [gap, end) of this thread's segment into the packer; returns
// how many.  *bad is set on a pattern no code matches.
__device__ __forceinline__ uint32_t segment(const uint64_t *win, const uint16_t *tree, uint32_t ntab,
                                            uint32_t r0, uint32_t r1, uint32_t r2, uint32_t pos,
                                            uint32_t end, BytePacker &out, uint32_t *bad) {
  // the next 64 bits of the stream are r0:r1 (r2 behind them); pos, end count from r0's top bit,
  // and the words slide up once pos passes 32, so every lookup is one funnel shift
  uint32_t cnt = 0;
  // body: every code found inside a whole 11-bit window starts before `end`.  A window whose
  // first code does not fit (or matches no code) is flagged long and goes to the tree, which
  // reports bad patterns.
  while (pos + kHuffWindowBits <= end) {
    if (pos >= 32) {
      r0 = r1;
      r1 = r2;
      r2 = 0;
      pos -= 32;
      end -= 32;
    }
    const uint32_t w = __funnelshift_l(r1, r0, pos);
    const uint64_t f = win[w >> (32 - kHuffWindowBits)];
    if (f & kHuffLong) {
      uint32_t sym;
      const uint32_t len = tree_decode(tree, ntab, w, &sym);
      if (!len) {
        *bad = EQ_DEV_BAD_CODE;
        break;
      }
      out.put(sym, 1);
      ++cnt;
      pos += len;
      continue;
    }
    const uint32_t hi = uint32_t(f >> 32);
    const uint32_t k = (hi >> 20) & 7u;
    out.put(uint32_t(f), k);
    cnt += k;
    pos += (hi >> 16) & 0xFu;
  }
  // tail: codes may reach past `end`; only those starting before it are this thread's
  while (pos < end && !*bad) {
    if (pos >= 32) {
      r0 = r1;
      r1 = r2;
      r2 = 0;
      pos -= 32;
      end -= 32;
    }
    const uint32_t w = __funnelshift_l(r1, r0, pos);
    const uint64_t f = win[w >> (32 - kHuffWindowBits)];
    if (f & kHuffLong) {
      uint32_t sym;
      const uint32_t len = tree_decode(tree, ntab, w, &sym);
      if (!len) {
        *bad = EQ_DEV_BAD_CODE;
        break;
      }
      out.put(sym, 1);
      ++cnt;
      pos += len;
      continue;
    }
    // the window's codes that start before `end` (the first always does)
    const uint32_t hi = uint32_t(f >> 32), k = (hi >> 20) & 7u;
    if (k == 0) {  // no code fits and the first is not long: no code matches
      *bad = EQ_DEV_BAD_CODE;
      break;
    }
    uint32_t kk = 1, p = pos + (hi & 0xFu);
#pragma unroll
    for (uint32_t i = 1; i < 4; ++i) {
      if (i < k && p < end) {
        ++kk;
        p += (hi >> (4 * i)) & 0xFu;
      }
    }
    out.put(uint32_t(f) & (0xFFFFFFFFu >> (32 - 8 * kk)), kk);
    cnt += kk;
    pos = p;
  }
  out.flush();
  return cnt;
}

// Move this thread's cnt packed bytes (column layout, at most 64) to ebuf[D .. D + cnt).  All
// threads first read their columns into registers; the caller's barrier separates that from the
// writes, since the compacted ranges overlap other threads' columns.
struct Staged {
  uint32_t w[17];
};

// NW: words read (16 for any segment; 8 when every lane of the warp holds at most 32 values)
template <uint32_t NW>
__device__ __forceinline__ void stage_read(const uint32_t *col, uint32_t T, uint32_t cnt, Staged &st) {
  const uint32_t nw = (cnt + 3) >> 2;
#pragma unroll
  for (uint32_t i = 0; i < NW; ++i) st.w[i] = i < nw ? col[i * T] : 0u;
  st.w[NW] = 0u;
}

template <uint32_t NW>
__device__ __forceinline__ void stage_write(uint8_t *ebuf, uint32_t D, uint32_t cnt, const Staged &st) {
  const uint32_t a = D & 3u, sh = 8 * a, nd = (a + cnt + 3) >> 2;
  uint32_t *dst = reinterpret_cast<uint32_t *>(ebuf + (D - a));
#pragma unroll
  for (uint32_t j = 0; j < NW + 1; ++j) {
    if (j < nd) {
      // destination word j holds source bytes 4j - a .. 4j - a + 3
      const uint32_t prev = j ? st.w[j - 1] : 0u;
      const uint32_t v = a ? __funnelshift_l(prev, st.w[j], sh) : st.w[j];
      const uint32_t b0 = j == 0 ? a : 0u, b1 = min(4u, a + cnt - 4 * j);
      if (b0 == 0 && b1 == 4) {
        dst[j] = v;
      } else {  // a word shared with a neighbouring thread's bytes: only ours
        for (uint32_t b = b0; b < b1; ++b) ebuf[D - a + 4 * j + b] = uint8_t(v >> (8 * b));
      }
    }
  }
}

// one integer code -> bf16 bits: (q - z) * s is exact in fp32, so the conversion is the rounding
__device__ __forceinline__ uint32_t int_code_bf16(uint32_t q, float s, int32_t z) {
  return pack_bf16x2(__int2float_rn(int32_t(q) - z) * s, 0.0f) & 0xFFFFu;
}

// At most 40 registers (3 CTAs of 512 or 6 of 256 threads per SM): the staging registers would
// otherwise cost more in occupancy than the single decode pass saves.
template <int MODE>
__global__ void __launch_bounds__(512, 3) huff_decode_kernel(const __grid_constant__ HuffParams P) {
  extern __shared__ __align__(16) unsigned char smem[];
  const uint32_t T = blockDim.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint64_t *win = reinterpret_cast<uint64_t *>(smem);
  uint8_t *ebuf = smem + kHuffWindow * 8;
  uint32_t *wsum = reinterpret_cast<uint32_t *>(ebuf + T * 64 + 16);
  const uint16_t *tree = reinterpret_cast<const uint16_t *>(P.table + kHuffTreeOffset);

  const HuffTableHeader hdr = *reinterpret_cast<const HuffTableHeader *>(P.table);
  if (hdr.magic != kHuffMagic || hdr.num_tables == 0 || hdr.num_tables > kHuffMaxTables) {
    if (tid == 0) report(P.status, EQ_DEV_BAD_CODE);
    return;
  }
  const uint32_t ntab = hdr.num_tables;
  {
    const uint4 *w4 = reinterpret_cast<const uint4 *>(P.table + kHuffWindowOffset);
    for (uint32_t i = tid; i < kHuffWindow / 2; i += T) reinterpret_cast<uint4 *>(win)[i] = __ldg(w4 + i);
  }
  __syncthreads();

  // a thread's 64-bit segment plus the 32 bits after it, and its Gap
  auto fetch = [&](uint64_t b, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &g) {
    const uint64_t t = b * T + tid;
    r0 = r1 = r2 = g = 0;
    if (b < P.blocks && t < P.threads) {
      const uint32_t *src = reinterpret_cast<const uint32_t *>(P.enc + 8 * t);
      r0 = __ldg(src);
      r1 = __ldg(src + 1);
      r2 = __ldg(src + 2);
      const uint64_t gbit = 5 * t;
      g = (uint32_t(__ldg(P.gaps + (gbit >> 3))) | (uint32_t(__ldg(P.gaps + (gbit >> 3) + 1)) << 8)) >>
          (gbit & 7);
    }
  };
  uint32_t err = 0;
  uint32_t n0, n1, n2, ng;
  fetch(blockIdx.x, n0, n1, n2, ng);
  for (uint64_t b = blockIdx.x; b < P.blocks; b += gridDim.x) {
    const uint64_t t = b * T + tid;
    const uint32_t r0 = bswap32(n0), r1 = bswap32(n1), r2 = bswap32(n2);
    uint32_t pos = ng & 31u, end = 0;
    if (t < P.threads) {
      const uint64_t left = P.total_bits - 64 * t;
      end = left < 64 ? uint32_t(left) : 64u;
    }
    fetch(b + gridDim.x, n0, n1, n2, ng);  // next block's bits, in flight during this one
    // ---- stage 1: decode once, the values packed into this thread's column of ebuf ----
    uint32_t bad = 0;
    BytePacker pk{reinterpret_cast<uint32_t *>(ebuf) + tid, T};
    const uint32_t cnt = segment(win, tree, ntab, r0, r1, r2, pos, end, pk, &bad);
    // the values leave this thread's column for registers now: the scan's barriers then also
    // order every column read before the compacting writes below
    Staged stg;
    // the common case (every lane of the warp at most 32 values) stages half the words
    const bool small = __all_sync(0xFFFFFFFFu, cnt <= 32);
    if (small) stage_read<8>(reinterpret_cast<const uint32_t *>(ebuf) + tid, T, cnt, stg);
    else stage_read<16>(reinterpret_cast<const uint32_t *>(ebuf) + tid, T, cnt, stg);
    const uint64_t o0 = __ldg(P.block_out + b), o1 = __ldg(P.block_out + b + 1);  // in flight
    // ---- block-wide exclusive scan of the counts ----
    uint32_t incl = cnt;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, d);
      if (lane >= uint32_t(d)) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const uint32_t nw = T / 32;
      uint32_t v = lane < nw ? wsum[lane] : 0u, s = v;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, s, d);
        if (lane >= uint32_t(d)) s += u;
      }
      if (lane < nw) wsum[lane] = s - v;  // exclusive prefix of the warp totals
      if (lane == nw - 1) wsum[32] = s;   // block total
    }
    __syncthreads();
    const uint32_t total = wsum[32];
    const uint32_t off = wsum[warp] + incl - cnt;

    uint64_t m = total;
    if (o1 < o0 || o1 > P.n) {
      err |= EQ_DEV_OVERRUN;
      m = 0;
    } else if (o1 - o0 != total) {
      err |= EQ_DEV_COUNT_MISMATCH;
      m = min(uint64_t(total), o1 - o0);
    }
    err |= bad;
    // ---- stage 2: every thread moves its values to their block positions (shifted so that
    //      8-aligned outputs are 8-aligned in shared memory) ----
    const uint32_t shift = uint32_t(o0 & 7);
    if (off + cnt <= m) {
      if (small) stage_write<8>(ebuf, shift + off, cnt, stg);
      else stage_write<16>(ebuf, shift + off, cnt, stg);
    }
    __syncthreads();

    // ---- merge with PackedSignMantissa and write the block's span ----
    const uint64_t ga = min((o0 + 7) & ~uint64_t(7), o0 + m);
    const uint64_t gb = max(ga, (o0 + m) & ~uint64_t(7));
    auto one = [&](uint64_t g) {
      const uint32_t x = ebuf[shift + (g - o0)];
      if constexpr (MODE == kHuffDf11) {
        const uint32_t s = P.sign_mant[g];
        P.out[g] = uint16_t(((s & 0x80u) << 8) | (x << 7) | (s & 0x7Fu));
      } else {
        if (x > P.code_limit) err |= EQ_DEV_BAD_CODE;
        P.out[g] = uint16_t(int_code_bf16(x, P.scale, P.zero));
      }
    };
    for (uint64_t g = o0 + tid; g < ga; g += T) one(g);  // unaligned head
    for (uint64_t g = ga + 8 * uint64_t(tid); g < gb; g += 8 * uint64_t(T)) {
      const uint2 x = *reinterpret_cast<const uint2 *>(ebuf + shift + (g - o0));
      uint32_t w[4];
      if constexpr (MODE == kHuffDf11) {
        const uint2 s = __ldg(reinterpret_cast<const uint2 *>(P.sign_mant + g));
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t sw = h ? s.y : s.x, xw = h ? x.y : x.x;
#pragma unroll
          for (int q = 0; q < 2; ++q) {  // bytes 2q, 2q+1 -> one bf16 pair
            const uint32_t s2 = __byte_perm(sw, 0, q ? 0x4342u : 0x4140u);
            const uint32_t x2 = __byte_perm(xw, 0, q ? 0x4342u : 0x4140u);
            w[2 * h + q] = ((s2 & 0x00800080u) << 8) | (x2 << 7) | (s2 & 0x007F007Fu);
          }
        }
      } else {
        // the limit is 2^bits - 1, so a byte above it has a bit outside the mask
        if ((x.x | x.y) & ~(0x01010101u * P.code_limit)) err |= EQ_DEV_BAD_CODE;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t xw = k < 2 ? x.x : x.y, sh = 16 * (k & 1);
          w[k] = pack_bf16x2(__int2float_rn(int32_t((xw >> sh) & 0xFFu) - P.zero) * P.scale,
                             __int2float_rn(int32_t((xw >> (sh + 8)) & 0xFFu) - P.zero) * P.scale);
        }
      }
      *reinterpret_cast<uint4 *>(P.out + g) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    for (uint64_t g = gb + tid; g < o0 + m; g += T) one(g);  // tail
    __syncthreads();  // ebuf and wsum are reused by the next block
  }
  report(P.status, err);
}

static std::atomic<bool> g_huff_attr[64][2];  // device, integer codes

// validation and launch shared by the DFloat11 and the integer decoders
template <int MODE>
static eq_status huff_launch(HuffParams &P, uint64_t n, uint64_t total_bits,
                             uint32_t bytes_per_thread, uint32_t T, const void *enc,
                             const void *gaps, const void *block_out, const void *tables,
                             uint16_t *d_out, uint32_t *d_status, void *stream) {
  if (!d_status) return EQ_ERR_ARG;
  if (bytes_per_thread != 8) return EQ_ERR_UNSUPPORTED;
  if (T < 32 || T > 512 || T % 32) return EQ_ERR_UNSUPPORTED;
  if (n == 0) return EQ_OK;
  if (n >= (1ull << 40) || total_bits == 0 || total_bits > 32 * n || total_bits < n)
    return EQ_ERR_ARG;
  if (!d_out || !enc || !gaps || !block_out || !tables) return EQ_ERR_ARG;
  if (!aligned(d_out, 16) || !aligned(enc, 8) || !aligned(tables, 16) || !aligned(block_out, 8))
    return EQ_ERR_ARG;
  const uint64_t threads = (total_bits + 63) / 64;
  const uint64_t blocks = (threads + T - 1) / T;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return EQ_ERR_CUDA;
  if (smem_optin_once(g_huff_attr[dev][MODE], reinterpret_cast<const void *>(huff_decode_kernel<MODE>),
                      huff_smem_bytes(512)) != EQ_OK)
    return EQ_ERR_CUDA;
  // persistent blocks: as many as fit on the device at once, each walking many blocks
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, huff_decode_kernel<MODE>, int(T),
                                                    huff_smem_bytes(T)) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const uint64_t grid = std::min<uint64_t>(blocks, uint64_t(per_sm) * device_sm_count());
  P.enc = static_cast<const uint8_t *>(enc);
  P.gaps = static_cast<const uint8_t *>(gaps);
  P.block_out = static_cast<const uint64_t *>(block_out);
  P.table = static_cast<const unsigned char *>(tables);
  P.out = d_out;
  P.status = d_status;
  P.n = n;
  P.total_bits = total_bits;
  P.threads = threads;
  P.blocks = blocks;
  huff_decode_kernel<MODE><<<uint32_t(grid), T, huff_smem_bytes(T), static_cast<cudaStream_t>(stream)>>>(P);
  return cuda_status(cudaGetLastError());
}

}  // namespace eq

using namespace eq;

extern "C" eq_status eq_huff_bf16_decode(const eq_huff_tensor *h, uint16_t *d_out,
                                         uint32_t *d_status, void *stream) {
  if (!h) return EQ_ERR_ARG;
  if (h->n && (!h->sign_mant || !aligned(h->sign_mant, 8))) return EQ_ERR_ARG;
  HuffParams P{};
  P.sign_mant = h->sign_mant;
  return huff_launch<kHuffDf11>(P, h->n, h->total_bits, h->bytes_per_thread, h->threads_per_block,
                                h->enc_exp, h->gaps, h->block_out, h->tables, d_out, d_status,
                                stream);
}

extern "C" eq_status eq_huff_int_decode(const eq_huff_int_tensor *h, uint16_t *d_out,
                                        uint32_t *d_status, void *stream) {
  if (!h) return EQ_ERR_ARG;
  if (h->bits != 8 && h->bits != 4) return EQ_ERR_UNSUPPORTED;
  const int32_t L = 1 << h->bits;
  if (h->zero < 0 || h->zero > L) return EQ_ERR_ARG;
  HuffParams P{};
  const uint32_t sbits = uint32_t(h->scale) << 16;
  std::memcpy(&P.scale, &sbits, 4);
  P.zero = h->zero;
  P.code_limit = uint32_t(L - 1);
  return huff_launch<kHuffInt>(P, h->n, h->total_bits, h->bytes_per_thread, h->threads_per_block,
                               h->enc, h->gaps, h->block_out, h->tables, d_out, d_status, stream);
}
