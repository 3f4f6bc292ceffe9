// eq_huff_bf16_decode: DFloat11 reconstruction of bf16 weights on sm_100a.
//
// Format and parallel decomposition follow the DFloat11 page ("Kernels GPU de 2 etapas y
// metadatos auxiliares"): thread t of the grid owns bytes [8t, 8t + 8) of EncodedExponent and
// decodes the codes that start there, beginning at its 5-bit Gap; one output position is stored
// per thread block; a block-wide prefix sum of the per-thread code counts gives every thread its
// output offset; exponents are gathered in shared memory and the block writes its span once,
// coalesced.  Codes are read through the hierarchical 256-entry lookup tables of "Decodificacion
// basada en LUT jerarquicas" (built by eq_build_tables(EQ_TABLE_HUFF)).
//
// Different from the page's kernel, which decodes every segment twice (count, then decode again
// and write): a B200 SM has room to keep the first pass, so each thread decodes once into a
// private 64-byte shared-memory slot (a 64-bit segment holds at most 64 code starts; the slots are
// interleaved so that a warp's byte stores fall in distinct banks), and after the scan copies its
// exponents to their block position.  The block scan is a warp-shuffle scan
// rather than Blelloch's tree.
#include "eq_internal.cuh"

namespace eq {

struct HuffParams {
  const uint8_t *enc;
  const uint8_t *sign_mant;
  const uint8_t *gaps;
  const uint64_t *block_out;
  const uint32_t *table;
  uint16_t *out;
  uint32_t *status;
  uint64_t n;
  uint64_t total_bits;
  uint64_t threads;
};

constexpr uint32_t kHuffLutBytes = kHuffMaxTables * 256 * 2;

__host__ __device__ constexpr size_t huff_smem_bytes(uint32_t tpb) {
  return kHuffLutBytes + size_t(tpb) * 64 + size_t(tpb) * 64 + 16 + 64 * 4;
}

__device__ __forceinline__ uint32_t bswap32(uint32_t v) { return __byte_perm(v, 0, 0x0123); }

__global__ void __launch_bounds__(1024) huff_decode_kernel(const __grid_constant__ HuffParams P) {
  extern __shared__ __align__(16) unsigned char smem[];
  const uint32_t T = blockDim.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint16_t *lut = reinterpret_cast<uint16_t *>(smem);
  uint8_t *priv = smem + kHuffLutBytes;
  uint8_t *ebuf = priv + T * 64;
  uint32_t *wsum = reinterpret_cast<uint32_t *>(ebuf + T * 64 + 16);

  const HuffTableHeader hdr = *reinterpret_cast<const HuffTableHeader *>(P.table);
  if (hdr.magic != kHuffMagic || hdr.num_tables == 0 || hdr.num_tables > kHuffMaxTables) {
    if (tid == 0) report(P.status, EQ_DEV_BAD_CODE);
    return;
  }
  const uint32_t ntab = hdr.num_tables;
  {
    const uint4 *src = reinterpret_cast<const uint4 *>(P.table + sizeof(HuffTableHeader) / 4);
    for (uint32_t i = tid; i < ntab * 32; i += T) reinterpret_cast<uint4 *>(lut)[i] = __ldg(src + i);
  }
  __syncthreads();

  // ---- decode this thread's segment once, into its private slot ----
  const uint64_t t = uint64_t(blockIdx.x) * T + tid;
  uint32_t cnt = 0, err = 0;
  if (t < P.threads) {
    const uint32_t *src = reinterpret_cast<const uint32_t *>(P.enc + 8 * t);
    uint64_t buf = (uint64_t(bswap32(__ldg(src))) << 32) | bswap32(__ldg(src + 1));
    const uint32_t nxt = bswap32(__ldg(src + 2));
    const uint64_t gbit = 5 * t;
    const uint32_t g2 = uint32_t(__ldg(P.gaps + (gbit >> 3))) |
                        (uint32_t(__ldg(P.gaps + (gbit >> 3) + 1)) << 8);
    const uint32_t gap = (g2 >> (gbit & 7)) & 31u;
    uint64_t pos = 64 * t + gap;
    const uint64_t end = min(64 * t + 64, P.total_bits);
    buf <<= gap;
    int valid = 64 - int(gap);
    bool more = true;
    uint8_t *mine = priv + tid;  // column-major: code k of thread t at priv[k * T + t]
    while (pos < end) {
      if (valid < 32 && more) {  // pull in the 32 bits after the segment (codes reach <= 31 past it)
        buf |= uint64_t(nxt) << (32 - valid);
        valid += 32;
        more = false;
      }
      uint32_t e = lut[buf >> 56];
      uint32_t used = 0;
      while ((e & 0x8000u) && e != kHuffInvalid) {  // pointer to the next 8-bit subtree
        const uint32_t tab = e & 0xFFu;
        used += 8;
        if (tab >= ntab || used > 24) {
          e = kHuffInvalid;
          break;
        }
        e = lut[tab * 256 + uint32_t((buf >> (56 - used)) & 0xFFu)];
      }
      const uint32_t rem = (e >> 8) & 0xFu;
      if (e == kHuffInvalid || rem == 0 || rem > 8 || cnt >= 64) {
        err |= EQ_DEV_BAD_CODE;
        break;
      }
      const uint32_t len = used + rem;
      mine[cnt * T] = uint8_t(e & 0xFFu);
      ++cnt;
      buf <<= len;
      valid -= int(len);
      pos += len;
    }
  }

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
    if (lane < nw) wsum[lane] = s - v;   // exclusive prefix of the warp totals
    if (lane == nw - 1) wsum[32] = s;    // block total
  }
  __syncthreads();
  const uint32_t total = wsum[32];
  const uint32_t off = wsum[warp] + incl - cnt;

  const uint64_t o0 = P.block_out[blockIdx.x], o1 = P.block_out[blockIdx.x + 1];
  uint64_t m = total;
  if (o1 < o0 || o1 > P.n) {
    err |= EQ_DEV_OVERRUN;
    m = 0;
  } else if (o1 - o0 != total) {
    err |= EQ_DEV_COUNT_MISMATCH;
    m = min(uint64_t(total), o1 - o0);
  }
  // ---- gather the exponents at their block positions (shifted so 8-aligned outputs are
  //      8-aligned in shared memory) ----
  const uint32_t shift = uint32_t(o0 & 7);
  for (uint32_t k = 0; k < cnt; ++k)
    if (off + k < m) ebuf[shift + off + k] = priv[k * T + tid];
  __syncthreads();

  // ---- merge with PackedSignMantissa and write the block's span ----
  const uint64_t ga = min((o0 + 7) & ~uint64_t(7), o0 + m);
  const uint64_t gb = max(ga, (o0 + m) & ~uint64_t(7));
  for (uint64_t g = o0 + tid; g < ga; g += T) {  // unaligned head
    const uint32_t s = P.sign_mant[g], x = ebuf[shift + (g - o0)];
    P.out[g] = uint16_t(((s & 0x80u) << 8) | (x << 7) | (s & 0x7Fu));
  }
  for (uint64_t g = ga + 8 * uint64_t(tid); g < gb; g += 8 * uint64_t(T)) {
    const uint2 s = __ldg(reinterpret_cast<const uint2 *>(P.sign_mant + g));
    const uint2 x = *reinterpret_cast<const uint2 *>(ebuf + shift + (g - o0));
    uint32_t w[4];
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
    *reinterpret_cast<uint4 *>(P.out + g) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  for (uint64_t g = gb + tid; g < o0 + m; g += T) {  // tail
    const uint32_t s = P.sign_mant[g], x = ebuf[shift + (g - o0)];
    P.out[g] = uint16_t(((s & 0x80u) << 8) | (x << 7) | (s & 0x7Fu));
  }
  report(P.status, err);
}

static bool g_huff_attr[64];

}  // namespace eq

using namespace eq;

extern "C" eq_status eq_huff_bf16_decode(const eq_huff_tensor *h, uint16_t *d_out,
                                         uint32_t *d_status, void *stream) {
  if (!h || !d_status) return EQ_ERR_ARG;
  if (h->bytes_per_thread != 8) return EQ_ERR_UNSUPPORTED;
  const uint32_t T = h->threads_per_block;
  if (T < 32 || T > 1024 || T % 32) return EQ_ERR_UNSUPPORTED;
  if (h->n == 0) return EQ_OK;
  if (h->n >= (1ull << 40) || h->total_bits == 0 || h->total_bits > 32 * h->n ||
      h->total_bits < h->n)
    return EQ_ERR_ARG;
  if (!d_out || !h->enc_exp || !h->sign_mant || !h->gaps || !h->block_out || !h->tables)
    return EQ_ERR_ARG;
  if (!aligned(d_out, 16) || !aligned(h->enc_exp, 8) || !aligned(h->sign_mant, 8) ||
      !aligned(h->tables, 16) || !aligned(h->block_out, 8))
    return EQ_ERR_ARG;
  const uint64_t threads = (h->total_bits + 63) / 64;
  const uint64_t blocks = (threads + T - 1) / T;
  if (blocks >= (1ull << 31)) return EQ_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return EQ_ERR_CUDA;
  if (!g_huff_attr[dev]) {
    if (cudaFuncSetAttribute(huff_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(huff_smem_bytes(1024))) != cudaSuccess)
      return EQ_ERR_CUDA;
    g_huff_attr[dev] = true;
  }
  HuffParams P;
  P.enc = h->enc_exp;
  P.sign_mant = h->sign_mant;
  P.gaps = h->gaps;
  P.block_out = h->block_out;
  P.table = static_cast<const uint32_t *>(h->tables);
  P.out = d_out;
  P.status = d_status;
  P.n = h->n;
  P.total_bits = h->total_bits;
  P.threads = threads;
  huff_decode_kernel<<<uint32_t(blocks), T, huff_smem_bytes(T), static_cast<cudaStream_t>(stream)>>>(P);
  return cuda_status(cudaGetLastError());
}
