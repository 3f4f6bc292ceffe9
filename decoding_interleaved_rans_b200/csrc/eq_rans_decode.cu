// eq_decode: interleaved-rANS decode + dequantisation to bf16 on sm_100a.
//
// What it computes is fixed by the format in eq.h ("Float8@2bits" summary: Float8-E4M3 / Int8
// symbols with per-channel scales, flattened and ANS-coded, decoded on the GPU into a buffer before
// the layer runs).  How, on B200:
//   * one warp decodes one chunk; lane l runs the K = streams/32 states l, l+32, ... so the K
//     dependency chains of a lane interleave and hide the shared-memory latency;
//   * the 4096-entry slot table (16 KiB) sits in shared memory, one 32-bit load per symbol;
//   * the chunk's 16-bit words stream through a per-warp shared-memory ring fed by 1-D bulk copies
//     (TMA engine, completion on an mbarrier), so HBM reads are large and asynchronous;
//   * renormalisation is warp-cooperative: a ballot of the states that need a word, a popcount
//     rank gives each its word, in stream order, from the ring;
//   * with run = 8 a lane emits eight consecutive bf16 per state and round: one 16-byte store,
//     a warp writes 512 contiguous bytes per state index;
//   * dequantisation (value * row scale, one rounding) happens in registers before the store.
// Many tensors go in one launch (the pages decode all weights of a transformer block together).
#include <algorithm>
#include <vector>

#include "eq_dequant.cuh"

namespace eq {

constexpr uint32_t kSegBytes = 1024;
constexpr uint32_t kNumSeg = 4;
constexpr uint32_t kRingBytes = kSegBytes * kNumSeg;
constexpr int kMaxDecodeTensors = 192;

struct RansDesc {
  const uint32_t *states;
  const uint64_t *word_off;
  const uint16_t *words;
  const uint16_t *scales;
  const uint32_t *table;  // RansTableHeader followed by the slot table
  uint16_t *out;
  uint64_t numel;
  uint64_t num_chunks;
  uint64_t row_magic;     // floor(j / cols) = __umul64hi(j, row_magic) (0: cols == 1)
  uint32_t cols;
  uint32_t chunk_symbols;
  uint32_t cta_begin;     // first CTA of this tensor in the launch
  uint32_t pad;
};

struct RansDecodeParams {
  uint32_t *status;
  uint32_t n;
  uint32_t warps;  // warps per CTA = chunks per CTA
  RansDesc d[kMaxDecodeTensors];
};

__host__ __device__ constexpr size_t decode_smem_bytes(uint32_t warps) {
  return kRansSlots * 4 + warps * (kRingBytes + kNumSeg * 8);
}

// ------------------------------------------------------------------------------------------------
// per-warp word ring: segment s of the chunk's (16-byte aligned) word span lives in slot s % 4
// ------------------------------------------------------------------------------------------------
struct WordRing {
  unsigned char *buf;
  uint64_t *bar;
  const unsigned char *A;  // chunk word span start, rounded down to 16 bytes
  uint32_t off0;           // bytes from A to the chunk's first word
  uint32_t span;           // bytes to copy (multiple of 16)
  uint32_t nseg;
  uint32_t issued;         // segments handed to the copy engine
  uint32_t ready;          // segments waited for

  __device__ __forceinline__ void issue(uint32_t lane) {
    if (lane == 0) {
      const uint32_t s = issued, slot = s % kNumSeg;
      const uint32_t bytes = min(kSegBytes, span - s * kSegBytes);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_expect_tx(&bar[slot], bytes);
      bulk_g2s(buf + slot * kSegBytes, A + size_t(s) * kSegBytes, bytes, &bar[slot]);
    }
    ++issued;
  }
  // make every segment up to `last` readable; false on timeout
  __device__ __forceinline__ bool wait_upto(uint32_t last) {
    while (ready <= last) {
      if (!mbar_wait_bounded(&bar[ready % kNumSeg], (ready / kNumSeg) & 1u)) return false;
      ++ready;
    }
    return true;
  }
  // refill slots whose segment lies entirely before word `ptr`
  __device__ __forceinline__ void refill(uint32_t ptr, uint32_t lane) {
    const uint32_t cur = (off0 + 2 * ptr) / kSegBytes;
    if (issued < nseg && issued < cur + kNumSeg) {
      __syncwarp();
      do issue(lane);
      while (issued < nseg && issued < cur + kNumSeg);
    }
  }
  __device__ __forceinline__ uint32_t word(uint32_t idx) const {
    return *reinterpret_cast<const uint16_t *>(buf + ((off0 + 2 * idx) & (kRingBytes - 1)));
  }
};

// ------------------------------------------------------------------------------------------------
// one chunk, K states per lane, run length G, symbol format FMT
// ------------------------------------------------------------------------------------------------
template <int K, int G, int FMT>
__device__ __forceinline__ uint32_t decode_chunk(const RansDesc &D, const uint32_t *lut,
                                                 uint32_t flags, uint32_t single_sym,
                                                 WordRing &R, uint64_t chunk, uint32_t lane) {
  constexpr uint32_t S = 32 * K;
  const uint64_t j0 = chunk * uint64_t(D.chunk_symbols);
  const uint32_t n = uint32_t(D.numel - j0 < D.chunk_symbols ? D.numel - j0 : D.chunk_symbols);
  const uint64_t w0 = D.word_off[chunk], w1 = D.word_off[chunk + 1];
  if (w1 < w0 || w1 - w0 >= (1ull << 31)) return EQ_DEV_OVERRUN;
  const uint32_t nwords = uint32_t(w1 - w0);
  uint32_t status = 0;

  uint32_t x[K];
#pragma unroll
  for (int k = 0; k < K; ++k) x[k] = D.states[chunk * S + lane + 32 * k];

  if (flags & kRansFlagSingle) {  // one symbol owns every slot: states never move, no words
    bool ok = nwords == 0;
#pragma unroll
    for (int k = 0; k < K; ++k) ok &= x[k] == kRansL;
    if (!__all_sync(0xFFFFFFFFu, ok)) status |= EQ_DEV_CORRUPT_STATE;
    for (uint32_t i = lane; i < n; i += 32) {
      const uint64_t j = j0 + i;
      const float sc = bf16_bits_to_float(D.scales[div_by_magic(j, D.row_magic)]);
      D.out[j] = dequant1<FMT>(single_sym, sc);
    }
    return status;
  }

  // word ring for this chunk
  const unsigned char *g = reinterpret_cast<const unsigned char *>(D.words + w0);
  R.A = reinterpret_cast<const unsigned char *>(reinterpret_cast<uintptr_t>(g) & ~uintptr_t(15));
  R.off0 = uint32_t(g - R.A);
  R.span = (R.off0 + 2 * nwords + 15u) & ~15u;
  R.nseg = (R.span + kSegBytes - 1) / kSegBytes;
  R.issued = 0;
  R.ready = 0;
  while (R.issued < min(R.nseg, kNumSeg)) R.issue(lane);

  const bool nan_codes = (FMT == EQ_SYM_E4M3) && (flags & (kRansFlagNaN7F | kRansFlagNaNFF));
  const uint32_t lt = lanemask_lt();
  const uint32_t runs = (n + G - 1) / G;
  const uint32_t rounds = (runs + S - 1) / S;
  uint32_t ptr = 0;

  for (uint32_t r = 0; r < rounds; ++r) {
    bool act[K];
#pragma unroll
    for (int k = 0; k < K; ++k) act[k] = r * S + lane + 32 * k < runs;
    uint32_t sym[K][(G + 3) / 4];
#pragma unroll
    for (int k = 0; k < K; ++k)
#pragma unroll
      for (int i = 0; i < (G + 3) / 4; ++i) sym[k][i] = 0;

#pragma unroll
    for (int p = 0; p < G; ++p) {
      // the words this step can read must have landed
      if (R.nseg) {
        const uint32_t last = min(R.nseg - 1, (R.off0 + 2 * (ptr + S) - 1) / kSegBytes);
        if (!R.wait_upto(last)) {
          status |= EQ_DEV_TIMEOUT;
          goto drain;
        }
      }
      uint32_t mask[K];
#pragma unroll
      for (int k = 0; k < K; ++k) {
        const uint32_t e = lut[x[k] & (kRansSlots - 1)];
        const uint32_t nx = ((e >> 12) & 0xFFFu) * (x[k] >> kRansProbBits) + (e & 0xFFFu);
        if (act[k]) x[k] = nx;
        // symbol byte -> byte p % 4 of sym[k][p / 4]
        sym[k][p >> 2] = __byte_perm(sym[k][p >> 2], e, (0x3210u & ~(0xFu << (4 * (p & 3)))) |
                                                            (0x7u << (4 * (p & 3))));
        mask[k] = __ballot_sync(0xFFFFFFFFu, act[k] && x[k] < kRansL);
      }
      uint32_t base = ptr;
#pragma unroll
      for (int k = 0; k < K; ++k) {
        if ((mask[k] >> lane) & 1u) x[k] = (x[k] << 16) | R.word(base + __popc(mask[k] & lt));
        base += __popc(mask[k]);
      }
      ptr = base;
      if (ptr > nwords) {
        status |= EQ_DEV_OVERRUN;
        goto drain;
      }
      R.refill(ptr, lane);

      if constexpr (G == 1) {
#pragma unroll
        for (int k = 0; k < K; ++k)
          if (act[k]) {
            const uint64_t j = j0 + uint64_t(r * S + lane + 32 * k);
            const float sc = bf16_bits_to_float(D.scales[div_by_magic(j, D.row_magic)]);
            D.out[j] = dequant1<FMT>(sym[k][0], sc);
          }
      }
    }
    if constexpr (G == 8) {
#pragma unroll
      for (int k = 0; k < K; ++k)
        if (act[k]) {
          const uint64_t j = j0 + uint64_t(r * S + lane + 32 * k) * 8;
          const float sc = bf16_bits_to_float(D.scales[div_by_magic(j, D.row_magic)]);
          const uint2 a = dequant4<FMT>(sym[k][0], sc, nan_codes);
          const uint2 b = dequant4<FMT>(sym[k][1], sc, nan_codes);
          *reinterpret_cast<uint4 *>(D.out + j) = make_uint4(a.x, a.y, b.x, b.y);
        }
    }
  }
  {
    bool ok = ptr == nwords;
#pragma unroll
    for (int k = 0; k < K; ++k) ok &= x[k] == kRansL;
    if (!__all_sync(0xFFFFFFFFu, ok)) status |= EQ_DEV_CORRUPT_STATE;
  }
drain:
  // every copy handed to the engine must land before the ring is reused or the CTA exits
  while (R.ready < R.issued) {
    if (!mbar_wait_bounded(&R.bar[R.ready % kNumSeg], (R.ready / kNumSeg) & 1u)) {
      status |= EQ_DEV_TIMEOUT;
      break;
    }
    ++R.ready;
  }
  return status;
}

template <int K, int G, int FMT>
__global__ void __launch_bounds__(256) rans_decode_kernel(const __grid_constant__ RansDecodeParams P) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint32_t *lut = reinterpret_cast<uint32_t *>(smem);
  unsigned char *rings = smem + kRansSlots * 4;
  uint64_t *bars = reinterpret_cast<uint64_t *>(rings + P.warps * kRingBytes);

  // tensor of this CTA: the last one whose first CTA is <= blockIdx.x
  uint32_t lo = 0, hi = P.n - 1;
  while (lo < hi) {
    const uint32_t mid = (lo + hi + 1) >> 1;
    if (P.d[mid].cta_begin <= blockIdx.x) lo = mid; else hi = mid - 1;
  }
  const RansDesc D = P.d[lo];
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const RansTableHeader hdr = *reinterpret_cast<const RansTableHeader *>(D.table);
  const uint4 *src = reinterpret_cast<const uint4 *>(D.table + sizeof(RansTableHeader) / 4);
  for (uint32_t i = threadIdx.x; i < kRansSlots / 4; i += blockDim.x)
    reinterpret_cast<uint4 *>(lut)[i] = __ldg(src + i);
  WordRing R;
  R.buf = rings + warp * kRingBytes;
  R.bar = bars + warp * kNumSeg;
  if (lane == 0) {
    for (uint32_t s = 0; s < kNumSeg; ++s) mbar_init(&R.bar[s], 1);
    fence_mbar_init();
  }
  __syncthreads();

  const uint64_t chunk = uint64_t(blockIdx.x - D.cta_begin) * P.warps + warp;
  if (chunk >= D.num_chunks) return;
  uint32_t status = 0;
  if (hdr.magic != kRansMagic) status = EQ_DEV_CORRUPT_STATE;
  else status = decode_chunk<K, G, FMT>(D, lut, hdr.flags, hdr.single_sym, R, chunk, lane);
  if (lane == 0) report(P.status, status);
}

// ------------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------------
using KernelFn = void (*)(RansDecodeParams);

template <int K, int G, int FMT>
static KernelFn kernel_for() {
  return rans_decode_kernel<K, G, FMT>;
}

template <int G, int FMT>
static KernelFn pick_k(uint32_t K) {
  switch (K) {
    case 1: return kernel_for<1, G, FMT>();
    case 2: return kernel_for<2, G, FMT>();
    case 4: return kernel_for<4, G, FMT>();
    case 8: return kernel_for<8, G, FMT>();
  }
  return nullptr;
}

static KernelFn pick_kernel(uint32_t symfmt, uint32_t streams, uint32_t run) {
  const uint32_t K = streams / 32;
  if (run == 8) return symfmt == EQ_SYM_E4M3 ? pick_k<8, EQ_SYM_E4M3>(K) : pick_k<8, EQ_SYM_INT8>(K);
  if (run == 1) return symfmt == EQ_SYM_E4M3 ? pick_k<1, EQ_SYM_E4M3>(K) : pick_k<1, EQ_SYM_INT8>(K);
  return nullptr;
}

// Host-side checks of one descriptor (shared with the fused GEMV).
eq_status validate_rans_tensor(const eq_rans_tensor &t) {
  if (t.version != EQ_ABI_VERSION) return EQ_ERR_ARG;
  if (t.symfmt != EQ_SYM_E4M3 && t.symfmt != EQ_SYM_INT8) return EQ_ERR_ARG;
  if (t.prob_bits != kRansProbBits) return EQ_ERR_UNSUPPORTED;
  if (t.run != 1 && t.run != 8) return EQ_ERR_UNSUPPORTED;
  const uint32_t K = t.streams / 32;
  if (t.streams % 32 || (K != 1 && K != 2 && K != 4 && K != 8)) return EQ_ERR_UNSUPPORTED;
  const uint64_t numel = uint64_t(t.rows) * t.cols;
  if (numel >= (1ull << 40)) return EQ_ERR_UNSUPPORTED;
  if (numel == 0) return t.num_chunks == 0 ? EQ_OK : EQ_ERR_ARG;
  if (t.chunk_symbols == 0 || t.chunk_symbols % t.run) return EQ_ERR_ARG;
  if (t.run == 8 && t.cols % 8) return EQ_ERR_UNSUPPORTED;
  if (t.num_chunks != (numel + t.chunk_symbols - 1) / t.chunk_symbols) return EQ_ERR_ARG;
  if (!t.states || !t.word_off || !t.words || !t.scales || !t.tables) return EQ_ERR_ARG;
  if (!aligned(t.words, 16) || !aligned(t.tables, 16) || !aligned(t.states, 4) ||
      !aligned(t.word_off, 8) || !aligned(t.scales, 2))
    return EQ_ERR_ARG;
  return EQ_OK;
}

static bool g_attr_set[64][2][2][9];

static eq_status launch_group(const eq_rans_tensor *ts, const std::vector<uint32_t> &idx,
                              uint16_t *const *d_out, uint32_t *d_status, cudaStream_t st) {
  const eq_rans_tensor &t0 = ts[idx[0]];
  KernelFn fn = pick_kernel(t0.symfmt, t0.streams, t0.run);
  if (!fn) return EQ_ERR_UNSUPPORTED;
  uint64_t total_chunks = 0;
  for (uint32_t i : idx) total_chunks += ts[i].num_chunks;
  // warps (= chunks) per CTA: enough CTAs to spread over every SM a few times
  const uint64_t sms = uint64_t(device_sm_count());
  uint32_t warps = 8;
  while (warps > 1 && (total_chunks + warps - 1) / warps < 3 * sms) warps >>= 1;
  const size_t smem = decode_smem_bytes(warps);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return EQ_ERR_CUDA;
  bool &attr = g_attr_set[dev][t0.symfmt - 1][t0.run == 8][t0.streams / 32];
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(decode_smem_bytes(8)));
    if (e != cudaSuccess) return EQ_ERR_CUDA;
    attr = true;
  }
  static thread_local RansDecodeParams P;
  for (size_t b = 0; b < idx.size(); b += kMaxDecodeTensors) {
    const size_t e = std::min(idx.size(), b + kMaxDecodeTensors);
    P.status = d_status;
    P.warps = warps;
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
      D.numel = uint64_t(t.rows) * t.cols;
      D.num_chunks = t.num_chunks;
      D.row_magic = div_magic(t.cols);
      D.cols = t.cols;
      D.chunk_symbols = t.chunk_symbols;
      D.cta_begin = uint32_t(ctas);
      D.pad = 0;
      ctas += (t.num_chunks + warps - 1) / warps;
    }
    if (P.n == 0) continue;
    if (ctas >= (1ull << 31)) return EQ_ERR_UNSUPPORTED;
    fn<<<uint32_t(ctas), 32 * warps, smem, st>>>(P);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return EQ_ERR_CUDA;
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
  // group by the compile-time parameters of the kernel
  std::vector<std::vector<uint32_t>> groups;
  std::vector<uint32_t> keys;
  for (uint32_t i = 0; i < n_tensors; ++i) {
    const uint32_t key = ts[i].symfmt * 10000 + ts[i].streams * 10 + ts[i].run;
    auto it = std::find(keys.begin(), keys.end(), key);
    if (it == keys.end()) {
      keys.push_back(key);
      groups.emplace_back();
      it = keys.end() - 1;
    }
    groups[it - keys.begin()].push_back(i);
  }
  for (auto &g : groups) {
    eq_status s = launch_group(ts, g, d_out, d_status, static_cast<cudaStream_t>(stream));
    if (s != EQ_OK) return s;
  }
  return EQ_OK;
}
