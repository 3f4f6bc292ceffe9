// eq_build_tables / eq_table_bytes and the small ABI utilities.
//
// The rANS slot table follows the decoding rule of the interleaved rANS format in eq.h
// ("Float8@2bits" summary, "Codificacion de Pesos": ANS over the flattened symbol stream).
// The Huffman tables follow the DFloat11 page, "Decodificacion basada en LUT jerarquicas": the
// canonical code tree is cut into height-8 subtrees, each a 256-entry lookup table; entries that
// lead deeper point at the child table.  The page reuses the never-seen exponents 240..255 as the
// pointers inside 8-bit entries; here entries are 16 bits wide (a pointer bit, the bits used at
// this level and the value), so every exponent value, including 240..255, stays decodable.
#include <algorithm>
#include <vector>

#include "eq_dequant.cuh"
#include "eq_internal.cuh"

namespace eq {

struct RansBuildArgs {
  uint32_t *dst;           // device table (header + 2^prob_bits entries)
  uint32_t flags, single;  // header fields
  uint32_t prob_bits;
  uint32_t symfmt;         // pair tables: the format of the values they carry
  uint16_t freq[256];
};

// one block of 256 threads: prefix sum of the frequencies, then every slot finds its symbol
__global__ void __launch_bounds__(256) rans_build_kernel(const __grid_constant__ RansBuildArgs a) {
  __shared__ uint32_t cum[257];
  const uint32_t t = threadIdx.x;
  if (t == 0) {
    uint32_t c = 0;
    for (int s = 0; s < 256; ++s) {
      cum[s] = c;
      c += a.freq[s];
    }
    cum[256] = c;
    const uint32_t magic = a.prob_bits == 12 ? kRansMagic
                           : a.symfmt == EQ_SYM_E4M3 ? kRans8MagicE4M3 : kRans8MagicInt8;
    RansTableHeader h{magic, a.flags, a.single, a.prob_bits};
    *reinterpret_cast<RansTableHeader *>(a.dst) = h;
  }
  __syncthreads();
  uint32_t *lut = a.dst + sizeof(RansTableHeader) / 4;
  const uint32_t pb = a.prob_bits, slots = 1u << pb;
  for (uint32_t slot = t; slot < slots; slot += blockDim.x) {
    // largest s with cum[s] <= slot: that symbol owns the slot
    int lo = 0, hi = 255;
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if (cum[mid] <= slot) lo = mid; else hi = mid - 1;
    }
    uint32_t f = a.freq[lo];
    uint32_t fe = (f >= slots) ? 0u : f;  // a one-symbol table is handled by the flag
    if (pb == 8) lut[slot] = (fe << 24) | (symbol_bf16(uint32_t(lo), a.symfmt) << 8) | (slot - cum[lo]);
    else lut[slot] = (fe << 20) | (uint32_t(lo) << 12) | (slot - cum[lo]);
  }
}

// The pair table of a 7-bit frequency table (layout in eq_internal.cuh): one block of 256
// threads, each entry from two slot -> symbol searches.
__global__ void __launch_bounds__(256) rans_pair_build_kernel(const __grid_constant__ RansBuildArgs a) {
  __shared__ uint32_t cum[257];
  const uint32_t t = threadIdx.x;
  if (t == 0) {
    uint32_t c = 0;
    for (int s = 0; s < 256; ++s) {
      cum[s] = c;
      c += a.freq[s];
    }
    cum[256] = c;
    RansTableHeader h{a.symfmt == EQ_SYM_E4M3 ? kRansPairMagicE4M3 : kRansPairMagicInt8, a.flags,
                      a.single, kRansPairBits};
    *reinterpret_cast<RansTableHeader *>(a.dst) = h;
  }
  __syncthreads();
  auto owner = [&](uint32_t slot) {  // largest s with cum[s] <= slot
    int lo = 0, hi = 255;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (cum[mid] <= slot) lo = mid; else hi = mid - 1;
    }
    return uint32_t(lo);
  };
  uint2 *ent = reinterpret_cast<uint2 *>(a.dst + sizeof(RansTableHeader) / 4);
  for (uint32_t i = t; i < kRansPairEntries; i += blockDim.x) {
    const uint32_t slot1 = i & 127u, L = i >> 7;
    const uint32_t s1 = owner(slot1), f1 = a.freq[s1];
    const uint32_t v = f1 * L + (slot1 - cum[s1]);
    const uint32_t slot2 = v & 127u, s2 = owner(slot2), f2 = a.freq[s2];
    const uint32_t F = f1 * f2, B = f2 * (v >> 7) + (slot2 - cum[s2]);
    // F = 2^14 only in a one-symbol table, which the decoders never look up
    ent[i] = make_uint2(symbol_bf16(s1, a.symfmt) | (symbol_bf16(s2, a.symfmt) << 16),
                        ((F & 0x3FFFu) << 14) | B);
  }
}

struct HuffBuildArgs {
  uint32_t *dst;
  HuffTableHeader h;
  uint16_t t[kHuffMaxTables][256];
};

// One code from the hierarchical tables, reading the 32 bits of w from the top.  Returns the
// length (0 for a bad pattern) and the value in *sym.
__device__ __forceinline__ uint32_t huff_tree_decode(const uint16_t *tree, uint32_t ntab, uint32_t w,
                                                     uint32_t *sym) {
  uint32_t e = tree[w >> 24], used = 0;
  while ((e & 0x8000u) && e != kHuffInvalid) {
    const uint32_t tab = e & 0xFFu;
    used += 8;
    if (tab >= ntab || used > 24) return 0;
    e = tree[tab * 256 + ((w >> (24 - used)) & 0xFFu)];
  }
  const uint32_t rem = (e >> 8) & 0xFu;
  if (e == kHuffInvalid || rem == 0 || rem > 8) return 0;
  *sym = e & 0xFFu;
  return used + rem;
}

// Copies the hierarchical tables and derives the 12-bit window table from them: window v lists
// the codes that a greedy decode of the 12 bits v finds wholly inside them (at most 4).
__global__ void __launch_bounds__(256) huff_build_kernel(const __grid_constant__ HuffBuildArgs a) {
  __shared__ uint16_t tree[kHuffMaxTables * 256];
  const uint32_t ntab = a.h.num_tables;
  unsigned char *base = reinterpret_cast<unsigned char *>(a.dst);
  uint16_t *gtree = reinterpret_cast<uint16_t *>(base + kHuffTreeOffset);
  for (uint32_t i = threadIdx.x; i < ntab * 256; i += blockDim.x) {
    tree[i] = a.t[i / 256][i % 256];
    gtree[i] = tree[i];
  }
  if (threadIdx.x == 0) *reinterpret_cast<HuffTableHeader *>(a.dst) = a.h;
  __syncthreads();
  uint64_t *win = reinterpret_cast<uint64_t *>(base + kHuffWindowOffset);
  for (uint32_t v = threadIdx.x; v < kHuffWindow; v += blockDim.x) {
    uint64_t entry = 0;
    uint32_t pos = 0, n = 0;
    while (n < 4) {
      uint32_t sym = 0;
      const uint32_t w = (v << (32 - kHuffWindowBits)) << pos;  // zeros past the window
      const uint32_t len = huff_tree_decode(tree, ntab, w, &sym);
      if (len == 0 || pos + len > kHuffWindowBits) {
        // the first code needs bits past the window (or the pattern is bad, which the full
        // decode on the real bits reports): the decoder takes the hierarchical path
        if (n == 0) entry |= kHuffLong;
        break;
      }
      entry |= uint64_t(sym) << (8 * n);
      entry |= uint64_t(len) << (32 + 4 * n);
      pos += len;
      ++n;
    }
    entry |= uint64_t(pos) << 48;
    entry |= uint64_t(n) << 52;
    win[v] = entry;
  }
}

// Hierarchical tables of a canonical code given by its lengths.  Returns EQ_OK and fills `a`.
static eq_status huff_tables_from_lengths(const uint32_t *len, HuffBuildArgs &a) {
  uint64_t kraft = 0;  // sum of 2^(32 - len), compared with 2^32
  uint32_t max_len = 0;
  for (int s = 0; s < 256; ++s) {
    if (len[s] > 32) return EQ_ERR_FORMAT;
    if (len[s]) kraft += 1ull << (32 - len[s]);
    max_len = std::max(max_len, len[s]);
  }
  if (kraft > (1ull << 32)) return EQ_ERR_FORMAT;
  for (auto &tbl : a.t) std::fill(std::begin(tbl), std::end(tbl), kHuffInvalid);
  uint32_t ntab = 1;
  // canonical order: by (length, value); code values increase by one, shifted as length grows
  uint64_t code = 0;
  uint32_t prev = 0;
  for (uint32_t l = 1; l <= 32; ++l)
    for (int s = 0; s < 256; ++s) {
      if (len[s] != l) continue;
      if (prev) code <<= (l - prev);
      prev = l;
      uint32_t table = 0, rem = l;
      while (rem > 8) {  // walk / create the pointer chain for the leading 8-bit groups
        uint32_t idx = uint32_t(code >> (rem - 8)) & 0xFFu;
        uint16_t &e = a.t[table][idx];
        if (e == kHuffInvalid) {
          if (ntab >= kHuffMaxTables) return EQ_ERR_UNSUPPORTED;
          e = uint16_t(0x8000u | ntab);
          ++ntab;
        } else if (!(e & 0x8000u)) {
          return EQ_ERR_FORMAT;  // a shorter code is a prefix of this one
        }
        table = e & 0xFFu;
        rem -= 8;
      }
      uint32_t lo = uint32_t(code & ((1ull << rem) - 1)) << (8 - rem);
      for (uint32_t k = 0; k < (1u << (8 - rem)); ++k) {
        uint16_t &e = a.t[table][lo + k];
        if (e != kHuffInvalid) return EQ_ERR_FORMAT;
        e = uint16_t((rem << 8) | uint32_t(s));
      }
      code += 1;
    }
  a.h = HuffTableHeader{kHuffMagic, ntab, max_len, 0u};
  return EQ_OK;
}

static std::atomic<int> g_sm_count[64];  // 0 until looked up; any host thread may call

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  if (dev < 64) {
    const int c = g_sm_count[dev].load(std::memory_order_relaxed);
    if (c) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  if (dev < 64) g_sm_count[dev].store(n, std::memory_order_relaxed);
  return n;
}

}  // namespace eq

using namespace eq;

extern "C" size_t eq_table_bytes(eq_table_kind kind) {
  if (kind == EQ_TABLE_RANS) return kRansTableBytes;
  if (kind == EQ_TABLE_RANS8_E4M3 || kind == EQ_TABLE_RANS8_INT8) return kRans8TableBytes;
  if (kind == EQ_TABLE_RANS_PAIR_E4M3 || kind == EQ_TABLE_RANS_PAIR_INT8) return kRansPairTableBytes;
  if (kind == EQ_TABLE_HUFF) return kHuffTableBytes;
  return 0;
}

extern "C" eq_status eq_build_tables(eq_table_kind kind, const uint32_t *host_in,
                                     uint32_t prob_bits, void *d_tables, void *stream) {
  if (!host_in || !d_tables || !aligned(d_tables, 16)) return EQ_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool pair = kind == EQ_TABLE_RANS_PAIR_E4M3 || kind == EQ_TABLE_RANS_PAIR_INT8;
  const bool rans8 = kind == EQ_TABLE_RANS8_E4M3 || kind == EQ_TABLE_RANS8_INT8;
  if (kind == EQ_TABLE_RANS || pair || rans8) {
    if (prob_bits != (pair ? kRansPairBits : rans8 ? 8u : 12u)) return EQ_ERR_UNSUPPORTED;
    const uint32_t slots = 1u << prob_bits;
    RansBuildArgs a;
    a.dst = static_cast<uint32_t *>(d_tables);
    a.prob_bits = prob_bits;
    a.symfmt = kind == EQ_TABLE_RANS_PAIR_E4M3 || kind == EQ_TABLE_RANS8_E4M3 ? EQ_SYM_E4M3 : EQ_SYM_INT8;
    uint64_t sum = 0;
    uint32_t used = 0, single = 0;
    for (int s = 0; s < 256; ++s) {
      if (host_in[s] > slots) return EQ_ERR_FORMAT;
      a.freq[s] = uint16_t(host_in[s]);
      sum += host_in[s];
      if (host_in[s]) {
        ++used;
        single = uint32_t(s);
      }
    }
    if (sum != slots) return EQ_ERR_FORMAT;
    a.flags = (host_in[0x7F] ? kRansFlagNaN7F : 0u) | (host_in[0xFF] ? kRansFlagNaNFF : 0u) |
              (used == 1 ? kRansFlagSingle : 0u);
    a.single = used == 1 ? single : 0u;
    if (pair) rans_pair_build_kernel<<<1, 256, 0, st>>>(a);
    else rans_build_kernel<<<1, 256, 0, st>>>(a);
    return cuda_status(cudaGetLastError());
  }
  if (kind == EQ_TABLE_HUFF) {
    static thread_local HuffBuildArgs a;  // 16 KB: too large for the stack of some callers
    a.dst = static_cast<uint32_t *>(d_tables);
    eq_status s = huff_tables_from_lengths(host_in, a);
    if (s != EQ_OK) return s;
    huff_build_kernel<<<1, 256, 0, st>>>(a);
    return cuda_status(cudaGetLastError());
  }
  return EQ_ERR_ARG;
}

extern "C" const char *eq_status_string(eq_status s) {
  switch (s) {
    case EQ_OK: return "ok";
    case EQ_ERR_ARG: return "invalid argument";
    case EQ_ERR_FORMAT: return "malformed coded tensor or table";
    case EQ_ERR_UNSUPPORTED: return "unsupported format parameters";
    case EQ_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

extern "C" uint32_t eq_abi_version(void) { return EQ_ABI_VERSION; }
