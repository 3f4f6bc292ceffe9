// Internal helpers shared by the library's CUDA sources (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "eq.h"

namespace eq {

// ------------------------------------------------------------------------------------------------
// device decode-table layouts written by eq_build_tables
// ------------------------------------------------------------------------------------------------

// rANS: 16-byte header, then one 32-bit entry per slot of the 2^pb-slot probability space
// (pb = prob_bits, 12 or 8), f = frequency of the slot's symbol (1 .. 2^pb - 1):
//   12-bit: bits 31..20 f, bits 19..12 symbol, bits 11..0 slot - cum;
//   8-bit:  bits 31..24 f, bits 23..8 the symbol's value as bf16, bits 7..0 slot - cum;
// so the decode step x' = f * floor(x / 2^pb) + slot - cum is (e >> (32 - pb)) * (x >> pb) +
// (e & (2^pb - 1)).
// A table whose single symbol owns every slot cannot store its frequency in pb bits; the header
// flags it instead and the decoders take a separate path.
constexpr uint32_t kRansProbBits = 12;                 // the larger table
constexpr uint32_t kRansSlots = 1u << kRansProbBits;  // entries the table allocation holds
constexpr uint32_t kRansL = 1u << 16;
struct RansTableHeader {
  uint32_t magic;        // kRansMagic, kRans8Magic*, kRansPairMagic*
  uint32_t flags;        // kRansFlag*
  uint32_t single_sym;   // symbol of a one-symbol table
  uint32_t prob_bits;    // 12 or 8
};
constexpr uint32_t kRansMagic = 0x52414E53u;  // "RANS" (12-bit slot table)
// 8-bit slot tables (EQ_TABLE_RANS8_E4M3 / _INT8) carry the symbol's value as bf16 bits (exact, as
// in the pair tables below) instead of the symbol, so they are specific to the symbol format.
constexpr uint32_t kRans8MagicE4M3 = 0x52563845u;  // "RV8E"
constexpr uint32_t kRans8MagicInt8 = 0x52563849u;  // "RV8I"
constexpr size_t kRans8TableBytes = 16 + 256 * 4;
// rANS pair table of a 7-bit frequency table (EQ_TABLE_RANS_PAIR_E4M3 / _INT8): two decode
// steps at once.  Entry i (i = x mod 2^14, the state's low 14 bits) for slot1 = i mod 128,
// L = i >> 7:
//   s1 = symbol of slot1, v = f1 * L + (slot1 - cum1), slot2 = v mod 128, s2 = its symbol,
//   F = f1 * f2, B = f2 * (v >> 7) + (slot2 - cum2);
//   word 0 = value(s1) | value(s2) << 16, each the symbol's value as bf16 bits (exact: an Int8
//            value has at most 8 significant bits, an E4M3 one 4 within bf16's exponent range;
//            the E4M3 NaN codes give 0x7FC0 / 0xFFC0),
//   word 1 = F << 14 | B.
// Then the two steps x -> x1 -> x2 are x2 = F * (x >> 14) + B: with x >> 7 = 128 H + L
// (H = x >> 14), x1 = f1 (x >> 7) + slot1 - cum1 = 128 f1 H + v, so x1 mod 128 = slot2 and
// x1 >> 7 = f1 H + (v >> 7).  B < F < 2^14 unless one symbol owns all 128 slots (F = 2^14), a
// table the header flags and the decoders never look up.  Dequantisation of the pair is one
// bf16x2 multiply of word 0 by the row scale: the product of two bf16 values is exact in fp32,
// so the multiply's one round-to-nearest-even gives bf16_rne(value * scale).
constexpr uint32_t kRansPairBits = 7;
constexpr uint32_t kRansPairEntries = 1u << (2 * kRansPairBits);
constexpr uint32_t kRansPairMagicE4M3 = 0x52504537u;  // "RPE7"
constexpr uint32_t kRansPairMagicInt8 = 0x52504937u;  // "RPI7"
constexpr size_t kRansPairTableBytes = 16 + size_t(kRansPairEntries) * 8;
constexpr uint32_t kRansFlagNaN7F = 1u;       // frequency of byte 0x7F is nonzero
constexpr uint32_t kRansFlagNaNFF = 2u;       // frequency of byte 0xFF is nonzero
constexpr uint32_t kRansFlagSingle = 4u;      // one symbol owns every slot
constexpr size_t kRansTableBytes = sizeof(RansTableHeader) + kRansSlots * 4;

// Huffman (DFloat11 exponent): 16-byte header, then
//   a window table W: 2048 x uint64, indexed by the next 11 code bits, listing the codes that lie
//   wholly inside those 11 bits (up to 4): bits 8i..8i+7 value of code i, bits 32+4i..35+4i its
//   length, bits 48..51 their total length, bits 52..54 how many (0 = no code fits, which is a
//   bad pattern unless bit 63 says the first code is longer than 12 bits);
//   then up to kHuffMaxTables hierarchical tables of 256 uint16 entries for codes of any length:
//   table 0 is indexed by the next 8 code bits; an entry is
//     a leaf    (bit 15 clear): bits 7..0 exponent value, bits 11..8 bits used at this level (1..8)
//     a pointer (bit 15 set):   bits 7..0 index of the child table, which reads the next 8 bits
//     0xFFFF: no code starts with this bit pattern.
constexpr uint32_t kHuffMaxTables = 32;
constexpr uint32_t kHuffWindowBits = 11;
constexpr uint32_t kHuffWindow = 1u << kHuffWindowBits;
constexpr uint64_t kHuffLong = 1ull << 63;
struct HuffTableHeader {
  uint32_t magic;        // kHuffMagic
  uint32_t num_tables;   // hierarchical tables in use
  uint32_t max_len;
  uint32_t reserved;
};
constexpr uint32_t kHuffMagic = 0x48554647u;  // "HUFG"
constexpr uint16_t kHuffInvalid = 0xFFFFu;
constexpr size_t kHuffWindowOffset = sizeof(HuffTableHeader);
constexpr size_t kHuffTreeOffset = kHuffWindowOffset + kHuffWindow * 8;
constexpr size_t kHuffTableBytes = kHuffTreeOffset + kHuffMaxTables * 256 * 2;

// ------------------------------------------------------------------------------------------------
// host helpers
// ------------------------------------------------------------------------------------------------

inline eq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? EQ_OK : EQ_ERR_CUDA; }

inline bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int device_sm_count();  // SMs of the current device (cached per device)

// A kernel's opt-in to more than 48 KiB of dynamic shared memory, set once per (device, kernel)
// flag.  Callers may issue library calls from several host threads at once: the flag is atomic,
// and two threads that both find it clear both make the (idempotent) attribute call.
inline eq_status smem_optin_once(std::atomic<bool> &done, const void *fn, size_t bytes) {
  if (done.load(std::memory_order_acquire)) return EQ_OK;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes)) !=
      cudaSuccess)
    return EQ_ERR_CUDA;
  done.store(true, std::memory_order_release);
  return EQ_OK;
}

// floor(n / d) for n < 2^40 and 1 <= d < 2^32 as __umul64hi(n, m) with m = ceil(2^64 / d).
inline uint64_t div_magic(uint64_t d) { return d <= 1 ? 0 : (~0ull) / d + 1; }

// ------------------------------------------------------------------------------------------------
// device helpers
// ------------------------------------------------------------------------------------------------

#ifdef __CUDACC__

__device__ __forceinline__ uint64_t div_by_magic(uint64_t n, uint64_t magic) {
  return magic ? __umul64hi(n, magic) : n;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// mbarrier + 1-D bulk copy (TMA engine, global -> this CTA's shared memory, no multicast)
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src_gmem, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_addr(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// try_wait / bounded wait on an mbarrier given by its shared address
__device__ __forceinline__ bool mbar_try_wait_s(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of an mbarrier, giving up after ~1 s (or 2^26 polls).  Returns false on
// timeout; the caller records EQ_DEV_TIMEOUT and stops using the buffer.
__device__ __forceinline__ bool mbar_wait_bounded_s(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait_s(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 0; i < (1u << 26); ++i) {
    if (mbar_try_wait_s(bar, parity)) return true;
    if ((i & 255u) == 255u && global_timer_ns() - t0 > 1000000000ull) break;
  }
  return false;
}
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity) {
  return mbar_wait_bounded_s(smem_addr(bar), parity);
}

// One 1-D bulk copy of `bytes` bytes (a multiple of 16) from global `src` to shared address
// `dst`, completing on the mbarrier at shared address `bar`, issued by the lanes with `issuer`
// set (one lane): the proxy fence that orders the warp's earlier reads of the destination before
// the copy engine's writes, the arrival with the expected byte count, the copy.  Predicated
// rather than branched, so the warp does not diverge around it.
__device__ __forceinline__ void bulk_g2s_issue(bool issuer, uint32_t dst, const void *src,
                                               uint32_t bytes, uint32_t bar) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.u32 p, %0, 0;\n"
      " @p fence.proxy.async.shared::cta;\n"
      " @p mbarrier.arrive.expect_tx.shared::cta.b64 _, [%4], %3;\n"
      " @p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%1], [%2], %3, [%4];\n"
      "}\n" ::"r"(uint32_t(issuer)),
      "r"(dst), "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void report(uint32_t *d_status, uint32_t bits) {
  if (bits) atomicOr(d_status, bits);
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

#endif  // __CUDACC__

}  // namespace eq
