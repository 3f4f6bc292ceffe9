// Shared core of the rANS kernels (decode and fused GEMV), for the format of eq_rans_tensor in
// eq.h: one warp decodes one group of 32 interleaved streams of a chunk (lane l = stream 32 g + l),
// reading the group's own word substream through a shared-memory ring fed by 1-D bulk copies.
#pragma once

#include "eq_internal.cuh"

namespace eq {

constexpr uint32_t kSegBytes = 512;  // one bulk copy; >= the 32 * 8 words a round can read
constexpr uint32_t kNumSeg = 4;
constexpr uint32_t kRingBytes = kSegBytes * kNumSeg;
constexpr uint32_t kRoundWords = 32 * 8;  // words a group reads at most per round of 8 steps

#ifdef __CUDACC__

// ------------------------------------------------------------------------------------------------
// Per-warp word ring.  Byte offsets are counted from A, the 16-byte-aligned start of the
// substream's span; segment s (bytes [s * 512, s * 512 + 512) of the span) lands in ring slot
// s % 4, i.e. at ring byte (offset mod 2048).  Copies are issued by lane 0; every lane waits.
// ------------------------------------------------------------------------------------------------
struct WordRing {
  unsigned char *buf;
  uint32_t ring_off;  // buf - shared-memory base (a multiple of kRingBytes)
  uint64_t *bar;
  const unsigned char *A;
  uint32_t off0;    // bytes from A to the first word
  uint32_t span;    // bytes to copy (multiple of 16)
  uint32_t nseg;
  uint32_t issued;  // segments handed to the copy engine
  uint32_t ready;   // segments waited for
  uint32_t ready_end;  // offsets below this have landed (ready segments)
  uint32_t refill_at;  // once q reaches this offset a slot can be refilled
  uint32_t phase;      // bit s: the phase the next wait on slot s's barrier waits for (it
                       // carries over from one substream to the next a warp decodes)

  __device__ __forceinline__ void issue(uint32_t lane) {
    if (lane == 0) {
      const uint32_t s = issued, slot = s % kNumSeg;
      const uint32_t bytes = min(kSegBytes, span - s * kSegBytes);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_expect_tx(&bar[slot], bytes);
      bulk_g2s(buf + slot * kSegBytes, A + size_t(s) * kSegBytes, bytes, &bar[slot]);
    }
    ++issued;
    refill_at = issued < nseg ? (issued - kNumSeg + 1) * kSegBytes : 0xFFFFFFFFu;
  }

  // point the ring at words [w0, w0 + nwords) and start the first copies
  __device__ __forceinline__ void start(const uint16_t *words, uint64_t w0, uint32_t nwords,
                                        uint32_t lane) {
    const unsigned char *g = reinterpret_cast<const unsigned char *>(words + w0);
    A = reinterpret_cast<const unsigned char *>(reinterpret_cast<uintptr_t>(g) & ~uintptr_t(15));
    off0 = uint32_t(g - A);
    span = (off0 + 2 * nwords + 15u) & ~15u;
    nseg = (span + kSegBytes - 1) / kSegBytes;
    issued = 0;
    ready = 0;
    ready_end = 0;
    refill_at = 0xFFFFFFFFu;
    while (issued < min(nseg, kNumSeg)) issue(lane);
  }

  // the copy into `slot` has landed (bounded wait); false on timeout
  __device__ __forceinline__ bool wait_slot(uint32_t slot) {
    if (!mbar_wait_bounded(&bar[slot], (phase >> slot) & 1u)) return false;
    phase ^= 1u << slot;
    return true;
  }

  // every byte below `end` (an offset from A) must have landed; false on timeout
  __device__ __forceinline__ bool wait_below(uint32_t end) {
    if (nseg == 0) return true;
    const uint32_t last = min(nseg - 1, (end - 1) / kSegBytes);
    while (ready <= last) {
      if (!wait_slot(ready % kNumSeg)) return false;
      ++ready;
    }
    ready_end = ready * kSegBytes;
    return true;
  }

  // the per-round checks: wait only when the round may read past the landed bytes, refill only
  // when a slot has been used up.  The wait covers one word beyond the round's last possible
  // word: lanes that need no word still load the one after the warp's words (and drop it).
  __device__ __forceinline__ bool round_wait(uint32_t q) {
    constexpr uint32_t kAhead = 2 * kRoundWords + 2;
    return (q + kAhead <= ready_end || ready >= nseg) ? true : wait_below(q + kAhead);
  }
  __device__ __forceinline__ void round_refill(uint32_t q, uint32_t lane) {
    if (q >= refill_at) refill(q, lane);
  }

  // The offset below which the per-round checks have nothing to do: no wait (the landed bytes
  // cover q plus a round's worth and one word), no refill (no slot used up) and no overrun
  // (q_end: one past the substream's last byte).
  __device__ __forceinline__ uint32_t quiet_until(uint32_t q_end) const {
    constexpr uint32_t kAhead = 2 * kRoundWords + 2;
    uint32_t t = ready >= nseg ? 0xFFFFFFFFu : (ready_end >= kAhead ? ready_end - kAhead + 1 : 0u);
    t = min(t, refill_at);
    return min(t, q_end + 1);
  }

  // hand out the slots of segments lying wholly below offset q
  __device__ __forceinline__ void refill(uint32_t q, uint32_t lane) {
    const uint32_t cur = q / kSegBytes;
    if (issued < nseg && issued < cur + kNumSeg) {
      __syncwarp();
      do issue(lane);
      while (issued < nseg && issued < cur + kNumSeg);
    }
  }

  // wait (bounded) for every copy handed to the engine; EQ_DEV_TIMEOUT or 0
  __device__ __forceinline__ uint32_t drain() {
    while (ready < issued) {
      if (!wait_slot(ready % kNumSeg)) return EQ_DEV_TIMEOUT;
      ++ready;
    }
    return 0;
  }

  __device__ __forceinline__ uint32_t word_at(uint32_t q) const {
    return *reinterpret_cast<const uint16_t *>(buf + (q & (kRingBytes - 1)));
  }
};

// ------------------------------------------------------------------------------------------------
// Decode steps of the lane's state x.  q is the byte offset (from the ring's A) of the group's
// next unread word; it advances by 2 bytes per word the warp reads.  Slot-table entry e of a
// 12-bit table: f in bits 31..20, symbol in 19..12, slot - cum in 11..0, so f * floor(x / 4096) +
// (slot - cum) is one multiply-high-add: hi32((e & 0xFFF00000) * (x & 0xFFFFF000)) + (e & 0xFFF)
// (an 8-bit table: the same with 8-bit fields).  At a renormalisation point a ballot finds the
// lanes whose state fell below 2^16; each takes the word at its rank among them, so words go out
// in stream order.  ring_off: shared-memory offset of this warp's ring (a multiple of its size),
// so the word address is one mask-and-or.
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t mad_hi(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("mad.hi.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t mad_lo(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// The decoding half of a step with a PB-bit table (entry: f in the top PB bits, the symbol
// above bit 8 or 12, slot - cum in the low PB bits; eq_internal.cuh); returns the entry.
// x' = f * (x >> PB) + (slot - cum) as shifts and a low multiply-add: x >> PB is computed while
// the table load is in flight, so the step's dependency chain is load -> shift -> multiply-add
// (a multiply-high form, fewer instructions, measured slower: the high product's latency sits
// on the chain).  One PTX block, so ptxas does not redo the address arithmetic; volatile, so it
// is never hoisted above the barrier that publishes the table.
template <bool FULL, uint32_t PB>
__device__ __forceinline__ uint32_t rans_decode_step(uint32_t &x, bool act, const uint32_t *lut) {
  static_assert(PB == 12 || PB == 8, "12- or 8-bit tables");
  const uint32_t base = uint32_t(__cvta_generic_to_shared(lut));
  uint32_t e, nx;
  asm volatile(
      "{\n\t.reg .b32 a, f, b, xs;\n\t"
      "and.b32 a, %2, %4;\n\t"
      "shl.b32 a, a, 2;\n\t"
      "add.u32 a, a, %3;\n\t"
      "shr.u32 xs, %2, %5;\n\t"
      "ld.shared.u32 %1, [a];\n\t"
      "shr.u32 f, %1, %6;\n\t"
      "and.b32 b, %1, %4;\n\t"
      "mad.lo.u32 %0, f, xs, b;\n\t}"
      : "=r"(nx), "=r"(e)
      : "r"(x), "r"(base), "n"((1u << PB) - 1), "n"(PB), "n"(32 - PB));
  if (FULL || act) x = nx;
  return e;
}

// Two decode steps of a 7-bit stream with one pair-table lookup (layout in eq_internal.cuh):
// x2 = F * (x >> 14) + B.  Returns the two symbols' values as bf16x2 (the first in the low half).
template <bool FULL>
__device__ __forceinline__ uint32_t rans_pair_step(uint32_t &x, bool act, const uint32_t *lut) {
  const uint32_t base = uint32_t(__cvta_generic_to_shared(lut));
  uint32_t w0, nx;
  asm volatile(
      "{\n\t.reg .b32 a, w1, f, xs;\n\t"
      "and.b32 a, %2, 16383;\n\t"
      "shl.b32 a, a, 3;\n\t"
      "add.u32 a, a, %3;\n\t"
      "shr.u32 xs, %2, 14;\n\t"
      "ld.shared.v2.u32 {%1, w1}, [a];\n\t"
      "shr.u32 f, w1, 14;\n\t"
      "and.b32 w1, w1, 16383;\n\t"
      "mad.lo.u32 %0, f, xs, w1;\n\t}"
      : "=r"(nx), "=r"(w0)
      : "r"(x), "r"(base));
  if (FULL || act) x = nx;
  return w0;
}

// the header magic of a PB-bit table for symbols of format FMT (8-bit slot tables and 7-bit pair
// tables carry the symbols' values, so they are specific to the format)
template <int FMT, uint32_t PB>
__device__ __forceinline__ constexpr uint32_t rans_table_magic() {
  return PB == 12 ? kRansMagic
         : PB == 8 ? (FMT == EQ_SYM_E4M3 ? kRans8MagicE4M3 : kRans8MagicInt8)
                   : (FMT == EQ_SYM_E4M3 ? kRansPairMagicE4M3 : kRansPairMagicInt8);
}

// the symbol byte of a PB-bit entry
template <uint32_t PB>
constexpr uint32_t kSymShift = PB;

// A renormalisation point: every lane below 2^16 takes the group's next word, in lane order.
// All lanes load (the others drop the word), which keeps the step free of branches; the load
// stays inside the landed part of the ring (see round_wait).
template <bool FULL>
__device__ __forceinline__ void rans_renorm(uint32_t &x, bool act, const unsigned char *smem,
                                            uint32_t ring_off, uint32_t &q, uint32_t lt) {
  const bool need = (FULL || act) && x < kRansL;
  const uint32_t m = __ballot_sync(0xFFFFFFFFu, need);
  const uint32_t a = (mad_lo(__popc(m & lt), 2u, q) & (kRingBytes - 1)) | ring_off;
  const uint32_t xr = mad_lo(x, 65536u, *reinterpret_cast<const uint16_t *>(smem + a));
  x = need ? xr : x;
  q = mad_lo(__popc(m), 2u, q);
}

// one full step of a 12-bit stream (a renormalisation point after every step)
template <bool FULL>
__device__ __forceinline__ uint32_t rans_step(uint32_t &x, bool act, const uint32_t *lut,
                                              const unsigned char *smem, uint32_t ring_off,
                                              uint32_t &q, uint32_t lt) {
  const uint32_t e = rans_decode_step<FULL, 12>(x, act, lut);
  rans_renorm<FULL>(x, act, smem, ring_off, q, lt);
  return e;
}

// first position of the sorted super-weight list idx[0, n) holding a value >= key
__device__ __forceinline__ uint64_t patch_lower_bound(const uint64_t *idx, uint64_t n,
                                                      uint64_t key) {
  uint64_t lo = 0, hi = n;
  while (lo < hi) {
    const uint64_t mid = (lo + hi) >> 1;
    if (__ldg(idx + mid) < key) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// symbols of two 12-bit slot-table entries as one 16-bit pair (first in the low byte)
__device__ __forceinline__ uint32_t sym_pair(uint32_t e0, uint32_t e1) {
  return ((e0 >> 12) & 0xFFu) | ((e1 >> 4) & 0xFF00u);
}

// Init the rings' mbarriers (lane 0 of each warp) -- call before the block-wide sync.
__device__ __forceinline__ void ring_init(WordRing &R, unsigned char *smem, unsigned char *rings,
                                          uint64_t *bars, uint32_t warp, uint32_t lane) {
  R.buf = rings + warp * kRingBytes;
  R.ring_off = uint32_t(R.buf - smem);
  R.bar = bars + warp * kNumSeg;
  R.phase = 0;
  if (lane == 0) {
    for (uint32_t s = 0; s < kNumSeg; ++s) mbar_init(&R.bar[s], 1);
    fence_mbar_init();
  }
}

#endif  // __CUDACC__

// bytes before the first ring: the slot table (2^pb entries; for 7-bit tables the pair table),
// padded so that every ring starts at a multiple of its own size (the word address is formed with
// an OR)
__host__ __device__ constexpr uint32_t rans_lut_bytes(uint32_t pb) {
  return pb == kRansPairBits ? kRansPairEntries * 8u
                             : ((4u << pb) + kRingBytes - 1) / kRingBytes * kRingBytes;
}

// shared memory of a CTA: the slot table, then one ring per warp, then the rings' barriers
__host__ __device__ constexpr size_t rans_smem_bytes(uint32_t warps, uint32_t pb = 12) {
  return rans_lut_bytes(pb) + warps * (kRingBytes + kNumSeg * 8);
}

}  // namespace eq
