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
// the 12-bit decode kernel's ring: 1 KiB copies, so that the ring work comes half as often
constexpr uint32_t kSegBytesWide = 1024;
constexpr uint32_t kRingBytesWide = kSegBytesWide * kNumSeg;

#ifdef __CUDACC__

// ------------------------------------------------------------------------------------------------
// Per-warp word ring.  Byte offsets are counted from A, the 16-byte-aligned start of the
// substream's span; segment s (bytes [s * SEG, s * SEG + SEG) of the span) lands in ring slot
// s % 4, i.e. at ring byte (offset mod 4 * SEG).  Copies are issued by lane 0; every lane waits.
// A slot is refilled only after the wait for its previous copy, so each of the four mbarriers has
// at most one copy in flight.  The ring and its barriers are held by their shared addresses.
// ------------------------------------------------------------------------------------------------
template <uint32_t SEG>
struct WordRingT {
  static constexpr uint32_t kSeg = SEG;
  static constexpr uint32_t kBytes = SEG * kNumSeg;
  uint32_t buf_s;     // shared address of the ring (a multiple of kBytes)
  uint32_t ring_off;  // the ring's offset from the shared-memory base (a multiple of kBytes)
  uint32_t bar_s;     // shared address of the ring's first mbarrier (four, 8 bytes apart)
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

  // hand segment `issued` to the copy engine (its slot's previous copy has been waited for):
  // predicated (the batch edges, where it keeps the warp from branching) or in a branch of lane 0
  // (the per-round checks, where the branch keeps the copy's operands out of the loop)
  __device__ __forceinline__ void issue_next(uint32_t lane) {
    const uint32_t s = issued, slot = s % kNumSeg;
    bulk_g2s_issue(lane == 0, buf_s + slot * SEG, A + size_t(s) * SEG, min(SEG, span - s * SEG),
                   bar_s + slot * 8u);
    ++issued;
  }
  __device__ __forceinline__ void issue(uint32_t lane) {
    if (lane == 0) {
      const uint32_t s = issued, slot = s % kNumSeg;
      bulk_g2s_issue(true, buf_s + slot * SEG, A + size_t(s) * SEG, min(SEG, span - s * SEG),
                     bar_s + slot * 8u);
    }
    ++issued;
    refill_at = issued < nseg ? (issued - kNumSeg + 1) * SEG : 0xFFFFFFFFu;
  }

  // point the ring at words [w0, w0 + nwords) and start the first copies
  __device__ __forceinline__ void start(const uint16_t *words, uint64_t w0, uint32_t nwords,
                                        uint32_t lane) {
    const unsigned char *g = reinterpret_cast<const unsigned char *>(words + w0);
    A = reinterpret_cast<const unsigned char *>(reinterpret_cast<uintptr_t>(g) & ~uintptr_t(15));
    off0 = uint32_t(g - A);
    span = (off0 + 2 * nwords + 15u) & ~15u;
    nseg = (span + SEG - 1) / SEG;
    issued = 0;
    ready = 0;
    ready_end = 0;
    refill_at = 0xFFFFFFFFu;
    while (issued < min(nseg, kNumSeg)) issue(lane);
  }

  // the copy into `slot` has landed (bounded wait); false on timeout
  __device__ __forceinline__ bool wait_slot(uint32_t slot) {
    if (!mbar_wait_bounded_s(bar_s + slot * 8u, (phase >> slot) & 1u)) return false;
    phase ^= 1u << slot;
    return true;
  }

  // every byte below `end` (an offset from A) must have landed; false on timeout
  __device__ __forceinline__ bool wait_below(uint32_t end) {
    if (nseg == 0) return true;
    const uint32_t last = min(nseg - 1, (end - 1) / SEG);
    while (ready <= last) {
      if (!wait_slot(ready % kNumSeg)) return false;
      ++ready;
    }
    ready_end = ready * SEG;
    return true;
  }

  // the per-round checks: wait only when the round may read past the landed bytes, refill only
  // when a slot has been used up.  The wait covers one word beyond the round's last possible
  // word: lanes that need no word still load the one after the warp's words (and drop it).
  __device__ __forceinline__ bool round_wait(uint32_t q) {
    constexpr uint32_t kAhead = 2 * kRoundWords + 2;
    return (q + kAhead <= ready_end || ready >= nseg) ? true : wait_below(q + kAhead);
  }
  // The batch protocol of the 12-bit decode's full rounds.  Once q (the warp's next word) has
  // entered segment cur, segments up to cur + 2 have landed and cur + 3 is in flight (or the
  // substream has no more), so every byte below safe_end = (cur + 3) * SEG can be read.  A round
  // of run G reads below q + 64 G + 2 and moves q by at most 64 G bytes, so the rounds of a batch
  // need no check: as many as keep their reads below safe_end, at least four with G = 8 and
  // SEG = 1024.  After a batch, each segment start q has passed (edge_next) is one edge: the slot
  // of the segment before it is used up and takes segment cur + 3, and segment cur + 2 (handed
  // out one segment earlier) is waited for.  batch_begin() sets this up from any state;
  // batch_end() restores the fields the per-round checks use.
  uint32_t edge_next;  // offset of the next segment start
  uint32_t safe_end;   // bytes below this offset have landed (0xFFFFFFFF: the whole substream)
  __device__ __forceinline__ void set_safe_end() {
    safe_end = ready >= nseg ? 0xFFFFFFFFu : ready * SEG;
  }
  __device__ __forceinline__ bool batch_begin(uint32_t q, uint32_t lane) {
    const uint32_t cur = q / SEG;
    while (issued < nseg && issued <= cur + 3) issue(lane);
    while (ready < nseg && ready <= cur + 2) {
      if (!wait_slot(ready % kNumSeg)) return false;
      ++ready;
    }
    edge_next = (cur + 1) * SEG;
    set_safe_end();
    return true;
  }
  // rounds of run G that can start at q without a check (at least 1 after batch_begin or the
  // edges of the last batch)
  template <int G>
  __device__ __forceinline__ uint32_t batch_rounds(uint32_t q) const {
    constexpr uint32_t kRound = 64u * G;
    return (safe_end - q - (kRound + 2u)) / kRound + 1u;
  }
  // one segment start passed: issued == cur + 3 and ready == cur + 2 whenever below nseg
  __device__ __forceinline__ bool batch_edge(uint32_t lane) {
    if (issued < nseg) {
      __syncwarp();
      issue_next(lane);
    }
    if (ready < nseg) {
      if (!wait_slot(ready % kNumSeg)) return false;
      ++ready;
    }
    edge_next += SEG;
    set_safe_end();
    return true;
  }
  __device__ __forceinline__ void batch_end() {
    ready_end = ready * SEG;
    refill_at = issued < nseg ? (issued - kNumSeg + 1) * SEG : 0xFFFFFFFFu;
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
    const uint32_t cur = q / SEG;
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
};
using WordRing = WordRingT<kSegBytes>;

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

// One step with the decode kernel's 12-bit table: 4-byte entries rearranged on load to
// [symbol:8 | f:12 | slot - cum:12] (bits 31..24, 23..12, 11..0; see decode_lut_bytes), at
// shared address `base`, so that the symbol byte lands where a byte-permute can take it.
// x' = f * (x >> 12) + (slot - cum).  Returns the entry.
template <bool FULL>
__device__ __forceinline__ uint32_t rans_sym_step(uint32_t &x, bool act, uint32_t base) {
  uint32_t e, nx;
  asm volatile(
      "{\n\t.reg .b32 a, f, b, xs;\n\t"
      "and.b32 a, %2, 4095;\n\t"
      "mad.lo.u32 a, a, 4, %3;\n\t"
      "shr.u32 xs, %2, 12;\n\t"
      "ld.shared.u32 %1, [a];\n\t"
      "shr.u32 f, %1, 12;\n\t"
      "and.b32 f, f, 4095;\n\t"
      "and.b32 b, %1, 4095;\n\t"
      "mad.lo.u32 %0, f, xs, b;\n\t}"
      : "=r"(nx), "=r"(e)
      : "r"(x), "r"(base));
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
template <bool FULL, uint32_t RING = kRingBytes>
__device__ __forceinline__ void rans_renorm(uint32_t &x, bool act, const unsigned char *smem,
                                            uint32_t ring_off, uint32_t &q, uint32_t lt) {
  const bool need = (FULL || act) && x < kRansL;
  const uint32_t m = __ballot_sync(0xFFFFFFFFu, need);
  const uint32_t a = (mad_lo(__popc(m & lt), 2u, q) & (RING - 1)) | ring_off;
  const uint32_t xr = mad_lo(x, 65536u, *reinterpret_cast<const uint16_t *>(smem + a));
  x = need ? xr : x;
  q = mad_lo(__popc(m), 2u, q);
}

// One round of a 12-bit stream (run 8) of Float8-E4M3 symbols in which every lane holds a run,
// as one PTX block: eight steps (rans_sym_step), each followed by its renormalisation point, and
// the round's dequantisation.  The dequantisation uses an exact identity of the E4M3 format: for
// every finite code c, the bf16 bit pattern (c & 0x80) << 8 | (c & 0x7F) << 4 is the value of c
// times 2^-120 (normal codes map to normal bf16 values, subnormal codes to subnormal ones, +-0 to
// +-0), so two codes become a bf16x2 pair with one byte-permute (the permute's sign-replicate
// mode supplies the sign bits) and two logic operations, and one bf16x2 multiply by the row scale
// times 2^120 gives bf16_rne(value * scale): both factors are exact and the product is rounded
// once.  Valid for tables without NaN codes and row scales below 2^8 in magnitude (the scale
// times 2^120 is then finite and exact).  One PTX block leaves ptxas no moves between the steps.
//   tb:   shared address of the table;
//   ring: shared address of this warp's word ring, a multiple of its size RING, so that a word's
//         address is one mask-and-or of q + 2 * rank;
//   lt:   the lanes below this one; sc2e: bf16 bits of scale * 2^120 in both halves.
// The lane's "needs a word" predicate feeds both the ballot and the predicated merge.
#define EQ_E4_STEP(V)                                  \
  "and.b32 t, %0, 4095;\n\t"                         \
  "mad.lo.u32 a, t, 4, %6;\n\t"                      \
  "shr.u32 xs, %0, 12;\n\t"                          \
  "ld.shared.u32 " V ", [a];\n\t"                    \
  "shr.u32 f, " V ", 12;\n\t"                        \
  "and.b32 f, f, 4095;\n\t"                          \
  "and.b32 t, " V ", 4095;\n\t"                      \
  "mad.lo.u32 %0, f, xs, t;\n\t"                     \
  "setp.lt.u32 p, %0, 65536;\n\t"                    \
  "vote.sync.ballot.b32 m, p, 0xffffffff;\n\t"       \
  "and.b32 r, m, %9;\n\t"                            \
  "popc.b32 r, r;\n\t"                               \
  "mad.lo.u32 a, r, 2, %1;\n\t"                      \
  "and.b32 a, a, %10;\n\t"                           \
  RING_JOIN " a, a, %8;\n\t"                         \
  "ld.shared.u16 w, [a];\n\t"                        \
  "@p mad.lo.u32 %0, %0, 65536, w;\n\t"              \
  "popc.b32 m, m;\n\t"                               \
  "mad.lo.u32 %1, m, 2, %1;\n\t"
#define EQ_E4_PAIR(OUT)                                \
  EQ_E4_STEP("va") EQ_E4_STEP("vb")                    \
  "prmt.b32 va, va, vb, 0xF7B3;\n\t"                 \
  "and.b32 vb, va, 0x007F007F;\n\t"                  \
  "shl.b32 vb, vb, 4;\n\t"                           \
  "and.b32 va, va, 0x80008000;\n\t"                  \
  "or.b32 va, va, vb;\n\t"                           \
  "mul.rn.bf16x2 " OUT ", va, %7;\n\t"

// ALIGNED: `ring` is a multiple of RING (the word address is then a mask-and-or); otherwise any
// shared address, and the masked offset is added to it.
template <uint32_t RING, bool ALIGNED = true>
__device__ __forceinline__ uint4 rans_round12_e4m3(uint32_t &x, uint32_t &q, uint32_t tb,
                                                   uint32_t ring, uint32_t lt, uint32_t sc2e) {
  uint4 o;
  if constexpr (ALIGNED) {
#define RING_JOIN "or.b32"
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b32 t, a, f, va, vb, xs, m, r, w;\n\t"
        EQ_E4_PAIR("%2") EQ_E4_PAIR("%3") EQ_E4_PAIR("%4") EQ_E4_PAIR("%5")
        "}"
        : "+r"(x), "+r"(q), "=r"(o.x), "=r"(o.y), "=r"(o.z), "=r"(o.w)
        : "r"(tb), "r"(sc2e), "r"(ring), "r"(lt), "n"(RING - 1));
#undef RING_JOIN
  } else {
#define RING_JOIN "add.u32"
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b32 t, a, f, va, vb, xs, m, r, w;\n\t"
        EQ_E4_PAIR("%2") EQ_E4_PAIR("%3") EQ_E4_PAIR("%4") EQ_E4_PAIR("%5")
        "}"
        : "+r"(x), "+r"(q), "=r"(o.x), "=r"(o.y), "=r"(o.z), "=r"(o.w)
        : "r"(tb), "r"(sc2e), "r"(ring), "r"(lt), "n"(RING - 1));
#undef RING_JOIN
  }
  return o;
}
#undef EQ_E4_PAIR
#undef EQ_E4_STEP

// [f:12 | symbol:8 | slot - cum:12] (the 12-bit table eq_build_tables writes) rearranged to the
// shared-memory layout [symbol:8 | f:12 | slot - cum:12] that rans_sym_step reads
__device__ __forceinline__ uint32_t sym_first_entry(uint32_t v) {
  return (v << 12 & 0xFF000000u) | (v >> 20) << 12 | (v & 0xFFFu);
}

// bf16 bits of scale * 2^120 in both halves (the factor of rans_round12_e4m3); exact for
// |scale| < 2^8 (a finite bf16 held exactly as fp32; the fp32 product is a power-of-two scaling)
__device__ __forceinline__ uint32_t scale_e4m3_offset(float sc) {
  return __byte_perm(__float_as_uint(sc * 1.329227995784916e36f), 0u, 0x3232u);
}

// A renormalisation point with the ring at absolute shared address `ring` (a multiple of RING):
// the general form of the one in rans_round12_e4m3, for rounds in which some lanes hold no run.
template <bool FULL, uint32_t RING>
__device__ __forceinline__ void rans_renorm_abs(uint32_t &x, bool act, uint32_t ring, uint32_t &q,
                                                uint32_t lt) {
  const bool need = (FULL || act) && x < kRansL;
  const uint32_t m = __ballot_sync(0xFFFFFFFFu, need);
  const uint32_t a = (mad_lo(__popc(m & lt), 2u, q) & (RING - 1)) | ring;
  uint32_t w;
  asm volatile("ld.shared.u16 %0, [%1];" : "=r"(w) : "r"(a));
  const uint32_t xr = mad_lo(x, 65536u, w);
  x = need ? xr : x;
  q = mad_lo(__popc(m), 2u, q);
}

// the lane mask below this lane, read once into a register (a volatile read, so that it is not
// re-read from the special register at every use)
__device__ __forceinline__ uint32_t lanemask_lt_once() {
  uint32_t m;
  asm volatile("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
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
template <class Ring>
__device__ __forceinline__ void ring_init(Ring &R, unsigned char *smem, unsigned char *rings,
                                          uint64_t *bars, uint32_t warp, uint32_t lane) {
  R.buf_s = smem_addr(rings) + warp * Ring::kBytes;
  R.ring_off = uint32_t(rings - smem) + warp * Ring::kBytes;
  R.bar_s = smem_addr(bars) + warp * kNumSeg * 8u;
  R.phase = 0;
  if (lane == 0) {
    for (uint32_t s = 0; s < kNumSeg; ++s) mbar_init(&bars[warp * kNumSeg + s], 1);
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

// The decode kernel's table: 12-bit entries are rearranged on load to [symbol | f | slot - cum]
// (16 KiB), the 8- and 7-bit tables are used as they are.  Its rings: 4 KiB (1 KiB copies) with
// 12-bit tables, placed at a shared address that is a multiple of their size (up to one ring of
// slack), else 2 KiB right after the table.
__host__ __device__ constexpr uint32_t decode_lut_bytes(uint32_t pb) {
  return rans_lut_bytes(pb);
}
__host__ __device__ constexpr uint32_t decode_ring_bytes(uint32_t pb) {
  return pb == 12 ? kRingBytesWide : kRingBytes;
}
__host__ __device__ constexpr size_t decode_smem_bytes(uint32_t warps, uint32_t pb) {
  return decode_lut_bytes(pb) + (pb == 12 ? kRingBytesWide : 0) +
         warps * (decode_ring_bytes(pb) + kNumSeg * 8);
}

}  // namespace eq
