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
  uint64_t *bar;
  const unsigned char *A;
  uint32_t off0;    // bytes from A to the first word
  uint32_t span;    // bytes to copy (multiple of 16)
  uint32_t nseg;
  uint32_t issued;  // segments handed to the copy engine
  uint32_t ready;   // segments waited for

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
    while (issued < min(nseg, kNumSeg)) issue(lane);
  }

  // every byte below `end` (an offset from A) must have landed; false on timeout
  __device__ __forceinline__ bool wait_below(uint32_t end) {
    if (nseg == 0) return true;
    const uint32_t last = min(nseg - 1, (end - 1) / kSegBytes);
    while (ready <= last) {
      if (!mbar_wait_bounded(&bar[ready % kNumSeg], (ready / kNumSeg) & 1u)) return false;
      ++ready;
    }
    return true;
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
      if (!mbar_wait_bounded(&bar[ready % kNumSeg], (ready / kNumSeg) & 1u)) return EQ_DEV_TIMEOUT;
      ++ready;
    }
    return 0;
  }

  __device__ __forceinline__ uint32_t word_at(uint32_t q) const {
    return *reinterpret_cast<const uint16_t *>(buf + (q & (kRingBytes - 1)));
  }
};

// ------------------------------------------------------------------------------------------------
// One decode step of the lane's state x.  q is the byte offset (from the ring's A) of the group's
// next unread word; it advances by 2 bytes per word the warp reads.  Slot-table entry: symbol in
// bits 31..24, frequency in 23..12, slot - cum in 11..0.  A ballot finds the lanes whose state
// fell below 2^16; each takes the word at its rank among them, so words go out in stream order.
// ------------------------------------------------------------------------------------------------
template <bool FULL>
__device__ __forceinline__ uint32_t rans_step(uint32_t &x, bool act, const uint32_t *lut,
                                              const WordRing &R, uint32_t &q, uint32_t lt) {
  const uint32_t e = lut[x & (kRansSlots - 1)];
  const uint32_t nx = ((e >> 12) & 0xFFFu) * (x >> kRansProbBits) + (e & 0xFFFu);
  const bool on = FULL || act;
  if (on) x = nx;
  const bool need = on && x < kRansL;
  const uint32_t m = __ballot_sync(0xFFFFFFFFu, need);
  if (need) x = (x << 16) | R.word_at(q + 2 * __popc(m & lt));
  q += 2 * __popc(m);
  return e;
}

// byte 3 of `e` into byte p of `acc`
__device__ __forceinline__ uint32_t put_sym(uint32_t acc, uint32_t e, int p) {
  return __byte_perm(acc, e, (0x3210u & ~(0xFu << (4 * p))) | (0x7u << (4 * p)));
}

// Init the rings' mbarriers (lane 0 of each warp) -- call before the block-wide sync.
__device__ __forceinline__ void ring_init(WordRing &R, unsigned char *rings, uint64_t *bars,
                                          uint32_t warp, uint32_t lane) {
  R.buf = rings + warp * kRingBytes;
  R.bar = bars + warp * kNumSeg;
  if (lane == 0) {
    for (uint32_t s = 0; s < kNumSeg; ++s) mbar_init(&R.bar[s], 1);
    fence_mbar_init();
  }
}

#endif  // __CUDACC__

__host__ __device__ constexpr size_t rans_smem_bytes(uint32_t warps) {
  return kRansSlots * 4 + warps * (kRingBytes + kNumSeg * 8);
}

}  // namespace eq
