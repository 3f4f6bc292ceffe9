// Dequantisation of decoded symbols: out = bf16_rne(value(symbol) * scale).
//
// value() is the Float8-E4M3 value of the byte or the byte read as int8 (the two base alphabets
// of "Float8@2bits", summary section "Concepto Central").  The scale is one bf16 per output
// channel (section "Optimizacion con Restriccion de Entropia": per-channel scales S).  Both
// factors are exact in fp32 and their product has at most 15 significant bits, so the fp32
// multiply is exact and the conversion to bf16 is the only rounding (round to nearest even).
// 8- and 7-bit tables carry the symbols' values as bf16 (exact): there one bf16x2 multiply
// computes two weights, its single rounding being the same round to nearest even.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "eq_internal.cuh"

namespace eq {

// two symbols (low byte first) -> two fp32 values
template <int FMT>
__device__ __forceinline__ float2 sym2_value(uint32_t two_bytes) {
  if constexpr (FMT == EQ_SYM_E4M3) {
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_bytes),
                                               __NV_E4M3);
    return __half22float2(*reinterpret_cast<__half2 *>(&h));
  } else {
    return make_float2(float(int32_t(two_bytes << 24) >> 24),
                       float(int32_t(two_bytes << 16) >> 24));
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&b);
}

// two symbols (16-bit pair, first in the low byte) scaled -> two bf16 in one 32-bit word.
// E4M3 NaN codes (0x7F, 0xFF) become the bf16 quiet NaN with the code's sign when nan_codes.
template <int FMT>
__device__ __forceinline__ uint32_t dequant2(uint32_t pair, float scale, bool nan_codes) {
  const float2 v = sym2_value<FMT>(pair);
  uint32_t o = pack_bf16x2(v.x * scale, v.y * scale);
  if constexpr (FMT == EQ_SYM_E4M3) {
    if (nan_codes) {
      if ((pair & 0x7Fu) == 0x7Fu) o = (o & 0xFFFF0000u) | 0x7FC0u | ((pair & 0x80u) << 8);
      if ((pair & 0x7F00u) == 0x7F00u)
        o = (o & 0x0000FFFFu) | ((0x7FC0u | (pair & 0x8000u)) << 16);
    }
  }
  return o;
}

// a symbol's value as bf16 bits, exactly (E4M3: at most 4 significant bits, exponent within
// bf16's range; Int8: at most 8 bits); the E4M3 NaN codes give the quiet NaN with their sign
__device__ __forceinline__ uint32_t symbol_bf16(uint32_t s, uint32_t symfmt) {
  if (symfmt == EQ_SYM_E4M3) {
    if ((s & 0x7Fu) == 0x7Fu) return 0x7FC0u | ((s & 0x80u) << 8);
    return __float_as_uint(sym2_value<EQ_SYM_E4M3>(s).x) >> 16;
  }
  return __float_as_uint(float(int32_t(s << 24) >> 24)) >> 16;
}

// A pair of symbol values from an 8-bit slot table or a 7-bit pair table (bf16x2, exact) times
// the row scale: one
// bf16x2 multiply, whose single round-to-nearest-even of the exact product is bf16_rne(value *
// scale).  sc2: the scale's bf16 bits in both halves.  Halves holding an E4M3 NaN code's value
// (the quiet NaN with the code's sign) pass through unscaled when nan_codes.
__device__ __forceinline__ uint32_t pair_dequant(uint32_t vals, uint32_t sc2, bool nan_codes) {
  uint32_t o;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(o) : "r"(vals), "r"(sc2));
  if (nan_codes) {
    if ((vals & 0x7FFFu) > 0x7F80u) o = (o & 0xFFFF0000u) | (vals & 0xFFFFu);
    if ((vals & 0x7FFF0000u) > 0x7F800000u) o = (o & 0x0000FFFFu) | (vals & 0xFFFF0000u);
  }
  return o;
}

// the values (bf16x2, first in the low half) of two expanded 12-bit entries' second words (value
// in bits 31..16)
__device__ __forceinline__ uint32_t value_pair12(uint32_t w0, uint32_t w1) {
  return __byte_perm(w0, w1, 0x7632u);
}

// the bf16 bits of a scale held as fp32 (converted exactly from bf16), in both halves
__device__ __forceinline__ uint32_t scale_bf16x2(float sc) {
  return __byte_perm(__float_as_uint(sc), 0u, 0x3232u);
}

// the values (bf16x2, first in the low half) of two 8-bit slot-table entries (value in bits 23..8)
__device__ __forceinline__ uint32_t value_pair8(uint32_t e0, uint32_t e1) {
  return __byte_perm(e0, e1, 0x6521u);
}

// the eight symbols of a round, taken from their PB-bit slot-table entries (12-bit: the symbol in
// bits 19..12; 8-bit: the symbol's value as bf16 in bits 23..8), scaled -> eight bf16 (one 16-byte
// store)
template <int FMT, uint32_t PB = 12>
__device__ __forceinline__ uint4 dequant8(const uint32_t (&e)[8], float scale, bool nan_codes) {
  uint32_t o[4];
  if constexpr (PB == 8) {
    const uint32_t sc2 = scale_bf16x2(scale);
#pragma unroll
    for (int k = 0; k < 4; ++k) o[k] = pair_dequant(value_pair8(e[2 * k], e[2 * k + 1]), sc2, nan_codes);
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if constexpr (FMT == EQ_SYM_INT8) {
        // the symbol byte sign-extended straight out of the entry
        const float v0 = float(int32_t(e[2 * k] << 12) >> 24);
        const float v1 = float(int32_t(e[2 * k + 1] << 12) >> 24);
        o[k] = pack_bf16x2(v0 * scale, v1 * scale);
      } else {
        o[k] = dequant2<FMT>(((e[2 * k] >> 12) & 0xFFu) | ((e[2 * k + 1] >> 4) & 0xFF00u), scale, nan_codes);
      }
    }
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// one symbol -> bf16 bits
template <int FMT>
__device__ __forceinline__ uint16_t dequant1(uint32_t sym, float scale) {
  float v = sym2_value<FMT>(sym & 0xFFu).x;
  uint32_t o = pack_bf16x2(v * scale, 0.0f) & 0xFFFFu;
  if constexpr (FMT == EQ_SYM_E4M3) {
    if ((sym & 0x7Fu) == 0x7Fu) o = 0x7FC0u | ((sym & 0x80u) << 8);
  }
  return static_cast<uint16_t>(o);
}

}  // namespace eq
