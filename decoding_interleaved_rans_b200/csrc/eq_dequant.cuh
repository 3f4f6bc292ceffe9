// Dequantisation of decoded symbols: out = bf16_rne(value(symbol) * scale).
//
// value() is the Float8-E4M3 value of the byte or the byte read as int8 (the two base alphabets
// of "Float8@2bits", summary section "Concepto Central").  The scale is one bf16 per output
// channel (section "Optimizacion con Restriccion de Entropia": per-channel scales S).  Both
// factors are exact in fp32 and their product has at most 15 significant bits, so the fp32
// multiply is exact and the conversion to bf16 is the only rounding (round to nearest even).
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

// E4M3 NaN codes (0x7F, 0xFF) -> bf16 quiet NaN keeping the sign.  `four` holds 4 symbols,
// `lo`/`hi` the two packed bf16 pairs computed for them.
__device__ __forceinline__ void fix_e4m3_nan(uint32_t four, uint32_t &lo, uint32_t &hi) {
  uint32_t r[2] = {lo, hi};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t b = (four >> (8 * i)) & 0xFFu;
    if ((b & 0x7Fu) == 0x7Fu) {
      uint32_t nan = 0x7FC0u | ((b & 0x80u) << 8);
      uint32_t sh = 16 * (i & 1);
      r[i >> 1] = (r[i >> 1] & ~(0xFFFFu << sh)) | (nan << sh);
    }
  }
  lo = r[0];
  hi = r[1];
}

// four symbols (low byte first) scaled -> four bf16 in two 32-bit words
template <int FMT>
__device__ __forceinline__ uint2 dequant4(uint32_t four, float scale, bool nan_codes) {
  float2 a = sym2_value<FMT>(four & 0xFFFFu);
  float2 b = sym2_value<FMT>(four >> 16);
  uint2 o;
  o.x = pack_bf16x2(a.x * scale, a.y * scale);
  o.y = pack_bf16x2(b.x * scale, b.y * scale);
  if constexpr (FMT == EQ_SYM_E4M3) {
    if (nan_codes) fix_e4m3_nan(four, o.x, o.y);
  }
  return o;
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
