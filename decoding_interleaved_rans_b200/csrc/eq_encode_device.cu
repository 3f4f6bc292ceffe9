// GPU compressor: per-channel AbsMax quantisation, symbol histogram and interleaved-rANS encoding
// on the device, producing exactly the containers the host compressor (eq_encode.cpp) and the
// decoders read.  The pages quantise and ANS-code the flattened weights offline ("Float8@2bits"
// summary, "Codificacion de Pesos"; compression of a 70B model in minutes, abstract and summary
// disagree on how many); doing it on the GPU makes that step a matter of milliseconds per layer.
//
// Encoding runs twice over the symbols: a plan pass (final states and each substream's word
// count, turned into offsets by a device scan) and a write pass that emits every word straight
// into its place.  One warp encodes one group of 32 streams, in exactly the reverse of the decode
// order: rounds and positions backwards; inside a step the words of the emitting lanes are placed,
// in stream order, just below those of the later steps (a ballot + popcount rank).
#include <algorithm>

#include "eq_encode.h"
#include "eq_internal.cuh"
#include <cuda_bf16.h>
#include <cuda_fp8.h>

namespace eq {

// ------------------------------------------------------------------------------------------------
// quantisation: one CTA per row
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quantize_kernel(const float *__restrict__ w, uint32_t cols,
                                                       uint32_t symfmt, float div,
                                                       uint8_t *__restrict__ sym,
                                                       uint16_t *__restrict__ scales) {
  __shared__ float red[8];
  __shared__ float s_sh;
  const uint64_t row = blockIdx.x;
  const float *wr = w + row * cols;
  float amax = 0.0f;
  for (uint32_t c = threadIdx.x; c < cols; c += blockDim.x) amax = fmaxf(amax, fabsf(wr[c]));
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, d));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.0f;
    for (uint32_t i = 0; i < blockDim.x / 32; ++i) m = fmaxf(m, red[i]);
    __nv_bfloat16 sb = __float2bfloat16_rn(__fdiv_rn(m, div));
    uint16_t bits = *reinterpret_cast<uint16_t *>(&sb);
    if (m == 0.0f || (bits & 0x7FFFu) == 0) bits = 0x3F80u;  // a row of zeros gets scale 1
    scales[row] = bits;
    s_sh = __uint_as_float(uint32_t(bits) << 16);
  }
  __syncthreads();
  const float s = s_sh;
  uint8_t *out = sym + row * cols;
  for (uint32_t c = threadIdx.x; c < cols; c += blockDim.x) {
    const float v = __fdiv_rn(wr[c], s);
    if (symfmt == EQ_SYM_E4M3) {
      out[c] = uint8_t(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
    } else {
      const float q = fminf(127.0f, fmaxf(-127.0f, rintf(v)));
      out[c] = uint8_t(int8_t(q));
    }
  }
}

// ------------------------------------------------------------------------------------------------
// histogram: per-CTA shared counts, then one atomic per symbol value
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) histogram_kernel(const uint8_t *__restrict__ sym, uint64_t n,
                                                        uint32_t *__restrict__ counts) {
  __shared__ uint32_t h[256];
  h[threadIdx.x] = 0;
  __syncthreads();
  const uint64_t stride = uint64_t(gridDim.x) * blockDim.x * 16;
  for (uint64_t base = (uint64_t(blockIdx.x) * blockDim.x + threadIdx.x) * 16; base < n;
       base += stride) {
    if (base + 16 <= n && (reinterpret_cast<uintptr_t>(sym + base) & 15) == 0) {
      const uint4 v = *reinterpret_cast<const uint4 *>(sym + base);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int b = 0; b < 4; ++b) atomicAdd(&h[(w[k] >> (8 * b)) & 0xFFu], 1u);
    } else {
      for (uint64_t j = base; j < n && j < base + 16; ++j) atomicAdd(&h[sym[j]], 1u);
    }
  }
  __syncthreads();
  if (h[threadIdx.x]) atomicAdd(&counts[threadIdx.x], h[threadIdx.x]);
}

// ------------------------------------------------------------------------------------------------
// rANS encoding
// ------------------------------------------------------------------------------------------------
struct EncodeParams {
  const uint8_t *sym;
  uint32_t *states;
  uint64_t *word_off;  // plan: counts land in word_off[u + 1]; encode: offsets
  uint16_t *words;
  uint32_t *status;
  uint64_t numel;
  uint64_t units;
  uint32_t chunk, streams, groups, run;
  uint32_t prob_bits;  // 12, or 8 / 7: renormalise after every second step (then run == 8)
  uint16_t freq[256];
};

template <bool WRITE>
__global__ void __launch_bounds__(256) rans_encode_kernel(const __grid_constant__ EncodeParams P) {
  __shared__ uint32_t fs[256], cs[256];
  __shared__ uint64_t rcp[256];  // ceil(2^64 / f): floor(x / f) = __umul64hi(x, rcp) for x < 2^32
  for (uint32_t s = threadIdx.x; s < 256; s += blockDim.x) {
    const uint32_t f = P.freq[s];
    uint32_t c = 0;
    for (uint32_t t = 0; t < s; ++t) c += P.freq[t];
    fs[s] = f;
    cs[s] = c;
    rcp[s] = f > 1 ? (~0ull) / f + 1 : 0;
  }
  __syncthreads();
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t unit = uint64_t(blockIdx.x) * (blockDim.x / 32) + warp;
  if (unit >= P.units) return;
  const uint64_t chunk = unit / P.groups;
  const uint32_t g = uint32_t(unit - chunk * P.groups);
  const uint32_t S = P.streams, s = 32 * g + lane, G = P.run;
  const uint64_t j0 = chunk * uint64_t(P.chunk);
  const uint32_t n = uint32_t(P.numel - j0 < P.chunk ? P.numel - j0 : P.chunk);
  const uint32_t runs = (n + G - 1) / G, rounds = (runs + S - 1) / S;
  const uint32_t lt = lanemask_lt();
  const uint8_t *src = P.sym + j0;
  uint32_t x = 1u << 16, bad = 0;
  uint64_t pos = WRITE ? P.word_off[unit + 1] : 0;  // words go below this, last step first
  uint64_t cnt = 0;
  for (uint32_t r = rounds; r-- > 0;) {
    const uint32_t run = r * S + s;
    for (uint32_t p = G; p-- > 0;) {
      const uint64_t j = uint64_t(run) * G + p;
      const bool on = run < runs && j < n;
      uint32_t f = 1, c = 0;
      uint64_t m = 0, xmax = 0;
      if (on) {
        const uint32_t q = src[j];
        f = fs[q];
        c = cs[q];
        m = rcp[q];
        if (f == 0) {
          bad = EQ_DEV_BAD_CODE;
          f = 1;
        }
        // flush bound of the renormalisation group that ends at this step: one step (12-bit
        // tables), or positions p - 1 and p of the run (8-bit tables, p odd)
        if (P.prob_bits == 12) xmax = uint64_t(f) << 20;
        else if (p & 1) xmax = (uint64_t(f) * max(fs[src[j - 1]], 1u)) << (32 - 2 * P.prob_bits);
      }
      const bool emit = on && xmax && uint64_t(x) >= xmax;
      const uint32_t em = __ballot_sync(0xFFFFFFFFu, emit);
      if (WRITE) {
        const uint32_t k = __popc(em);
        if (emit) P.words[pos - k + __popc(em & lt)] = uint16_t(x);
        pos -= k;
      } else {
        cnt += __popc(em);
      }
      if (emit) x >>= 16;
      if (on) {
        const uint32_t qt = f > 1 ? uint32_t(__umul64hi(uint64_t(x), m)) : x;
        x = (qt << P.prob_bits) + (x - qt * f) + c;
      }
    }
  }
  if (WRITE) {
    if (lane == 0 && pos != P.word_off[unit]) bad |= EQ_DEV_COUNT_MISMATCH;
  } else {
    P.states[chunk * S + s] = x;
    if (lane == 0) P.word_off[unit + 1] = cnt;
  }
  if (bad) atomicOr(P.status, bad);
}

// exclusive prefix over word_off[1 .. units] (the counts), in place; word_off[0] = 0
__global__ void __launch_bounds__(1024) offsets_scan_kernel(uint64_t *word_off, uint64_t units) {
  __shared__ uint64_t wsum[32];
  __shared__ uint64_t carry;
  const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    carry = 0;
    word_off[0] = 0;
  }
  __syncthreads();
  for (uint64_t base = 0; base < units; base += blockDim.x) {
    const uint64_t i = base + threadIdx.x;
    uint64_t v = i < units ? word_off[i + 1] : 0, incl = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint64_t u = __shfl_up_sync(0xFFFFFFFFu, incl, d);
      if (lane >= uint32_t(d)) incl += u;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      uint64_t w = lane < blockDim.x / 32 ? wsum[lane] : 0, s = w;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const uint64_t u = __shfl_up_sync(0xFFFFFFFFu, s, d);
        if (lane >= uint32_t(d)) s += u;
      }
      wsum[lane] = s - w;
    }
    __syncthreads();
    const uint64_t c0 = carry;
    if (i < units) word_off[i + 1] = c0 + wsum[warp] + incl;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = c0 + wsum[warp] + incl;
    __syncthreads();
  }
}

static eq_status check_encode_args(const uint8_t *d_sym, uint32_t rows, uint32_t cols,
                                   const uint32_t *host_freqs, uint32_t chunk_symbols,
                                   uint32_t streams, uint32_t run, EncodeParams &P) {
  if (!host_freqs) return EQ_ERR_ARG;
  const uint64_t numel = uint64_t(rows) * cols;
  if (numel >= (1ull << 40)) return EQ_ERR_UNSUPPORTED;
  if (streams == 0 || streams % 32 || streams > 1024 || (run != 1 && run != 8)) return EQ_ERR_UNSUPPORTED;
  const uint32_t chunk = chunk_symbols ? chunk_symbols : cols;
  if (numel && (!d_sym || chunk == 0 || chunk % run)) return EQ_ERR_ARG;
  uint64_t sum = 0;
  for (int s = 0; s < 256; ++s) {
    if (host_freqs[s] > kRansSlots) return EQ_ERR_FORMAT;
    sum += host_freqs[s];
    P.freq[s] = uint16_t(host_freqs[s]);
  }
  if (sum != 128 && sum != 256 && sum != kRansSlots) return EQ_ERR_FORMAT;
  P.prob_bits = sum == 128 ? 7 : sum == 256 ? 8 : 12;
  // pairs of steps stay inside runs only when every run is whole
  if (P.prob_bits != 12 && (run != 8 || cols % 8)) return EQ_ERR_UNSUPPORTED;
  P.sym = d_sym;
  P.numel = numel;
  P.chunk = chunk;
  P.streams = streams;
  P.groups = streams / 32;
  P.run = run;
  P.units = numel ? (numel + chunk - 1) / chunk * P.groups : 0;
  return EQ_OK;
}

}  // namespace eq

using namespace eq;

extern "C" eq_status eq_quantize_device(const float *d_w, uint32_t rows, uint32_t cols,
                                        uint32_t symfmt, float int8_div, uint8_t *d_sym,
                                        uint16_t *d_scales, void *stream) {
  if (symfmt != EQ_SYM_E4M3 && symfmt != EQ_SYM_INT8) return EQ_ERR_ARG;
  if (symfmt == EQ_SYM_INT8 && !(int8_div > 0.0f)) return EQ_ERR_ARG;
  if (uint64_t(rows) * cols == 0) return EQ_OK;
  if (!d_w || !d_sym || !d_scales || rows >= (1u << 31)) return EQ_ERR_ARG;
  quantize_kernel<<<rows, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      d_w, cols, symfmt, symfmt == EQ_SYM_E4M3 ? 448.0f : int8_div, d_sym, d_scales);
  return cuda_status(cudaGetLastError());
}

extern "C" eq_status eq_histogram_device(const uint8_t *d_sym, uint64_t n, uint32_t *d_counts,
                                         void *stream) {
  if (!d_counts || (n && !d_sym)) return EQ_ERR_ARG;
  if (n == 0) return EQ_OK;
  const uint64_t per = 256ull * 16;
  const uint64_t blocks = std::min<uint64_t>((n + per - 1) / per, uint64_t(device_sm_count()) * 8);
  histogram_kernel<<<uint32_t(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(d_sym, n, d_counts);
  return cuda_status(cudaGetLastError());
}

extern "C" eq_status eq_rans_plan_device(const uint8_t *d_sym, uint32_t rows, uint32_t cols,
                                         const uint32_t *host_freqs, uint32_t chunk_symbols,
                                         uint32_t streams, uint32_t run, uint32_t *d_states,
                                         uint64_t *d_word_off, uint32_t *d_status, void *stream) {
  static thread_local EncodeParams P;
  eq_status s = check_encode_args(d_sym, rows, cols, host_freqs, chunk_symbols, streams, run, P);
  if (s != EQ_OK) return s;
  if (!d_word_off || !d_status || (P.units && !d_states)) return EQ_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  P.states = d_states;
  P.word_off = d_word_off;
  P.words = nullptr;
  P.status = d_status;
  if (P.units) {
    rans_encode_kernel<false><<<uint32_t((P.units + 7) / 8), 256, 0, st>>>(P);
    if (cudaGetLastError() != cudaSuccess) return EQ_ERR_CUDA;
  }
  offsets_scan_kernel<<<1, 1024, 0, st>>>(d_word_off, P.units);
  return cuda_status(cudaGetLastError());
}

extern "C" eq_status eq_rans_encode_device(const uint8_t *d_sym, uint32_t rows, uint32_t cols,
                                           const uint32_t *host_freqs, uint32_t chunk_symbols,
                                           uint32_t streams, uint32_t run,
                                           const uint64_t *d_word_off, uint16_t *d_words,
                                           uint32_t *d_status, void *stream) {
  static thread_local EncodeParams P;
  eq_status s = check_encode_args(d_sym, rows, cols, host_freqs, chunk_symbols, streams, run, P);
  if (s != EQ_OK) return s;
  if (!d_word_off || !d_status || (P.units && !d_words)) return EQ_ERR_ARG;
  if (!P.units) return EQ_OK;
  P.states = nullptr;
  P.word_off = const_cast<uint64_t *>(d_word_off);
  P.words = d_words;
  P.status = d_status;
  rans_encode_kernel<true><<<uint32_t((P.units + 7) / 8), 256, 0, static_cast<cudaStream_t>(stream)>>>(P);
  return cuda_status(cudaGetLastError());
}
