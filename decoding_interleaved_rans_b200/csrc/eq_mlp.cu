// eq_mlp_decode: a LLaMA-style MLP block y = W_down (silu(W_gate x) * (W_up x)) straight from the
// rANS-coded weights.  The pages name fused decode + compute kernels as the next step ("Float8@2bits"
// summary, closing section); no decoded weight ever reaches memory.  For batch <= 4 one kernel
// takes each row of gate and up in the same warp and writes the gated hidden vector h =
// bf16(silu(g) * u) directly (rans_gate_up_kernel); otherwise the gate and up products run in
// eq_decode_gemv's kernels and the SiLU gate in one small kernel that also rounds h to bf16 (the
// dtype the down projection reads).  Either way the down product then runs in eq_decode_gemv.
// The caller provides the scratch for the intermediate vectors (eq_mlp_scratch_bytes).
#include <algorithm>

#include "eq_internal.cuh"

#include <cuda_bf16.h>

namespace eq {

eq_status validate_rans_tensor(const eq_rans_tensor &t);  // eq_rans_decode.cu
eq_status gate_up_launch(const eq_rans_tensor *g, const eq_rans_tensor *u, const uint16_t *d_x,
                         uint32_t batch, uint16_t *d_h, uint32_t *d_status,
                         cudaStream_t st);  // eq_rans_gemv.cu

// h = bf16( silu(g) * u ), silu(v) = v / (1 + e^-v)
__global__ void __launch_bounds__(256) silu_mul_kernel(const float *__restrict__ g,
                                                       const float *__restrict__ u,
                                                       __nv_bfloat16 *__restrict__ h, uint64_t n) {
  for (uint64_t i = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += uint64_t(gridDim.x) * blockDim.x) {
    const float v = g[i];
    h[i] = __float2bfloat16_rn(v / (1.0f + expf(-v)) * u[i]);
  }
}

inline size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

size_t mlp_scratch_bytes(uint64_t inter, uint64_t batch) {
  return 2 * align256(inter * batch * 4) + align256(inter * batch * 2);
}

// the three products and the gate, given scratch already split into g, u, h.  With batch <= 4
// and gate/up in the fused kernel's layout, gate, up and the gate are one launch writing h (the
// products never leave the warps); otherwise two products, the gate kernel, and h.
eq_status mlp_run(const eq_rans_tensor *gate, const eq_rans_tensor *up,
                  const eq_rans_tensor *down, const uint16_t *d_x, uint32_t batch, float *d_y,
                  float *g, float *u, uint16_t *h, uint32_t *d_status, void *stream) {
  const eq_status f = gate_up_launch(gate, up, d_x, batch, h, d_status,
                                     static_cast<cudaStream_t>(stream));
  if (f == EQ_OK) return eq_decode_gemv(down, h, batch, d_y, d_status, stream);
  if (f != EQ_ERR_UNSUPPORTED) return f;
  eq_status s = eq_decode_gemv(gate, d_x, batch, g, d_status, stream);
  if (s != EQ_OK) return s;
  s = eq_decode_gemv(up, d_x, batch, u, d_status, stream);
  if (s != EQ_OK) return s;
  const uint64_t n = uint64_t(gate->rows) * batch;
  const uint64_t blocks = std::min<uint64_t>((n + 255) / 256, uint64_t(device_sm_count()) * 8);
  silu_mul_kernel<<<uint32_t(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      g, u, reinterpret_cast<__nv_bfloat16 *>(h), n);
  if (cudaGetLastError() != cudaSuccess) return EQ_ERR_CUDA;
  return eq_decode_gemv(down, h, batch, d_y, d_status, stream);
}

// shapes and descriptors of the three tensors, checked before anything launches
eq_status mlp_validate(const eq_rans_tensor *gate, const eq_rans_tensor *up,
                       const eq_rans_tensor *down, uint32_t batch) {
  if (!gate || !up || !down) return EQ_ERR_ARG;
  for (const eq_rans_tensor *t : {gate, up, down}) {
    const eq_status s = validate_rans_tensor(*t);
    if (s != EQ_OK) return s;
  }
  if (batch < 1 || batch > 16) return EQ_ERR_ARG;
  if (gate->rows != up->rows || gate->cols != up->cols || down->cols != gate->rows ||
      down->rows != gate->cols || gate->rows == 0 || gate->cols == 0)
    return EQ_ERR_ARG;
  if (gate->rows % 8) return EQ_ERR_UNSUPPORTED;  // h rows are 16-byte aligned vectors
  return EQ_OK;
}

}  // namespace eq

using namespace eq;

extern "C" size_t eq_mlp_scratch_bytes(uint32_t inter, uint32_t batch) {
  return mlp_scratch_bytes(inter, batch);
}

extern "C" eq_status eq_mlp_decode(const eq_rans_tensor *gate, const eq_rans_tensor *up,
                                   const eq_rans_tensor *down, const uint16_t *d_x, uint32_t batch,
                                   float *d_y, void *d_scratch, size_t scratch_bytes,
                                   uint32_t *d_status, void *stream) {
  eq_status s = mlp_validate(gate, up, down, batch);
  if (s != EQ_OK) return s;
  if (!d_x || !d_y || !d_status || !d_scratch || !aligned(d_scratch, 256)) return EQ_ERR_ARG;
  const uint64_t inter = gate->rows;
  if (scratch_bytes < mlp_scratch_bytes(inter, batch)) return EQ_ERR_ARG;
  unsigned char *p = static_cast<unsigned char *>(d_scratch);
  float *g = reinterpret_cast<float *>(p);
  float *u = reinterpret_cast<float *>(p + align256(inter * batch * 4));
  uint16_t *h = reinterpret_cast<uint16_t *>(p + 2 * align256(inter * batch * 4));
  return mlp_run(gate, up, down, d_x, batch, d_y, g, u, h, d_status, stream);
}
