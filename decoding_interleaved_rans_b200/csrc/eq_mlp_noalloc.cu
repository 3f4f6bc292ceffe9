// eq_mlp_decode_noalloc: eq_mlp_decode for callers that cannot allocate device memory.
//
// Some callers can hand this library no scratch buffer: a serving engine or framework that has
// reserved (nearly) all of HBM for its own allocator up front, so that a cudaMalloc from here
// would fail or eat into its pool, and hot loops that must not pay for cudaMalloc / cudaFree,
// which can synchronise the device.  For them the intermediate vectors of the MLP block (the two
// fp32 products and the bf16 hidden vector) live in one file-scope device array sized for
// EQ_MLP_NOALLOC_MAX_ELEMS = inter x batch elements (5 MiB); the CUDA runtime places it when it
// loads this module on a device, and nothing here calls an allocating routine.
//
// There is one array per device, shared by every call on that device: calls whose work may
// overlap on the GPU (unordered streams) race on it.  Nothing in it needs to start at zero:
// each call writes every element it later reads.
#include "eq_internal.cuh"

namespace eq {

// eq_mlp.cu
eq_status mlp_validate(const eq_rans_tensor *gate, const eq_rans_tensor *up,
                       const eq_rans_tensor *down, uint32_t batch);
size_t mlp_scratch_bytes(uint64_t inter, uint64_t batch);
eq_status mlp_run(const eq_rans_tensor *gate, const eq_rans_tensor *up,
                  const eq_rans_tensor *down, const uint16_t *d_x, uint32_t batch, float *d_y,
                  float *g, float *u, uint16_t *h, uint32_t *d_status, void *stream);

namespace {

constexpr uint64_t round256(uint64_t b) { return (b + 255) & ~uint64_t(255); }

// [g fp32 | u fp32 | h bf16], each part 256-byte aligned, for inter x batch <= the maximum
constexpr uint64_t kNoallocBytes = 2 * round256(uint64_t(EQ_MLP_NOALLOC_MAX_ELEMS) * 4) +
                                   round256(uint64_t(EQ_MLP_NOALLOC_MAX_ELEMS) * 2);

__device__ __align__(256) unsigned char mlp_noalloc_scratch[kNoallocBytes];

// The array's address on the device of the call's stream, which must be the current device
// (the array exists once per device; a stream of another device gets EQ_ERR_ARG).  The address is
// looked up on every call rather than cached: cudaGetSymbolAddress is a host-side lookup that
// allocates nothing, and a fresh lookup stays right when the device's context has been reset and
// the module loaded again at another address.
eq_status scratch_for_stream(cudaStream_t stream, unsigned char **out) {
  int dev = -1, stream_dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return EQ_ERR_CUDA;
  if (cudaStreamGetDevice(stream, &stream_dev) != cudaSuccess) return EQ_ERR_CUDA;
  if (stream_dev != dev) return EQ_ERR_ARG;
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, mlp_noalloc_scratch) != cudaSuccess || !p) return EQ_ERR_CUDA;
  *out = static_cast<unsigned char *>(p);
  return EQ_OK;
}

}  // namespace
}  // namespace eq

using namespace eq;

extern "C" eq_status eq_mlp_decode_noalloc(const eq_rans_tensor *gate, const eq_rans_tensor *up,
                                           const eq_rans_tensor *down, const uint16_t *d_x,
                                           uint32_t batch, float *d_y, uint32_t *d_status,
                                           void *stream) {
  eq_status s = mlp_validate(gate, up, down, batch);
  if (s != EQ_OK) return s;
  if (!d_x || !d_y || !d_status) return EQ_ERR_ARG;
  const uint64_t inter = gate->rows;
  if (inter * batch > EQ_MLP_NOALLOC_MAX_ELEMS) return EQ_ERR_UNSUPPORTED;
  unsigned char *p = nullptr;
  s = scratch_for_stream(static_cast<cudaStream_t>(stream), &p);
  if (s != EQ_OK) return s;
  const uint64_t n = inter * batch;
  float *g = reinterpret_cast<float *>(p);
  float *u = reinterpret_cast<float *>(p + round256(n * 4));
  uint16_t *h = reinterpret_cast<uint16_t *>(p + 2 * round256(n * 4));
  return mlp_run(gate, up, down, d_x, batch, d_y, g, u, h, d_status, stream);
}
