// Entry points not built yet: they report EQ_ERR_UNSUPPORTED.
#include "eq_internal.cuh"

extern "C" eq_status eq_decode_gemv(const eq_rans_tensor *, const uint16_t *, uint32_t, float *,
                                    uint32_t *, void *) {
  return EQ_ERR_UNSUPPORTED;
}
