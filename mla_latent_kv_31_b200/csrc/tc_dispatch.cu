// Which ops take the tensor-core kernels in this build.
#include <cuda_runtime.h>

#include "tc.cuh"

namespace mla {

bool tc_available(mla_op_t op) {
  (void)op;
  return false;
}

size_t tc_decode_scratch_bytes(int64_t B, int32_t tq) {
  (void)B; (void)tq;
  return 0;
}

cudaError_t tc_cache_append(const mla_dims_t&, const mla_weights_t&, const void*, const int64_t*, const int64_t*,
                            int64_t, void*, int64_t, uint32_t*, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t tc_latent_core(const mla_dims_t&, const void*, const void*, int64_t, int32_t, const int64_t*,
                           const void*, int64_t, void*, bool, float*, void*, int, uint32_t*, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t tc_decode(const mla_dims_t&, const mla_weights_t&, const void*, int64_t, int32_t, const int64_t*,
                      const int64_t*, const void*, int64_t, void*, void*, void*, void*, void*, void*, void*,
                      float*, void*, int, uint32_t*, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t tc_prefill(const mla_dims_t&, const mla_weights_t&, const void*, int64_t, const int64_t*, int64_t,
                       int64_t, const int64_t*, void*, int64_t, void*, void*, void*, void*, void*, void*, void*,
                       uint32_t*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace mla
