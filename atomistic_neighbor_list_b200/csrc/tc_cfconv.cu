// Tensor-core path (tcgen05 / TMEM): not enabled yet; every configuration runs the SIMT kernels.
#include "tc_api.cuh"

namespace mp {
bool tc_supported(const mp_ctx*) { return false; }
int tc_prepare(mp_ctx*, cudaStream_t) { return MP_OK; }
int tc_cfconv_fwd(mp_ctx*, int, int, long long, const float*, const int*, const int*, const void*,
                  void*, cudaStream_t) {
  return MP_ERR_UNIMPLEMENTED;
}
int tc_cfconv_bwd(mp_ctx*, int, int, long long, const float*, const int*, const int*, const void*,
                  const void*, float*, float*, bool, cudaStream_t) {
  return MP_ERR_UNIMPLEMENTED;
}
}  // namespace mp
