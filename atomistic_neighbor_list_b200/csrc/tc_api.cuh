// Interface of the tensor-core (tcgen05 / TMEM) kernels of tc_cfconv.cu.
#pragma once
#include "mp_internal.cuh"

namespace mp {
// True when the context's configuration runs on the tensor-core kernels (bf16, F = 128).
bool tc_supported(const mp_ctx* ctx);
// True when the fused backward also runs on the tensor-core kernel.
bool tc_bwd_supported(const mp_ctx* ctx);
// Build the packed 16-bit operand images of the filter weights (called once by mp_init).
int tc_prepare(mp_ctx* ctx, cudaStream_t s);
int tc_cfconv_fwd(mp_ctx* ctx, int block, int N, long long E, const float* pos, const int* row_ptr,
                  const int* col_idx, const void* x, void* out, cudaStream_t s);
int tc_cfconv_bwd(mp_ctx* ctx, int block, int N, long long E, const float* pos, const int* row_ptr,
                  const int* col_idx, const void* h, const void* g, float* grad_h, float* forces,
                  bool accumulate, cudaStream_t s);
}  // namespace mp
