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
// Warp-specialised pipelined variant of tc_cfconv_fwd (tc_cfconv_ws.cu).
int tc_cfconv_fwd_ws(mp_ctx* ctx, int block, int N, long long E, const float* pos,
                     const int* row_ptr, const int* col_idx, const void* x, void* out,
                     cudaStream_t s);
// Warp-specialised pipelined variant of tc_cfconv_bwd (tc_cfconv_bwd_ws.cu).
int tc_cfconv_bwd_ws(mp_ctx* ctx, int block, int N, long long E, const float* pos,
                     const int* row_ptr, const int* col_idx, const void* h, const void* g,
                     float* grad_h, float* forces, bool accumulate, cudaStream_t s);
int tc_cfconv_bwd(mp_ctx* ctx, int block, int N, long long E, const float* pos, const int* row_ptr,
                  const int* col_idx, const void* h, const void* g, float* grad_h, float* forces,
                  bool accumulate, cudaStream_t s);
// Neighbor attention on the tensor cores (tc_attn.cu): 16 heads of 8, K a multiple of 128, x
// 16-byte aligned; q (fp32 [N][F]) and k (fp16 [N][F], attn_project with k_f16) must already be in
// ctx->q, ctx->k.
bool tc_attn_supported(const mp_ctx* ctx, int K);
int tc_attn_fwd(mp_ctx* ctx, int N, int K, const float* pos, const int* nbr,
                const unsigned char* mask, const void* x, void* out, cudaStream_t s);
// The attention with the equivariant value path (9 solid harmonics, out [N][9][F]) on the same
// tensor-core kernel, one weighted-sum MMA per harmonic (tc_attn.cu).
bool tc_attn_eq_supported(const mp_ctx* ctx, int K);
int tc_attn_eq_fwd(mp_ctx* ctx, int N, int K, const float* pos, const int* nbr,
                   const unsigned char* mask, const void* x, void* out, cudaStream_t s);
// Destination pass of the attention backward on the tensor cores (tc_attn_bwd.cu): writes dL/dq
// (scaled) into gq, the row side of dL/dr into grad_pos, and the rows' softmax statistics.
bool tc_attn_bwd_supported(const mp_ctx* ctx, int K);
int tc_attn_bwd_dst(mp_ctx* ctx, int N, int K, const float* pos, const int* nbr,
                    const unsigned char* mask, const void* x, const float* g, float* gq,
                    float* grad_pos, cudaStream_t s);
// Its source pass (needs the destination pass's statistics): writes the value path of dL/dx
// into grad_x, dL/dk into gk, and adds the source side of dL/dr to grad_pos.
int tc_attn_bwd_src(mp_ctx* ctx, int N, int K, const float* pos, const int* rev_ptr,
                    const int* rev, const void* x, const float* g, float* grad_x, float* gk,
                    float* grad_pos, cudaStream_t s);
// Atomwise layer on the tensor cores: out = in . W + b over rows (see tc_dense.cu for the modes).
enum { TC_DENSE_STORE = 0, TC_DENSE_RESIDUAL = 1, TC_DENSE_READOUT = 2, TC_DENSE_STORE_F16 = 3 };
size_t tc_dense_bytes(int n_blocks);
int tc_dense_pack(const float* W, int rows, int cols, bool transpose, uint8_t* dst);
int tc_dense(mp_ctx* ctx, int N, int Kin, int Nout, const void* in, bool in_bf16,
             const uint8_t* wimg, const float* bias, void* out, bool out_bf16, int mode,
             cudaStream_t s);
// Two dependent atomwise layers per 128-row tile (see tc_dense.cu): the first (STORE or RESIDUAL
// into the fp32 out1), then the updated row through W2 (STORE as bf16 with N2 = 128, or READOUT
// with N2 = 64).
int tc_dense2(mp_ctx* ctx, int N, int K1, const void* in1, bool in1_bf16, const uint8_t* w1,
              const float* b1, float* out1, int mode1, const uint8_t* w2, const float* b2, int N2,
              void* out2, int mode2, cudaStream_t s);
// Offsets of the packed dense images inside ctx->tc_dense_img.
inline size_t tc_dense_off(int kind, int block, int n_blocks) {
  // kind: 0 W_in, 1 W_out, 2 W_out^T, 3 W_in^T (per block), 4 B1, 5 B1^T, 6 Wq, 7 Wk
  const size_t sq = (size_t)128 * 128 * 2;
  if (kind < 4) return ((size_t)block * 4 + kind) * sq;
  if (kind >= 6) return ((size_t)n_blocks * 4 + 1 + (kind - 6)) * sq;
  return (size_t)n_blocks * 4 * sq + (kind == 4 ? 0 : sq / 2);
}
// The attention's query and key rows q = x Wq, k = x Wk (fp32 [N][F] in ctx->q, ctx->k): on the
// tensor cores when the context holds their packed images (bf16 path, F = 128), else on the CUDA
// cores (tc_dense.cu). k_f16: k stored as fp16 [N][F] instead (the tensor-core attention forward's
// operand; needs the tensor-core projection).
int attn_project(mp_ctx* ctx, int N, const void* x, cudaStream_t s, bool k_f16 = false);
}  // namespace mp
