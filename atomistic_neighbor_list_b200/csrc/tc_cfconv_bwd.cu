// Tensor-core (tcgen05 / TMEM) fused cfconv backward for the bf16 path, F = 128 (the kernel is the
// warp-specialised one of tc_cfconv_bwd_ws.cu): the gradient with respect to the block input h and
// the block's contribution to the forces, in one pass over the
// symmetric CSR (FlashSchNet page, technical summary s.2.3: the backward reduces by source; on a
// symmetric cutoff graph the edges of source k are the edges of row k, so every output row is
// again written once, with no atomics).
//
// For each row k and edge j of row k (d = |r_k - r_j|, e the Gaussian row, e' = de/dd):
//   z1 = e . A1ext, t = e' . A1                                      (MMA1, two accumulators)
//   Q = sigmoid(z1) (.) t  ->  v = Q . A2                            (MMA2b)
//   P = ssp(z1)            ->  u = P . A2                            (MMA2a)
//   W = f_c (u + c2),   W' = dW/dd = f_c' (u + c2) + f_c v            (filter and its d-derivative)
//   grad_h[k] += g_j (.) W                                           (MMA3 segment sum, 0/1 matrix)
//   s_kj = sum_f (g_k h_j + g_j h_k)_f W'_f                          (in registers, per edge)
//   forces[k] -= sum_j s_kj (r_k - r_j) / d                          (per-row sum in shared memory)
// The filter is recomputed instead of stored (no edge-sized tensor).
#include "tc_common.cuh"

namespace mp {

bool tc_bwd_supported(const mp_ctx* ctx) { return tc_supported(ctx); }

int tc_cfconv_bwd(mp_ctx* ctx, int block, int N, long long E, const float* pos, const int* row_ptr,
                  const int* col_idx, const void* h, const void* g, float* grad_h, float* forces,
                  bool accumulate, cudaStream_t s) {
  return tc_cfconv_bwd_ws(ctx, block, N, E, pos, row_ptr, col_idx, h, g, grad_h, forces, accumulate,
                          s);
}

}  // namespace mp
