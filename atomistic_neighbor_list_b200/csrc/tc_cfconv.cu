// Tensor-core (tcgen05 / TMEM) fused cfconv for the bf16 path, F = 128: the packed operand images of
// the filter weights, the dispatch, and a layout self-check of the MMA building blocks. The kernel
// is the warp-specialised one of tc_cfconv_ws.cu.
//
// The arithmetic of one tile (FlashSchNet page, technical summary s.2.1-2.4, restated for sm_100a).
// A persistent CTA owns a contiguous range of destination rows (balanced by edge count) and streams
// its edges in CSR order, 128 at a time (one MMA M-tile):
//   prep   distance, cosine envelope f_c and the Gaussian basis of each edge, written once as the
//          bf16 A operand [edge][k] (a constant-1 column folds the first-layer bias c1)   (s.2.1)
//   MMA1   z1 = e . A1ext                     -> TMEM (fp32)                               (s.2.4)
//   epi-1  h' = f_c * ssp(z1)                 -> bf16 A operand (shared memory)
//   MMA2   u = h' . A2                        -> TMEM; W = u + f_c c2 = f_c (ssp(z1) A2 + c2)
//   epi-2  msg = x_j (.) W (x_j gathered from global memory, L2-resident) -> bf16, stored MN-major
//   MMA3   the segment sum on the tensor core: D^T[f][row] = sum_e msg[e][f] S[e][row], with S the
//          0/1 edge-to-row matrix of the tile                                            (s.2.3)
//   drain  one thread per feature reads its TMEM lane and writes each finished row once; a row cut
//          by the tile boundary is carried in registers to the next tile. No atomics, no edge-sized
//          tensor in global memory                                                      (s.2.2)
#include <cstring>
#include <vector>

#include "tc_common.cuh"

namespace mp {
// ---------------------------------------------------------------------------------------------
using namespace tcc;

bool tc_supported(const mp_ctx* ctx) {
  // the tensor-core kernels are built for Gaussian operands of 32 to 80 columns (n_rbf 16 to 64);
  // fewer radial functions run on the CUDA-core kernels
  return ctx->cfg.dtype == MP_BF16 && ctx->cfg.F == FT && ctx->tc_weights != nullptr &&
         k1_of(ctx->cfg.n_rbf) >= 32 && k1_of(ctx->cfg.n_rbf) <= 80;
}

int tc_prepare(mp_ctx* ctx, cudaStream_t s) {
  const mp_config& c = ctx->cfg;
  if (c.dtype != MP_BF16 || c.F != FT) return MP_OK;
  const int R = c.n_rbf, K1 = k1_of(R), B = c.n_blocks;
  const ImgLayout IL = img_layout(K1);
  std::vector<uint8_t> host(IL.bytes * B, 0);
  std::vector<float> A1((size_t)R * FT), c1(FT), A2((size_t)FT * FT), c2(FT);
  auto bf16_bits = [](float v) -> uint16_t {  // values are already bf16-rounded: truncate exactly
    uint32_t u;
    std::memcpy(&u, &v, 4);
    return (uint16_t)(u >> 16);
  };
  for (int b = 0; b < B; ++b) {
    if (cudaMemcpy(A1.data(), ctx->A1[b], A1.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(c1.data(), ctx->c1[b], FT * 4, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(A2.data(), ctx->A2[b], A2.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(c2.data(), ctx->c2[b], FT * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
      return MP_ERR_CUDA;
    uint8_t* base = host.data() + IL.bytes * b;
    for (int f = 0; f < FT; ++f) {
      for (int k = 0; k < K1; ++k) {
        float v = k < R ? A1[(size_t)k * FT + f] : (k == R ? c1[f] : 0.f);
        const uint16_t bits = bf16_bits(v);
        std::memcpy(base + IL.w1 + kmaj(f, k, K1), &bits, 2);
      }
      for (int g = 0; g < K2; ++g) {
        const uint16_t bits = bf16_bits(A2[(size_t)g * FT + f]);
        std::memcpy(base + IL.w2 + kmaj(f, g, K2), &bits, 2);
      }
    }
    std::memcpy(base + IL.c2, c2.data(), FT * 4);
  }
  // atomwise layers: W_in, W_out, W_out^T, W_in^T per block, then B1 and B1^T
  {
    std::vector<uint8_t> dimg(tc_dense_bytes(B), 0);
    std::vector<float> Wi((size_t)FT * FT), Wo((size_t)FT * FT), B1((size_t)FT * (FT / 2));
    for (int b = 0; b < B; ++b) {
      if (cudaMemcpy(Wi.data(), ctx->W_in[b], Wi.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess ||
          cudaMemcpy(Wo.data(), ctx->W_out[b], Wo.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
        return MP_ERR_CUDA;
      tc_dense_pack(Wi.data(), FT, FT, false, dimg.data() + tc_dense_off(0, b, B));
      tc_dense_pack(Wo.data(), FT, FT, false, dimg.data() + tc_dense_off(1, b, B));
      tc_dense_pack(Wo.data(), FT, FT, true, dimg.data() + tc_dense_off(2, b, B));
      tc_dense_pack(Wi.data(), FT, FT, true, dimg.data() + tc_dense_off(3, b, B));
    }
    if (cudaMemcpy(B1.data(), ctx->B1, B1.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
      return MP_ERR_CUDA;
    tc_dense_pack(B1.data(), FT, FT / 2, false, dimg.data() + tc_dense_off(4, 0, B));
    tc_dense_pack(B1.data(), FT, FT / 2, true, dimg.data() + tc_dense_off(5, 0, B));
    if (c.n_heads > 0 && ctx->Wq && ctx->Wk) {  // the attention's query and key projections
      if (cudaMemcpy(Wi.data(), ctx->Wq, Wi.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess ||
          cudaMemcpy(Wo.data(), ctx->Wk, Wo.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
        return MP_ERR_CUDA;
      tc_dense_pack(Wi.data(), FT, FT, false, dimg.data() + tc_dense_off(6, 0, B));
      tc_dense_pack(Wo.data(), FT, FT, false, dimg.data() + tc_dense_off(7, 0, B));
      ctx->tc_qk = true;
    }
    if (cudaMalloc(&ctx->tc_dense_img, dimg.size()) != cudaSuccess) return MP_ERR_CUDA;
    if (cudaMemcpy(ctx->tc_dense_img, dimg.data(), dimg.size(), cudaMemcpyHostToDevice) != cudaSuccess)
      return MP_ERR_CUDA;
  }
  // attention (16 heads of 8): B rows 128..143 of its first MMA, P^T with the bias p on column R
  if (c.n_heads == 16 && c.head_dim == 8 && ctx->P && ctx->p) {
    const int H = c.n_heads;
    std::vector<float> P((size_t)R * H), pb(H);
    if (cudaMemcpy(P.data(), ctx->P, P.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(pb.data(), ctx->p, H * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
      return MP_ERR_CUDA;
    std::vector<uint8_t> pimg((size_t)H * K1 * 2, 0);
    for (int h = 0; h < H; ++h)
      for (int k = 0; k < K1; ++k) {
        const float v = k < R ? P[(size_t)k * H + h] : (k == R ? pb[h] : 0.f);
        const uint16_t bits = bf16_bits(v);
        std::memcpy(pimg.data() + kmaj(h, k, K1), &bits, 2);
      }
    if (cudaMalloc(&ctx->tc_attn_p, pimg.size()) != cudaSuccess ||
        cudaMemcpy(ctx->tc_attn_p, pimg.data(), pimg.size(), cudaMemcpyHostToDevice) != cudaSuccess)
      return MP_ERR_CUDA;
  }
  if (cudaMalloc(&ctx->tc_weights, host.size()) != cudaSuccess) return MP_ERR_CUDA;
  ctx->tc_weights_bytes = host.size();
  if (cudaMemcpyAsync(ctx->tc_weights, host.data(), host.size(), cudaMemcpyHostToDevice, s) !=
      cudaSuccess)
    return MP_ERR_CUDA;
  return cudaStreamSynchronize(s) == cudaSuccess ? MP_OK : MP_ERR_CUDA;
}

int tc_cfconv_fwd(mp_ctx* ctx, int block, int N, long long E, const float* pos, const int* row_ptr,
                  const int* col_idx, const void* x, void* out, cudaStream_t s) {
  return tc_cfconv_fwd_ws(ctx, block, N, E, pos, row_ptr, col_idx, x, out, s);
}

}  // namespace mp

// ---------------------------------------------------------------------------------------------
// Layout self-check of the tensor-core building blocks, on small-integer matrices whose products
// are exact in fp32: (1) K-major A [128 x 64] times K-major B [128 x 64], N = 128, the layout of
// MMA1/MMA2; (2) MN-major A [128 x 128] times K-major B [16 x 128], N = 16, the layout of the
// segment-sum MMA. Each thread checks one output row against a direct sum.
namespace mp {
namespace {
using namespace tcc;

__device__ __forceinline__ float st_a1(int m, int k) { return (float)(((m * 7 + k * 3) % 9) - 4); }
__device__ __forceinline__ float st_b1(int n, int k) { return (float)(((n * 5 + k) % 7) - 3); }
__device__ __forceinline__ float st_a2(int m, int k) { return (float)(((m + 3 * k) % 5) - 2); }
__device__ __forceinline__ float st_b2(int n, int k) { return (float)(((n * 3 + k * 7) % 4) - 1); }

__global__ void __launch_bounds__(128) k_selftest_tc(int* mismatches) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = sm;               // 128 x 128 x 2 = 32 KB (test 1 uses the first 16 KB)
  uint8_t* sB = sm + 32768;       // 128 x 64 x 2 = 16 KB
  __shared__ uint64_t mbar;
  __shared__ uint32_t tslot;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (warp == 0) tc::tmem_alloc(&tslot, 128);
  if (tid == 0) tc::mbar_init(&mbar, 1);
  // test 1 operands
  for (int k = 0; k < 64; ++k) {
    *(__nv_bfloat16*)(sA + kmaj(tid, k, 64)) = __float2bfloat16_rn(st_a1(tid, k));
    *(__nv_bfloat16*)(sB + kmaj(tid, k, 64)) = __float2bfloat16_rn(st_b1(tid, k));
  }
  tc::fence_proxy_async();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = tslot;
  if (tid == 0) {
    for (int ks = 0; ks < 4; ++ks)
      tc::mma(tmem, tc::sdesc(tc::smem_u32(sA) + ks * 256, 128, 1024),
              tc::sdesc(tc::smem_u32(sB) + ks * 256, 128, 1024), tc::idesc(128, 128, 1, false, false),
              ks > 0);
    tc::commit(&mbar);
  }
  int bad1 = 0, bad2 = 0;
  const bool ok1 = tc::mbar_wait(&mbar, 0, 1u << 22);
  tc::fence_after();
  if (ok1) {
    for (int c0 = 0; c0 < 128; c0 += 32) {
      uint32_t r[32];
      tc::ld32(tmem + ((uint32_t)(32 * warp) << 16) + c0, r);
      tc::ld_wait();
      for (int i = 0; i < 32; ++i) {
        float ref = 0.f;
        for (int k = 0; k < 64; ++k) ref += st_a1(tid, k) * st_b1(c0 + i, k);
        bad1 += __uint_as_float(r[i]) != ref;
      }
    }
  } else {
    bad1 = -1000000;
  }
  tc::fence_before();
  __syncthreads();
  // test 2 operands: A MN-major (m contiguous), B K-major with 16 rows
  for (int k = 0; k < 128; ++k)
    *(__nv_bfloat16*)(sA + (tid >> 3) * 2048 + (k >> 3) * 128 + (k & 7) * 16 + (tid & 7) * 2) =
        __float2bfloat16_rn(st_a2(tid, k));
  if (tid < 16)
    for (int k = 0; k < 128; ++k)
      *(__nv_bfloat16*)(sB + kmaj(tid, k, 128)) = __float2bfloat16_rn(st_b2(tid, k));
  tc::fence_proxy_async();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (tid == 0 && ok1) {
    for (int ks = 0; ks < 8; ++ks)
      tc::mma(tmem, tc::sdesc(tc::smem_u32(sA) + ks * 256, 128, 2048),
              tc::sdesc(tc::smem_u32(sB) + ks * 256, 128, 2048), tc::idesc(128, 16, 1, true, false),
              ks > 0);
    tc::commit(&mbar);
  }
  const bool ok2 = ok1 && tc::mbar_wait(&mbar, 1, 1u << 22);
  tc::fence_after();
  if (ok2) {
    uint32_t r[16];
    tc::ld16(tmem + ((uint32_t)(32 * warp) << 16), r);
    tc::ld_wait();
    for (int i = 0; i < 16; ++i) {
      float ref = 0.f;
      for (int k = 0; k < 128; ++k) ref += st_a2(tid, k) * st_b2(i, k);
      bad2 += __uint_as_float(r[i]) != ref;
    }
  } else {
    bad2 = -1000000;
  }
  atomicAdd(&mismatches[0], bad1);
  atomicAdd(&mismatches[1], bad2);
  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 128);
  (void)lane;
}

}  // namespace
}  // namespace mp

extern "C" int mp_selftest_tc(int* mismatches) {
  if (!mismatches) return MP_ERR_INVALID_ARG;
  int* d = nullptr;
  if (cudaMalloc(&d, 2 * sizeof(int)) != cudaSuccess) return MP_ERR_CUDA;
  cudaMemset(d, 0, 2 * sizeof(int));
  const size_t smem = 32768 + 32768 + 1024;
  cudaFuncSetAttribute(mp::k_selftest_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  mp::k_selftest_tc<<<1, 128, smem>>>(d);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(mismatches, d, 2 * sizeof(int), cudaMemcpyDeviceToHost);
  cudaFree(d);
  return e == cudaSuccess ? MP_OK : MP_ERR_CUDA;
}
