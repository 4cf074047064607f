// Tensor-core (tcgen05 / TMEM) fused cfconv for the bf16 path, F = 128.
//
// FlashSchNet page, technical summary s.2.1-2.4, restated for sm_100a. A persistent CTA owns a
// contiguous range of destination rows (balanced by edge count) and streams its edges in CSR order,
// 128 at a time (one MMA M-tile):
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
// Two CTAs share an SM (about 100-110 KB of shared memory and 128 TMEM columns each), so one CTA's
// MMAs overlap the other's epilogue.
#include <cstring>
#include <vector>

#include "tc_common.cuh"

namespace mp {
namespace {
using namespace tcc;

constexpr int SLOT_PASS = 64;      // destination rows per segment-sum MMA
constexpr int THREADS = 256;

// Shared-memory carve-up (offsets from a 1024-aligned base).
struct Smem {
  uint32_t w1, w2, ae, h, c2, meta, total;
};
__host__ __device__ inline Smem smem_layout(int K1) {
  Smem s;
  s.w1 = 0;
  s.w2 = s.w1 + FT * K1 * 2;
  s.ae = s.w2 + FT * K2 * 2;
  const uint32_t ae_bytes = (uint32_t)(TM * K1 * 2 > SLOT_PASS * TM * 2 ? TM * K1 * 2
                                                                        : SLOT_PASS * TM * 2);
  s.h = s.ae + ae_bytes;
  s.c2 = s.h + TM * K2 * 2;
  s.meta = s.c2 + FT * 4;
  s.total = s.meta + 6 * TM * 4 + 64;
  return s;
}

__global__ void __launch_bounds__(THREADS, 2) k_cfconv_fwd_tc(
    int N, long long E, const float* __restrict__ pos, const int* __restrict__ row_ptr,
    const int* __restrict__ col_idx, const __nv_bfloat16* __restrict__ x,
    __nv_bfloat16* __restrict__ out, const uint8_t* __restrict__ img, Radial rp, int K1,
    int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const Smem L = smem_layout(K1);
  uint8_t* sW1 = sm + L.w1;
  uint8_t* sW2 = sm + L.w2;
  uint8_t* sAe = sm + L.ae;
  uint8_t* sH = sm + L.h;
  float* sc2 = (float*)(sm + L.c2);
  int* s_src = (int*)(sm + L.meta);
  int* s_dst = s_src + TM;
  float* s_fc = (float*)(s_dst + TM);
  int* s_slot = (int*)(s_fc + TM);
  int* s_slot_row = s_slot + TM;
  int* s_wsum = s_slot_row + TM;                 // 4 warp totals
  int* s_misc = s_wsum + 8;                      // [0] nslots, [1] range rows
  uint64_t* s_mbar = (uint64_t*)(s_misc + 8);
  uint32_t* s_tmem = (uint32_t*)(s_mbar + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;

  // ---- this CTA's destination rows: those whose first edge lies in [E c / G, E (c+1) / G)
  if (tid == 0) {
    const long long b_lo = E * cta / G, b_hi = E * (cta + 1) / G;
    const int r0 = lower_row(row_ptr, N, b_lo);
    const int r1 = (cta == G - 1) ? N : lower_row(row_ptr, N, b_hi);
    s_misc[2] = r0;
    s_misc[3] = r1 > r0 ? r1 : r0;
  }
  __syncthreads();
  const int r_begin = s_misc[2], r_end = s_misc[3];
  if (r_begin >= r_end) return;
  long long e_begin = clamp_off(row_ptr[r_begin], E);
  long long e_end = clamp_off(row_ptr[r_end], E);
  if (e_end < e_begin) e_end = e_begin;

  // ---- setup: TMEM (128 columns), mbarrier, weights into shared memory
  if (warp == 0) tc::tmem_alloc(s_tmem, 128);
  if (tid == 0) tc::mbar_init(s_mbar, 1);
  {
    const ImgLayout IL = img_layout(K1);
    const uint4* g1 = (const uint4*)(img + IL.w1);
    uint4* d1 = (uint4*)sW1;
    for (int i = tid; i < FT * K1 * 2 / 16; i += THREADS) d1[i] = g1[i];
    const uint4* g2 = (const uint4*)(img + IL.w2);
    uint4* d2 = (uint4*)sW2;
    for (int i = tid; i < FT * K2 * 2 / 16; i += THREADS) d2[i] = g2[i];
    const float* gc2 = (const float*)(img + IL.c2);
    for (int i = tid; i < FT; i += THREADS) sc2[i] = gc2[i];
  }
  tc::fence_proxy_async();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t idesc_fc = tc::idesc(TM, FT, 1, false, false);
  uint32_t phase = 0;
  bool aborted = false;

  // drain state (threads 0..127: feature f = tid)
  float carry = 0.f;
  int carry_row = -1;
  int next_row = r_begin;

  auto wait_mma = [&]() -> bool {
    const int bad = tc::mbar_wait(s_mbar, phase, WAIT_LIMIT) ? 0 : 1;
    phase ^= 1u;
    tc::fence_after();
    return __syncthreads_or(bad) == 0;
  };
  auto write_row = [&](int row, float v) {  // called by the 128 drain threads
    for (int rr = next_row; rr < row; ++rr) out[(size_t)rr * FT + tid] = __float2bfloat16_rn(0.f);
    out[(size_t)row * FT + tid] = __float2bfloat16_rn(v);
    next_row = row + 1;
  };

  const uint32_t sAe_a = tc::smem_u32(sAe), sW1_a = tc::smem_u32(sW1);
  const uint32_t sH_a = tc::smem_u32(sH), sW2_a = tc::smem_u32(sW2);
  const float nglog2e = -rp.gamma * LOG2E;

  for (long long tb = e_begin; tb < e_end && !aborted; tb += TM) {
    const int ne = (int)((e_end - tb) < TM ? (e_end - tb) : TM);
    // ------------------------------------------------------------------ prep (warps 0-3)
    int my_dst = -1;
    if (tid < TM) {
      const int t = tid;
      float fc = 0.f, d = 0.f;
      int j = 0;
      bool ok = false;
      if (t < ne) {
        const long long g = tb + t;
        my_dst = row_of(row_ptr, r_begin, r_end, g);
        j = col_idx[g];
        if ((unsigned)j < (unsigned)N) {
          const float dx = pos[3 * my_dst] - pos[3 * j], dy = pos[3 * my_dst + 1] - pos[3 * j + 1],
                      dz = pos[3 * my_dst + 2] - pos[3 * j + 2];
          d = sqrtf(dx * dx + dy * dy + dz * dz);
          fc = cutoff_f(d, rp.r_c);
          ok = true;
        } else {
          raise_status(status, kStatusBounds);
          j = 0;
        }
      }
      s_src[t] = j;
      s_dst[t] = my_dst;
      s_fc[t] = fc;
      // Gaussian row (bf16), bias column R = 1, zero padding
      for (int k0 = 0; k0 < K1; k0 += 8) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float v[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int k = k0 + 2 * q + h;
            float val = 0.f;
            if (ok) {
              if (k < rp.R) {
                const float dd = d - (rp.mu_min + k * rp.dmu);
                val = tc::ex2f(nglog2e * dd * dd);
              } else if (k == rp.R) {
                val = 1.f;
              }
            }
            v[h] = val;
          }
          w[q] = tc::pack_bf16(v[0], v[1]);
        }
        *(uint4*)(sAe + kmaj(t, k0, K1)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    __syncthreads();
    // slots: the edges of one destination row inside the tile share a slot (0, 1, 2, ...)
    bool flag = false;
    int incl = 0;
    if (tid < TM) {
      const int t = tid;
      flag = (t < ne) && (t == 0 || s_dst[t - 1] != my_dst);
      const unsigned b = __ballot_sync(0xffffffffu, flag);
      if (lane == 0) s_wsum[warp] = __popc(b);
      incl = __popc(b & ((2u << lane) - 1u));  // inclusive count of row starts within the warp
    }
    tc::fence_proxy_async();  // the Gaussian rows are read by the tensor core
    __syncthreads();
    if (tid < TM) {
      const int t = tid;
      int off = 0;
      for (int w2 = 0; w2 < warp; ++w2) off += s_wsum[w2];
      const int slot = (t < ne) ? off + incl - 1 : -1;
      if (flag) s_slot_row[slot] = my_dst;
      s_slot[t] = slot;
      if (t == 0) s_misc[0] = s_wsum[0] + s_wsum[1] + s_wsum[2] + s_wsum[3];
    }
    __syncthreads();
    const int nslots = s_misc[0];

    // ------------------------------------------------------------------ MMA1
    if (tid == 0) {
      tc::fence_after();
      for (int ks = 0; ks < K1 / 16; ++ks)
        tc::mma(tmem, tc::sdesc(sAe_a + ks * 256, 128, K1 * 16),
                tc::sdesc(sW1_a + ks * 256, 128, K1 * 16), idesc_fc, ks > 0);
      tc::commit(s_mbar);
    }
    if (!wait_mma()) {
      aborted = true;
      break;
    }
    // ------------------------------------------------------------------ epilogue 1
    {
      const int q4 = warp & 3, half = warp >> 2;
      const int e = 32 * q4 + lane;
      const float fc = s_fc[e], fcln2 = fc * LN2;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int f0 = 64 * half + 32 * c;
        uint32_t r[32];
        tc::ld32(tmem + ((uint32_t)(32 * q4) << 16) + f0, r);
        tc::ld_wait();
#pragma unroll
        for (int g8 = 0; g8 < 4; ++g8) {
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float a = ssp_scaled(__uint_as_float(r[8 * g8 + 2 * q]), fc, fcln2);
            const float b = ssp_scaled(__uint_as_float(r[8 * g8 + 2 * q + 1]), fc, fcln2);
            w[q] = tc::pack_bf16(a, b);
          }
          *(uint4*)(sH + kmaj(e, f0 + 8 * g8, K2)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
    tc::fence_proxy_async();
    tc::fence_before();
    __syncthreads();
    // ------------------------------------------------------------------ MMA2
    if (tid == 0) {
      tc::fence_after();
      for (int ks = 0; ks < K2 / 16; ++ks)
        tc::mma(tmem, tc::sdesc(sH_a + ks * 256, 128, K2 * 16),
                tc::sdesc(sW2_a + ks * 256, 128, K2 * 16), idesc_fc, ks > 0);
      tc::commit(s_mbar);
    }
    if (!wait_mma()) {
      aborted = true;
      break;
    }
    // ------------------------------------------------------------------ epilogue 2
    {
      const int q4 = warp & 3, half = warp >> 2;
      const int e = 32 * q4 + lane;
      const float fc = s_fc[e];
      const uint4* xr = (const uint4*)(x + (size_t)s_src[e] * FT);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int f0 = 64 * half + 32 * c;
        uint32_t r[32];
        tc::ld32(tmem + ((uint32_t)(32 * q4) << 16) + f0, r);
        uint4 xv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) xv[q] = __ldg(xr + (f0 >> 3) + q);
        tc::ld_wait();
#pragma unroll
        for (int g8 = 0; g8 < 4; ++g8) {
          const uint32_t xw[4] = {xv[g8].x, xv[g8].y, xv[g8].z, xv[g8].w};
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int f = f0 + 8 * g8 + 2 * q;
            const float W0 = fmaf(fc, sc2[f], __uint_as_float(r[8 * g8 + 2 * q]));
            const float W1 = fmaf(fc, sc2[f + 1], __uint_as_float(r[8 * g8 + 2 * q + 1]));
            w[q] = tc::pack_bf16(W0 * bf_lo(xw[q]), W1 * bf_hi(xw[q]));
          }
          // msg^T, MN-major: (f, e) at (f/8)*2048 + (e/8)*128 + (e%8)*16 + (f%8)*2
          const int f8 = f0 + 8 * g8;
          *(uint4*)(sH + (f8 >> 3) * 2048 + (e >> 3) * 128 + (e & 7) * 16) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
    tc::fence_before();
    // ------------------------------------------------------------------ MMA3: segment sum
    for (int p = 0; p * SLOT_PASS < nslots; ++p) {
      const int ns = nslots - p * SLOT_PASS < SLOT_PASS ? nslots - p * SLOT_PASS : SLOT_PASS;
      const int n16 = (ns + 15) & ~15;
      __syncthreads();  // previous users of sAe (MMA1 / previous pass) are done
      {
        uint4* z = (uint4*)sAe;
        for (int i = tid; i < n16 * TM * 2 / 16; i += THREADS) z[i] = make_uint4(0, 0, 0, 0);
      }
      __syncthreads();
      if (tid < TM) {
        const int sl = s_slot[tid] - p * SLOT_PASS;
        if (s_slot[tid] >= 0 && sl >= 0 && sl < ns)
          *(uint16_t*)(sAe + kmaj(sl, tid, TM)) = (uint16_t)0x3F80;  // bf16 1.0
      }
      tc::fence_proxy_async();
      tc::fence_before();
      __syncthreads();
      if (tid == 0) {
        tc::fence_after();
        const uint32_t id3 = tc::idesc(TM, n16, 1, true, false);
        for (int ks = 0; ks < TM / 16; ++ks)
          tc::mma(tmem + p * SLOT_PASS, tc::sdesc(sH_a + ks * 256, 128, 2048),
                  tc::sdesc(sAe_a + ks * 256, 128, TM * 16), id3, ks > 0);
        tc::commit(s_mbar);
      }
      if (!wait_mma()) {
        aborted = true;
        break;
      }
    }
    if (aborted) break;
    // ------------------------------------------------------------------ drain
    if (tid < TM) {
      const int q4 = warp;  // warps 0-3 own TMEM lanes 32*warp .. +31 = features
      for (int c0 = 0; c0 < nslots; c0 += 16) {
        uint32_t r[16];
        tc::ld16(tmem + ((uint32_t)(32 * q4) << 16) + c0, r);
        tc::ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int s = c0 + i;
          if (s < nslots) {
            const int row = s_slot_row[s];
            float v = __uint_as_float(r[i]);
            if (row == carry_row) {
              v += carry;
            } else if (carry_row >= 0) {
              write_row(carry_row, carry);
            }
            carry_row = -1;
            if (s == nslots - 1) {
              carry = v;
              carry_row = row;
            } else {
              write_row(row, v);
            }
          }
        }
      }
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
  }

  if (aborted) {
    if (tid == 0) {
      raise_status(status, kStatusTimeout);
      tc::mbar_wait(s_mbar, phase ^ 1u, WAIT_LIMIT);  // let an MMA still in flight finish
    }
  } else if (tid < TM) {
    if (carry_row >= 0) write_row(carry_row, carry);
    for (int rr = next_row; rr < r_end; ++rr) out[(size_t)rr * FT + tid] = __float2bfloat16_rn(0.f);
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 128);
}

}  // namespace

// ---------------------------------------------------------------------------------------------
using namespace tcc;

bool tc_supported(const mp_ctx* ctx) {
  return ctx->cfg.dtype == MP_BF16 && ctx->cfg.F == FT && ctx->tc_weights != nullptr;
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
  if (cudaMalloc(&ctx->tc_weights, host.size()) != cudaSuccess) return MP_ERR_CUDA;
  ctx->tc_weights_bytes = host.size();
  if (cudaMemcpyAsync(ctx->tc_weights, host.data(), host.size(), cudaMemcpyHostToDevice, s) !=
      cudaSuccess)
    return MP_ERR_CUDA;
  return cudaStreamSynchronize(s) == cudaSuccess ? MP_OK : MP_ERR_CUDA;
}

int tc_cfconv_fwd(mp_ctx* ctx, int block, int N, long long E, const float* pos, const int* row_ptr,
                  const int* col_idx, const void* x, void* out, cudaStream_t s) {
  const int K1 = k1_of(ctx->cfg.n_rbf);
  const Smem L = smem_layout(K1);
  const size_t smem = L.total + 1024;
  auto kern = k_cfconv_fwd_tc;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const ImgLayout IL = img_layout(K1);
  const uint8_t* img = (const uint8_t*)ctx->tc_weights + IL.bytes * block;
  long long tiles = (E + TM - 1) / TM;
  int grid = 2 * ctx->num_sms;
  if (tiles < grid) grid = (int)(tiles > 0 ? tiles : 1);
  return launch(ctx, K_CFCONV_FWD_TC, kern, dim3(grid), dim3(THREADS), smem, s, N, E, pos, row_ptr,
                col_idx, (const __nv_bfloat16*)x, (__nv_bfloat16*)out, img, radial_of(ctx), K1,
                ctx->status_d);
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
