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
__host__ __device__ constexpr Smem smem_layout(int K1) {
  return Smem{0u,
              (uint32_t)(FT * K1 * 2),
              (uint32_t)(FT * K1 * 2 + FT * K2 * 2),
              (uint32_t)(FT * K1 * 2 + FT * K2 * 2 +
                         (TM * K1 * 2 > SLOT_PASS * TM * 2 ? TM * K1 * 2 : SLOT_PASS * TM * 2)),
              (uint32_t)(FT * K1 * 2 + FT * K2 * 2 +
                         (TM * K1 * 2 > SLOT_PASS * TM * 2 ? TM * K1 * 2 : SLOT_PASS * TM * 2) +
                         TM * K2 * 2),
              (uint32_t)(FT * K1 * 2 + FT * K2 * 2 +
                         (TM * K1 * 2 > SLOT_PASS * TM * 2 ? TM * K1 * 2 : SLOT_PASS * TM * 2) +
                         TM * K2 * 2 + FT * 4),
              (uint32_t)(FT * K1 * 2 + FT * K2 * 2 +
                         (TM * K1 * 2 > SLOT_PASS * TM * 2 ? TM * K1 * 2 : SLOT_PASS * TM * 2) +
                         TM * K2 * 2 + FT * 4 + 7 * TM * 4 + 128)};
}

// Destination row of edge g: the largest r with row_ptr[r] <= g. s_rp caches row_ptr[r_lo + i],
// i = 0..TM (clamped at r_end); edges beyond the window fall back to a search in global memory.
__device__ __forceinline__ int dst_of(const int* __restrict__ s_rp, int r_lo, int r_end,
                                      const int* __restrict__ row_ptr, long long g) {
  if ((long long)s_rp[TM] <= g) return row_of(row_ptr, r_lo + TM, r_end, g);
  int lo = 0, hi = TM;  // s_rp[lo] <= g < s_rp[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((long long)s_rp[mid] <= g) lo = mid; else hi = mid;
  }
  return r_lo + lo;
}

template <int K1>
__global__ void __launch_bounds__(THREADS, 2) k_cfconv_fwd_tc(
    int N, long long E, const float* __restrict__ pos, const int* __restrict__ row_ptr,
    const int* __restrict__ col_idx, const __nv_bfloat16* __restrict__ x,
    __nv_bfloat16* __restrict__ out, const uint8_t* __restrict__ img, Radial rp, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr Smem L = smem_layout(K1);
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
  int* s_rp = s_slot_row + TM;                   // TM + 1 used (2 TM reserved)
  int* s_wsum = s_rp + 2 * TM;                   // 8
  int* s_misc = s_wsum + 8;                      // 8: nslots, -, r_begin, r_end, next r_lo
  uint64_t* s_mbar = (uint64_t*)(s_misc + 8);    // [0] MMA completion, [1] weight copy
  uint32_t* s_tmem = (uint32_t*)(s_mbar + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;

  // ---- this CTA's destination rows: those whose first edge lies in [E c / G, E (c+1) / G)
  E = clamp_off(row_ptr[N], E);  // the edges the list holds (E may be an upper bound of them)
  if (tid == 0) {
    const long long b_lo = E * cta / G, b_hi = E * (cta + 1) / G;
    const int r0 = lower_row(row_ptr, N, b_lo);
    const int r1 = (cta == G - 1) ? N : lower_row(row_ptr, N, b_hi);
    s_misc[2] = r0;
    s_misc[3] = r1 > r0 ? r1 : r0;
    s_misc[4] = r0;
  }
  __syncthreads();
  const int r_begin = s_misc[2], r_end = s_misc[3];
  if (r_begin >= r_end) return;
  long long e_begin = clamp_off(row_ptr[r_begin], E);
  long long e_end = clamp_off(row_ptr[r_end], E);
  if (e_end < e_begin) e_end = e_begin;

  // ---- setup: TMEM (128 columns), mbarriers, weights into shared memory by one bulk copy each
  if (warp == 0) tc::tmem_alloc(s_tmem, 128);
  if (tid == 0) {
    tc::mbar_init(&s_mbar[0], 1);
    tc::mbar_init(&s_mbar[1], 1);
    const ImgLayout IL = img_layout(K1);
    tc::mbar_expect_tx(&s_mbar[1], FT * K1 * 2 + FT * K2 * 2 + FT * 4);
    tc::bulk_g2s(sW1, img + IL.w1, FT * K1 * 2, &s_mbar[1]);
    tc::bulk_g2s(sW2, img + IL.w2, FT * K2 * 2, &s_mbar[1]);
    tc::bulk_g2s(sc2, img + IL.c2, FT * 4, &s_mbar[1]);
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t idesc_fc = tc::idesc(TM, FT, 1, false, false);
  uint32_t phase = 0;
  bool aborted = __syncthreads_or(tc::mbar_wait(&s_mbar[1], 0, WAIT_LIMIT) ? 0 : 1) != 0;

  // drain state (threads 0..127: feature f = tid)
  float carry = 0.f;
  int carry_row = -1;
  int next_row = r_begin;

  auto wait_mma = [&]() -> bool {
    const int bad = tc::mbar_wait(&s_mbar[0], phase, WAIT_LIMIT) ? 0 : 1;
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
  const int q4 = warp & 3, half = warp >> 2;
  const int e_me = 32 * q4 + lane;  // this thread's edge (TMEM lane) in every phase below
  const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);

  for (long long tb = e_begin; tb < e_end && !aborted; tb += TM) {
    const int ne = (int)((e_end - tb) < TM ? (e_end - tb) : TM);
    const int r_lo = s_misc[4];
    // ------------------------------------------------------------------ row window
    for (int i = tid; i <= TM; i += THREADS) s_rp[i] = row_ptr[min(r_lo + i, r_end)];
    __syncthreads();
    // ------------------------------------------------------------------ prep (all warps)
    int my_dst = -1;
    {
      const int t = e_me;
      float fc = 0.f, d = 0.f;
      int j = 0;
      bool ok = false;
      if (t < ne) {
        const long long g = tb + t;
        my_dst = dst_of(s_rp, r_lo, r_end, row_ptr, g);
        j = col_idx[g];
        if ((unsigned)j < (unsigned)N) {
          const float dx = pos[3 * my_dst] - pos[3 * j], dy = pos[3 * my_dst + 1] - pos[3 * j + 1],
                      dz = pos[3 * my_dst + 2] - pos[3 * j + 2];
          d = sqrtf(dx * dx + dy * dy + dz * dz);
          fc = cutoff_f(d, rp.r_c);
          ok = true;
        } else {
          if (half == 0) raise_status(status, kStatusBounds);
          j = 0;
        }
      }
      if (half == 0) {
        s_src[t] = j;
        s_dst[t] = my_dst;
        s_fc[t] = fc;
      }
      // Gaussian row (bf16), bias column R = 1, zero padding; each half writes K1/2 columns
      const float d0 = d - rp.mu_min;
#pragma unroll
      for (int c = 0; c < K1 / 16; ++c) {
        const int k0 = half * (K1 / 2) + 8 * c;
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float v[2];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int k = k0 + 2 * q + hh;
            const float dd = fmaf(-(float)k, rp.dmu, d0);
            float val = tc::ex2f(nglog2e * dd * dd);
            val = k < rp.R ? val : (k == rp.R ? 1.f : 0.f);
            v[hh] = ok ? val : 0.f;
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
      incl = __popc(b & ((2u << lane) - 1u));
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
      if (t == ne - 1) s_misc[4] = my_dst;  // the next tile starts in this row or later
    }
    // ------------------------------------------------------------------ MMA1
    if (tid == 0) {
      tc::fence_after();
      for (int ks = 0; ks < K1 / 16; ++ks)
        tc::mma(tmem, tc::sdesc(sAe_a + ks * 256, 128, K1 * 16),
                tc::sdesc(sW1_a + ks * 256, 128, K1 * 16), idesc_fc, ks > 0);
      tc::commit(&s_mbar[0]);
    }
    if (!wait_mma()) {
      aborted = true;
      break;
    }
    const int nslots = s_misc[0];
    // ------------------------------------------------------------------ epilogue 1
    const float fc_me = s_fc[e_me];
    {
      const float fcln2 = fc_me * LN2;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int f0 = 64 * half + 32 * c;
        uint32_t r[32];
        tc::ld32(lane_base + f0, r);
        tc::ld_wait();
#pragma unroll
        for (int g8 = 0; g8 < 4; ++g8) {
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float a = ssp_scaled(__uint_as_float(r[8 * g8 + 2 * q]), fc_me, fcln2);
            const float b = ssp_scaled(__uint_as_float(r[8 * g8 + 2 * q + 1]), fc_me, fcln2);
            w[q] = tc::pack_bf16(a, b);
          }
          *(uint4*)(sH + kmaj(e_me, f0 + 8 * g8, K2)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
    // this thread's half-row of x_j, loaded while the second MMA runs
    uint4 xv[8];
    {
      const uint4* xr = (const uint4*)(x + (size_t)s_src[e_me] * FT) + 8 * half;
#pragma unroll
      for (int q = 0; q < 8; ++q) xv[q] = __ldg(xr + q);
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
      tc::commit(&s_mbar[0]);
    }
    if (!wait_mma()) {
      aborted = true;
      break;
    }
    // ------------------------------------------------------------------ epilogue 2
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int f0 = 64 * half + 32 * c;
      uint32_t r[32];
      tc::ld32(lane_base + f0, r);
      tc::ld_wait();
#pragma unroll
      for (int g8 = 0; g8 < 4; ++g8) {
        const uint4 xq = xv[4 * c + g8];
        const uint32_t xw[4] = {xq.x, xq.y, xq.z, xq.w};
        const int f8 = f0 + 8 * g8;
        const float4 ca = *(const float4*)(sc2 + f8);
        const float4 cb = *(const float4*)(sc2 + f8 + 4);
        const float cc[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float W0 = fmaf(fc_me, cc[2 * q], __uint_as_float(r[8 * g8 + 2 * q]));
          const float W1 = fmaf(fc_me, cc[2 * q + 1], __uint_as_float(r[8 * g8 + 2 * q + 1]));
          w[q] = tc::pack_bf16(W0 * bf_lo(xw[q]), W1 * bf_hi(xw[q]));
        }
        // msg^T, MN-major: (f, e) at (f/8)*2048 + (e/8)*128 + (e%8)*16 + (f%8)*2
        *(uint4*)(sH + (f8 >> 3) * 2048 + (e_me >> 3) * 128 + (e_me & 7) * 16) =
            make_uint4(w[0], w[1], w[2], w[3]);
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
        tc::commit(&s_mbar[0]);
      }
      if (!wait_mma()) {
        aborted = true;
        break;
      }
    }
    if (aborted) break;
    // ------------------------------------------------------------------ drain
    if (tid < TM) {
      for (int c0 = 0; c0 < nslots; c0 += 16) {
        uint32_t r[16];
        tc::ld16(tmem + ((uint32_t)(32 * warp) << 16) + c0, r);
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
      tc::mbar_wait(&s_mbar[0], phase ^ 1u, WAIT_LIMIT);  // let an MMA still in flight finish
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

int tc_cfconv_fwd_sequential(mp_ctx* ctx, int block, int N, long long E, const float* pos,
                             const int* row_ptr, const int* col_idx, const void* x, void* out,
                             cudaStream_t s) {
  const int K1 = k1_of(ctx->cfg.n_rbf);
  const ImgLayout IL = img_layout(K1);
  const uint8_t* img = (const uint8_t*)ctx->tc_weights + IL.bytes * block;
  long long tiles = (E + TM - 1) / TM;
  int grid = 2 * ctx->num_sms;
  if (tiles < grid) grid = (int)(tiles > 0 ? tiles : 1);
  auto go = [&](auto kern, int k1) {
    const size_t smem = smem_layout(k1).total + 1024;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return launch(ctx, K_CFCONV_FWD_TC_LS, kern, dim3(grid), dim3(THREADS), smem, s, N, E, pos,
                  row_ptr, col_idx, (const __nv_bfloat16*)x, (__nv_bfloat16*)out, img,
                  radial_of(ctx), ctx->status_d);
  };
  if (K1 == 64) return go(k_cfconv_fwd_tc<64>, 64);
  if (K1 == 80) return go(k_cfconv_fwd_tc<80>, 80);
  if (K1 == 48) return go(k_cfconv_fwd_tc<48>, 48);
  if (K1 == 32) return go(k_cfconv_fwd_tc<32>, 32);
  return MP_ERR_INVALID_ARG;
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
