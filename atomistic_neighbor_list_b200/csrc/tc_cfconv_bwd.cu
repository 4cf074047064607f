// Tensor-core (tcgen05 / TMEM) fused cfconv backward for the bf16 path, F = 128: the gradient with
// respect to the block input h and the block's contribution to the forces, in one pass over the
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
// The filter is recomputed instead of stored (no edge-sized tensor). Two CTAs share an SM (256 TMEM
// columns and about 100-110 KB of shared memory each).
#include "tc_common.cuh"

namespace mp {
namespace {
using namespace tcc;

constexpr int THREADS = 256;
constexpr int SLOT_PASS = 32;  // destination rows per segment-sum MMA

struct SmemB {
  uint32_t w1, w2, x, y, c2, meta, total;
};
__host__ __device__ constexpr uint32_t xbytes_b(int K1) {
  return (uint32_t)(2 * TM * K1 * 2 > TM * K2 * 2 ? 2 * TM * K1 * 2 : TM * K2 * 2);
}
__host__ __device__ constexpr SmemB smem_layout_b(int K1) {
  return SmemB{0u, (uint32_t)(FT * K1 * 2), (uint32_t)(FT * K1 * 2 + FT * K2 * 2),
               (uint32_t)(FT * K1 * 2 + FT * K2 * 2) + xbytes_b(K1),
               (uint32_t)(FT * K1 * 2 + FT * K2 * 2) + xbytes_b(K1) + SLOT_PASS * TM * 2,
               (uint32_t)(FT * K1 * 2 + FT * K2 * 2) + xbytes_b(K1) + SLOT_PASS * TM * 2 + FT * 4,
               (uint32_t)(FT * K1 * 2 + FT * K2 * 2) + xbytes_b(K1) + SLOT_PASS * TM * 2 + FT * 4 +
                   9216};
}

__device__ __forceinline__ int dst_of_b(const int* __restrict__ s_rp, int r_lo, int r_end,
                                        const int* __restrict__ row_ptr, long long g) {
  if ((long long)s_rp[TM] <= g) return row_of(row_ptr, r_lo + TM, r_end, g);
  int lo = 0, hi = TM;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((long long)s_rp[mid] <= g) lo = mid; else hi = mid;
  }
  return r_lo + lo;
}

__device__ __forceinline__ float rcpf(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

template <int K1>
__global__ void __launch_bounds__(THREADS, 2) k_cfconv_bwd_tc(
    int N, long long E, const float* __restrict__ pos, const int* __restrict__ row_ptr,
    const int* __restrict__ col_idx, const __nv_bfloat16* __restrict__ hin,
    const __nv_bfloat16* __restrict__ gin, float* __restrict__ grad_h, float* __restrict__ forces,
    int accumulate, const uint8_t* __restrict__ img, Radial rp, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr SmemB L = smem_layout_b(K1);
  uint8_t* sW1 = sm + L.w1;
  uint8_t* sW2 = sm + L.w2;
  uint8_t* sX = sm + L.x;
  uint8_t* sY = sm + L.y;
  float* sc2 = (float*)(sm + L.c2);
  int* s_src = (int*)(sm + L.meta);
  int* s_dst = s_src + TM;
  float* s_fc = (float*)(s_dst + TM);
  float* s_dfc = s_fc + TM;
  float* s_ux = s_dfc + TM;
  float* s_uy = s_ux + TM;
  float* s_uz = s_uy + TM;
  int* s_slot = (int*)(s_uz + TM);
  int* s_slot_row = s_slot + TM;
  int* s_slot_start = s_slot_row + TM;           // TM + 1 used
  float* s_part = (float*)(s_slot_start + TM + 4);  // [2][TM]
  float* s_force = s_part + 2 * TM;              // [TM][3]
  int* s_rp = (int*)(s_force + 3 * TM);          // TM + 1 used (2 TM reserved)
  int* s_wsum = s_rp + 2 * TM;                   // 8
  int* s_misc = s_wsum + 8;                      // 8: nslots, -, r_begin, r_end, next r_lo
  uint64_t* s_mbar = (uint64_t*)(s_misc + 8);    // [0] MMA completion, [1] weight copy
  uint32_t* s_tmem = (uint32_t*)(s_mbar + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
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

  if (warp == 0) tc::tmem_alloc(s_tmem, 256);
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
  const uint32_t idesc_ff = tc::idesc(TM, FT, 1, false, false);
  uint32_t phase = 0;
  bool aborted = __syncthreads_or(tc::mbar_wait(&s_mbar[1], 0, WAIT_LIMIT) ? 0 : 1) != 0;

  float carry = 0.f, fcarry = 0.f;
  int carry_row = -1;
  int next_row = r_begin;

  auto wait_mma = [&]() -> bool {
    const int bad = tc::mbar_wait(&s_mbar[0], phase, WAIT_LIMIT) ? 0 : 1;
    phase ^= 1u;
    tc::fence_after();
    return __syncthreads_or(bad) == 0;
  };
  auto write_row = [&](int row, float v, float fv) {  // drain threads (tid < 128 = feature)
    for (int rr = next_row; rr < row; ++rr) {
      grad_h[(size_t)rr * FT + tid] = 0.f;
      if (tid < 3 && !accumulate) forces[(size_t)rr * 3 + tid] = 0.f;
    }
    grad_h[(size_t)row * FT + tid] = v;
    if (tid < 3) {
      float* fp = forces + (size_t)row * 3 + tid;
      *fp = (accumulate ? *fp : 0.f) - fv;
    }
    next_row = row + 1;
  };

  const uint32_t sX_a = tc::smem_u32(sX), sY_a = tc::smem_u32(sY);
  const uint32_t sW1_a = tc::smem_u32(sW1), sW2_a = tc::smem_u32(sW2);
  const uint32_t sXe2_a = sX_a + TM * K1 * 2;  // second Gaussian-derivative operand
  const float nglog2e = -rp.gamma * LOG2E;

  for (long long tb = e_begin; tb < e_end && !aborted; tb += TM) {
    const int ne = (int)((e_end - tb) < TM ? (e_end - tb) : TM);
    const int r_lo = s_misc[4];
    for (int i = tid; i <= TM; i += THREADS) s_rp[i] = row_ptr[min(r_lo + i, r_end)];
    __syncthreads();
    // ------------------------------------------------------------------ prep (all warps)
    // half 0 writes the Gaussian row e, half 1 its d-derivative e'
    int my_dst = -1;
    {
      const int t = 32 * (warp & 3) + lane;
      const int hf = warp >> 2;
      float fc = 0.f, dfc = 0.f, d = 0.f, ux = 0.f, uy = 0.f, uz = 0.f;
      int j = 0;
      bool ok = false;
      if (t < ne) {
        const long long gidx = tb + t;
        my_dst = dst_of_b(s_rp, r_lo, r_end, row_ptr, gidx);
        j = col_idx[gidx];
        if ((unsigned)j < (unsigned)N) {
          const float dx = pos[3 * my_dst] - pos[3 * j], dy = pos[3 * my_dst + 1] - pos[3 * j + 1],
                      dz = pos[3 * my_dst + 2] - pos[3 * j + 2];
          d = sqrtf(dx * dx + dy * dy + dz * dz);
          fc = cutoff_f(d, rp.r_c);
          dfc = cutoff_grad_f(d, rp.r_c);
          if (d > 0.f) {
            const float inv = 1.f / d;
            ux = dx * inv;
            uy = dy * inv;
            uz = dz * inv;
          }
          ok = true;
        } else {
          if (hf == 0) raise_status(status, kStatusBounds);
          j = 0;
        }
      }
      if (hf == 0) {
        s_src[t] = j;
        s_dst[t] = my_dst;
        s_fc[t] = fc;
        s_dfc[t] = dfc;
        s_ux[t] = ux;
        s_uy[t] = uy;
        s_uz[t] = uz;
      }
      const float d0 = d - rp.mu_min;
      uint8_t* dstA = sX + hf * (TM * K1 * 2);
#pragma unroll
      for (int k0 = 0; k0 < K1; k0 += 8) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float v[2];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int k = k0 + 2 * q + hh;
            const float dd = fmaf(-(float)k, rp.dmu, d0);
            const float ek = tc::ex2f(nglog2e * dd * dd);
            float val;
            if (hf == 0) val = k < rp.R ? ek : (k == rp.R ? 1.f : 0.f);  // bias column: z1 only
            else val = k < rp.R ? -2.f * rp.gamma * dd * ek : 0.f;
            v[hh] = ok ? val : 0.f;
          }
          w[q] = tc::pack_bf16(v[0], v[1]);
        }
        *(uint4*)(dstA + kmaj(t, k0, K1)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    __syncthreads();
    bool flag = false;
    int incl = 0;
    if (tid < TM) {
      const int t = tid;
      flag = (t < ne) && (t == 0 || s_dst[t - 1] != my_dst);
      const unsigned b = __ballot_sync(0xffffffffu, flag);
      if (lane == 0) s_wsum[warp] = __popc(b);
      incl = __popc(b & ((2u << lane) - 1u));
    }
    tc::fence_proxy_async();
    __syncthreads();
    if (tid < TM) {
      const int t = tid;
      int off = 0;
      for (int w2 = 0; w2 < warp; ++w2) off += s_wsum[w2];
      const int slot = (t < ne) ? off + incl - 1 : -1;
      if (flag) {
        s_slot_row[slot] = my_dst;
        s_slot_start[slot] = t;
      }
      s_slot[t] = slot;
      if (t == 0) {
        const int ns = s_wsum[0] + s_wsum[1] + s_wsum[2] + s_wsum[3];
        s_misc[0] = ns;
        s_slot_start[ns] = ne;
      }
      if (t == ne - 1) s_misc[4] = my_dst;  // the next tile starts in this row or later
    }
    __syncthreads();
    const int nslots = s_misc[0];

    // ------------------------------------------------------------------ MMA1: z1 and t
    if (tid == 0) {
      tc::fence_after();
      for (int ks = 0; ks < K1 / 16; ++ks)
        tc::mma(tmem, tc::sdesc(sX_a + ks * 256, 128, K1 * 16),
                tc::sdesc(sW1_a + ks * 256, 128, K1 * 16), idesc_ff, ks > 0);
      for (int ks = 0; ks < K1 / 16; ++ks)
        tc::mma(tmem + 128, tc::sdesc(sXe2_a + ks * 256, 128, K1 * 16),
                tc::sdesc(sW1_a + ks * 256, 128, K1 * 16), idesc_ff, ks > 0);
      tc::commit(&s_mbar[0]);
    }
    if (!wait_mma()) {
      aborted = true;
      break;
    }
    const int q4 = warp & 3, half = warp >> 2;
    const int e = 32 * q4 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
    // ------------------------------------------------------------------ epi-1a: Q = sigmoid(z1) t
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int f0 = 64 * half + 32 * c;
      uint32_t rz[32], rt[32];
      tc::ld32(lane_base + f0, rz);
      tc::ld32(lane_base + 128 + f0, rt);
      tc::ld_wait();
#pragma unroll
      for (int g8 = 0; g8 < 4; ++g8) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float o[2];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int i = 8 * g8 + 2 * q + hh;
            const float z = __uint_as_float(rz[i]);
            const float sg = rcpf(1.f + tc::ex2f(-z * LOG2E));
            o[hh] = sg * __uint_as_float(rt[i]);
          }
          w[q] = tc::pack_bf16(o[0], o[1]);
        }
        *(uint4*)(sX + kmaj(e, f0 + 8 * g8, K2)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    tc::fence_proxy_async();
    tc::fence_before();
    __syncthreads();
    if (tid == 0) {  // MMA2b: v = Q . A2 into columns 128..255
      tc::fence_after();
      for (int ks = 0; ks < K2 / 16; ++ks)
        tc::mma(tmem + 128, tc::sdesc(sX_a + ks * 256, 128, K2 * 16),
                tc::sdesc(sW2_a + ks * 256, 128, K2 * 16), idesc_ff, ks > 0);
      tc::commit(&s_mbar[0]);
    }
    if (!wait_mma()) {
      aborted = true;
      break;
    }
    // ------------------------------------------------------------------ epi-1b: P = ssp(z1)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int f0 = 64 * half + 32 * c;
      uint32_t rz[32];
      tc::ld32(lane_base + f0, rz);
      tc::ld_wait();
#pragma unroll
      for (int g8 = 0; g8 < 4; ++g8) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float a = ssp_scaled(__uint_as_float(rz[8 * g8 + 2 * q]), 1.f, LN2);
          const float b = ssp_scaled(__uint_as_float(rz[8 * g8 + 2 * q + 1]), 1.f, LN2);
          w[q] = tc::pack_bf16(a, b);
        }
        *(uint4*)(sX + kmaj(e, f0 + 8 * g8, K2)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    // first 16-column chunk of the four gathered rows, loaded while MMA2a runs
    const int j_me = s_src[e];
    const int k_me = s_dst[e] >= 0 ? s_dst[e] : 0;
    const uint4* gj = (const uint4*)(gin + (size_t)j_me * FT);
    const uint4* hj = (const uint4*)(hin + (size_t)j_me * FT);
    const uint4* gk = (const uint4*)(gin + (size_t)k_me * FT);
    const uint4* hk = (const uint4*)(hin + (size_t)k_me * FT);
    uint4 vgj[2], vhj[2], vgk[2], vhk[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int o = 8 * half + q;
      vgj[q] = __ldg(gj + o);
      vhj[q] = __ldg(hj + o);
      vgk[q] = __ldg(gk + o);
      vhk[q] = __ldg(hk + o);
    }
    tc::fence_proxy_async();
    tc::fence_before();
    __syncthreads();
    if (tid == 0) {  // MMA2a: u = P . A2 into columns 0..127
      tc::fence_after();
      for (int ks = 0; ks < K2 / 16; ++ks)
        tc::mma(tmem, tc::sdesc(sX_a + ks * 256, 128, K2 * 16),
                tc::sdesc(sW2_a + ks * 256, 128, K2 * 16), idesc_ff, ks > 0);
      tc::commit(&s_mbar[0]);
    }
    if (!wait_mma()) {
      aborted = true;
      break;
    }
    // ------------------------------------------------------------------ epi-2
    {
      const float fc = s_fc[e], dfc = s_dfc[e];
      float s_acc = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int f0 = 64 * half + 16 * c;
        uint32_t ru[16], rv[16];
        tc::ld16(lane_base + f0, ru);
        tc::ld16(lane_base + 128 + f0, rv);
        float c2v[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 t4 = *(const float4*)(sc2 + f0 + 4 * q);
          c2v[4 * q] = t4.x;
          c2v[4 * q + 1] = t4.y;
          c2v[4 * q + 2] = t4.z;
          c2v[4 * q + 3] = t4.w;
        }
        if (c > 0) {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            vgj[q] = __ldg(gj + (f0 >> 3) + q);
            vhj[q] = __ldg(hj + (f0 >> 3) + q);
            vgk[q] = __ldg(gk + (f0 >> 3) + q);
            vhk[q] = __ldg(hk + (f0 >> 3) + q);
          }
        }
        tc::ld_wait();
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const uint32_t a_gj[4] = {vgj[q].x, vgj[q].y, vgj[q].z, vgj[q].w};
          const uint32_t a_hj[4] = {vhj[q].x, vhj[q].y, vhj[q].z, vhj[q].w};
          const uint32_t a_gk[4] = {vgk[q].x, vgk[q].y, vgk[q].z, vgk[q].w};
          const uint32_t a_hk[4] = {vhk[q].x, vhk[q].y, vhk[q].z, vhk[q].w};
          uint32_t w[4];
#pragma unroll
          for (int p2 = 0; p2 < 4; ++p2) {
            float m2[2];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int i = 8 * q + 2 * p2 + hh;
              const int f = f0 + i;
              const float U = __uint_as_float(ru[i]) + c2v[i];
              const float Wv = fc * U;
              const float Wp = fmaf(dfc, U, fc * __uint_as_float(rv[i]));
              const float vgj_f = hh ? bf_hi(a_gj[p2]) : bf_lo(a_gj[p2]);
              const float vhj_f = hh ? bf_hi(a_hj[p2]) : bf_lo(a_hj[p2]);
              const float vgk_f = hh ? bf_hi(a_gk[p2]) : bf_lo(a_gk[p2]);
              const float vhk_f = hh ? bf_hi(a_hk[p2]) : bf_lo(a_hk[p2]);
              m2[hh] = vgj_f * Wv;
              s_acc = fmaf(fmaf(vgk_f, vhj_f, vgj_f * vhk_f), Wp, s_acc);
            }
            w[p2] = tc::pack_bf16(m2[0], m2[1]);
          }
          const int f8 = f0 + 8 * q;
          *(uint4*)(sX + (f8 >> 3) * 2048 + (e >> 3) * 128 + (e & 7) * 16) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      s_part[half * TM + e] = s_acc;
    }
    tc::fence_before();
    __syncthreads();
    // ------------------------------------------------------------------ per-row force sums
    if (tid >= TM) {
      const int s = tid - TM;
      if (s < nslots) {
        float fx = 0.f, fy = 0.f, fz = 0.f;
        for (int t = s_slot_start[s]; t < s_slot_start[s + 1]; ++t) {
          const float sv = s_part[t] + s_part[TM + t];
          fx = fmaf(sv, s_ux[t], fx);
          fy = fmaf(sv, s_uy[t], fy);
          fz = fmaf(sv, s_uz[t], fz);
        }
        s_force[3 * s] = fx;
        s_force[3 * s + 1] = fy;
        s_force[3 * s + 2] = fz;
      }
    }
    // ------------------------------------------------------------------ MMA3: grad_h segment sum
    for (int p = 0; p * SLOT_PASS < nslots; ++p) {
      const int ns = nslots - p * SLOT_PASS < SLOT_PASS ? nslots - p * SLOT_PASS : SLOT_PASS;
      const int n16 = (ns + 15) & ~15;
      __syncthreads();
      {
        uint4* z = (uint4*)sY;
        for (int i = tid; i < n16 * TM * 2 / 16; i += THREADS) z[i] = make_uint4(0, 0, 0, 0);
      }
      __syncthreads();
      if (tid < TM) {
        const int sl = s_slot[tid] - p * SLOT_PASS;
        if (s_slot[tid] >= 0 && sl >= 0 && sl < ns)
          *(uint16_t*)(sY + kmaj(sl, tid, TM)) = (uint16_t)0x3F80;
      }
      tc::fence_proxy_async();
      tc::fence_before();
      __syncthreads();
      if (tid == 0) {
        tc::fence_after();
        const uint32_t id3 = tc::idesc(TM, n16, 1, true, false);
        for (int ks = 0; ks < TM / 16; ++ks)
          tc::mma(tmem + p * SLOT_PASS, tc::sdesc(sX_a + ks * 256, 128, 2048),
                  tc::sdesc(sY_a + ks * 256, 128, TM * 16), id3, ks > 0);
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
            float fv = tid < 3 ? s_force[3 * s + tid] : 0.f;
            if (row == carry_row) {
              v += carry;
              fv += fcarry;
            } else if (carry_row >= 0) {
              write_row(carry_row, carry, fcarry);
            }
            carry_row = -1;
            if (s == nslots - 1) {
              carry = v;
              fcarry = fv;
              carry_row = row;
            } else {
              write_row(row, v, fv);
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
      tc::mbar_wait(&s_mbar[0], phase ^ 1u, WAIT_LIMIT);
    }
  } else if (tid < TM) {
    if (carry_row >= 0) write_row(carry_row, carry, fcarry);
    for (int rr = next_row; rr < r_end; ++rr) {
      grad_h[(size_t)rr * FT + tid] = 0.f;
      if (tid < 3 && !accumulate) forces[(size_t)rr * 3 + tid] = 0.f;
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 256);
}

}  // namespace

bool tc_bwd_supported(const mp_ctx* ctx) { return tc_supported(ctx); }

int tc_cfconv_bwd(mp_ctx* ctx, int block, int N, long long E, const float* pos, const int* row_ptr,
                  const int* col_idx, const void* h, const void* g, float* grad_h, float* forces,
                  bool accumulate, cudaStream_t s) {
  return tc_cfconv_bwd_ws(ctx, block, N, E, pos, row_ptr, col_idx, h, g, grad_h, forces, accumulate,
                          s);
}

int tc_cfconv_bwd_sequential(mp_ctx* ctx, int block, int N, long long E, const float* pos,
                             const int* row_ptr, const int* col_idx, const void* h, const void* g,
                             float* grad_h, float* forces, bool accumulate, cudaStream_t s) {
  const int K1 = k1_of(ctx->cfg.n_rbf);
  const ImgLayout IL = img_layout(K1);
  const uint8_t* img = (const uint8_t*)ctx->tc_weights + IL.bytes * block;
  long long tiles = (E + TM - 1) / TM;
  int grid = 2 * ctx->num_sms;
  if (tiles < grid) grid = (int)(tiles > 0 ? tiles : 1);
  auto go = [&](auto kern, int k1) {
    const size_t smem = smem_layout_b(k1).total + 1024;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return launch(ctx, K_CFCONV_BWD_TC_LS, kern, dim3(grid), dim3(THREADS), smem, s, N, E, pos,
                  row_ptr, col_idx, (const __nv_bfloat16*)h, (const __nv_bfloat16*)g, grad_h,
                  forces, (int)accumulate, img, radial_of(ctx), ctx->status_d);
  };
  if (K1 == 64) return go(k_cfconv_bwd_tc<64>, 64);
  if (K1 == 80) return go(k_cfconv_bwd_tc<80>, 80);
  if (K1 == 48) return go(k_cfconv_bwd_tc<48>, 48);
  if (K1 == 32) return go(k_cfconv_bwd_tc<32>, 32);
  return MP_ERR_INVALID_ARG;
}

}  // namespace mp
