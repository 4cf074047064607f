// Tensor-core destination pass of the attention backward (bf16 path, F = 128, 16 heads x 8, K a
// multiple of 128). E2Former-V2 page s.3.2 for the aggregation it differentiates; the arithmetic
// is that of the CUDA-core destination pass (attn_bwd.cu), with the filter and its distance
// derivative on the tensor cores as in the cfconv backward (FlashSchNet page s.2.3):
//   [z1 | bias] = e [A1ext | P],  [t | b'] = e' [A1 | P]                  (MMA1, N = 144 each)
//   v = (sigmoid(z1) t) A2,  u = ssp(z1) A2                              (MMA2b, MMA2a)
//   W = f_c (u + c2),  W' = f_c' (u + c2) + f_c v
// and, per slot s of row i and head h, in the epilogue (thread = slot, a quarter of the features):
//   l = q_i . k_j / sqrt(8) + bias,  dalpha = sum g_i x_j W,  beta = sum g_i x_j W',  b'.
// Once the row's K / 128 tiles are done: the row's softmax statistics (max, sum, D = sum alpha
// dalpha), dL/dq_i = sum_s dl k_j / sqrt(8) and the row side of dL/dr_i, as the CUDA-core pass.
// One CTA of 512 threads per SM (four warps per TMEM lane quarter), lock-step tiles; every wait
// is bounded.
#include "tc_common.cuh"

namespace mp {
namespace {
using namespace tcc;

constexpr int BT = 512;          // threads: four warps per TMEM lane quarter
constexpr int BH = 16, BD = 8;   // heads, head width
constexpr int BN1 = FT + BH;     // MMA1 columns: the filter's first layer and the radial bias
constexpr int KMAX = 256;        // slots per row this kernel keeps on chip
constexpr int SLS = KMAX + 16;   // row stride of the per-head slot arrays (rows of consecutive
                                 // heads start on different banks)

struct BwSmem {
  uint32_t w1, w2, c2, x, row, total;
};
__host__ __device__ constexpr BwSmem bw_layout(int K1) {
  // W1 | P (144 rows) | W2 | c2 | operand area (e and e', then Q, then P) | per-row slot data
  BwSmem L{};
  uint32_t o = 0;
  L.w1 = o;  o += BN1 * K1 * 2;
  L.w2 = o;  o += FT * K2 * 2;
  L.c2 = o;  o += 1024;
  L.x = o;   o += (2 * TM * K1 * 2 > TM * K2 * 2 ? 2 * TM * K1 * 2 : TM * K2 * 2);
  L.row = o;
  // per slot: logit, dalpha, beta, b' [16] each, unit vector [3], source; q_i, g_i; statistics;
  // per-tile geometry (fc, f_c', source) and reduction scratch
  o += (4 * BH * SLS + 4 * KMAX) * 4 + 2 * FT * 4 + 3 * BH * 4 + 3 * TM * 4 + 64 * 4;
  o += 64;  // mbarriers and the TMEM slot
  L.total = o;
  return L;
}
__host__ __device__ constexpr bool bw_fits_attn(int K1) {
  return bw_layout(K1).total + 1024 <= 227 * 1024;
}

// The filter of a tile's 128 entries and its d-derivative on the tensor cores. Every thread of
// the CTA calls it with its entry e (TMEM lane), feature quarter, distance d and validity; on return
// (all MMAs complete) TMEM holds u = ssp(z1) A2 in columns [0,128), the radial bias of the 16
// heads in [128,144), v = (sigmoid(z1) t) A2 in [256,384) and the bias's d-derivative in
// [384,400). The operand area sX is free again. False when a bounded wait ran out.
template <int K1>
__device__ __forceinline__ bool filter_tile(uint8_t* sX, uint32_t sX_a, uint32_t sW1_a,
                                            uint32_t sW2_a, uint32_t tmem, uint32_t lane_base,
                                            int e, int part, float d, bool ok, const Radial& rp,
                                            uint64_t* mbar, uint32_t& phase) {
  const int tid = threadIdx.x;
  auto wait_mma = [&]() -> bool {
    const int bad = tc::mbar_wait(mbar, phase, WAIT_LIMIT) ? 0 : 1;
    phase ^= 1u;
    tc::fence_after();
    return __syncthreads_or(bad) == 0;
  };
  const uint32_t id1 = tc::idesc(TM, BN1, 1, false, false);
  const uint32_t id2 = tc::idesc(TM, FT, 1, false, false);
  const float nglog2e = -rp.gamma * LOG2E;
  // parts 0 and 1 write the two halves of the Gaussian row e (with the constant bias column),
  // parts 2 and 3 those of e' = de/dd
  {
    const float d0 = d - rp.mu_min;
    const bool deriv = part >= 2;
    uint8_t* dstA = sX + (deriv ? TM * K1 * 2 : 0);
    const int kb = (part & 1) * (K1 / 2);
#pragma unroll
    for (int c8 = 0; c8 < K1 / 16; ++c8) {
      const int k0 = kb + 8 * c8;
      uint32_t w[4];
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        float v[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int k = k0 + 2 * qq + hh;
          const float dd = fmaf(-(float)k, rp.dmu, d0);
          const float ek = tc::ex2f(nglog2e * dd * dd);
          float val;
          if (!deriv) val = k < rp.R ? ek : (k == rp.R ? 1.f : 0.f);
          else val = k < rp.R ? -2.f * rp.gamma * dd * ek : 0.f;
          v[hh] = ok ? val : 0.f;
        }
        w[qq] = tc::pack_bf16(v[0], v[1]);
      }
      *(uint4*)(dstA + kmaj(e, k0, K1)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  tc::fence_proxy_async();
  tc::fence_before();
  __syncthreads();
  // MMA1: [z1 | bias] into columns [0,144), [t | b'] into [256,400)
  if (tid == 0) {
    tc::fence_after();
    const uint32_t sXe2_a = sX_a + TM * K1 * 2;
    for (int ks = 0; ks < K1 / 16; ++ks)
      tc::mma(tmem, tc::sdesc(sX_a + ks * 256, 128, K1 * 16),
              tc::sdesc(sW1_a + ks * 256, 128, K1 * 16), id1, ks > 0);
    for (int ks = 0; ks < K1 / 16; ++ks)
      tc::mma(tmem + 256, tc::sdesc(sXe2_a + ks * 256, 128, K1 * 16),
              tc::sdesc(sW1_a + ks * 256, 128, K1 * 16), id1, ks > 0);
    tc::commit(mbar);
  }
  if (!wait_mma()) return false;
  // E1a: Q = sigmoid(z1) t
  {
    const int f0 = 32 * part;
    uint32_t rz[32], rt[32];
    tc::ld32(lane_base + f0, rz);
    tc::ld32(lane_base + 256 + f0, rt);
    tc::ld_wait();
#pragma unroll
    for (int g8 = 0; g8 < 4; ++g8) {
      uint32_t w[4];
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        float o[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int ii = 8 * g8 + 2 * qq + hh;
          const float sg = tc::rcpf(1.f + tc::ex2f(-__uint_as_float(rz[ii]) * LOG2E));
          o[hh] = sg * __uint_as_float(rt[ii]);
        }
        w[qq] = tc::pack_bf16(o[0], o[1]);
      }
      *(uint4*)(sX + kmaj(e, f0 + 8 * g8, K2)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  tc::fence_proxy_async();
  tc::fence_before();
  __syncthreads();
  if (tid == 0) {  // MMA2b: v = Q A2 into columns 256..383 (t is consumed; b' stays)
    tc::fence_after();
    for (int ks = 0; ks < K2 / 16; ++ks)
      tc::mma(tmem + 256, tc::sdesc(sX_a + ks * 256, 128, K2 * 16),
              tc::sdesc(sW2_a + ks * 256, 128, K2 * 16), id2, ks > 0);
    tc::commit(mbar);
  }
  if (!wait_mma()) return false;
  // E1b: P = ssp(z1)
  {
    const int f0 = 32 * part;
    uint32_t rz[32];
    tc::ld32(lane_base + f0, rz);
    tc::ld_wait();
#pragma unroll
    for (int g8 = 0; g8 < 4; ++g8) {
      uint32_t w[4];
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        const float a = ssp_scaled(__uint_as_float(rz[8 * g8 + 2 * qq]), 1.f, LN2);
        const float b = ssp_scaled(__uint_as_float(rz[8 * g8 + 2 * qq + 1]), 1.f, LN2);
        w[qq] = tc::pack_bf16(a, b);
      }
      *(uint4*)(sX + kmaj(e, f0 + 8 * g8, K2)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  tc::fence_proxy_async();
  tc::fence_before();
  __syncthreads();
  if (tid == 0) {  // MMA2a: u = P A2 into columns 0..127 (z1 is consumed; the bias stays)
    tc::fence_after();
    for (int ks = 0; ks < K2 / 16; ++ks)
      tc::mma(tmem, tc::sdesc(sX_a + ks * 256, 128, K2 * 16),
              tc::sdesc(sW2_a + ks * 256, 128, K2 * 16), id2, ks > 0);
    tc::commit(mbar);
  }
  return wait_mma();
}

template <int K1>
__global__ void __launch_bounds__(BT, 1) k_attn_bwd_dst_tc(
    int N, int K, const float* __restrict__ pos, const int* __restrict__ nbr,
    const unsigned char* __restrict__ mask, const __nv_bfloat16* __restrict__ x,
    const float* __restrict__ g, const float* __restrict__ q, const float* __restrict__ kx,
    const uint8_t* __restrict__ img, const uint8_t* __restrict__ pimg, Radial rp, float qscale,
    float* __restrict__ gq, float* __restrict__ grad_pos, float* __restrict__ stats,
    int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr BwSmem L = bw_layout(K1);
  uint8_t* sW1 = sm + L.w1;
  uint8_t* sW2 = sm + L.w2;
  float* sc2 = (float*)(sm + L.c2);
  uint8_t* sX = sm + L.x;
  float* s_l = (float*)(sm + L.row);         // [16][SLS]: per head, per slot
  float* s_da = s_l + BH * SLS;              // [16][SLS]
  float* s_be = s_da + BH * SLS;             // [16][SLS]
  float* s_bp = s_be + BH * SLS;             // [16][SLS]
  float* s_u = s_bp + BH * SLS;              // [KMAX][3]
  int* s_src = (int*)(s_u + 3 * KMAX);       // [KMAX], -1: no valid neighbor in the slot
  float* s_q = (float*)(s_src + KMAX);       // [F], scaled by qscale
  float* s_g = s_q + FT;                     // [F]
  float* s_st = s_g + FT;                    // [3][16]: max, 1 / sum, D
  float* s_fc = s_st + 3 * BH;               // [TM] the tile's envelope
  float* s_dfc = s_fc + TM;                  // [TM]
  int* s_tj = (int*)(s_dfc + TM);            // [TM] the tile's sources (0 when empty)
  float* s_red = (float*)(s_tj + TM);        // [64]
  uint64_t* s_mbar = (uint64_t*)(s_red + 64);  // [0] MMA completion, [1] weight copy
  uint32_t* s_tmem = (uint32_t*)(s_mbar + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int TPA = K / TM;
  if (warp == 0) tc::tmem_alloc(s_tmem, 512);
  if (tid == 0) {
    tc::mbar_init(&s_mbar[0], 1);
    tc::mbar_init(&s_mbar[1], 1);
    const ImgLayout IL = img_layout(K1);
    tc::mbar_expect_tx(&s_mbar[1], FT * K1 * 2 + BH * K1 * 2 + FT * K2 * 2 + FT * 4);
    tc::bulk_g2s(sW1, img + IL.w1, FT * K1 * 2, &s_mbar[1]);
    tc::bulk_g2s(sW1 + FT * K1 * 2, pimg, BH * K1 * 2, &s_mbar[1]);
    tc::bulk_g2s(sW2, img + IL.w2, FT * K2 * 2, &s_mbar[1]);
    tc::bulk_g2s(sc2, img + IL.c2, FT * 4, &s_mbar[1]);
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *s_tmem;
  uint32_t phase = 0;
  bool aborted = __syncthreads_or(tc::mbar_wait(&s_mbar[1], 0, WAIT_LIMIT) ? 0 : 1) != 0;
  const uint32_t sX_a = tc::smem_u32(sX), sW1_a = tc::smem_u32(sW1), sW2_a = tc::smem_u32(sW2);
  // TMEM columns: [0,144) z1 | bias, then u in [0,128); [256,400) t | b', then v in [256,384)
  const int q4 = warp & 3, part = warp >> 2;  // lane quarter; features [32 part, 32 part + 32)
  const int e = 32 * q4 + lane;               // the tile's slot this thread works on
  const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);

  for (int i = blockIdx.x; i < N && !aborted; i += gridDim.x) {
    if (tid < FT) {
      s_q[tid] = q[(size_t)i * FT + tid] * qscale;
      s_g[tid] = g[(size_t)i * FT + tid];
    }
    const float pix = pos[3 * i], piy = pos[3 * i + 1], piz = pos[3 * i + 2];
    for (int tt = 0; tt < TPA && !aborted; ++tt) {
      const int s0 = tt * TM;
      // ---------------------------------------------------------------- prep (all threads)
      {
        const size_t slot = (size_t)i * K + s0 + e;
        int j = nbr[slot];
        bool ok = mask[slot] != 0;
        if (ok && (unsigned)j >= (unsigned)N) {
          if (part == 0) raise_status(status, kStatusBounds);
          ok = false;
        }
        if (!ok) j = 0;
        float d = 0.f, fc = 0.f, dfc = 0.f, ux = 0.f, uy = 0.f, uz = 0.f;
        if (ok) {
          const float dx = pix - pos[3 * j], dy = piy - pos[3 * j + 1], dz = piz - pos[3 * j + 2];
          d = sqrtf(dx * dx + dy * dy + dz * dz);
          fc = cutoff_f(d, rp.r_c);
          dfc = cutoff_grad_f(d, rp.r_c);
          if (d > 0.f) {
            const float inv = 1.f / d;
            ux = dx * inv;
            uy = dy * inv;
            uz = dz * inv;
          }
        }
        if (part == 0) {
          s_src[s0 + e] = ok ? j : -1;
          s_u[3 * (s0 + e)] = ux;
          s_u[3 * (s0 + e) + 1] = uy;
          s_u[3 * (s0 + e) + 2] = uz;
          s_fc[e] = fc;
          s_dfc[e] = dfc;
          s_tj[e] = j;
        }
        if (!filter_tile<K1>(sX, sX_a, sW1_a, sW2_a, tmem, lane_base, e, part, d, ok, rp,
                             &s_mbar[0], phase)) {
          aborted = true;
          break;
        }
      }
      // ---------------------------------------------------------------- E2: per slot and head
      {
        const int j = s_tj[e];
        const float fc = s_fc[e], dfc = s_dfc[e];
        const bool ok = s_src[s0 + e] >= 0;
        uint32_t rb[8], rp8[8];
        tc::ld8(lane_base + FT + 8 * (part >> 1), rb);        // the radial bias of 8 heads ..
        tc::ld8(lane_base + 256 + FT + 8 * (part >> 1), rp8);  // and its d-derivative b'
        tc::ld_wait(rb, rp8);
        const __nv_bfloat16* xr = x + (size_t)j * FT;
        const float* kr = kx + (size_t)j * FT;
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {  // head 4 part + hh: features f0 .. f0 + 7
          const int f0 = 32 * part + 8 * hh;
          const float bias_h = __uint_as_float((part & 1) ? rb[4 + hh] : rb[hh]);
          const float bp_h = __uint_as_float((part & 1) ? rp8[4 + hh] : rp8[hh]);
          uint32_t ru[8], rv[8];
          tc::ld8(lane_base + f0, ru);
          tc::ld8(lane_base + 256 + f0, rv);
          const uint4 xq = *(const uint4*)(xr + f0);
          const float4 ka = *(const float4*)(kr + f0);
          const float4 kb = *(const float4*)(kr + f0 + 4);
          tc::ld_wait(ru, rv);
          const uint32_t xw[4] = {xq.x, xq.y, xq.z, xq.w};
          const float kk[8] = {ka.x, ka.y, ka.z, ka.w, kb.x, kb.y, kb.z, kb.w};
          float l = 0.f, da = 0.f, be = 0.f;
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const float xv = (cc & 1) ? bf_hi(xw[cc >> 1]) : bf_lo(xw[cc >> 1]);
            const float uc = __uint_as_float(ru[cc]) + sc2[f0 + cc];
            const float W = fc * uc;
            const float Wp = fmaf(dfc, uc, fc * __uint_as_float(rv[cc]));
            const float gx = s_g[f0 + cc] * xv;
            l = fmaf(s_q[f0 + cc], kk[cc], l);
            da = fmaf(gx, W, da);
            be = fmaf(gx, Wp, be);
          }
          if (ok) {
            const int o = (4 * part + hh) * SLS + s0 + e;
            s_l[o] = l + bias_h;
            s_da[o] = da;
            s_be[o] = be;
            s_bp[o] = bp_h;
          }
        }
      }
      tc::fence_before();
      __syncthreads();  // the next tile's prep rewrites the operand area and the tile geometry
    }
    if (aborted) break;
    // ------------------------------------------------------------------ the row's statistics
    // one warp per head, slots strided over its lanes
    {
      const int h = warp, c = lane;
      float m = -INFINITY;
      for (int s = c; s < K; s += 32)
        if (s_src[s] >= 0) m = fmaxf(m, s_l[h * SLS + s]);
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float z = 0.f;
      for (int s = c; s < K; s += 32)
        if (s_src[s] >= 0) z += tc::ex2f((s_l[h * SLS + s] - m) * LOG2E);
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
      const float iz = z > 0.f ? 1.f / z : 0.f;
      float D = 0.f;
      for (int s = c; s < K; s += 32)
        if (s_src[s] >= 0) D += tc::ex2f((s_l[h * SLS + s] - m) * LOG2E) * iz * s_da[h * SLS + s];
      for (int o = 16; o > 0; o >>= 1) D += __shfl_xor_sync(0xffffffffu, D, o);
      if (c == 0) {
        s_st[h] = m;
        s_st[BH + h] = iz;
        s_st[2 * BH + h] = D;
        stats[(size_t)i * 3 * BH + h] = m;
        stats[(size_t)i * 3 * BH + BH + h] = z;
        stats[(size_t)i * 3 * BH + 2 * BH + h] = D;
      }
    }
    __syncthreads();
    // dL/dq_i: thread (feature f, residue r of the slot mod 4) sums a quarter of the slots; the
    // four partial sums meet in shared memory and are added in a fixed order
    {
      const int f = tid & (FT - 1), par = tid >> 7, h = f >> 3;
      const float m = s_st[h], iz = s_st[BH + h], D = s_st[2 * BH + h];
      float acc = 0.f;
      for (int s0 = par; s0 < K; s0 += 32) {  // eight independent gathers in flight
        float kv[8];
#pragma unroll
        for (int u8 = 0; u8 < 8; ++u8) {
          const int s = s0 + 4 * u8;
          const int j = s < K ? s_src[s] : -1;
          kv[u8] = j >= 0 ? kx[(size_t)j * FT + f] : 0.f;
        }
#pragma unroll
        for (int u8 = 0; u8 < 8; ++u8) {
          const int s = s0 + 4 * u8;
          if (s < K && s_src[s] >= 0) {
            const int o = h * SLS + s;
            const float a = tc::ex2f((s_l[o] - m) * LOG2E) * iz;
            acc = fmaf(a * (s_da[o] - D), kv[u8], acc);
          }
        }
      }
      float* pacc = (float*)sX;      // the operand area is free between rows
      if (par > 0) pacc[par * FT + f] = acc;
      __syncthreads();
      if (par == 0)
        gq[(size_t)i * FT + f] = (((acc + pacc[FT + f]) + pacc[2 * FT + f]) + pacc[3 * FT + f]) * qscale;
    }
    // dL/dr_i, row side: each slot's dL/dd over the heads times (r_i - r_j) / d
    {
      float gp0 = 0.f, gp1 = 0.f, gp2 = 0.f;
      for (int s = tid; s < K; s += BT) {
        if (s_src[s] < 0) continue;
        float sd = 0.f;
        for (int h = 0; h < BH; ++h) {
          const int o = h * SLS + s;
          const float a = tc::ex2f((s_l[o] - s_st[h]) * LOG2E) * s_st[BH + h];
          sd = fmaf(a, s_be[o], sd);
          sd = fmaf(a * (s_da[o] - s_st[2 * BH + h]), s_bp[o], sd);
        }
        gp0 = fmaf(sd, s_u[3 * s], gp0);
        gp1 = fmaf(sd, s_u[3 * s + 1], gp1);
        gp2 = fmaf(sd, s_u[3 * s + 2], gp2);
      }
      for (int o = 16; o > 0; o >>= 1) {
        gp0 += __shfl_xor_sync(0xffffffffu, gp0, o);
        gp1 += __shfl_xor_sync(0xffffffffu, gp1, o);
        gp2 += __shfl_xor_sync(0xffffffffu, gp2, o);
      }
      if (lane == 0) {
        s_red[16 + warp] = gp0;
        s_red[32 + warp] = gp1;
        s_red[48 + warp] = gp2;
      }
      __syncthreads();
      if (tid < 3) {
        float v = 0.f;
        for (int w = 0; w < BT / 32; ++w) v += s_red[16 * (tid + 1) + w];
        grad_pos[3 * i + tid] = v;
      }
      __syncthreads();  // s_q, s_g, the slot data and the operand area are reused by the next row
    }
  }
  tc::fence_before();
  __syncthreads();
  if (tid == 0 && aborted) raise_status(status, kStatusTimeout);
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------------------ source pass
// One CTA of 512 threads per SM; per source atom j, its transposed entries (row i, slot), in
// ascending order, in tiles of 128: the filter as in the destination pass; then per entry and head
// (thread = entry, a quarter of the features) alpha = e^(l - m_ih) / z_ih from the row's statistics,
// dalpha, beta and dl = alpha (dalpha - D_ih); per feature the entry's terms dl q_i / sqrt(8) (of
// dL/dk_j) and alpha g_i W (the value path of dL/dx_j), summed over the entries by two MMAs of
// bf16 message tiles against a column of ones, accumulated in TMEM over the source's tiles; and
// the entry's dL/dd = sum_h (alpha beta + dl b') times -(r_i - r_j) / d, summed on chip.
struct SrSmem {
  uint32_t w1, w2, c2, x, m1, m2, ones, misc, total;
};
__host__ __device__ constexpr SrSmem sr_layout(int K1) {
  SrSmem L{};
  uint32_t o = 0;
  L.w1 = o;   o += BN1 * K1 * 2;
  L.w2 = o;   o += FT * K2 * 2;
  L.c2 = o;   o += 1024;
  L.x = o;    o += (2 * TM * K1 * 2 > TM * K2 * 2 ? 2 * TM * K1 * 2 : TM * K2 * 2);
  L.m1 = o;   o += FT * TM * 2;
  L.m2 = o;   o += FT * TM * 2;
  L.ones = o; o += 16 * TM * 2;
  L.misc = o;
  // k_j, x_j [F]; per entry: row, envelope, its derivative, unit vector [3], four dL/dd parts;
  // reduction scratch; mbarriers and the TMEM slot
  o += 2 * FT * 4 + TM * (1 + 2 + 3 + 4) * 4 + 64 * 4 + 64;
  L.total = o;
  return L;
}
__host__ __device__ constexpr bool sr_fits(int K1) { return sr_layout(K1).total + 1024 <= 227 * 1024; }

template <int K1>
__global__ void __launch_bounds__(BT, 1) k_attn_bwd_src_tc(
    int N, int K, const float* __restrict__ pos, const int* __restrict__ rev_ptr,
    const int* __restrict__ rev, const __nv_bfloat16* __restrict__ x,
    const float* __restrict__ g, const float* __restrict__ q, const float* __restrict__ kx,
    const float* __restrict__ stats, const uint8_t* __restrict__ img,
    const uint8_t* __restrict__ pimg, Radial rp, float qscale, float* __restrict__ grad_x,
    float* __restrict__ gk, float* __restrict__ grad_pos, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr SrSmem L = sr_layout(K1);
  uint8_t* sW1 = sm + L.w1;
  uint8_t* sW2 = sm + L.w2;
  float* sc2 = (float*)(sm + L.c2);
  uint8_t* sX = sm + L.x;
  uint8_t* sM1 = sm + L.m1;
  uint8_t* sM2 = sm + L.m2;
  uint8_t* sOnes = sm + L.ones;
  float* s_k = (float*)(sm + L.misc);  // [F] k_j
  float* s_xj = s_k + FT;              // [F] x_j
  int* s_row = (int*)(s_xj + FT);      // [TM] the entry's row i (0 when empty)
  float* s_fc = (float*)(s_row + TM);  // [TM]
  float* s_dfc = s_fc + TM;            // [TM]
  float* s_u = s_dfc + TM;             // [TM][3]
  float* s_sd = s_u + 3 * TM;          // [4][TM] dL/dd of the entry, per feature quarter
  float* s_red = s_sd + 4 * TM;        // [64]
  uint64_t* s_mbar = (uint64_t*)(s_red + 64);
  uint32_t* s_tmem = (uint32_t*)(s_mbar + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (warp == 0) tc::tmem_alloc(s_tmem, 512);
  for (int k = tid; k < 16 * TM * 2 / 4; k += BT) ((uint32_t*)sOnes)[k] = 0u;  // rows 1..15 stay 0
  if (tid == 0) {
    tc::mbar_init(&s_mbar[0], 1);
    tc::mbar_init(&s_mbar[1], 1);
    const ImgLayout IL = img_layout(K1);
    tc::mbar_expect_tx(&s_mbar[1], FT * K1 * 2 + BH * K1 * 2 + FT * K2 * 2 + FT * 4);
    tc::bulk_g2s(sW1, img + IL.w1, FT * K1 * 2, &s_mbar[1]);
    tc::bulk_g2s(sW1 + FT * K1 * 2, pimg, BH * K1 * 2, &s_mbar[1]);
    tc::bulk_g2s(sW2, img + IL.w2, FT * K2 * 2, &s_mbar[1]);
    tc::bulk_g2s(sc2, img + IL.c2, FT * 4, &s_mbar[1]);
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *s_tmem;
  uint32_t phase = 0;
  bool aborted = __syncthreads_or(tc::mbar_wait(&s_mbar[1], 0, WAIT_LIMIT) ? 0 : 1) != 0;
  const uint32_t sX_a = tc::smem_u32(sX), sW1_a = tc::smem_u32(sW1), sW2_a = tc::smem_u32(sW2);
  const uint32_t sM1_a = tc::smem_u32(sM1), sM2_a = tc::smem_u32(sM2);
  const uint32_t sOnes_a = tc::smem_u32(sOnes);
  const uint32_t id3 = tc::idesc(TM, 16, 1, true, false);
  const int q4 = warp & 3, part = warp >> 2;
  const int e = 32 * q4 + lane;
  const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
  // TMEM columns [400,416): dL/dk_j per feature (lane); [416,432): the value path of dL/dx_j

  for (int j = blockIdx.x; j < N && !aborted; j += gridDim.x) {
    const int r0 = rev_ptr[j], r1 = rev_ptr[j + 1];
    if (r1 <= r0) {  // no row reads atom j: its source-side terms are zero
      if (tid < FT) {
        grad_x[(size_t)j * FT + tid] = 0.f;
        gk[(size_t)j * FT + tid] = 0.f;
      }
      continue;
    }
    if (tid < FT) {
      s_k[tid] = kx[(size_t)j * FT + tid];
      s_xj[tid] = __bfloat162float(x[(size_t)j * FT + tid]);
    }
    const float pjx = pos[3 * j], pjy = pos[3 * j + 1], pjz = pos[3 * j + 2];
    float gp0 = 0.f, gp1 = 0.f, gp2 = 0.f;
    const int ntile = (r1 - r0 + TM - 1) / TM;
    for (int tt = 0; tt < ntile && !aborted; ++tt) {
      // ---------------------------------------------------------------- prep
      const int idx = r0 + tt * TM + e;
      bool ok = idx < r1;
      int i = 0;
      if (ok) {
        i = rev[idx] / K;
        if ((unsigned)i >= (unsigned)N) {
          if (part == 0) raise_status(status, kStatusBounds);
          ok = false;
          i = 0;
        }
      }
      float d = 0.f, fc = 0.f, dfc = 0.f, ux = 0.f, uy = 0.f, uz = 0.f;
      if (ok) {
        const float dx = pos[3 * i] - pjx, dy = pos[3 * i + 1] - pjy, dz = pos[3 * i + 2] - pjz;
        d = sqrtf(dx * dx + dy * dy + dz * dz);
        fc = cutoff_f(d, rp.r_c);
        dfc = cutoff_grad_f(d, rp.r_c);
        if (d > 0.f) {
          const float inv = 1.f / d;
          ux = dx * inv;
          uy = dy * inv;
          uz = dz * inv;
        }
      }
      if (part == 0) {
        s_row[e] = ok ? i : -1;
        s_fc[e] = fc;
        s_dfc[e] = dfc;
        s_u[3 * e] = ux;
        s_u[3 * e + 1] = uy;
        s_u[3 * e + 2] = uz;
        // the ones column: entry e of row 0 of the (slot x entry) matrix
        *(__nv_bfloat16*)(sOnes + kmaj(0, e, TM)) = __float2bfloat16_rn(ok ? 1.f : 0.f);
      }
      if (!filter_tile<K1>(sX, sX_a, sW1_a, sW2_a, tmem, lane_base, e, part, d, ok, rp,
                           &s_mbar[0], phase)) {
        aborted = true;
        break;
      }
      // ---------------------------------------------------------------- E2: per entry and head
      {
        const int row = s_row[e];
        const bool eok = row >= 0;
        const int ii = eok ? row : 0;
        const float efc = s_fc[e], edfc = s_dfc[e];
        uint32_t rb[8], rp8[8];
        tc::ld8(lane_base + FT + 8 * (part >> 1), rb);
        tc::ld8(lane_base + 256 + FT + 8 * (part >> 1), rp8);
        tc::ld_wait(rb, rp8);
        const float* qr = q + (size_t)ii * FT;
        const float* gr = g + (size_t)ii * FT;
        const float* st = stats + (size_t)ii * 3 * BH;
        float sd = 0.f;
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
          const int h = 4 * part + hh, f0 = 8 * h;
          const float bias_h = __uint_as_float((part & 1) ? rb[4 + hh] : rb[hh]);
          const float bp_h = __uint_as_float((part & 1) ? rp8[4 + hh] : rp8[hh]);
          uint32_t ru[8], rv[8];
          tc::ld8(lane_base + f0, ru);
          tc::ld8(lane_base + 256 + f0, rv);
          const float4 qa = *(const float4*)(qr + f0), qb = *(const float4*)(qr + f0 + 4);
          const float4 ga = *(const float4*)(gr + f0), gb = *(const float4*)(gr + f0 + 4);
          const float m = st[h], z = st[BH + h], D = st[2 * BH + h];
          tc::ld_wait(ru, rv);
          const float qq[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
          const float gg[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
          float l = 0.f, da = 0.f, be = 0.f, W[8];
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const float uc = __uint_as_float(ru[cc]) + sc2[f0 + cc];
            W[cc] = efc * uc;
            const float Wp = fmaf(edfc, uc, efc * __uint_as_float(rv[cc]));
            const float gx = gg[cc] * s_xj[f0 + cc];
            l = fmaf(qq[cc] * qscale, s_k[f0 + cc], l);
            da = fmaf(gx, W[cc], da);
            be = fmaf(gx, Wp, be);
          }
          l += bias_h;
          const float a = (eok && z > 0.f) ? tc::ex2f((l - m) * LOG2E) * (1.f / z) : 0.f;
          const float dl = a * (da - D);
          sd = fmaf(a, be, fmaf(dl, bp_h, sd));
          uint32_t w1[4], w2[4];
#pragma unroll
          for (int c2i = 0; c2i < 4; ++c2i) {
            const int c0 = 2 * c2i;
            w1[c2i] = tc::pack_bf16(dl * qq[c0] * qscale, dl * qq[c0 + 1] * qscale);
            w2[c2i] = tc::pack_bf16(a * gg[c0] * W[c0], a * gg[c0 + 1] * W[c0 + 1]);
          }
          const uint32_t mo = (uint32_t)(h * 2048 + (e >> 3) * 128 + (e & 7) * 16);
          *(uint4*)(sM1 + mo) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
          *(uint4*)(sM2 + mo) = make_uint4(w2[0], w2[1], w2[2], w2[3]);
        }
        s_sd[part * TM + e] = eok ? sd : 0.f;
      }
      tc::fence_proxy_async();
      tc::fence_before();
      __syncthreads();
      // ---------------------------------------------------------------- MMA3: sums over entries
      if (tid == 0) {
        tc::fence_after();
        for (int ks = 0; ks < TM / 16; ++ks) {
          tc::mma(tmem + 400, tc::sdesc(sM1_a + ks * 256, 128, 2048),
                  tc::sdesc(sOnes_a + ks * 256, 128, TM * 16), id3, (tt > 0 || ks > 0) ? 1u : 0u);
          tc::mma(tmem + 416, tc::sdesc(sM2_a + ks * 256, 128, 2048),
                  tc::sdesc(sOnes_a + ks * 256, 128, TM * 16), id3, (tt > 0 || ks > 0) ? 1u : 0u);
        }
        tc::commit(&s_mbar[0]);
      }
      {
        const int bad = tc::mbar_wait(&s_mbar[0], phase, WAIT_LIMIT) ? 0 : 1;
        phase ^= 1u;
        tc::fence_after();
        if (__syncthreads_or(bad) != 0) {
          aborted = true;
          break;
        }
      }
      if (part == 0 && s_row[e] >= 0) {  // -dL/dd (r_i - r_j) / d of this entry
        const float sdd = ((s_sd[e] + s_sd[TM + e]) + s_sd[2 * TM + e]) + s_sd[3 * TM + e];
        gp0 = fmaf(-sdd, s_u[3 * e], gp0);
        gp1 = fmaf(-sdd, s_u[3 * e + 1], gp1);
        gp2 = fmaf(-sdd, s_u[3 * e + 2], gp2);
      }
    }
    if (aborted) break;
    // ------------------------------------------------------------------ source j's outputs
    if (tid < FT) {  // warps 0-3: TMEM lane = feature
      uint32_t vk, vx;
      tc::ld1(lane_base + 400, vk);
      tc::ld1(lane_base + 416, vx);
      tc::ld_wait();
      gk[(size_t)j * FT + tid] = __uint_as_float(vk);
      grad_x[(size_t)j * FT + tid] = __uint_as_float(vx);
    }
    for (int o = 16; o > 0; o >>= 1) {
      gp0 += __shfl_xor_sync(0xffffffffu, gp0, o);
      gp1 += __shfl_xor_sync(0xffffffffu, gp1, o);
      gp2 += __shfl_xor_sync(0xffffffffu, gp2, o);
    }
    if (lane == 0) {
      s_red[16 + warp] = gp0;
      s_red[32 + warp] = gp1;
      s_red[48 + warp] = gp2;
    }
    tc::fence_before();
    __syncthreads();
    if (tid < 3) {
      float v = 0.f;
      for (int w = 0; w < BT / 32; ++w) v += s_red[16 * (tid + 1) + w];
      grad_pos[3 * j + tid] += v;  // the destination pass wrote the row side
    }
    __syncthreads();
  }
  tc::fence_before();
  __syncthreads();
  if (tid == 0 && aborted) raise_status(status, kStatusTimeout);
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

}  // namespace

bool tc_attn_bwd_supported(const mp_ctx* ctx, int K) {
  const mp_config& c = ctx->cfg;
  return tc_supported(ctx) && ctx->tc_attn_p && c.n_heads == BH && c.head_dim == BD &&
         K % TM == 0 && K <= KMAX && k1_of(c.n_rbf) <= 64 &&  // built for 32-64 operand columns
         bw_fits_attn(k1_of(c.n_rbf)) && sr_fits(k1_of(c.n_rbf));
}

int tc_attn_bwd_dst(mp_ctx* ctx, int N, int K, const float* pos, const int* nbr,
                    const unsigned char* mask, const void* x, const float* g, float* gq,
                    float* grad_pos, cudaStream_t s) {
  const int K1 = k1_of(ctx->cfg.n_rbf);
  const uint8_t* img = (const uint8_t*)ctx->tc_weights;  // the filter of block 0
  int grid = ctx->num_sms;
  if (N < grid) grid = N > 0 ? N : 1;
  const float qscale = 1.f / sqrtf((float)BD);
  auto go = [&](auto kern, int k1) {
    const size_t smem = bw_layout(k1).total + 1024;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return launch(ctx, K_ATTN_BWD_TC, kern, dim3(grid), dim3(BT), smem, s, N, K, pos, nbr, mask,
                  (const __nv_bfloat16*)x, g, (const float*)ctx->q, (const float*)ctx->k, img,
                  (const uint8_t*)ctx->tc_attn_p, radial_of(ctx), qscale, gq, grad_pos,
                  ctx->attn_stats, ctx->status_d);
  };
  if (K1 == 64) return go(k_attn_bwd_dst_tc<64>, 64);
  if (K1 == 48) return go(k_attn_bwd_dst_tc<48>, 48);
  if (K1 == 32) return go(k_attn_bwd_dst_tc<32>, 32);
  return MP_ERR_INVALID_ARG;
}

}  // namespace mp

namespace mp {

int tc_attn_bwd_src(mp_ctx* ctx, int N, int K, const float* pos, const int* rev_ptr,
                    const int* rev, const void* x, const float* g, float* grad_x, float* gk,
                    float* grad_pos, cudaStream_t s) {
  const int K1 = k1_of(ctx->cfg.n_rbf);
  const uint8_t* img = (const uint8_t*)ctx->tc_weights;
  int grid = ctx->num_sms;
  if (N < grid) grid = N > 0 ? N : 1;
  const float qscale = 1.f / sqrtf((float)BD);
  auto go = [&](auto kern, int k1) {
    const size_t smem = sr_layout(k1).total + 1024;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return launch(ctx, K_ATTN_BWD_SRC_TC, kern, dim3(grid), dim3(BT), smem, s, N, K, pos, rev_ptr,
                  rev, (const __nv_bfloat16*)x, g, (const float*)ctx->q, (const float*)ctx->k,
                  (const float*)ctx->attn_stats, img, (const uint8_t*)ctx->tc_attn_p,
                  radial_of(ctx), qscale, grad_x, gk, grad_pos, ctx->status_d);
  };
  if (K1 == 64) return go(k_attn_bwd_src_tc<64>, 64);
  if (K1 == 48) return go(k_attn_bwd_src_tc<48>, 48);
  if (K1 == 32) return go(k_attn_bwd_src_tc<32>, 32);
  return MP_ERR_INVALID_ARG;
}

}  // namespace mp
