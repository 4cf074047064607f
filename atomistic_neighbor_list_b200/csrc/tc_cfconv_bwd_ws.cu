// Warp-specialised, double-buffered tensor-core cfconv backward (bf16 path, F = 128): grad_h and
// the block's force contribution in one pass over the symmetric CSR, with the same arithmetic as the
// tile description in tc_cfconv_bwd.cu (FlashSchNet page, technical summary s.2.3: the backward
// reduces by source; every output row is written once, no atomics; the filter is recomputed).
//
// Roles of one persistent CTA per SM (13 warps):
//   prep (warps 0-3)      tile i+1: rows, distances, envelope and its derivative, unit vectors,
//                         the Gaussian operand e and its d-derivative e'
//   epilogue (warps 4-11) in the order E2(i), E1a(i+1), force sums(i), E1b(i+1), drain(i):
//                           E1a  Q = sigmoid(z1) t  (stored) and P = ssp(z1) (kept in registers)
//                           E1b  P stored once MMA2b has consumed Q
//                           E2   W = f_c (u + c2), W' = f_c' (u + c2) + f_c v; msg = g_j W for the
//                                segment-sum MMA; s_kj = sum_f (g_k h_j + g_j h_k) W' per edge
//                           drain grad_h rows and forces (per-row sums), written once
//   MMA (warp 12)         MMA1 (z1 and t), MMA2b (v = Q A2), MMA2a (u = P A2), MMA3 (segment sum)
// TMEM: two 256-column buffers (z1 | t, then u | v, then the segment sums); mbarriers carry every
// hand-off with bounded waits and uniform abort votes.
#include "tc_common.cuh"

namespace mp {
namespace {
using namespace tcc;

constexpr int BW_THREADS = 416;
constexpr int BW_PREP_WARPS = 4, BW_EPI_WARP0 = 4, BW_MMA_WARP = 12;
constexpr int SMB = 128;  // destination rows per tile

struct BwMeta {  // written by prep (triple-buffered)
  int src[TM];
  int dst[TM];
  float fc[TM], dfc[TM], ux[TM], uy[TM], uz[TM];
  int slot[TM];
  int slot_row[SMB];
  int slot_start[SMB + 4];
  int nslots, ne, pad0, pad1;
};
struct BwEpi {  // epilogue scratch (double-buffered)
  float spart[2][TM];
  float force[SMB][3];
};
__host__ __device__ constexpr uint32_t ee_bytes(int K1) {
  return (uint32_t)(2 * TM * K1 * 2 > SMB * TM * 2 ? 2 * TM * K1 * 2 : SMB * TM * 2);
}
struct BwSmem {
  uint32_t w1, w2, c2, ee0, qp0, meta0, epi0, rp, misc, bars, total;
};
__host__ __device__ constexpr BwSmem bw_layout(int K1) {
  return BwSmem{0u,
                (uint32_t)(FT * K1 * 2),
                (uint32_t)(FT * K1 * 2 + FT * K2 * 2),
                (uint32_t)(FT * K1 * 2 + FT * K2 * 2 + 1024),
                (uint32_t)(FT * K1 * 2 + FT * K2 * 2 + 1024 + 2 * ee_bytes(K1)),
                (uint32_t)(FT * K1 * 2 + FT * K2 * 2 + 1024 + 2 * ee_bytes(K1) + 2 * TM * K2 * 2),
                (uint32_t)(FT * K1 * 2 + FT * K2 * 2 + 1024 + 2 * ee_bytes(K1) + 2 * TM * K2 * 2 +
                           3 * (uint32_t)sizeof(BwMeta)),
                (uint32_t)(FT * K1 * 2 + FT * K2 * 2 + 1024 + 2 * ee_bytes(K1) + 2 * TM * K2 * 2 +
                           3 * (uint32_t)sizeof(BwMeta) + 2 * (uint32_t)sizeof(BwEpi)),
                (uint32_t)(FT * K1 * 2 + FT * K2 * 2 + 1024 + 2 * ee_bytes(K1) + 2 * TM * K2 * 2 +
                           3 * (uint32_t)sizeof(BwMeta) + 2 * (uint32_t)sizeof(BwEpi) + 2 * TM * 4 +
                           64),
                (uint32_t)(FT * K1 * 2 + FT * K2 * 2 + 1024 + 2 * ee_bytes(K1) + 2 * TM * K2 * 2 +
                           3 * (uint32_t)sizeof(BwMeta) + 2 * (uint32_t)sizeof(BwEpi) + 2 * TM * 4 +
                           128),
                (uint32_t)(FT * K1 * 2 + FT * K2 * 2 + 1024 + 2 * ee_bytes(K1) + 2 * TM * K2 * 2 +
                           3 * (uint32_t)sizeof(BwMeta) + 2 * (uint32_t)sizeof(BwEpi) + 2 * TM * 4 +
                           128 + 256)};
}

enum { Q_FULL_A = 0, Q_DONE1, Q_FULL_Q, Q_DONE2B, Q_FULL_P, Q_DONE2A, Q_FULL_M, Q_DONE3, Q_FREE_T,
       Q_W };

template <int K1>
__global__ void __launch_bounds__(BW_THREADS, 1) k_cfconv_bwd_ws(
    int N, long long E, const float* __restrict__ pos, const int* __restrict__ row_ptr,
    const int* __restrict__ col_idx, const __nv_bfloat16* __restrict__ hin,
    const __nv_bfloat16* __restrict__ gin, float* __restrict__ grad_h, float* __restrict__ forces,
    int accumulate, const uint8_t* __restrict__ img, Radial rp, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr BwSmem L = bw_layout(K1);
  uint8_t* sW1 = sm + L.w1;
  uint8_t* sW2 = sm + L.w2;
  float* sc2 = (float*)(sm + L.c2);
  auto EE = [&](int b) { return sm + L.ee0 + (uint32_t)b * ee_bytes(K1); };
  auto QP = [&](int b) { return sm + L.qp0 + (uint32_t)b * (TM * K2 * 2); };
  auto MB = [&](int k) { return (BwMeta*)(sm + L.meta0) + k; };
  auto EP = [&](int b) { return (BwEpi*)(sm + L.epi0) + b; };
  int* s_rp = (int*)(sm + L.rp);
  int* s_pdst = s_rp + TM + 4;
  int* s_misc = (int*)(sm + L.misc);
  uint64_t* bars = (uint64_t*)(sm + L.bars);
  uint32_t* s_tmem = (uint32_t*)(bars + 20);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  if (tid == 0) {
    const long long b_lo = E * cta / G, b_hi = E * (cta + 1) / G;
    const int r0 = lower_row(row_ptr, N, b_lo);
    const int r1 = (cta == G - 1) ? N : lower_row(row_ptr, N, b_hi);
    s_misc[8] = r0;
    s_misc[9] = r1 > r0 ? r1 : r0;
    s_misc[10] = 0;
  }
  __syncthreads();
  const int r_begin = s_misc[8], r_end = s_misc[9];
  if (r_begin >= r_end) return;
  const long long e_begin = clamp_off(row_ptr[r_begin], E);
  long long e_end = clamp_off(row_ptr[r_end], E);
  if (e_end < e_begin) e_end = e_begin;
  const int ntiles = (int)((e_end - e_begin + TM - 1) / TM);

  if (warp == 0) tc::tmem_alloc(s_tmem, 512);
  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&bars[2 * Q_FULL_A + b], 128);
      tc::mbar_init(&bars[2 * Q_DONE1 + b], 1);
      tc::mbar_init(&bars[2 * Q_FULL_Q + b], 256);
      tc::mbar_init(&bars[2 * Q_DONE2B + b], 1);
      tc::mbar_init(&bars[2 * Q_FULL_P + b], 256);
      tc::mbar_init(&bars[2 * Q_DONE2A + b], 1);
      tc::mbar_init(&bars[2 * Q_FULL_M + b], 256);
      tc::mbar_init(&bars[2 * Q_DONE3 + b], 1);
      tc::mbar_init(&bars[2 * Q_FREE_T + b], 256);
    }
    tc::mbar_init(&bars[2 * Q_W], 1);
    const ImgLayout IL = img_layout(K1);
    tc::mbar_expect_tx(&bars[2 * Q_W], FT * K1 * 2 + FT * K2 * 2 + FT * 4);
    tc::bulk_g2s(sW1, img + IL.w1, FT * K1 * 2, &bars[2 * Q_W]);
    tc::bulk_g2s(sW2, img + IL.w2, FT * K2 * 2, &bars[2 * Q_W]);
    tc::bulk_g2s(sc2, img + IL.c2, FT * 4, &bars[2 * Q_W]);
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *s_tmem;
  volatile int* abort_flag = &s_misc[10];
  auto wait_bar = [&](int idx, int b, uint32_t parity) -> bool {
    if (tc::mbar_wait(&bars[2 * idx + b], parity, WAIT_LIMIT)) return true;
    *abort_flag = 1;
    return false;
  };

  if (warp < BW_PREP_WARPS) {
    // =============================================================== prep role (128 threads)
    const int t = tid;
    const float nglog2e = -rp.gamma * LOG2E;
    int r_lo = r_begin;
    for (int it = 0; it < ntiles; ++it) {
      const int b = it & 1;
      const long long tb = e_begin + (long long)it * TM;
      const int ne = (int)((e_end - tb) < TM ? (e_end - tb) : TM);
      const long long g = tb + t;
      int j = t < ne ? col_idx[g] : 0;
      const bool jok = (unsigned)j < (unsigned)N;
      if (!jok) j = 0;
      const int rpv = row_ptr[min(r_lo + t, r_end)];
      const int rpv_last = row_ptr[min(r_lo + TM, r_end)];
      const float pjx = pos[3 * j], pjy = pos[3 * j + 1], pjz = pos[3 * j + 2];
      // operand buffer b is free once the segment-sum MMA of tile it-2 completed
      const bool free_ok = it < 2 || wait_bar(Q_DONE3, b, ((it - 2) >> 1) & 1);
      if (bar_sync_or(1, 128, !free_ok || *abort_flag)) break;
      s_rp[t] = rpv;
      if (t == 0) s_rp[TM] = rpv_last;
      bar_sync(1, 128);
      BwMeta* M = MB(it % 3);
      int my_dst = -1;
      float fc = 0.f, dfc = 0.f, d = 0.f, ux = 0.f, uy = 0.f, uz = 0.f;
      bool ok = false;
      if (t < ne) {
        if ((long long)s_rp[TM] <= g) {
          my_dst = row_of(row_ptr, r_lo + TM, r_end, g);
        } else {
          int lo = 0, hi = TM;
          while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if ((long long)s_rp[mid] <= g) lo = mid; else hi = mid;
          }
          my_dst = r_lo + lo;
        }
        if (jok) {
          const float dx = pos[3 * my_dst] - pjx, dy = pos[3 * my_dst + 1] - pjy,
                      dz = pos[3 * my_dst + 2] - pjz;
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
          raise_status(status, kStatusBounds);
        }
      }
      M->src[t] = j;
      M->dst[t] = my_dst >= 0 ? my_dst : 0;
      M->fc[t] = fc;
      M->dfc[t] = dfc;
      M->ux[t] = ux;
      M->uy[t] = uy;
      M->uz[t] = uz;
      s_pdst[t] = my_dst;
      // the Gaussian row e (bias column R = 1) and its d-derivative e' (no bias)
      const float d0 = d - rp.mu_min;
      uint8_t* A = EE(b);
#pragma unroll 2
      for (int k0 = 0; k0 < K1; k0 += 8) {
        uint32_t w[4], wd[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float v[2], vd[2];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int k = k0 + 2 * q + hh;
            const float dd = fmaf(-(float)k, rp.dmu, d0);
            const float ek = tc::ex2f(nglog2e * dd * dd);
            float val = ek, dval = -2.f * rp.gamma * dd * ek;
            if (k >= rp.R) {
              val = k == rp.R ? 1.f : 0.f;
              dval = 0.f;
            }
            v[hh] = ok ? val : 0.f;
            vd[hh] = ok ? dval : 0.f;
          }
          w[q] = tc::pack_bf16(v[0], v[1]);
          wd[q] = tc::pack_bf16(vd[0], vd[1]);
        }
        *(uint4*)(A + kmaj(t, k0, K1)) = make_uint4(w[0], w[1], w[2], w[3]);
        *(uint4*)(A + TM * K1 * 2 + kmaj(t, k0, K1)) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
      }
      bar_sync(1, 128);  // s_pdst complete
      const bool flag = (t < ne) && (t == 0 || s_pdst[t - 1] != my_dst);
      const unsigned bal = __ballot_sync(0xffffffffu, flag);
      if (lane == 0) s_misc[warp] = __popc(bal);
      bar_sync(1, 128);
      int off = 0;
      for (int w2 = 0; w2 < warp; ++w2) off += s_misc[w2];
      const int slot = (t < ne) ? off + __popc(bal & ((2u << lane) - 1u)) - 1 : -1;
      if (flag) {
        M->slot_row[slot] = my_dst;
        M->slot_start[slot] = t;
      }
      M->slot[t] = slot;
      if (t == 0) {
        const int ns = s_misc[0] + s_misc[1] + s_misc[2] + s_misc[3];
        M->nslots = ns;
        M->ne = ne;
        M->slot_start[ns] = ne;
      }
      if (t == ne - 1) s_rp[TM + 1] = my_dst;
      tc::fence_proxy_async();
      bar_sync(1, 128);
      r_lo = s_rp[TM + 1];
      mbar_arrive1(&bars[2 * Q_FULL_A + b]);
    }
  } else if (warp == BW_MMA_WARP) {
    // =============================================================== MMA role (one thread)
    if (lane == 0) {
      bool ok = tc::mbar_wait(&bars[2 * Q_W], 0, WAIT_LIMIT);
      if (!ok) *abort_flag = 1;
      const uint32_t id = tc::idesc(TM, FT, 1, false, false);
      const uint32_t sW1_a = tc::smem_u32(sW1), sW2_a = tc::smem_u32(sW2);
      int n1 = 0, n2b = 0, n2a = 0, n3 = 0;
      uint32_t spins = 0;
      while (ok && n3 < ntiles && !*abort_flag) {
        bool issued = false;
        if (n3 < n2a) {  // MMA3: segment sums of g_j W
          const int b = n3 & 1;
          if (tc::mbar_test(&bars[2 * Q_FULL_M + b], (n3 >> 1) & 1)) {
            tc::fence_after();
            const int ns = MB(n3 % 3)->nslots;
            const int n16 = ns > 0 ? (ns + 15) & ~15 : 16;
            const uint32_t id3 = tc::idesc(TM, n16, 1, true, false);
            const uint32_t qa = tc::smem_u32(QP(b)), sa = tc::smem_u32(EE(b));
            for (int ks = 0; ks < TM / 16; ++ks)
              tc::mma(tmem + 256 * b, tc::sdesc(qa + ks * 256, 128, 2048),
                      tc::sdesc(sa + ks * 256, 128, TM * 16), id3, ks > 0);
            tc::commit(&bars[2 * Q_DONE3 + b]);
            ++n3;
            issued = true;
          }
        }
        if (!issued && n2a < n2b) {  // MMA2a: u = P A2 -> columns 0..127
          const int b = n2a & 1;
          if (tc::mbar_test(&bars[2 * Q_FULL_P + b], (n2a >> 1) & 1)) {
            tc::fence_after();
            const uint32_t qa = tc::smem_u32(QP(b));
            for (int ks = 0; ks < K2 / 16; ++ks)
              tc::mma(tmem + 256 * b, tc::sdesc(qa + ks * 256, 128, K2 * 16),
                      tc::sdesc(sW2_a + ks * 256, 128, K2 * 16), id, ks > 0);
            tc::commit(&bars[2 * Q_DONE2A + b]);
            ++n2a;
            issued = true;
          }
        }
        if (!issued && n2b < n1) {  // MMA2b: v = Q A2 -> columns 128..255
          const int b = n2b & 1;
          if (tc::mbar_test(&bars[2 * Q_FULL_Q + b], (n2b >> 1) & 1)) {
            tc::fence_after();
            const uint32_t qa = tc::smem_u32(QP(b));
            for (int ks = 0; ks < K2 / 16; ++ks)
              tc::mma(tmem + 256 * b + 128, tc::sdesc(qa + ks * 256, 128, K2 * 16),
                      tc::sdesc(sW2_a + ks * 256, 128, K2 * 16), id, ks > 0);
            tc::commit(&bars[2 * Q_DONE2B + b]);
            ++n2b;
            issued = true;
          }
        }
        if (!issued && n1 < ntiles && n1 < n3 + 2) {  // MMA1: z1 = e A1ext, t = e' A1
          const int b = n1 & 1;
          if (tc::mbar_test(&bars[2 * Q_FULL_A + b], (n1 >> 1) & 1) &&
              (n1 < 2 || tc::mbar_test(&bars[2 * Q_FREE_T + b], ((n1 - 2) >> 1) & 1))) {
            tc::fence_after();
            const uint32_t ea = tc::smem_u32(EE(b));
            for (int ks = 0; ks < K1 / 16; ++ks)
              tc::mma(tmem + 256 * b, tc::sdesc(ea + ks * 256, 128, K1 * 16),
                      tc::sdesc(sW1_a + ks * 256, 128, K1 * 16), id, ks > 0);
            for (int ks = 0; ks < K1 / 16; ++ks)
              tc::mma(tmem + 256 * b + 128, tc::sdesc(ea + TM * K1 * 2 + ks * 256, 128, K1 * 16),
                      tc::sdesc(sW1_a + ks * 256, 128, K1 * 16), id, ks > 0);
            tc::commit(&bars[2 * Q_DONE1 + b]);
            ++n1;
            issued = true;
          }
        }
        if (issued) {
          spins = 0;
        } else if (++spins > (WAIT_LIMIT >> 2)) {
          *abort_flag = 1;
        } else {
          __nanosleep(64);
        }
      }
      if (n3 > 0)
        tc::mbar_wait(&bars[2 * Q_DONE3 + ((n3 - 1) & 1)], ((n3 - 1) >> 1) & 1, WAIT_LIMIT);
    }
  } else {
    // =============================================================== epilogue role (256 threads)
    const int ew = warp - BW_EPI_WARP0;
    const int q4 = warp & 3, half = ew >> 2;
    const int e_me = 32 * q4 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
    float carry = 0.f, fcarry = 0.f;
    int carry_row = -1, next_row = r_begin;
    uint32_t ppk[32];  // P = ssp(z1) of this thread's 64 columns, bf16 pairs, between E1a and E1b
    auto emit = [&](int row, float v, float fv) {
      for (int rr = next_row; rr < row; ++rr) {
        grad_h[(size_t)rr * FT + e_me] = 0.f;
        if (e_me < 3 && !accumulate) forces[(size_t)rr * 3 + e_me] = 0.f;
      }
      grad_h[(size_t)row * FT + e_me] = v;
      if (e_me < 3) {
        float* fp = forces + (size_t)row * 3 + e_me;
        *fp = (accumulate ? *fp : 0.f) - fv;
      }
      next_row = row + 1;
    };
    auto E1a = [&](int i) -> bool {
      const int b = i & 1;
      if (bar_sync_or(2, 256, !wait_bar(Q_DONE1, b, (i >> 1) & 1))) return false;
      tc::fence_after();
      uint8_t* Qb = QP(b);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int f0 = 64 * half + 16 * c;
        uint32_t rz[16], rt[16];
        tc::ld16(lane_base + 256 * b + f0, rz);
        tc::ld16(lane_base + 256 * b + 128 + f0, rt);
        tc::ld_wait();
        uint32_t wq[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float qo[2], po[2];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const float z = __uint_as_float(rz[2 * q + hh]);
            const float tn = tc::ex2f(-fabsf(z) * LOG2E);  // e^-|z|
            const float inv = inv_one_plus(tn);
            const float sg = z >= 0.f ? inv : tn * inv;     // sigmoid(z)
            qo[hh] = sg * __uint_as_float(rt[2 * q + hh]);
            po[hh] = fmaxf(z, 0.f) + ln_half_one_plus(tn);  // ssp(z)
          }
          wq[q] = tc::pack_bf16(qo[0], qo[1]);
          ppk[8 * c + q] = tc::pack_bf16(po[0], po[1]);
        }
        *(uint4*)(Qb + kmaj(e_me, f0, K2)) = make_uint4(wq[0], wq[1], wq[2], wq[3]);
        *(uint4*)(Qb + kmaj(e_me, f0 + 8, K2)) = make_uint4(wq[4], wq[5], wq[6], wq[7]);
      }
      // clear the rows of the 0/1 matrix this tile uses (e and e' are consumed)
      const int ns = MB(i % 3)->nslots;
      const int n16 = ns > 0 ? (ns + 15) & ~15 : 16;
      uint4* zz = (uint4*)EE(b);
      for (int k = e_me + 128 * half; k < n16 * TM * 2 / 16; k += 256) zz[k] = make_uint4(0, 0, 0, 0);
      tc::fence_proxy_async();
      tc::fence_before();
      mbar_arrive1(&bars[2 * Q_FULL_Q + b]);
      return true;
    };
    auto E1b = [&](int i) -> bool {
      const int b = i & 1;
      if (bar_sync_or(2, 256, !wait_bar(Q_DONE2B, b, (i >> 1) & 1))) return false;
      uint8_t* Pb = QP(b);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int f0 = 64 * half + 16 * c;
        *(uint4*)(Pb + kmaj(e_me, f0, K2)) =
            make_uint4(ppk[8 * c], ppk[8 * c + 1], ppk[8 * c + 2], ppk[8 * c + 3]);
        *(uint4*)(Pb + kmaj(e_me, f0 + 8, K2)) =
            make_uint4(ppk[8 * c + 4], ppk[8 * c + 5], ppk[8 * c + 6], ppk[8 * c + 7]);
      }
      tc::fence_proxy_async();
      mbar_arrive1(&bars[2 * Q_FULL_P + b]);
      return true;
    };
    auto E2 = [&](int i) -> bool {
      const int b = i & 1;
      const BwMeta* M = MB(i % 3);
      const float fc = M->fc[e_me], dfc = M->dfc[e_me];
      const uint4* gj = (const uint4*)(gin + (size_t)M->src[e_me] * FT) + 8 * half;
      const uint4* hj = (const uint4*)(hin + (size_t)M->src[e_me] * FT) + 8 * half;
      const uint4* gk = (const uint4*)(gin + (size_t)M->dst[e_me] * FT) + 8 * half;
      const uint4* hk = (const uint4*)(hin + (size_t)M->dst[e_me] * FT) + 8 * half;
      uint4 vgj[2], vhj[2], vgk[2], vhk[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        vgj[q] = __ldg(gj + q);
        vhj[q] = __ldg(hj + q);
        vgk[q] = __ldg(gk + q);
        vhk[q] = __ldg(hk + q);
      }
      if (bar_sync_or(2, 256, !wait_bar(Q_DONE2A, b, (i >> 1) & 1))) return false;
      tc::fence_after();
      uint8_t* Mb = QP(b);
      float s_acc = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int f0 = 64 * half + 16 * c;
        uint32_t ru[16], rv[16];
        tc::ld16(lane_base + 256 * b + f0, ru);
        tc::ld16(lane_base + 256 * b + 128 + f0, rv);
        if (c > 0) {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            vgj[q] = __ldg(gj + 2 * c + q);
            vhj[q] = __ldg(hj + 2 * c + q);
            vgk[q] = __ldg(gk + 2 * c + q);
            vhk[q] = __ldg(hk + 2 * c + q);
          }
        }
        tc::ld_wait();
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const uint32_t a_gj[4] = {vgj[q].x, vgj[q].y, vgj[q].z, vgj[q].w};
          const uint32_t a_hj[4] = {vhj[q].x, vhj[q].y, vhj[q].z, vhj[q].w};
          const uint32_t a_gk[4] = {vgk[q].x, vgk[q].y, vgk[q].z, vgk[q].w};
          const uint32_t a_hk[4] = {vhk[q].x, vhk[q].y, vhk[q].z, vhk[q].w};
          const int f8 = f0 + 8 * q;
          const float4 ca = *(const float4*)(sc2 + f8);
          const float4 cb = *(const float4*)(sc2 + f8 + 4);
          const float cc[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
          uint32_t w[4];
#pragma unroll
          for (int p2 = 0; p2 < 4; ++p2) {
            float m2[2];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int ii = 8 * q + 2 * p2 + hh;
              const float U = __uint_as_float(ru[ii]) + cc[2 * p2 + hh];
              const float Wv = fc * U;
              const float Wp = fmaf(dfc, U, fc * __uint_as_float(rv[ii]));
              const float xgj = hh ? bf_hi(a_gj[p2]) : bf_lo(a_gj[p2]);
              const float xhj = hh ? bf_hi(a_hj[p2]) : bf_lo(a_hj[p2]);
              const float xgk = hh ? bf_hi(a_gk[p2]) : bf_lo(a_gk[p2]);
              const float xhk = hh ? bf_hi(a_hk[p2]) : bf_lo(a_hk[p2]);
              m2[hh] = xgj * Wv;
              s_acc = fmaf(fmaf(xgk, xhj, xgj * xhk), Wp, s_acc);
            }
            w[p2] = tc::pack_bf16(m2[0], m2[1]);
          }
          *(uint4*)(Mb + (f8 >> 3) * 2048 + (e_me >> 3) * 128 + (e_me & 7) * 16) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      EP(b)->spart[half][e_me] = s_acc;
      bar_sync(2, 256);  // every thread's clearing of the 0/1 matrix (in E1a) is done
      if (half == 0) {
        const int sl = M->slot[e_me];
        if (sl >= 0) *(uint16_t*)(EE(b) + kmaj(sl, e_me, TM)) = (uint16_t)0x3F80;  // bf16 1.0
      }
      tc::fence_proxy_async();
      tc::fence_before();
      mbar_arrive1(&bars[2 * Q_FULL_M + b]);
      return true;
    };
    auto FS = [&](int i) {  // per-row force sums of tile i (after a barrier over the epilogue)
      const int b = i & 1;
      const BwMeta* M = MB(i % 3);
      BwEpi* P = EP(b);
      const int s = tid - 128;
      if (s < M->nslots) {
        float fx = 0.f, fy = 0.f, fz = 0.f;
        for (int t = M->slot_start[s]; t < M->slot_start[s + 1]; ++t) {
          const float sv = P->spart[0][t] + P->spart[1][t];
          fx = fmaf(sv, M->ux[t], fx);
          fy = fmaf(sv, M->uy[t], fy);
          fz = fmaf(sv, M->uz[t], fz);
        }
        P->force[s][0] = fx;
        P->force[s][1] = fy;
        P->force[s][2] = fz;
      }
    };
    auto DR = [&](int i) -> bool {
      const int b = i & 1;
      if (bar_sync_or(2, 256, !wait_bar(Q_DONE3, b, (i >> 1) & 1))) return false;
      tc::fence_after();
      const BwMeta* M = MB(i % 3);
      const BwEpi* P = EP(b);
      const int ns = M->nslots;
      if (half == 0) {
        if (ns > 0 && carry_row >= 0 && M->slot_row[0] != carry_row) {
          emit(carry_row, carry, fcarry);
          carry_row = -1;
        }
#pragma unroll 1
        for (int s = 0; s < ns; ++s) {
          uint32_t rv;
          tc::ld1(lane_base + 256 * b + s, rv);
          tc::ld_wait();
          const int row = M->slot_row[s];
          float v = __uint_as_float(rv);
          float fv = e_me < 3 ? P->force[s][e_me] : 0.f;
          if (row == carry_row) {
            v += carry;
            fv += fcarry;
          }
          carry_row = -1;
          if (s == ns - 1) {
            carry = v;
            fcarry = fv;
            carry_row = row;
          } else {
            emit(row, v, fv);
          }
        }
      }
      tc::fence_before();
      mbar_arrive1(&bars[2 * Q_FREE_T + b]);
      return true;
    };
    bool ok = true;
    if (ntiles > 0) ok = E1a(0) && E1b(0);
    for (int i = 0; ok && i < ntiles; ++i) {
      ok = E2(i);
      if (ok && i + 1 < ntiles) ok = E1a(i + 1);
      if (ok) {
        bar_sync(2, 256);  // the per-edge dot products of tile i are complete
        FS(i);
      }
      if (ok && i + 1 < ntiles) ok = E1b(i + 1);
      if (ok) ok = DR(i);
    }
    if (ok && half == 0) {
      if (carry_row >= 0) emit(carry_row, carry, fcarry);
      for (int rr = next_row; rr < r_end; ++rr) {
        grad_h[(size_t)rr * FT + e_me] = 0.f;
        if (e_me < 3 && !accumulate) forces[(size_t)rr * 3 + e_me] = 0.f;
      }
    }
  }
  tc::fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag) raise_status(status, kStatusTimeout);
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

}  // namespace

int tc_cfconv_bwd_ws(mp_ctx* ctx, int block, int N, long long E, const float* pos,
                     const int* row_ptr, const int* col_idx, const void* h, const void* g,
                     float* grad_h, float* forces, bool accumulate, cudaStream_t s) {
  const int K1 = k1_of(ctx->cfg.n_rbf);
  const ImgLayout IL = img_layout(K1);
  const uint8_t* img = (const uint8_t*)ctx->tc_weights + IL.bytes * block;
  long long tiles = (E + TM - 1) / TM;
  int grid = ctx->num_sms;
  if (tiles < grid) grid = (int)(tiles > 0 ? tiles : 1);
  auto go = [&](auto kern, int k1) {
    const size_t smem = bw_layout(k1).total + 1024;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return launch(ctx, K_CFCONV_BWD_TC, kern, dim3(grid), dim3(BW_THREADS), smem, s, N, E, pos,
                  row_ptr, col_idx, (const __nv_bfloat16*)h, (const __nv_bfloat16*)g, grad_h,
                  forces, (int)accumulate, img, radial_of(ctx), ctx->status_d);
  };
  if (K1 == 64) return go(k_cfconv_bwd_ws<64>, 64);
  if (K1 == 80) return go(k_cfconv_bwd_ws<80>, 80);
  if (K1 == 48) return go(k_cfconv_bwd_ws<48>, 48);
  if (K1 == 32) return go(k_cfconv_bwd_ws<32>, 32);
  return MP_ERR_INVALID_ARG;
}

}  // namespace mp
