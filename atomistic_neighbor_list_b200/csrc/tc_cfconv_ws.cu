// Warp-specialised, double-buffered tensor-core cfconv forward (bf16 path, F = 128).
//
// Same arithmetic as the tile description in tc_cfconv.cu (FlashSchNet page, technical summary
// s.2.1-2.4): Gaussian basis with the bias folded into MMA1, f_c * ssp epilogue, MMA2, x_j (.) W
// epilogue, the segment sum as MMA3 with a 0/1 edge-to-row matrix, one write per row. The tile loop
// is pipelined across three warp roles of one persistent CTA per SM:
//   prep (warps 0-3)      tile t+1: row of each edge, distance, envelope, Gaussian operand, slots
//   epilogue (warps 4-11) in the order epi-2(t), epi-1(t+1), drain(t), so that MMA3(t) and MMA2(t+1)
//                         run on the tensor core while the other epilogue step runs
//   MMA (warp 12)         one thread issues MMA1/MMA2/MMA3 as their inputs become ready
// Two TMEM accumulators of 128 columns and two sets of shared-memory operands alternate between
// tiles; mbarriers carry every hand-off (bounded waits: on expiry the kernel raises a status bit,
// waits for what it issued, frees TMEM and returns).
#include "tc_common.cuh"

namespace mp {
namespace {
using namespace tcc;

constexpr int WS_THREADS = 416;  // 13 warps
constexpr int PREP_WARPS = 4, EPI_WARP0 = 4, MMA_WARP = 12;  // epilogue: warps 4-11
constexpr int SMAX = 128;        // destination rows per tile (one segment-sum MMA, N <= 128)

// shared memory: W1 [F][K1], W2 [F][128], c2, then per buffer b: AS[b] (Gaussian operand, later
// the 0/1 matrix, max(TM*K1*2, SMAX*TM*2) bytes), H[b] (h' then msg^T, TM*K2*2), MB(b).
struct WsMeta {
  int src[TM];
  float fc[TM];
  int slot[TM];
  int slot_row[SMAX];
  int nslots, ne, pad0, pad1;
};
__host__ __device__ constexpr uint32_t as_bytes(int K1) {
  return (uint32_t)(TM * K1 * 2 > SMAX * TM * 2 ? TM * K1 * 2 : SMAX * TM * 2);
}
struct WsSmem {
  uint32_t w1, w2, c2, as0, h0, meta0, rp, misc, bars, total;
};
__host__ __device__ constexpr WsSmem ws_layout(int K1) {
  // all offsets multiples of 1024 up to meta
  return WsSmem{0u,
                (uint32_t)(FT * K1 * 2),
                (uint32_t)(FT * K1 * 2 + FT * K2 * 2),
                (uint32_t)(FT * K1 * 2 + FT * K2 * 2 + 1024),
                (uint32_t)(FT * K1 * 2 + FT * K2 * 2 + 1024 + 2 * as_bytes(K1)),
                (uint32_t)(FT * K1 * 2 + FT * K2 * 2 + 1024 + 2 * as_bytes(K1) + 2 * TM * K2 * 2),
                (uint32_t)(FT * K1 * 2 + FT * K2 * 2 + 1024 + 2 * as_bytes(K1) + 2 * TM * K2 * 2 +
                           3 * (uint32_t)sizeof(WsMeta)),
                (uint32_t)(FT * K1 * 2 + FT * K2 * 2 + 1024 + 2 * as_bytes(K1) + 2 * TM * K2 * 2 +
                           3 * (uint32_t)sizeof(WsMeta) + 2 * TM * 4 + 64),
                (uint32_t)(FT * K1 * 2 + FT * K2 * 2 + 1024 + 2 * as_bytes(K1) + 2 * TM * K2 * 2 +
                           3 * (uint32_t)sizeof(WsMeta) + 2 * TM * 4 + 128),
                (uint32_t)(FT * K1 * 2 + FT * K2 * 2 + 1024 + 2 * as_bytes(K1) + 2 * TM * K2 * 2 +
                           3 * (uint32_t)sizeof(WsMeta) + 2 * TM * 4 + 128 + 256)};
}

// mbarrier indices (each double-buffered: index*2 + b)
enum { B_FULL_A = 0, B_DONE1 = 1, B_FULL_H = 2, B_DONE2 = 3, B_FULL_M = 4, B_DONE3 = 5,
       B_FREE_T = 6, B_W = 7 };

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Barrier over `n` threads that also returns the OR of `pred` over them (a uniform decision).
__device__ __forceinline__ bool named_sync_or(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n.reg .pred p, q;\nsetp.ne.b32 p, %1, 0;\nbar.red.or.pred q, %2, %3, p;\n"
      "selp.b32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void mbar_arrive(uint64_t* m) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_u32(m)) : "memory");
}

template <int K1>
__global__ void __launch_bounds__(WS_THREADS, 1) k_cfconv_fwd_ws(
    int N, long long E, const float* __restrict__ pos, const int* __restrict__ row_ptr,
    const int* __restrict__ col_idx, const __nv_bfloat16* __restrict__ x,
    __nv_bfloat16* __restrict__ out, const uint8_t* __restrict__ img, Radial rp, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr WsSmem L = ws_layout(K1);
  uint8_t* sW1 = sm + L.w1;
  uint8_t* sW2 = sm + L.w2;
  float* sc2 = (float*)(sm + L.c2);
  auto AS = [&](int b) { return sm + L.as0 + (uint32_t)b * as_bytes(K1); };
  auto HB = [&](int b) { return sm + L.h0 + (uint32_t)b * (TM * K2 * 2); };
  auto MB = [&](int b) { return (WsMeta*)(sm + L.meta0) + b; };
  int* s_rp = (int*)(sm + L.rp);           // prep-private row window (TM + 1)
  int* s_pdst = s_rp + TM + 4;             // prep-private: dst of each edge of the tile
  int* s_misc = (int*)(sm + L.misc);       // [0..3] prep warp totals, [8] r_begin, [9] r_end, [10] abort
  uint64_t* bars = (uint64_t*)(sm + L.bars);
  uint32_t* s_tmem = (uint32_t*)(bars + 16);

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

  if (warp == 0) tc::tmem_alloc(s_tmem, 256);
  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&bars[2 * B_FULL_A + b], 128);
      tc::mbar_init(&bars[2 * B_DONE1 + b], 1);
      tc::mbar_init(&bars[2 * B_FULL_H + b], 256);
      tc::mbar_init(&bars[2 * B_DONE2 + b], 1);
      tc::mbar_init(&bars[2 * B_FULL_M + b], 256);
      tc::mbar_init(&bars[2 * B_DONE3 + b], 1);
      tc::mbar_init(&bars[2 * B_FREE_T + b], 256);
    }
    tc::mbar_init(&bars[2 * B_W], 1);
    const ImgLayout IL = img_layout(K1);
    tc::mbar_expect_tx(&bars[2 * B_W], FT * K1 * 2 + FT * K2 * 2 + FT * 4);
    tc::bulk_g2s(sW1, img + IL.w1, FT * K1 * 2, &bars[2 * B_W]);
    tc::bulk_g2s(sW2, img + IL.w2, FT * K2 * 2, &bars[2 * B_W]);
    tc::bulk_g2s(sc2, img + IL.c2, FT * 4, &bars[2 * B_W]);
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

  if (warp < PREP_WARPS) {
    // =============================================================== prep role (128 threads)
    const int t = tid;
    const float nglog2e = -rp.gamma * LOG2E;
    int r_lo = r_begin;
    for (int it = 0; it < ntiles; ++it) {
      const int b = it & 1;
      const long long tb = e_begin + (long long)it * TM;
      const int ne = (int)((e_end - tb) < TM ? (e_end - tb) : TM);
      // loads that need no buffer go first: they overlap the wait below
      const long long g = tb + t;
      int j = t < ne ? col_idx[g] : 0;
      const bool jok = (unsigned)j < (unsigned)N;
      if (!jok) j = 0;
      const int rpv = row_ptr[min(r_lo + t, r_end)];
      const int rpv_last = row_ptr[min(r_lo + TM, r_end)];
      const float pjx = pos[3 * j], pjy = pos[3 * j + 1], pjz = pos[3 * j + 2];
      // operand buffer b is free once the segment-sum MMA of tile it-2 completed
      const bool free_ok = it < 2 || wait_bar(B_DONE3, b, ((it - 2) >> 1) & 1);
      if (named_sync_or(1, 128, !free_ok || *abort_flag)) break;  // uniform over the prep warps
      s_rp[t] = rpv;
      if (t == 0) s_rp[TM] = rpv_last;
      named_sync(1, 128);
      WsMeta* M = MB(it % 3);
      int my_dst = -1;
      float fc = 0.f, d = 0.f;
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
          ok = true;
        } else {
          raise_status(status, kStatusBounds);
        }
      }
      M->src[t] = j;
      M->fc[t] = fc;
      s_pdst[t] = my_dst;
      // Gaussian operand row (bf16), bias column R = 1, zero padding
      const float d0 = d - rp.mu_min;
      uint8_t* A = AS(b);
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
            float val = tc::ex2f(nglog2e * dd * dd);
            if (k >= K1 - 16) val = k < rp.R ? val : (k == rp.R ? 1.f : 0.f);
            v[hh] = ok ? val : 0.f;
          }
          w[q] = tc::pack_bf16(v[0], v[1]);
        }
        *(uint4*)(A + kmaj(t, k0, K1)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      named_sync(1, 128);  // s_pdst complete
      const bool flag = (t < ne) && (t == 0 || s_pdst[t - 1] != my_dst);
      const unsigned bal = __ballot_sync(0xffffffffu, flag);
      if (lane == 0) s_misc[warp] = __popc(bal);
      named_sync(1, 128);
      int off = 0;
      for (int w2 = 0; w2 < warp; ++w2) off += s_misc[w2];
      const int slot = (t < ne) ? off + __popc(bal & ((2u << lane) - 1u)) - 1 : -1;
      if (flag) M->slot_row[slot] = my_dst;
      M->slot[t] = slot;
      if (t == 0) {
        M->nslots = s_misc[0] + s_misc[1] + s_misc[2] + s_misc[3];
        M->ne = ne;
      }
      if (t == ne - 1) s_rp[TM + 1] = my_dst;
      tc::fence_proxy_async();
      named_sync(1, 128);
      r_lo = s_rp[TM + 1];
      mbar_arrive(&bars[2 * B_FULL_A + b]);
    }
  } else if (warp == MMA_WARP) {
    // =============================================================== MMA role (one thread)
    if (lane == 0) {
      bool ok = tc::mbar_wait(&bars[2 * B_W], 0, WAIT_LIMIT);
      if (!ok) *abort_flag = 1;
      const uint32_t id12 = tc::idesc(TM, FT, 1, false, false);
      const uint32_t sW1_a = tc::smem_u32(sW1), sW2_a = tc::smem_u32(sW2);
      int n1 = 0, n2 = 0, n3 = 0;  // next tile for MMA1 / MMA2 / MMA3
      uint32_t spins = 0;
      while (ok && n3 < ntiles && !*abort_flag) {
        bool issued = false;
        // MMA3(n3): messages and 0/1 matrix written
        if (n3 < n2) {
          const int b = n3 & 1;
          if (tc::mbar_test(&bars[2 * B_FULL_M + b], (n3 >> 1) & 1)) {
            tc::fence_after();
            const int ns = MB(n3 % 3)->nslots;
            const int n16 = ns > 0 ? (ns + 15) & ~15 : 16;
            const uint32_t id3 = tc::idesc(TM, n16, 1, true, false);
            const uint32_t sH_a = tc::smem_u32(HB(b)), sS_a = tc::smem_u32(AS(b));
            for (int ks = 0; ks < TM / 16; ++ks)
              tc::mma(tmem + 128 * b, tc::sdesc(sH_a + ks * 256, 128, 2048),
                      tc::sdesc(sS_a + ks * 256, 128, TM * 16), id3, ks > 0);
            tc::commit(&bars[2 * B_DONE3 + b]);
            ++n3;
            issued = true;
          }
        }
        // MMA2(n2): h' written
        if (!issued && n2 < n1) {
          const int b = n2 & 1;
          if (tc::mbar_test(&bars[2 * B_FULL_H + b], (n2 >> 1) & 1)) {
            tc::fence_after();
            const uint32_t sH_a = tc::smem_u32(HB(b));
            for (int ks = 0; ks < K2 / 16; ++ks)
              tc::mma(tmem + 128 * b, tc::sdesc(sH_a + ks * 256, 128, K2 * 16),
                      tc::sdesc(sW2_a + ks * 256, 128, K2 * 16), id12, ks > 0);
            tc::commit(&bars[2 * B_DONE2 + b]);
            ++n2;
            issued = true;
          }
        }
        // MMA1(n1): Gaussian operand written and accumulator b free
        if (!issued && n1 < ntiles && n1 < n3 + 2) {
          const int b = n1 & 1;
          if (tc::mbar_test(&bars[2 * B_FULL_A + b], (n1 >> 1) & 1) &&
              (n1 < 2 || tc::mbar_test(&bars[2 * B_FREE_T + b], ((n1 - 2) >> 1) & 1))) {
            tc::fence_after();
            const uint32_t sA_a = tc::smem_u32(AS(b));
            for (int ks = 0; ks < K1 / 16; ++ks)
              tc::mma(tmem + 128 * b, tc::sdesc(sA_a + ks * 256, 128, K1 * 16),
                      tc::sdesc(sW1_a + ks * 256, 128, K1 * 16), id12, ks > 0);
            tc::commit(&bars[2 * B_DONE1 + b]);
            ++n1;
            issued = true;
          }
        }
        if (issued) {
          spins = 0;
        } else if (++spins > (WAIT_LIMIT >> 2)) {
          *abort_flag = 1;
        } else {
          __nanosleep(64);  // leave the issue slots of this scheduler to the epilogue warps
        }
      }
      // let the last MMA finish before the CTA frees its TMEM
      if (n3 > 0) tc::mbar_wait(&bars[2 * B_DONE3 + ((n3 - 1) & 1)], ((n3 - 1) >> 1) & 1, WAIT_LIMIT);
    }
  } else {
    // =============================================================== epilogue role (256 threads)
    const int ew = warp - EPI_WARP0;        // 0..7
    const int q4 = warp & 3, half = ew >> 2;
    const int e_me = 32 * q4 + lane;        // edge = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
    float carry = 0.f;
    int carry_row = -1, next_row = r_begin;
    auto write_row = [&](int row, float v) {  // drain threads: half 0, feature f = e_me
      for (int rr = next_row; rr < row; ++rr) out[(size_t)rr * FT + e_me] = __float2bfloat16_rn(0.f);
      out[(size_t)row * FT + e_me] = __float2bfloat16_rn(v);
      next_row = row + 1;
    };
    // epi-1 of tile i: h' = f_c ssp(z1) -> H[b]; the 0/1 matrix area is cleared
    auto epi1 = [&](int i) -> bool {
      const int b = i & 1;
      if (named_sync_or(2, 256, !wait_bar(B_DONE1, b, (i >> 1) & 1))) return false;
      tc::fence_after();
      const WsMeta* M = MB(i % 3);
      const float fc = M->fc[e_me];
      uint8_t* H = HB(b);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int f0 = 64 * half + 32 * c;
        uint32_t r[32];
        tc::ld32(lane_base + 128 * b + f0, r);
        tc::ld_wait();
#pragma unroll
        for (int g8 = 0; g8 < 4; ++g8) {
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float a = ssp_fc_poly(__uint_as_float(r[8 * g8 + 2 * q]), fc);
            const float bb = ssp_fc_poly(__uint_as_float(r[8 * g8 + 2 * q + 1]), fc);
            w[q] = tc::pack_bf16(a, bb);
          }
          *(uint4*)(H + kmaj(e_me, f0 + 8 * g8, K2)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      // clear the 0/1 matrix rows this tile uses (the Gaussian operand is consumed)
      const int ns = M->nslots;
      const int n16 = ns > 0 ? (ns + 15) & ~15 : 16;
      uint4* z = (uint4*)AS(b);
      for (int k = e_me + 128 * half; k < n16 * TM * 2 / 16; k += 256) z[k] = make_uint4(0, 0, 0, 0);
      tc::fence_proxy_async();
      tc::fence_before();
      mbar_arrive(&bars[2 * B_FULL_H + b]);
      return true;
    };
    // epi-2 of tile i: msg = x_j (.) (u + f_c c2) -> H[b] (MN-major); 0/1 matrix ones
    auto epi2 = [&](int i) -> bool {
      const int b = i & 1;
      const WsMeta* M = MB(i % 3);
      const float fc = M->fc[e_me];
      const uint4* xr = (const uint4*)(x + (size_t)M->src[e_me] * FT) + 8 * half;
      uint4 xv[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) xv[q] = __ldg(xr + q);
      if (named_sync_or(2, 256, !wait_bar(B_DONE2, b, (i >> 1) & 1))) return false;
      tc::fence_after();
      uint8_t* H = HB(b);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int f0 = 64 * half + 32 * c;
        uint32_t r[32];
        tc::ld32(lane_base + 128 * b + f0, r);
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
            const float W0 = fmaf(fc, cc[2 * q], __uint_as_float(r[8 * g8 + 2 * q]));
            const float W1 = fmaf(fc, cc[2 * q + 1], __uint_as_float(r[8 * g8 + 2 * q + 1]));
            w[q] = tc::pack_bf16(W0 * bf_lo(xw[q]), W1 * bf_hi(xw[q]));
          }
          *(uint4*)(H + (f8 >> 3) * 2048 + (e_me >> 3) * 128 + (e_me & 7) * 16) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      named_sync(2, 256);  // every thread's clearing of the 0/1 matrix is done
      if (half == 0) {
        const int sl = M->slot[e_me];
        if (sl >= 0) *(uint16_t*)(AS(b) + kmaj(sl, e_me, TM)) = (uint16_t)0x3F80;  // bf16 1.0
      }
      tc::fence_proxy_async();
      tc::fence_before();
      mbar_arrive(&bars[2 * B_FULL_M + b]);
      return true;
    };
    // drain of tile i: the segment sums of each destination row, written once (half 0 threads)
    auto drain = [&](int i) -> bool {
      const int b = i & 1;
      if (named_sync_or(2, 256, !wait_bar(B_DONE3, b, (i >> 1) & 1))) return false;
      tc::fence_after();
      const WsMeta* M = MB(i % 3);
      const int ns = M->nslots;
      if (half == 0) {
#pragma unroll 1
        for (int sidx = 0; sidx < ns; ++sidx) {
          uint32_t rv;
          tc::ld1(lane_base + 128 * b + sidx, rv);
          tc::ld_wait();
          const int row = M->slot_row[sidx];
          float v = __uint_as_float(rv);
          if (row == carry_row) {
            v += carry;
          } else if (carry_row >= 0) {
            write_row(carry_row, carry);
          }
          carry_row = -1;
          if (sidx == ns - 1) {
            carry = v;
            carry_row = row;
          } else {
            write_row(row, v);
          }
        }
      }
      tc::fence_before();
      mbar_arrive(&bars[2 * B_FREE_T + b]);
      return true;
    };
    bool ok = ntiles > 0 ? epi1(0) : true;
    for (int i = 0; ok && i < ntiles; ++i) {
      ok = epi2(i);
      if (ok && i + 1 < ntiles) ok = epi1(i + 1);
      if (ok) ok = drain(i);
    }
    if (ok && half == 0) {
      if (carry_row >= 0) write_row(carry_row, carry);
      for (int rr = next_row; rr < r_end; ++rr) out[(size_t)rr * FT + e_me] = __float2bfloat16_rn(0.f);
    }
  }
  tc::fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag) raise_status(status, kStatusTimeout);
  if (warp == 0) tc::tmem_dealloc(tmem, 256);
}

}  // namespace

int tc_cfconv_fwd_ws(mp_ctx* ctx, int block, int N, long long E, const float* pos,
                     const int* row_ptr, const int* col_idx, const void* x, void* out,
                     cudaStream_t s) {
  const int K1 = k1_of(ctx->cfg.n_rbf);
  const ImgLayout IL = img_layout(K1);
  const uint8_t* img = (const uint8_t*)ctx->tc_weights + IL.bytes * block;
  long long tiles = (E + TM - 1) / TM;
  int grid = ctx->num_sms;
  if (tiles < grid) grid = (int)(tiles > 0 ? tiles : 1);
  auto go = [&](auto kern, int k1) {
    const size_t smem = ws_layout(k1).total + 1024;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return launch(ctx, K_CFCONV_FWD_TC, kern, dim3(grid), dim3(WS_THREADS), smem, s, N, E, pos,
                  row_ptr, col_idx, (const __nv_bfloat16*)x, (__nv_bfloat16*)out, img,
                  radial_of(ctx), ctx->status_d);
  };
  if (K1 == 64) return go(k_cfconv_fwd_ws<64>, 64);
  if (K1 == 80) return go(k_cfconv_fwd_ws<80>, 80);
  if (K1 == 48) return go(k_cfconv_fwd_ws<48>, 48);
  if (K1 == 32) return go(k_cfconv_fwd_ws<32>, 32);
  return MP_ERR_INVALID_ARG;
}

}  // namespace mp
