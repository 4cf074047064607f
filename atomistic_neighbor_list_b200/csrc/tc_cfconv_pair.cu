// Undirected-pair cfconv forward on the tensor cores (bf16 path, F = 128): the filter once per
// pair {i, j}, both messages from it (FlashSchNet page, 2.3: the symmetric list; 2.4: the filter
// MLP on the tensor cores). The plan (pairs.cu) hands each CTA a contiguous run of tiles; a tile
// holds 128 pairs (i, j), i < j, of one block pair (I, J) of 128-atom blocks. Per tile:
//   MMA1   z1 = e . [A1; c1]                                   (the Gaussian operand of the pairs)
//   E1     h' = f_c ssp(z1)
//   MMA2   u = h' A2;  W = u + f_c c2 (one filter per pair)
//   E2     msg_I = x_j (.) W   ->  MMA3_I: m_I^T += msg_I^T S_I^T  (S_I: pair -> i mod 128)
//          msg_J = x_i (.) W   ->  MMA3_J: m_J^T += msg_J^T S_J^T  (m_I when I = J), from the
//          same W once MMA3_I has read the message buffer
//   DR     when a run of m_I or m_J ends (block row or block pair changes, or the CTA's run
//          ends), the rows it touched are written as one fp32 partial block with a row mask;
//          k_pair_sum adds them per row in a fixed order. No atomics, no edge-sized tensor.
// Roles (22 warps, as in the directed kernel of tc_cfconv_ws.cu): prep 0-3, epilogue 4-19 (four
// warps per TMEM lane quarter, 32 features each; per warp E2(i), E1(i+1), DR(i)), MMA1
// warp 20, MMA2/MMA3 warp 21. TMEM: z1/u of two tiles (2 x 128 columns), m_I, m_J (128 each).
// The 0/1 matrix S stays zero but for one entry per pair: each pair's thread clears the entry it
// set for the previous product and sets the next one. Every wait is bounded.
#include "tc_common.cuh"

namespace mp {
namespace {
using namespace tcc;

constexpr int NEPI = 16;
constexpr int FPT = FT * 4 / NEPI;  // 32 features per epilogue thread
constexpr int PREP_WARPS = 4, EPI_WARP0 = 4, MMA1_WARP = EPI_WARP0 + NEPI, MMA23_WARP = MMA1_WARP + 1;
constexpr int PW_THREADS = 32 * (MMA23_WARP + 1);  // 22 warps
constexpr int NMETA = 4;
constexpr unsigned FULL = 0xffffffffu;
constexpr uint32_t COL_MI = 256, COL_MJ = 384;  // TMEM columns of m_I^T and m_J^T

struct PairMeta {
  int srcJ[TM];  // j of each pair slot (0 on padding): x_j for the message to row i
  int srcI[TM];  // i: x_i for the message to row j
  float fc[TM];  // envelope (0 on padding)
  int rI[TM];    // i mod 128, -1 on padding: the pair's row in S_I
  int rJ[TM];    // j mod 128: its row in S_J
  // rows of the tile's pairs, per prep warp: words 0-3 the i rows, 4-7 the j rows (bit r & 31 of
  // word r >> 5)
  uint32_t rows[PREP_WARPS][8];
  int flags, slotI, slotJ, pad;
};
struct PwSmem {
  uint32_t w1, w2, c2, a0, s, h0, x, meta0, misc, bars, total;
};
__host__ __device__ constexpr int pw_nbuf_a(int K1) { return K1 <= 64 ? 2 : 1; }
__host__ __device__ constexpr PwSmem pw_layout(int K1) {
  // W1, W2, c2 | Gaussian operand x NA | S | h' / msg^T x2 | x_j rows | metadata x4 | misc | bars
  PwSmem L{};
  uint32_t o = 0;
  L.w1 = o;    o += FT * K1 * 2;
  L.w2 = o;    o += FT * K2 * 2;
  L.c2 = o;    o += 1024;
  L.a0 = o;    o += pw_nbuf_a(K1) * TM * K1 * 2;
  L.s = o;     o += TM * TM * 2;
  L.h0 = o;    o += 2 * TM * K2 * 2;
  L.x = o;     o += TM * FT * 2;
  L.meta0 = o; o += NMETA * (uint32_t)sizeof(PairMeta);
  L.misc = o;  o += 64;
  L.bars = o;  o += 256;
  L.total = o;
  return L;
}
__host__ __device__ constexpr bool pw_fits(int K1) {
  return pw_layout(K1).total + 1024 <= 227 * 1024 && pw_layout(K1).x % 1024 == 0;
}
// staged x_j rows, as in the directed kernel: chunks permuted within each half row
__device__ __forceinline__ uint32_t xoff(int r, int c) {
  return (uint32_t)(r * (FT * 2) + ((c ^ (r & 7)) << 4));
}

enum {
  B_FULL_A = 0,     // prep -> MMA1: Gaussian operand and metadata (128 arrivals)
  B_DONE1 = 2,      // MMA1 complete
  B_FULL_H = 4,     // h' written (one arrival per epilogue warp)
  B_DONE2 = 6,      // MMA2 complete
  B_FULL_M = 8,     // msg_I^T and S_I written
  B_DONE3A = 10,    // MMA3_I complete
  B_FULL_M2 = 12,   // msg_J^T and S_J written
  B_DONE3B = 14,    // MMA3_J complete
  B_FREE_T = 16,    // the tile's z1/u columns free (and its partials written)
  B_W = 18, B_XFULL = 19, B_XFREE = 20, B_FIN1 = 21, B_FIN2 = 22,
  N_BARS = 24
};

template <int K1>
__global__ void __launch_bounds__(PW_THREADS, 1) k_cfconv_pair_fwd(
    int N, int T, const PairTile* __restrict__ tiles, const int2* __restrict__ tpairs,
    const float* __restrict__ pos, const __nv_bfloat16* __restrict__ x,
    float* __restrict__ partial, uint32_t* __restrict__ pmask,
    const uint8_t* __restrict__ img, Radial rp, int* status, unsigned long long wait_ns) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr PwSmem L = pw_layout(K1);
  constexpr int NA = pw_nbuf_a(K1);
  uint8_t* sW1 = sm + L.w1;
  uint8_t* sW2 = sm + L.w2;
  float* sc2 = (float*)(sm + L.c2);
  uint8_t* sS = sm + L.s;
  uint8_t* sX = sm + L.x;
  auto AB = [&](int b) { return sm + L.a0 + (uint32_t)b * (TM * K1 * 2); };
  auto HB = [&](int b) { return sm + L.h0 + (uint32_t)b * (TM * K2 * 2); };
  auto MB = [&](int k) { return (PairMeta*)(sm + L.meta0) + k; };
  int* s_misc = (int*)(sm + L.misc);  // [10] abort
  uint64_t* bars = (uint64_t*)(sm + L.bars);
  uint32_t* s_tmem = (uint32_t*)(bars + N_BARS);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int t_begin = (int)((long long)T * cta / G), t_end = (int)((long long)T * (cta + 1) / G);
  const int ntiles = t_end - t_begin;
  if (ntiles <= 0) return;

  if (warp == 0) tc::tmem_alloc(s_tmem, 512);
  if (tid == 0) {
    s_misc[10] = 0;
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&bars[B_FULL_A + b], 128);
      tc::mbar_init(&bars[B_DONE1 + b], 1);
      tc::mbar_init(&bars[B_FULL_H + b], NEPI);
      tc::mbar_init(&bars[B_DONE2 + b], 1);
      tc::mbar_init(&bars[B_FULL_M + b], NEPI);
      tc::mbar_init(&bars[B_DONE3A + b], 1);
      tc::mbar_init(&bars[B_FULL_M2 + b], NEPI);
      tc::mbar_init(&bars[B_DONE3B + b], 1);
      tc::mbar_init(&bars[B_FREE_T + b], NEPI);
    }
    tc::mbar_init(&bars[B_W], 1);
    tc::mbar_init(&bars[B_XFULL], 128);
    tc::mbar_init(&bars[B_XFREE], NEPI);
    tc::mbar_init(&bars[B_FIN1], 1);
    tc::mbar_init(&bars[B_FIN2], 1);
    const ImgLayout IL = img_layout(K1);
    tc::mbar_expect_tx(&bars[B_W], FT * K1 * 2 + FT * K2 * 2 + FT * 4);
    tc::bulk_g2s(sW1, img + IL.w1, FT * K1 * 2, &bars[B_W]);
    tc::bulk_g2s(sW2, img + IL.w2, FT * K2 * 2, &bars[B_W]);
    tc::bulk_g2s(sc2, img + IL.c2, FT * 4, &bars[B_W]);
  }
  // S starts at zero; from then on only single entries change
  for (int k = tid; k < TM * TM * 2 / 16; k += PW_THREADS)
    *(uint4*)(sS + 16 * k) = make_uint4(0u, 0u, 0u, 0u);
  tc::fence_proxy_async();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *s_tmem;
  volatile int* abort_flag = &s_misc[10];
  auto wait_bar = [&](int idx, uint32_t parity) -> bool {
    if (tc::mbar_wait_ns(&bars[idx], parity, WAIT_LIMIT, wait_ns)) return true;
    *abort_flag = 1;
    return false;
  };
  const uint32_t id12 = tc::idesc(TM, FT, 1, false, false);

  if (warp < PREP_WARPS) {
    // =============================================================== prep role (128 threads)
    const int t = tid;
    const float xs = sqrtf(rp.gamma * LOG2E), dmu_x = rp.dmu * xs;
    const float rstep = tc::ex2f(-2.f * dmu_x * dmu_x), pi_rc = 3.14159265358979f / rp.r_c;
    // the x_j rows of tile k, once every epilogue warp has read those of tile k-1
    auto gather = [&](int k) -> bool {
      const bool ok = k < 1 || wait_bar(B_XFREE, (k - 1) & 1);
      if (bar_sync_or(1, 128, !ok || *abort_flag)) return false;
      const int* src = MB(k % NMETA)->srcJ;
      const int c = t & 15;
#pragma unroll 4
      for (int p = 0; p < TM / 8; ++p) {
        const int r = 8 * p + (t >> 4);
        tc::cp_async16(sX + xoff(r, c), x + (size_t)src[r] * FT + 8 * c);
      }
      tc::cp_async_arrive(&bars[B_XFULL]);
      return true;
    };
    // loads run ahead of their tile: the pair slot two tiles ahead, its positions one tile ahead
    auto load_pair = [&](int k) -> int2 {
      return k < ntiles ? tpairs[(size_t)(t_begin + k) * TM + t] : make_int2(-1, -1);
    };
    auto valid = [&](int2 pr) {
      return pr.x >= 0 && pr.x < N && pr.y >= 0 && pr.y < N;
    };
    struct PPos { float ix, iy, iz, jx, jy, jz; };
    auto load_pos = [&](int2 pr) {
      PPos P{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (valid(pr)) {
        P.ix = pos[3 * pr.x]; P.iy = pos[3 * pr.x + 1]; P.iz = pos[3 * pr.x + 2];
        P.jx = pos[3 * pr.y]; P.jy = pos[3 * pr.y + 1]; P.jz = pos[3 * pr.y + 2];
      } else if (pr.x != -1 || pr.y != -1) {
        raise_status(status, kStatusBounds);
      }
      return P;
    };
    int2 pr0 = load_pair(0), pr1 = load_pair(1);
    PPos P0 = load_pos(pr0);
    bool live = true;
    for (int it = 0; it < ntiles; ++it) {
      const int b = it & 1;
      const int2 pr2 = load_pair(it + 2);
      const PPos P1 = load_pos(pr1);
      const PairTile D = tiles[t_begin + it];
      // Gaussian operand buffer it % NA is free once MMA1 of tile it - NA completed (and with it
      // the metadata slot of tile it-4: its partials were written before that MMA1)
      const bool free_ok =
          it < NA || wait_bar(B_DONE1 + ((it - NA) & 1), ((it - NA) >> 1) & 1);
      if (bar_sync_or(1, 128, !free_ok || *abort_flag)) {
        live = false;
        break;
      }
      // the x_j rows of the previous tile first: they are needed one tile sooner than this one
      if (it > 0 && !gather(it - 1)) {
        live = false;
        break;
      }
      PairMeta* M = MB(it % NMETA);
      const bool ok = valid(pr0);
      float d = 0.f, fc = 0.f;
      if (ok) {
        const float dx = P0.ix - P0.jx, dy = P0.iy - P0.jy, dz = P0.iz - P0.jz;
        d = sqrtf(dx * dx + dy * dy + dz * dz);
        if (d < rp.r_c) fc = 0.5f * (__cosf(pi_rc * d) + 1.f);  // argument in [0, pi)
      }
      M->srcJ[t] = ok ? pr0.y : 0;
      M->srcI[t] = ok ? pr0.x : 0;
      M->fc[t] = fc;
      M->rI[t] = ok ? (pr0.x & 127) : -1;
      M->rJ[t] = ok ? (pr0.y & 127) : -1;
      {  // this warp's share of the tile's row sets
        const int wi = ok ? (pr0.x & 127) : -1, wj = ok ? (pr0.y & 127) : -1;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t mi = __reduce_or_sync(FULL, (wi >> 5) == q ? 1u << (wi & 31) : 0u);
          const uint32_t mj = __reduce_or_sync(FULL, (wj >> 5) == q ? 1u << (wj & 31) : 0u);
          if (lane == 0) {
            M->rows[warp][q] = mi;
            M->rows[warp][4 + q] = mj;
          }
        }
      }
      if (t == 0) {
        M->flags = D.flags;
        M->slotI = D.slotI;
        M->slotJ = D.slotJ;
      }
      // Gaussian operand row (bf16), bias column R = 1; zero on a padding slot. e_k = 2^(-x_k^2)
      // on the scaled distance by the two-ex2-per-eight-centres recurrence of the directed kernel
      const float xk00 = (d - rp.mu_min) * xs;
      uint8_t* A = AB(it % NA);
#pragma unroll
      for (int k0 = 0; k0 < K1; k0 += 8) {
        const float xk0 = fmaf(-(float)k0, dmu_x, xk00);
        float ek = tc::ex2f(-(xk0 * xk0));
        float rk = tc::ex2f(dmu_x * fmaf(2.f, xk0, -dmu_x));
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float v[2];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int k = k0 + 2 * q + hh;
            float val = ek;
            if (k >= K1 - 16) val = k < rp.R ? val : (k == rp.R ? 1.f : 0.f);
            v[hh] = ok ? val : 0.f;
            ek *= rk;
            rk *= rstep;
          }
          w[q] = tc::pack_bf16(v[0], v[1]);
        }
        *(uint4*)(A + kmaj(t, k0, K1)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      tc::fence_proxy_async();
      bar_sync(1, 128);
      mbar_arrive1(&bars[B_FULL_A + b]);
      // the loads issued at the top of this tile are consumed from here on
      pr0 = pr1;
      P0 = P1;
      pr1 = pr2;
    }
    if (live) gather(ntiles - 1);
    tc::cp_async_wait_all();  // nothing in flight when the CTA exits
  } else if (warp == MMA1_WARP) {
    // =============================================================== MMA1 (lane 0 issues)
    auto wait_w = [&](int idx, uint32_t parity) -> bool {
      return !__any_sync(FULL, !wait_bar(idx, parity));
    };
    bool ok = wait_w(B_W, 0);
    const uint32_t sW1_a = tc::smem_u32(sW1);
    for (int n = 0; ok && n < ntiles; ++n) {
      if (__any_sync(FULL, *abort_flag != 0)) break;
      const int b = n & 1;
      ok = wait_w(B_FULL_A + b, (n >> 1) & 1) &&
           (n < 2 || wait_w(B_FREE_T + b, ((n - 2) >> 1) & 1));
      if (!ok) break;
      tc::fence_after();
      if (lane == 0) {
        const uint32_t sA_a = tc::smem_u32(AB(n % NA));
        for (int ks = 0; ks < K1 / 16; ++ks)
          tc::mma(tmem + 128 * b, tc::sdesc(sA_a + ks * 256, 128, K1 * 16),
                  tc::sdesc(sW1_a + ks * 256, 128, K1 * 16), id12, ks > 0);
        tc::commit(&bars[B_DONE1 + b]);
      }
      __syncwarp();
    }
    if (!ok) *abort_flag = 1;
    if (lane == 0) {
      tc::commit(&bars[B_FIN1]);
      tc::mbar_wait(&bars[B_FIN1], 0, WAIT_LIMIT);
    }
  } else if (warp == MMA23_WARP) {
    // =============================================================== MMA2, MMA3_I, MMA3_J
    if (lane == 0) {
      bool ok = wait_bar(B_W, 0);
      const uint32_t sW2_a = tc::smem_u32(sW2), sS_a = tc::smem_u32(sS);
      const uint32_t id3 = tc::idesc(TM, TM, 1, true, false);
      for (int i = 0; ok && i < ntiles && !*abort_flag; ++i) {
        const int b = i & 1;
        const uint32_t par = (i >> 1) & 1;
        if (!(ok = wait_bar(B_FULL_H + b, par))) break;
        tc::fence_after();
        const uint32_t sH_a = tc::smem_u32(HB(b));
        for (int ks = 0; ks < K2 / 16; ++ks)
          tc::mma(tmem + 128 * b, tc::sdesc(sH_a + ks * 256, 128, K2 * 16),
                  tc::sdesc(sW2_a + ks * 256, 128, K2 * 16), id12, ks > 0);
        tc::commit(&bars[B_DONE2 + b]);
        const int flags = MB(i % NMETA)->flags;
        // D^T[F x 128 rows] (+)= msg^T (MN-major) . S^T (K-major); a run starts without the add
        if (!(ok = wait_bar(B_FULL_M + b, par))) break;
        tc::fence_after();
        for (int ks = 0; ks < TM / 16; ++ks)
          tc::mma(tmem + COL_MI, tc::sdesc(sH_a + ks * 256, 128, 2048),
                  tc::sdesc(sS_a + ks * 256, 128, TM * 16), id3,
                  ks > 0 || (flags & kPairAccI) != 0);
        tc::commit(&bars[B_DONE3A + b]);
        if (!(ok = wait_bar(B_FULL_M2 + b, par))) break;
        tc::fence_after();
        const bool diag = (flags & kPairDiag) != 0;
        for (int ks = 0; ks < TM / 16; ++ks)
          tc::mma(tmem + (diag ? COL_MI : COL_MJ), tc::sdesc(sH_a + ks * 256, 128, 2048),
                  tc::sdesc(sS_a + ks * 256, 128, TM * 16), id3,
                  ks > 0 || diag || (flags & kPairAccJ) != 0);
        tc::commit(&bars[B_DONE3B + b]);
      }
      if (!ok) *abort_flag = 1;
      tc::commit(&bars[B_FIN2]);
      tc::mbar_wait(&bars[B_FIN2], 0, WAIT_LIMIT);
    }
  } else {
    // =============================================================== epilogue (16 warps)
    const int ew = warp - EPI_WARP0;          // 0..15
    const int q4 = warp & 3, part = ew >> 2;  // TMEM lane quarter, feature quarter
    const int f0 = FPT * part;
    const int e_me = 32 * q4 + lane;          // pair slot = TMEM lane (DR: feature)
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
    int rJ_prev = -1;  // part 0: the S entry this pair slot set for the previous MMA3_J
    // rows [32 part, 32 part + 32) that the current runs of m_I and m_J have touched
    uint32_t runI = 0u, runJ = 0u;
    auto wait_warp = [&](int idx, uint32_t parity) -> bool {
      return !__any_sync(FULL, !wait_bar(idx, parity));
    };
    auto arrive_warp = [&](int idx) {
      tc::fence_proxy_async();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive1(&bars[idx]);
    };
    auto setS = [&](int row, uint16_t v) {
      if (row >= 0) *(uint16_t*)(sS + kmaj(row, e_me, TM)) = v;
    };
    // E1 of tile i: h' = f_c ssp(z1) -> H[b]
    auto E1 = [&](int i) -> bool {
      const int b = i & 1;
      if (!wait_warp(B_DONE1 + b, (i >> 1) & 1)) return false;
      tc::fence_after();
      const float fc = MB(i % NMETA)->fc[e_me], fcln2 = fc * LN2;
      uint8_t* H = HB(b);
      uint32_t r[32];
      tc::ld32(lane_base + 128 * b + f0, r);
      tc::ld_wait();
#pragma unroll
      for (int g8 = 0; g8 < 4; ++g8) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int k = 8 * g8 + 2 * q;
          w[q] = ssp_scaled_bf16x2(__uint_as_float(r[k]), __uint_as_float(r[k + 1]), fc, fcln2);
        }
        *(uint4*)(H + kmaj(e_me, f0 + 8 * g8, K2)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      arrive_warp(B_FULL_H + b);
      return true;
    };
    // W = u + f_c c2 of tile i for this thread's 32 features (u read from TMEM)
    auto filter = [&](int i, float* W) {
      const int b = i & 1;
      const float fc = MB(i % NMETA)->fc[e_me];
      uint32_t r[32];
      tc::ld32(lane_base + 128 * b + f0, r);
      tc::ld_wait();
#pragma unroll
      for (int g8 = 0; g8 < 4; ++g8) {
        const float4 ca = *(const float4*)(sc2 + f0 + 8 * g8);
        const float4 cb = *(const float4*)(sc2 + f0 + 8 * g8 + 4);
        const float cc[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) W[8 * g8 + k] = fmaf(fc, cc[k], __uint_as_float(r[8 * g8 + k]));
      }
    };
    // a message y (.) W into H[b] as msg^T (MN-major)
    auto message = [&](int i, const uint4* yv, const float* W) {
      uint8_t* H = HB(i & 1);
#pragma unroll
      for (int g8 = 0; g8 < 4; ++g8) {
        const uint4 yq = yv[g8];
        const uint32_t yw[4] = {yq.x, yq.y, yq.z, yq.w};
        const int f8 = f0 + 8 * g8;
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          w[q] = tc::pack_bf16(W[8 * g8 + 2 * q] * bf_lo(yw[q]),
                               W[8 * g8 + 2 * q + 1] * bf_hi(yw[q]));
        *(uint4*)(H + (f8 >> 3) * 2048 + (e_me >> 3) * 128 + (e_me & 7) * 16) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
    };
    // E2 of tile i: msg_I = x_j (.) W and S_I -> MMA3_I; once MMA3_I has read H[b] and S,
    // msg_J = x_i (.) W (the same W, kept in registers) and S_J -> MMA3_J
    auto E2 = [&](int i) -> bool {
      const int b = i & 1;
      const PairMeta* M = MB(i % NMETA);
      if (!wait_warp(B_XFULL, i & 1)) return false;
      uint4 xv[FPT / 8];
#pragma unroll
      for (int q = 0; q < FPT / 8; ++q) xv[q] = *(const uint4*)(sX + xoff(e_me, f0 / 8 + q));
      __syncwarp();
      if (lane == 0) mbar_arrive1(&bars[B_XFREE]);
      if (!wait_warp(B_DONE2 + b, (i >> 1) & 1)) return false;
      tc::fence_after();
      float W[32];
      filter(i, W);
      message(i, xv, W);
      // W kept for the second message as fp16 pairs (10-bit mantissa, below the message's bf16
      // rounding), so that it holds 16 registers across the wait
      uint32_t Wh[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const __half2 h = __floats2half2_rn(W[2 * k], W[2 * k + 1]);
        Wh[k] = *(const uint32_t*)&h;
      }
      if (part == 0) {  // MMA3_J of tile i-1 has completed (this warp saw it in DR(i-1))
        setS(rJ_prev, 0);
        setS(M->rI[e_me], 0x3F80);
      }
      arrive_warp(B_FULL_M + b);
      uint4 xi[FPT / 8];  // x_i, requested while MMA3_I runs
      {
        const uint4* xr = (const uint4*)(x + (size_t)M->srcI[e_me] * FT + f0);
#pragma unroll
        for (int q = 0; q < FPT / 8; ++q) xi[q] = __ldg(xr + q);
      }
      if (!wait_warp(B_DONE3A + b, (i >> 1) & 1)) return false;
      tc::fence_after();
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const float2 w2 = __half22float2(*(const __half2*)&Wh[k]);
        W[2 * k] = w2.x;
        W[2 * k + 1] = w2.y;
      }
      message(i, xi, W);
      if (part == 0) {
        setS(M->rI[e_me], 0);
        rJ_prev = M->rJ[e_me];
        setS(rJ_prev, 0x3F80);
      }
      arrive_warp(B_FULL_M2 + b);
      return true;
    };
    // DR of tile i: partial rows of the runs that end here (thread = feature 32 q4 + lane; the
    // four warps of a lane quarter take 32 rows each), then the tile's columns are free
    auto DR = [&](int i) -> bool {
      const int b = i & 1;
      if (!wait_warp(B_DONE3B + b, (i >> 1) & 1)) return false;
      tc::fence_after();
      const PairMeta* M = MB(i % NMETA);
      const int flags = M->flags;
      const int f = 32 * q4 + lane;
      uint32_t ti = 0u, tj = 0u;
#pragma unroll
      for (int w = 0; w < PREP_WARPS; ++w) {
        ti |= M->rows[w][part];
        tj |= M->rows[w][4 + part];
      }
      if (flags & kPairDiag) {
        ti |= tj;
        tj = 0u;
      }
      runI = ((flags & kPairAccI) ? runI : 0u) | ti;
      if (!(flags & kPairDiag)) runJ = ((flags & kPairAccJ) ? runJ : 0u) | tj;
#pragma unroll 1
      for (int side = 0; side < 2; ++side) {
        const bool go = side == 0 ? (flags & kPairFlushI) != 0 : (flags & kPairFlushJ) != 0;
        if (!go) continue;
        const int slot = side == 0 ? M->slotI : M->slotJ;
        const uint32_t rows = side == 0 ? runI : runJ;
        if (lane == 0) pmask[(size_t)slot * 4 + part] = rows;
        if (rows == 0u) continue;  // none of this warp's 32 rows was touched
        uint32_t r[32];
        tc::ld32(lane_base + (side == 0 ? COL_MI : COL_MJ) + 32 * part, r);
        tc::ld_wait();
        float* dst = partial + ((size_t)slot * TM + 32 * part) * FT + f;
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if ((rows >> k) & 1u) dst[(size_t)k * FT] = __uint_as_float(r[k]);
      }
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive1(&bars[B_FREE_T + b]);
      return true;
    };
    bool ok = wait_warp(B_W, 0);  // c2 is read in the messages
    if (ok) ok = E1(0);
    for (int i = 0; ok && i < ntiles; ++i) {
      ok = E2(i);
      if (ok && i + 1 < ntiles) ok = E1(i + 1);
      if (ok) ok = DR(i);
    }
  }
  // the weight copy has landed before the CTA exits, whatever the roles gave up on (full budget)
  if (tid == 0) tc::mbar_wait(&bars[B_W], 0, WAIT_LIMIT);
  tc::fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag) raise_status(status, kStatusTimeout);
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

}  // namespace

int tc_cfconv_fwd_pairs(mp_ctx* ctx, int block, int N, const float* pos, const void* x, void* out,
                        cudaStream_t s) {
  const PairPlan& P = ctx->pair;
  if (!P.valid || P.N != N || P.G != ctx->num_sms) return MP_ERR_INVALID_ARG;
  const int K1 = k1_of(ctx->cfg.n_rbf);
  const ImgLayout IL = img_layout(K1);
  const uint8_t* img = (const uint8_t*)ctx->tc_weights + IL.bytes * block;
  int rc = MP_OK;
  if (P.T > 0) {
    auto go = [&](auto kern, int k1) {
      const size_t smem = pw_layout(k1).total + 1024;
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      return launch(ctx, K_CFCONV_PAIR_TC, kern, dim3(P.G), dim3(PW_THREADS), smem, s, N, P.T,
                    (const PairTile*)P.tiles, (const int2*)P.tpairs, pos,
                    (const __nv_bfloat16*)x, P.part, P.pmask, img, radial_of(ctx), ctx->status_d,
                    (unsigned long long)ctx->wait_ns);
    };
    static_assert(pw_fits(80) && pw_fits(64) && pw_fits(48) && pw_fits(32), "shared memory plan");
    if (K1 == 80) rc = go(k_cfconv_pair_fwd<80>, 80);
    else if (K1 == 64) rc = go(k_cfconv_pair_fwd<64>, 64);
    else if (K1 == 48) rc = go(k_cfconv_pair_fwd<48>, 48);
    else if (K1 == 32) rc = go(k_cfconv_pair_fwd<32>, 32);
    else rc = MP_ERR_INVALID_ARG;
  }
  if (rc != MP_OK) return rc;
  return pair_sum_launch(ctx, N, out, s);
}

}  // namespace mp
