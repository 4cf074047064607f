// Warp-specialised, double-buffered tensor-core cfconv forward (bf16 path, F = 128).
//
// Arithmetic as in the tile description of tc_cfconv.cu (FlashSchNet page, technical summary
// s.2.1-2.4): Gaussian basis with the bias folded into MMA1, f_c * ssp epilogue, MMA2, x_j (.) W
// epilogue, the segment sum as MMA3 with a 0/1 edge-to-row matrix, one write per row.
// Roles of one persistent CTA per SM (22 warps):
//   prep (warps 0-3)       up to two tiles ahead: row of each edge, distance, envelope, Gaussian
//                          operand, slots (tile metadata in a ring of four); then the x_j rows of
//                          the previous tile copied into a swizzled buffer (asynchronous 16-byte
//                          copies, whole rows per half warp)
//   epilogue (warps 4-19)  four warps per TMEM lane quarter, 32 features each; per warp, in the
//                          order E2(i), E1(i+1), drain(i); the warps do not meet each other:
//                          every hand-off is an mbarrier (one arrival per warp)
//   MMA1 (warp 20)         MMA1 of each tile once its Gaussian operand is written
//   MMA2/3 (warp 21)       MMA2 and MMA3 in the order the epilogue produces their operands
// Two TMEM accumulators of 128 columns and two Gaussian (one for 64 radial functions) and two h'
// operand buffers alternate between tiles; the 0/1 matrix and the x_j rows have one buffer each. Every wait is bounded; a warp that
// gives up votes so within the warp, and the other roles then run out their own bounded waits.
#include "tc_common.cuh"

namespace mp {
namespace {
using namespace tcc;

constexpr int NEPI = 16;         // epilogue warps: 4 per TMEM lane quarter
constexpr int FPT = FT * 4 / NEPI;  // features per epilogue thread (32)
constexpr int PREP_WARPS = 4, EPI_WARP0 = 4, MMA1_WARP = EPI_WARP0 + NEPI, MMA23_WARP = MMA1_WARP + 1;
constexpr int WS_THREADS = 32 * (MMA23_WARP + 1);  // 22 warps
constexpr int SMAX = 128;        // destination rows per tile (one segment-sum MMA, N <= 128)
constexpr int NMETA = 4;         // tile-metadata ring
constexpr unsigned FULL = 0xffffffffu;

struct WsMeta {
  int src[TM];
  float fc[TM];
  int slot[TM];
  int slot_row[SMAX];
  int nslots, ne, pad0, pad1;
};
struct WsSmem {
  uint32_t w1, w2, c2, a0, s, h0, x, meta0, rp, misc, bars, total;
};
// Gaussian operand buffers: two (the prep runs two tiles ahead) where they fit beside the staged
// x_j rows, one for the wider operand of 64 radial functions (K1 = 80; the prep then runs one
// tile ahead)
__host__ __device__ constexpr int ws_nbuf_a(int K1) { return K1 <= 64 ? 2 : 1; }
__host__ __device__ constexpr WsSmem ws_layout(int K1) {
  // W1, W2, c2 | Gaussian operand x2 | 0/1 matrix | h' / msg^T x2 | x_j rows | metadata x4 |
  // prep | misc | mbarriers
  WsSmem L{};
  uint32_t o = 0;
  L.w1 = o;    o += FT * K1 * 2;
  L.w2 = o;    o += FT * K2 * 2;
  L.c2 = o;    o += 1024;
  L.a0 = o;    o += ws_nbuf_a(K1) * TM * K1 * 2;
  L.s = o;     o += SMAX * TM * 2;
  L.h0 = o;    o += 2 * TM * K2 * 2;
  L.x = o;     o += TM * FT * 2;
  L.meta0 = o; o += NMETA * (uint32_t)sizeof(WsMeta);
  L.rp = o;    o += 2 * TM * 4 + 64 + 3 * TM * 4;
  L.misc = o;  o += 64;
  L.bars = o;  o += 256;
  L.total = o;
  return L;
}
constexpr int WS_SMEM_LIMIT = 227 * 1024;
__host__ __device__ constexpr bool ws_fits(int K1) {
  return ws_layout(K1).total + 1024 <= WS_SMEM_LIMIT && ws_layout(K1).x % 1024 == 0;
}
// Staged x_j rows: row r (edge of the tile), 16-byte chunk c (0..15) of its 256 bytes, chunks
// permuted within each half row so that eight consecutive rows reading the same chunk hit
// distinct banks.
__device__ __forceinline__ uint32_t xoff(int r, int c) {
  return (uint32_t)(r * (FT * 2) + ((c ^ (r & 7)) << 4));
}

// Feature f of the output rows [r0, r1) set to 0 (rows with no edges); kept out of line, it is
// rarely taken and would otherwise be inlined at every row write.
__device__ __noinline__ void zero_rows(__nv_bfloat16* out, int r0, int r1, int f) {
  for (int r = r0; r < r1; ++r) out[(size_t)r * FT + f] = __float2bfloat16_rn(0.f);
}

// mbarriers; the double-buffered ones at index + b
enum {
  B_FULL_A = 0,   // prep -> MMA1: Gaussian operand and metadata written (128 arrivals)
  B_DONE1 = 2,    // MMA1 complete
  B_FULL_H = 4,   // epilogue -> MMA2: h' written (one arrival per epilogue warp)
  B_DONE2 = 6,    // MMA2 complete
  B_FULL_M = 8,   // epilogue -> MMA3: msg^T and 0/1 matrix written (one per epilogue warp)
  B_DONE3 = 10,   // MMA3 complete
  B_FREE_T = 12,  // epilogue done with the tile's TMEM accumulator (one per epilogue warp)
  B_W = 14,       // weight images landed
  B_XFULL = 15,   // x_j rows of the tile landed (one arrival per prep thread)
  B_XFREE = 16,   // every epilogue warp has read its x_j values (one per epilogue warp)
  B_FIN1 = 17,    // completion of everything the MMA1 warp issued
  B_FIN2 = 18,    // completion of everything the MMA2/3 warp issued
  N_BARS = 20
};

template <int K1>
__global__ void __launch_bounds__(WS_THREADS, 1) k_cfconv_fwd_ws(
    int N, long long E, const float* __restrict__ pos, const int* __restrict__ row_ptr,
    const int* __restrict__ col_idx, const __nv_bfloat16* __restrict__ x,
    __nv_bfloat16* __restrict__ out, const uint8_t* __restrict__ img, Radial rp, int* status,
    unsigned long long wait_ns) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr WsSmem L = ws_layout(K1);
  constexpr int NA = ws_nbuf_a(K1);
  uint8_t* sW1 = sm + L.w1;
  uint8_t* sW2 = sm + L.w2;
  float* sc2 = (float*)(sm + L.c2);
  uint8_t* sS = sm + L.s;
  uint8_t* sX = sm + L.x;
  auto AB = [&](int b) { return sm + L.a0 + (uint32_t)b * (TM * K1 * 2); };
  auto HB = [&](int b) { return sm + L.h0 + (uint32_t)b * (TM * K2 * 2); };
  auto MB = [&](int k) { return (WsMeta*)(sm + L.meta0) + k; };
  int* s_rp = (int*)(sm + L.rp);  // prep-private row window (TM + 1), next row at [TM + 1]
  int* s_pdst = s_rp + TM + 4;    // prep-private: dst of each edge of the tile
  float* s_wpos = (float*)(s_pdst + TM + 12);  // prep-private: positions of the row window
  int* s_misc = (int*)(sm + L.misc);  // [0..3] prep warp totals, [8] r_begin, [9] r_end, [10] abort
  uint64_t* bars = (uint64_t*)(sm + L.bars);
  uint32_t* s_tmem = (uint32_t*)(bars + N_BARS);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  E = clamp_off(row_ptr[N], E);  // the edges the list holds (E may be an upper bound of them)
  if (warp < 2) {  // this CTA's rows: an edge-balanced split, both ends searched at once
    const long long bnd = E * (cta + warp) / G;
    const int r = (warp == 1 && cta == G - 1) ? N : warp_lower_row(row_ptr, N, bnd);
    if (lane == 0) s_misc[8 + warp] = r;
    if (tid == 0) s_misc[10] = 0;
  }
  __syncthreads();
  const int r_begin = s_misc[8], r_end = max(s_misc[9], s_misc[8]);
  if (r_begin >= r_end) return;
  const long long e_begin = clamp_off(row_ptr[r_begin], E);
  long long e_end = clamp_off(row_ptr[r_end], E);
  if (e_end < e_begin) e_end = e_begin;
  const int ntiles = (int)((e_end - e_begin + TM - 1) / TM);

  if (warp == 0) tc::tmem_alloc(s_tmem, 256);
  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&bars[B_FULL_A + b], 128);
      tc::mbar_init(&bars[B_DONE1 + b], 1);
      tc::mbar_init(&bars[B_FULL_H + b], NEPI);
      tc::mbar_init(&bars[B_DONE2 + b], 1);
      tc::mbar_init(&bars[B_FULL_M + b], NEPI);
      tc::mbar_init(&bars[B_DONE3 + b], 1);
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
    int r_lo = r_begin;
    // the x_j rows of tile k, once every epilogue warp has read those of tile k-1 (16 threads per
    // 256-byte row); false on abort, uniformly over the prep warps
    auto gather = [&](int k) -> bool {
      const bool ok = k < 1 || wait_bar(B_XFREE, (k - 1) & 1);
      if (bar_sync_or(1, 128, !ok || *abort_flag)) return false;
      const int* src = MB(k % NMETA)->src;
      const int c = t & 15;
#pragma unroll 4
      for (int p = 0; p < TM / 8; ++p) {
        const int r = 8 * p + (t >> 4);
        tc::cp_async16(sX + xoff(r, c), x + (size_t)src[r] * FT + 8 * c);
      }
      tc::cp_async_arrive(&bars[B_XFULL]);
      return true;
    };
    bool live = true;
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
      const int wr = min(r_lo + t, N - 1);  // the window's rows hold this tile's destinations
      const float wx = pos[3 * wr], wy = pos[3 * wr + 1], wz = pos[3 * wr + 2];
      // Gaussian operand buffer it % NA is free once MMA1 of tile it - NA completed (and with it
      // the metadata slot of tile it-4: its drain preceded that MMA1)
      const bool free_ok =
          it < NA || wait_bar(B_DONE1 + ((it - NA) & 1), ((it - NA) >> 1) & 1);
      if (bar_sync_or(1, 128, !free_ok || *abort_flag)) {  // uniform over the prep warps
        live = false;
        break;
      }
      // the x_j rows of the previous tile first: they are needed one tile sooner than this one
      if (it > 0 && !gather(it - 1)) {
        live = false;
        break;
      }
      s_rp[t] = rpv;
      if (t == 0) s_rp[TM] = rpv_last;
      s_wpos[3 * t] = wx;
      s_wpos[3 * t + 1] = wy;
      s_wpos[3 * t + 2] = wz;
      bar_sync(1, 128);
      WsMeta* M = MB(it % NMETA);
      int my_dst = -1;
      float fc = 0.f, d = 0.f;
      bool ok = false;
      if (t < ne) {
        float pix, piy, piz;
        if ((long long)s_rp[TM] <= g) {  // beyond the window (rows with many edges)
          my_dst = row_of(row_ptr, r_lo + TM, r_end, g);
          pix = pos[3 * my_dst];
          piy = pos[3 * my_dst + 1];
          piz = pos[3 * my_dst + 2];
        } else {
          int lo = 0, hi = TM;
          while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if ((long long)s_rp[mid] <= g) lo = mid; else hi = mid;
          }
          my_dst = r_lo + lo;
          pix = s_wpos[3 * lo];
          piy = s_wpos[3 * lo + 1];
          piz = s_wpos[3 * lo + 2];
        }
        if (jok) {
          const float dx = pix - pjx, dy = piy - pjy, dz = piz - pjz;
          d = sqrtf(dx * dx + dy * dy + dz * dz);
          if (d < rp.r_c) fc = 0.5f * (__cosf(pi_rc * d) + 1.f);  // argument in [0, pi)
          ok = true;
        } else {
          raise_status(status, kStatusBounds);
        }
      }
      M->src[t] = j;
      M->fc[t] = fc;
      s_pdst[t] = my_dst;
      // Gaussian operand row (bf16), bias column R = 1, zero padding. On the scaled distance
      // x_k = (d - mu_k) sqrt(gamma log2 e), e_k = 2^(-x_k^2); within a chunk of eight centres
      // e_{k+1} = e_k r_k, r_k = 2^(2 x_k dx - dx^2), r_{k+1} = r_k 2^(-2 dx^2): two ex2 per chunk
      // (the relative error grows by a few ulp per step, far below the operand's bf16 rounding;
      // where e_k0 underflows to 0 the chunk is below 2^-70, and r stays finite for |x| <= 80)
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
      bar_sync(1, 128);  // s_pdst complete
      const bool flag = (t < ne) && (t == 0 || s_pdst[t - 1] != my_dst);
      const unsigned bal = __ballot_sync(FULL, flag);
      if (lane == 0) s_misc[warp] = __popc(bal);
      bar_sync(1, 128);
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
      bar_sync(1, 128);
      r_lo = s_rp[TM + 1];
      mbar_arrive1(&bars[B_FULL_A + b]);
    }
    if (live && ntiles > 0) gather(ntiles - 1);
    tc::cp_async_wait_all();  // nothing in flight when the CTA exits
  } else if (warp == MMA1_WARP) {
    // =============================================================== MMA1 (lane 0 issues)
    auto wait_w = [&](int idx, uint32_t parity) -> bool {
      return !__any_sync(FULL, !wait_bar(idx, parity));
    };
    bool ok = wait_w(B_W, 0);
    const uint32_t sW1_a = tc::smem_u32(sW1);
    for (int n = 0; ok && n < ntiles; ++n) {
      if (__any_sync(FULL, *abort_flag != 0)) break;  // uniform over the warp
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
    // =============================================================== MMA2 and MMA3, in order
    if (lane == 0) {
      bool ok = wait_bar(B_W, 0);
      const uint32_t sW2_a = tc::smem_u32(sW2), sS_a = tc::smem_u32(sS);
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
        if (!(ok = wait_bar(B_FULL_M + b, par))) break;
        tc::fence_after();
        // D^T[F x slots] = msg^T (MN-major) . S^T (K-major), N = slots rounded up to 16
        const int ns = MB(i % NMETA)->nslots;
        const int n16 = ns > 0 ? (ns + 15) & ~15 : 16;
        const uint32_t id3 = tc::idesc(TM, n16, 1, true, false);
        for (int ks = 0; ks < TM / 16; ++ks)
          tc::mma(tmem + 128 * b, tc::sdesc(sH_a + ks * 256, 128, 2048),
                  tc::sdesc(sS_a + ks * 256, 128, TM * 16), id3, ks > 0);
        tc::commit(&bars[B_DONE3 + b]);
      }
      if (!ok) *abort_flag = 1;
      tc::commit(&bars[B_FIN2]);
      tc::mbar_wait(&bars[B_FIN2], 0, WAIT_LIMIT);
    }
  } else {
    // =============================================================== epilogue (8 warps)
    const int ew = warp - EPI_WARP0;        // 0..15
    const int q4 = warp & 3, part = ew >> 2;  // lane quarter, feature quarter
    const int f0 = FPT * part;
    const int e_me = 32 * q4 + lane;        // edge = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
    float carry = 0.f;
    int carry_row = -1, next_row = r_begin;
    auto write_row = [&](int row, float v) {  // drain threads: part 0, feature f = e_me
      if (row != next_row) zero_rows(out, next_row, row, e_me);  // rows without edges
      out[(size_t)row * FT + e_me] = __float2bfloat16_rn(v);
      next_row = row + 1;
    };
    auto wait_warp = [&](int idx, uint32_t parity) -> bool {  // the outcome is uniform in the warp
      return !__any_sync(FULL, !wait_bar(idx, parity));
    };
    // this warp's operand writes made visible to the tensor core, then one arrival for the warp
    auto arrive_warp = [&](int idx) {
      tc::fence_proxy_async();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive1(&bars[idx]);
    };
    // E1 of tile i: h' = f_c ssp(z1) -> H[b]
    auto epi1 = [&](int i) -> bool {
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
    // E2 of tile i: msg = x_j (.) (u + f_c c2) -> H[b] (MN-major), and the 0/1 matrix
    auto epi2 = [&](int i) -> bool {
      const int b = i & 1;
      const WsMeta* M = MB(i % NMETA);
      if (!wait_warp(B_XFULL, i & 1)) return false;
      uint4 xv[FPT / 8];
#pragma unroll
      for (int q = 0; q < FPT / 8; ++q) xv[q] = *(const uint4*)(sX + xoff(e_me, f0 / 8 + q));
      __syncwarp();
      if (lane == 0) mbar_arrive1(&bars[B_XFREE]);
      if (!wait_warp(B_DONE2 + b, (i >> 1) & 1)) return false;
      tc::fence_after();
      const float fc = M->fc[e_me];
      uint8_t* H = HB(b);
      uint32_t r[32];
      tc::ld32(lane_base + 128 * b + f0, r);
      tc::ld_wait();
#pragma unroll
      for (int g8 = 0; g8 < 4; ++g8) {
        const uint4 xq = xv[g8];
        const uint32_t xw[4] = {xq.x, xq.y, xq.z, xq.w};
        const int f8 = f0 + 8 * g8;
        const float4 ca = *(const float4*)(sc2 + f8);
        const float4 cb = *(const float4*)(sc2 + f8 + 4);
        const float cc[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int k = 8 * g8 + 2 * q;
          const float W0 = fmaf(fc, cc[2 * q], __uint_as_float(r[k]));
          const float W1 = fmaf(fc, cc[2 * q + 1], __uint_as_float(r[k + 1]));
          w[q] = tc::pack_bf16(W0 * bf_lo(xw[q]), W1 * bf_hi(xw[q]));
        }
        *(uint4*)(H + (f8 >> 3) * 2048 + (e_me >> 3) * 128 + (e_me & 7) * 16) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
      // rows s < n16 of the 0/1 matrix, 16 bytes (slot s, edges 8m..8m+7) per store; MMA3 of
      // tile i-1 has completed (this warp waited for it in that tile's drain)
      const int ns = M->nslots;
      const int n16 = ns > 0 ? (ns + 15) & ~15 : 16;
      for (int k = 32 * ew + lane; k < n16 * 16; k += 32 * NEPI) {
        const int s = k >> 4, m = k & 15;
        const int4 sa = *(const int4*)(M->slot + 8 * m);
        const int4 sb = *(const int4*)(M->slot + 8 * m + 4);
        uint4 w;
        w.x = (sa.x == s ? 0x3F80u : 0u) | (sa.y == s ? 0x3F800000u : 0u);
        w.y = (sa.z == s ? 0x3F80u : 0u) | (sa.w == s ? 0x3F800000u : 0u);
        w.z = (sb.x == s ? 0x3F80u : 0u) | (sb.y == s ? 0x3F800000u : 0u);
        w.w = (sb.z == s ? 0x3F80u : 0u) | (sb.w == s ? 0x3F800000u : 0u);
        *(uint4*)(sS + kmaj(s, 8 * m, TM)) = w;
      }
      arrive_warp(B_FULL_M + b);
      return true;
    };
    // drain of tile i: the segment sums of each destination row, written once (part 0 warps)
    auto drain = [&](int i) -> bool {
      const int b = i & 1;
      if (!wait_warp(B_DONE3 + b, (i >> 1) & 1)) return false;
      tc::fence_after();
      const WsMeta* M = MB(i % NMETA);
      const int ns = M->nslots;
      if (part == 0) {
        if (ns > 0 && carry_row >= 0 && M->slot_row[0] != carry_row) {
          write_row(carry_row, carry);
          carry_row = -1;
        }
        // four slot columns per TMEM load; a row's sum is written once it is complete (the
        // tile's last slot may continue into the next tile: it is carried)
#pragma unroll 1
        for (int s0 = 0; s0 < ns; s0 += 4) {
          uint32_t v4[4];
          tc::ld4(lane_base + 128 * b + s0, v4);
          tc::ld_wait();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int s = s0 + k;
            if (s < ns) {
              const int row = M->slot_row[s];
              float v = __uint_as_float(v4[k]);
              if (row == carry_row) v += carry;
              carry_row = -1;
              if (s == ns - 1) {
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
      __syncwarp();
      if (lane == 0) mbar_arrive1(&bars[B_FREE_T + b]);
      return true;
    };
    // the weight images (c2 is read here) have landed
    bool ok = wait_warp(B_W, 0);
    if (ok && ntiles > 0) ok = epi1(0);
    for (int i = 0; ok && i < ntiles; ++i) {
      ok = epi2(i);
      if (ok && i + 1 < ntiles) ok = epi1(i + 1);
      if (ok) ok = drain(i);
    }
    if (ok && part == 0) {
      if (carry_row >= 0) write_row(carry_row, carry);
      zero_rows(out, next_row, r_end, e_me);
    }
  }
  // the weight copy has landed before the CTA exits, whatever the roles gave up on (full budget)
  if (tid == 0) tc::mbar_wait(&bars[B_W], 0, WAIT_LIMIT);
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
                  row_ptr, col_idx, (const __nv_bfloat16*)x, (__nv_bfloat16*)out, img, radial_of(ctx),
                  ctx->status_d, (unsigned long long)ctx->wait_ns);
  };
  static_assert(ws_fits(80) && ws_fits(64) && ws_fits(48) && ws_fits(32), "shared memory plan");
  if (K1 == 80) return go(k_cfconv_fwd_ws<80>, 80);
  if (K1 == 64) return go(k_cfconv_fwd_ws<64>, 64);
  if (K1 == 48) return go(k_cfconv_fwd_ws<48>, 48);
  if (K1 == 32) return go(k_cfconv_fwd_ws<32>, 32);
  return MP_ERR_INVALID_ARG;
}

}  // namespace mp
