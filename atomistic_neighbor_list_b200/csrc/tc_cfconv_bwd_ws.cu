// Warp-specialised, double-buffered tensor-core cfconv backward (bf16 path, F = 128): grad_h and
// the block's force contribution in one pass over the symmetric CSR, with the same arithmetic as the
// tile description in tc_cfconv_bwd.cu (FlashSchNet page, technical summary s.2.3: the backward
// reduces by source; every output row is written once, no atomics; the filter is recomputed).
//
// Roles of one persistent CTA per SM (20 warps, five per SM sub-partition, so each thread may
// hold 96 registers):
//   prep (warps 0-2)        up to two tiles ahead: per edge the row, distance, envelope and its
//                           derivative, unit vector; per (edge, 8 columns) the Gaussian operand e
//                           and its d-derivative e'; the row segments
//   epilogue (warps 3-18)   four warps per TMEM lane quarter, 32 features each; per warp, in the
//                           order E2(i), E1a(i+1), FS(i), E1b(i+1), DR(i):
//                             E1a  Q = sigmoid(z1) t stored; P = ssp(z1) kept in registers
//                             E1b  P stored once MMA2b has consumed Q
//                             E2   W = f_c (u + c2), W' = f_c' (u + c2) + f_c v; msg = g_j W for
//                                  the segment-sum MMA; per-edge partial of
//                                  s_kj = sum_f (g_k h_j + g_j h_k) W'; the 0/1 matrix
//                             FS   (one warp per lane quarter) s_kj u_kj summed per row by a
//                                  segmented shuffle scan over the warp's edges
//                             DR   (one warp per lane quarter) grad_h rows, written once
//                             FP   (part 1 of lane quarter 0, in DR's place) forces of the rows
//                                  completed in the tile, ten rows x 3 components per pass
//   MMA (warp 19)           z1 = e A1ext, t = e' A1; v = Q A2, u = P A2; the segment sums; all in
//                           the fixed order in which their operands become ready
// TMEM: two 256-column buffers (z1 | t, then u | v, then the segment sums). The epilogue warps
// meet only through mbarriers; every wait is bounded and a warp that gives up votes so within
// the warp.
#include "tc_common.cuh"

namespace mp {
namespace {
using namespace tcc;

constexpr int NEPI = 16;               // epilogue warps: 4 per TMEM lane quarter
constexpr int FPT = FT * 4 / NEPI;     // features per epilogue thread (32)
constexpr int BW_PREP_WARPS = 3, PREP_T = 32 * BW_PREP_WARPS, BW_EPI_WARP0 = BW_PREP_WARPS,
              BW_MMA_WARP = BW_EPI_WARP0 + NEPI;
constexpr int BW_THREADS = 32 * (BW_MMA_WARP + 1);  // 20 warps: five per sub-partition
constexpr int EPT = (TM + PREP_T - 1) / PREP_T;     // edges per prep thread in the per-edge phase
constexpr int SMB = 128;               // destination rows per tile
constexpr int NMETA = 5;               // tile-metadata ring
constexpr unsigned FULL = 0xffffffffu;

struct BwMeta {  // written by prep
  int src[TM];
  int dst[TM];
  float fc[TM], dfc[TM], ux[TM], uy[TM], uz[TM];
  int slot[TM];
  int slot_row[SMB];
  int slot_start[SMB + 4];
  int nslots, ne, pad0, pad1;
};
struct BwEpi {  // epilogue scratch (double-buffered)
  float spart[4][TM];      // per-edge partial dot products, one per feature quarter
  float fseg[4][32][4];    // per lane quarter and row segment in it: partial force (x, y, z, -)
};
__host__ __device__ constexpr uint32_t ee_bytes(int K1) { return (uint32_t)(2 * TM * K1 * 2); }
struct BwSmem {
  uint32_t w1, w2, c2, ee0, s, qp, meta0, epi0, rp, misc, bars, total;
};
__host__ __device__ constexpr BwSmem bw_layout(int K1) {
  // W1, W2, c2 | e, e' x2 | 0/1 matrix | Q (then P, then msg^T) | metadata x4 |
  // epilogue scratch x2 | prep | misc | mbarriers
  BwSmem L{};
  uint32_t o = 0;
  L.w1 = o;    o += FT * K1 * 2;
  L.w2 = o;    o += FT * K2 * 2;
  L.c2 = o;    o += 1024;
  L.ee0 = o;   o += 2 * ee_bytes(K1);
  L.s = o;     o += SMB * TM * 2;
  L.qp = o;    o += TM * K2 * 2;
  L.meta0 = o; o += NMETA * (uint32_t)sizeof(BwMeta);
  L.epi0 = o;  o += 2 * (uint32_t)sizeof(BwEpi);
  L.rp = o;    o += 2 * TM * 4 + 64 + 3 * TM * 4 + TM * 4 + 64;
  L.misc = o;  o += 64;
  L.bars = o;  o += 512;
  L.total = o;
  return L;
}
constexpr int BW_SMEM_LIMIT = 227 * 1024;
__host__ __device__ constexpr bool bw_fits(int K1) { return bw_layout(K1).total + 1024 <= BW_SMEM_LIMIT; }

// mbarriers; the double-buffered ones at index + b
enum {
  Q_FULL_A = 0,    // prep -> MMA1 (one arrival per prep thread)
  Q_DONE1 = 2,
  Q_FULL_Q = 4,    // epilogue -> MMA2b: Q written (one arrival per epilogue warp)
  Q_DONE2B = 6,
  Q_FULL_P = 8,    // epilogue -> MMA2a: P written
  Q_DONE2A = 10,
  Q_FULL_M = 12,   // epilogue -> MMA3: msg^T and the 0/1 matrix written
  Q_DONE3 = 14,
  Q_FREE_T = 16,   // epilogue done with the tile's TMEM buffer
  Q_SPART = 18,    // 18 + 4 b + lane quarter: the three other feature quarters' partials written
  Q_FORCE = 26,    // per-row force partials of every lane quarter written (4 arrivals)
  Q_W = 28,        // weight images landed
  Q_FIN1 = 29,     // completion of everything the MMA thread issued
  Q_NBARS = 32
};

// grad_h feature f and (f < 3, not accumulating) force component f of rows [r0, r1) set to 0:
// rows without edges; out of line, it is rarely taken.
__device__ __noinline__ void zero_rows_bwd(float* grad_h, float* forces, int accumulate, int r0,
                                           int r1, int f) {
  for (int r = r0; r < r1; ++r) {
    grad_h[(size_t)r * FT + f] = 0.f;
    if (f < 3 && !accumulate) forces[(size_t)r * 3 + f] = 0.f;
  }
}

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
  uint8_t* sQP = sm + L.qp;  // Q, then P, then msg^T of one tile at a time
  uint8_t* sS = sm + L.s;    // the 0/1 segment matrix of one tile at a time
  auto MB = [&](int k) { return (BwMeta*)(sm + L.meta0) + k; };
  auto EP = [&](int b) { return (BwEpi*)(sm + L.epi0) + b; };
  int* s_rp = (int*)(sm + L.rp);               // prep: row window (TM + 1), next row at [TM + 1]
  int* s_pdst = s_rp + TM + 4;                 // prep: dst of each edge of the tile
  float* s_wpos = (float*)(s_pdst + TM + 12);  // prep: positions of the row window
  float* s_pd = s_wpos + 3 * TM;               // prep: distance of each edge (< 0: none)
  unsigned* s_bal = (unsigned*)(s_pd + TM);    // prep: row-segment starts of each 32-edge group
  int* s_misc = (int*)(sm + L.misc);  // [0..3] prep warp totals, [8] r_begin, [9] r_end, [10] abort
  uint64_t* bars = (uint64_t*)(sm + L.bars);
  uint32_t* s_tmem = (uint32_t*)(bars + Q_NBARS);

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

  if (warp == 0) tc::tmem_alloc(s_tmem, 512);
  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&bars[Q_FULL_A + b], PREP_T);
      tc::mbar_init(&bars[Q_DONE1 + b], 1);
      tc::mbar_init(&bars[Q_FULL_Q + b], NEPI);
      tc::mbar_init(&bars[Q_DONE2B + b], 1);
      tc::mbar_init(&bars[Q_FULL_P + b], NEPI);
      tc::mbar_init(&bars[Q_DONE2A + b], 1);
      tc::mbar_init(&bars[Q_FULL_M + b], NEPI);
      tc::mbar_init(&bars[Q_DONE3 + b], 1);
      tc::mbar_init(&bars[Q_FREE_T + b], NEPI);
      for (int q = 0; q < 4; ++q) tc::mbar_init(&bars[Q_SPART + 4 * b + q], 3);
      tc::mbar_init(&bars[Q_FORCE + b], 4);
    }
    tc::mbar_init(&bars[Q_W], 1);
    tc::mbar_init(&bars[Q_FIN1], 1);
    const ImgLayout IL = img_layout(K1);
    tc::mbar_expect_tx(&bars[Q_W], FT * K1 * 2 + FT * K2 * 2 + FT * 4);
    tc::bulk_g2s(sW1, img + IL.w1, FT * K1 * 2, &bars[Q_W]);
    tc::bulk_g2s(sW2, img + IL.w2, FT * K2 * 2, &bars[Q_W]);
    tc::bulk_g2s(sc2, img + IL.c2, FT * 4, &bars[Q_W]);
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *s_tmem;
  volatile int* abort_flag = &s_misc[10];
  auto wait_bar = [&](int idx, uint32_t parity) -> bool {
    if (tc::mbar_wait(&bars[idx], parity, WAIT_LIMIT)) return true;
    *abort_flag = 1;
    return false;
  };
  auto wait_warp = [&](int idx, uint32_t parity) -> bool {  // the outcome is uniform in the warp
    return !__any_sync(FULL, !wait_bar(idx, parity));
  };
  const uint32_t id12 = tc::idesc(TM, FT, 1, false, false);

  if (warp < BW_PREP_WARPS) {
    // =============================================================== prep role (PREP_T threads)
    // per edge: destination row, distance, envelope and its derivative, unit vector; then per
    // (edge, 8-column chunk): the Gaussian operand e and its d-derivative e'; then row segments
    const int t = tid;
    // Gaussians on a scaled distance x = (d - mu_k) sqrt(gamma log2 e): e_k = 2^(-x^2) and
    // e'_k = -2 gamma (d - mu_k) e_k = (-2 gamma / sqrt(gamma log2 e)) x e_k
    const float xs = sqrtf(rp.gamma * LOG2E), dmu_x = rp.dmu * xs, cdx = -2.f * rp.gamma / xs;
    const float pi_rc = 3.14159265358979f / rp.r_c;
    // chunks that hold a Gaussian or the bias column (R + 1 columns); the rest of K1 is zero
    const int nchunk = min(K1 / 8, rp.R / 8 + 1);
    int r_lo = r_begin;
    for (int it = 0; it < ntiles; ++it) {
      const int b = it & 1;
      const long long tb = e_begin + (long long)it * TM;
      const int ne = (int)((e_end - tb) < TM ? (e_end - tb) : TM);
      // loads that need no buffer go first: they overlap the wait below
      int jj[EPT];
      float pj[EPT][3], wp[EPT][3];
      int rpv[EPT];
#pragma unroll
      for (int h = 0; h < EPT; ++h) {
        const int e = t + PREP_T * h;
        int j = (e < ne) ? col_idx[tb + e] : 0;
        jj[h] = j;
        if ((unsigned)j >= (unsigned)N) j = 0;
        pj[h][0] = pos[3 * j];
        pj[h][1] = pos[3 * j + 1];
        pj[h][2] = pos[3 * j + 2];
        const int wr = min(r_lo + e, N - 1);  // the row window: its rows hold this tile's rows
        rpv[h] = row_ptr[min(r_lo + e, r_end)];
        wp[h][0] = pos[3 * wr];
        wp[h][1] = pos[3 * wr + 1];
        wp[h][2] = pos[3 * wr + 2];
      }
      const int rpv_last = row_ptr[min(r_lo + TM, r_end)];
      // operand buffer b (e, e') is free once MMA1 of tile it-2 completed; that MMA1 was issued
      // after every epilogue warp released tile it-4, and each warp had finished reading the
      // metadata of tile it-5 (the last slot this tile reuses) before that release
      const bool free_ok = it < 2 || wait_bar(Q_DONE1 + b, ((it - 2) >> 1) & 1);
      if (bar_sync_or(1, PREP_T, !free_ok || *abort_flag)) break;  // uniform over the prep warps
#pragma unroll
      for (int h = 0; h < EPT; ++h) {
        const int e = t + PREP_T * h;
        if (e < TM) {
          s_rp[e] = rpv[h];
          s_wpos[3 * e] = wp[h][0];
          s_wpos[3 * e + 1] = wp[h][1];
          s_wpos[3 * e + 2] = wp[h][2];
        }
      }
      if (t == 0) s_rp[TM] = rpv_last;
      bar_sync(1, PREP_T);
      BwMeta* M = MB(it % NMETA);
      // ---- per edge
#pragma unroll
      for (int h = 0; h < EPT; ++h) {
        const int e = t + PREP_T * h;
        if (e >= TM) continue;
        const long long g = tb + e;
        int my_dst = -1, j = jj[h];
        float fc = 0.f, dfc = 0.f, d = -1.f, ux = 0.f, uy = 0.f, uz = 0.f;
        if (e < ne) {
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
          if ((unsigned)j < (unsigned)N) {
            const float dx = pix - pj[h][0], dy = piy - pj[h][1], dz = piz - pj[h][2];
            const float d2 = dx * dx + dy * dy + dz * dz;
            const float inv = d2 > 0.f ? rsqrtf(d2) : 0.f;
            const float dd = d2 * inv;
            d = dd;
            if (dd < rp.r_c) {  // cosine envelope and its derivative from one sine/cosine
              float sn, cs;
              sincospif(dd / rp.r_c, &sn, &cs);
              fc = 0.5f * (cs + 1.f);
              dfc = -0.5f * pi_rc * sn;
            }
            ux = dx * inv;
            uy = dy * inv;
            uz = dz * inv;
          } else {
            raise_status(status, kStatusBounds);
            j = 0;
          }
        } else {
          j = 0;
        }
        M->src[e] = j;
        M->dst[e] = my_dst >= 0 ? my_dst : 0;
        M->fc[e] = fc;
        M->dfc[e] = dfc;
        M->ux[e] = ux;
        M->uy[e] = uy;
        M->uz[e] = uz;
        s_pdst[e] = my_dst;
        s_pd[e] = d;  // < 0: the edge contributes nothing (padding or a rejected index)
      }
      bar_sync(1, PREP_T);
      // ---- per (edge, chunk): the Gaussian row e (bias column R = 1) and e' (no bias)
      uint8_t* A = EE(b);
#pragma unroll 1
      for (int item = t; item < TM * (K1 / 8); item += PREP_T) {
        const int e = item & (TM - 1), k0 = 8 * (item >> 7);
        uint4 wv = make_uint4(0, 0, 0, 0), wdv = make_uint4(0, 0, 0, 0);
        const float d = s_pd[e];
        if (k0 < 8 * nchunk && d >= 0.f) {
          const float x0 = (d - rp.mu_min) * xs;
          const bool full = k0 + 8 <= rp.R;  // no bias or padding column in this chunk
          uint32_t w[4], wd[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float v[2], vd[2];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int k = k0 + 2 * q + hh;
              const float x = fmaf(-(float)k, dmu_x, x0);
              const float ek = tc::ex2f(-(x * x));
              v[hh] = ek;
              vd[hh] = cdx * x * ek;
              if (!full) {
                v[hh] = k < rp.R ? ek : (k == rp.R ? 1.f : 0.f);
                vd[hh] = k < rp.R ? vd[hh] : 0.f;
              }
            }
            w[q] = tc::pack_bf16(v[0], v[1]);
            wd[q] = tc::pack_bf16(vd[0], vd[1]);
          }
          wv = make_uint4(w[0], w[1], w[2], w[3]);
          wdv = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        }
        *(uint4*)(A + kmaj(e, k0, K1)) = wv;
        *(uint4*)(A + TM * K1 * 2 + kmaj(e, k0, K1)) = wdv;
      }
      // ---- row segments ("slots"): edges grouped by destination; group g = edges 32g..32g+31
#pragma unroll
      for (int gq = 0; gq < 4; gq += BW_PREP_WARPS) {
        const int grp = gq + warp;
        if (grp < 4) {
          const int e = 32 * grp + lane;
          const bool flag = (e < ne) && (e == 0 || s_pdst[e - 1] != s_pdst[e]);
          const unsigned bal = __ballot_sync(FULL, flag);
          if (lane == 0) {
            s_misc[grp] = __popc(bal);
            s_bal[grp] = bal;
          }
        }
      }
      bar_sync(1, PREP_T);
#pragma unroll
      for (int gq = 0; gq < 4; gq += BW_PREP_WARPS) {
        const int grp = gq + warp;
        if (grp < 4) {
          const int e = 32 * grp + lane;
          const unsigned bal = s_bal[grp];
          int off = 0;
          for (int g2 = 0; g2 < grp; ++g2) off += s_misc[g2];
          const int slot = (e < ne) ? off + __popc(bal & ((2u << lane) - 1u)) - 1 : -1;
          if ((bal >> lane) & 1u) {
            M->slot_row[slot] = s_pdst[e];
            M->slot_start[slot] = e;
          }
          M->slot[e] = slot;
          if (e == ne - 1) s_rp[TM + 1] = s_pdst[e];
        }
      }
      if (t == 0) {
        const int ns = s_misc[0] + s_misc[1] + s_misc[2] + s_misc[3];
        M->nslots = ns;
        M->ne = ne;
        M->slot_start[ns] = ne;
      }
      tc::fence_proxy_async();
      bar_sync(1, PREP_T);
      r_lo = s_rp[TM + 1];
      mbar_arrive1(&bars[Q_FULL_A + b]);
    }
  } else if (warp == BW_MMA_WARP) {
    // =============================================================== every MMA, in one order
    // The epilogue produces the operands in the order Q(i), P(i), [msg, 0/1](i), and releases a
    // tile's TMEM after that, so one thread can wait for each in turn: MMA1(0), MMA1(1), MMA2b(0),
    // MMA2a(0), then per tile i: MMA3(i), MMA2b(i+1), MMA2a(i+1), MMA1(i+2).
    if (lane == 0) {
      const uint32_t sW1_a = tc::smem_u32(sW1), sW2_a = tc::smem_u32(sW2);
      auto mma1 = [&](int n) -> bool {  // z1 = e A1ext -> columns 0..127, t = e' A1 -> 128..255
        const int b = n & 1;
        if (!wait_bar(Q_FULL_A + b, (n >> 1) & 1)) return false;
        if (n >= 2 && !wait_bar(Q_FREE_T + b, ((n - 2) >> 1) & 1)) return false;
        tc::fence_after();
        const uint32_t ea = tc::smem_u32(EE(b));
        for (int ks = 0; ks < K1 / 16; ++ks)
          tc::mma(tmem + 256 * b, tc::sdesc(ea + ks * 256, 128, K1 * 16),
                  tc::sdesc(sW1_a + ks * 256, 128, K1 * 16), id12, ks > 0);
        for (int ks = 0; ks < K1 / 16; ++ks)
          tc::mma(tmem + 256 * b + 128, tc::sdesc(ea + TM * K1 * 2 + ks * 256, 128, K1 * 16),
                  tc::sdesc(sW1_a + ks * 256, 128, K1 * 16), id12, ks > 0);
        tc::commit(&bars[Q_DONE1 + b]);
        return true;
      };
      auto mma2 = [&](int i, int full, int done, uint32_t col) -> bool {  // (Q or P) A2
        const int b = i & 1;
        if (!wait_bar(full + b, (i >> 1) & 1)) return false;
        tc::fence_after();
        const uint32_t qa = tc::smem_u32(sQP);
        for (int ks = 0; ks < K2 / 16; ++ks)
          tc::mma(tmem + 256 * b + col, tc::sdesc(qa + ks * 256, 128, K2 * 16),
                  tc::sdesc(sW2_a + ks * 256, 128, K2 * 16), id12, ks > 0);
        tc::commit(&bars[done + b]);
        return true;
      };
      auto mma3 = [&](int i) -> bool {  // segment sums of g_j W: msg^T (MN-major) . S^T
        const int b = i & 1;
        if (!wait_bar(Q_FULL_M + b, (i >> 1) & 1)) return false;
        tc::fence_after();
        const int ns = MB(i % NMETA)->nslots;
        const int n16 = ns > 0 ? (ns + 15) & ~15 : 16;
        const uint32_t id3 = tc::idesc(TM, n16, 1, true, false);
        const uint32_t qa = tc::smem_u32(sQP), sa = tc::smem_u32(sS);
        for (int ks = 0; ks < TM / 16; ++ks)
          tc::mma(tmem + 256 * b, tc::sdesc(qa + ks * 256, 128, 2048),
                  tc::sdesc(sa + ks * 256, 128, TM * 16), id3, ks > 0);
        tc::commit(&bars[Q_DONE3 + b]);
        return true;
      };
      bool ok = wait_bar(Q_W, 0) && (ntiles < 1 || mma1(0)) && (ntiles < 2 || mma1(1)) &&
                (ntiles < 1 || (mma2(0, Q_FULL_Q, Q_DONE2B, 128) && mma2(0, Q_FULL_P, Q_DONE2A, 0)));
      for (int i = 0; ok && i < ntiles && !*abort_flag; ++i) {
        ok = mma3(i);
        if (ok && i + 1 < ntiles)
          ok = mma2(i + 1, Q_FULL_Q, Q_DONE2B, 128) && mma2(i + 1, Q_FULL_P, Q_DONE2A, 0);
        if (ok && i + 2 < ntiles) ok = mma1(i + 2);
      }
      if (!ok) *abort_flag = 1;
      tc::commit(&bars[Q_FIN1]);
      tc::mbar_wait(&bars[Q_FIN1], 0, WAIT_LIMIT);
    }
  } else {
    // =============================================================== epilogue (16 warps)
    const int ew = warp - BW_EPI_WARP0;       // 0..15
    const int q4 = warp & 3, part = ew >> 2;  // TMEM lane quarter (warp % 4), feature quarter
    const int f0 = FPT * part;
    const int e_me = 32 * q4 + lane;          // edge = TMEM lane (drain: feature)
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
    float carry = 0.f;
    int carry_row = -1, next_row = r_begin;
    float fcarry = 0.f;  // lanes 0-2 of the force warp (part 1, quarter 0): carried component
    int fcarry_row = -1;
    uint32_t ppk[FPT / 2];  // P = ssp(z1) of this thread's features, bf16 pairs, E1a -> E1b
    uint32_t wq[FPT / 2];   // Q = sigmoid(z1) t, bf16 pairs, until the operand buffer is free
    // this warp's operand writes made visible to the tensor core, then one arrival for the warp
    auto arrive_warp = [&](int idx) {
      tc::fence_proxy_async();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive1(&bars[idx]);
    };
    auto emit = [&](int row, float v) {  // drain threads: part 0, feature f = e_me
      if (row != next_row) zero_rows_bwd(grad_h, forces, accumulate, next_row, row, e_me);
      grad_h[(size_t)row * FT + e_me] = v;
      next_row = row + 1;
    };
    auto put_force = [&](int row, int c, float fv) {  // force = -dE/dr, summed over the blocks
      float* fp = forces + (size_t)row * 3 + c;
      *fp = (accumulate ? *fp : 0.f) - fv;
    };
    // E1a of tile i: Q = sigmoid(z1) t -> QP[b]; P = ssp(z1) kept packed in registers
    auto E1a = [&](int i) -> bool {
      const int b = i & 1;
      if (!wait_warp(Q_DONE1 + b, (i >> 1) & 1)) return false;
      tc::fence_after();
      {  // this tile's destination rows of g and h (this thread's 64 bytes of each) into L1;
         // the metadata is complete: the prep wrote it before MMA1 of this tile was issued
        const size_t ok = (size_t)MB(i % NMETA)->dst[e_me] * FT + f0;
        tc::prefetch_l1(gin + ok);
        tc::prefetch_l1(gin + ok + FPT - 1);
        tc::prefetch_l1(hin + ok);
        tc::prefetch_l1(hin + ok + FPT - 1);
      }
      // eight columns of z1 and of t per TMEM load; the next pair is requested before this one is
      // used, so only the first load's latency is exposed
      const uint32_t zb = lane_base + 256 * b + f0;
      uint32_t rz[8], rt[8];
      tc::ld8(zb, rz);
      tc::ld8(zb + 128, rt);
#pragma unroll
      for (int c = 0; c < FPT / 8; ++c) {
        tc::ld_wait(rz, rt);
        uint32_t cz[8], ct[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          cz[k] = rz[k];
          ct[k] = rt[k];
        }
        if (c + 1 < FPT / 8) {
          tc::ld8(zb + 8 * (c + 1), rz);
          tc::ld8(zb + 128 + 8 * (c + 1), rt);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float qo[2], po[2];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const float z = __uint_as_float(cz[2 * q + hh]);
            const float tn = tc::ex2f(-fabsf(z) * LOG2E);              // e^-|z|
            const float sg = fmaf(0.5f, tc::tanhf_approx(0.5f * z), 0.5f);  // sigmoid(z)
            qo[hh] = sg * __uint_as_float(ct[2 * q + hh]);
            // ssp(z) = max(z, 0) + ln((1 + e^-|z|) / 2)
            po[hh] = fmaf(LN2, tc::lg2f(fmaf(tn, 0.5f, 0.5f)), fmaxf(z, 0.f));
          }
          wq[4 * c + q] = tc::pack_bf16(qo[0], qo[1]);
          ppk[4 * c + q] = tc::pack_bf16(po[0], po[1]);
        }
      }
      // the single operand buffer holds msg^T of tile i-1 until its segment-sum MMA completes
      if (i > 0 && !wait_warp(Q_DONE3 + ((i - 1) & 1), ((i - 1) >> 1) & 1)) return false;
#pragma unroll
      for (int c = 0; c < FPT / 8; ++c)
        *(uint4*)(sQP + kmaj(e_me, f0 + 8 * c, K2)) =
            make_uint4(wq[4 * c], wq[4 * c + 1], wq[4 * c + 2], wq[4 * c + 3]);
      arrive_warp(Q_FULL_Q + b);
      return true;
    };
    // E1b of tile i: P -> QP[b] once MMA2b has read Q
    auto E1b = [&](int i) -> bool {
      const int b = i & 1;
      if (!wait_warp(Q_DONE2B + b, (i >> 1) & 1)) return false;
      uint8_t* Pb = sQP;
#pragma unroll
      for (int c = 0; c < FPT / 8; ++c)
        *(uint4*)(Pb + kmaj(e_me, f0 + 8 * c, K2)) =
            make_uint4(ppk[4 * c], ppk[4 * c + 1], ppk[4 * c + 2], ppk[4 * c + 3]);
      arrive_warp(Q_FULL_P + b);
      return true;
    };
    // E2 of tile i, eight features per pass (the next pass's rows are loaded a pass ahead)
    auto E2 = [&](int i) -> bool {
      const int b = i & 1;
      const BwMeta* M = MB(i % NMETA);
      const float fc = M->fc[e_me], dfc = M->dfc[e_me];
      // row offsets in 16-byte units (N * F / 8 < 2^31)
      const uint32_t oj = (uint32_t)M->src[e_me] * (FT / 8) + f0 / 8;
      const uint32_t ok = (uint32_t)M->dst[e_me] * (FT / 8) + f0 / 8;
      const uint4* g4 = (const uint4*)gin;
      const uint4* h4 = (const uint4*)hin;
      // the rows g_j, h_j and g_k, h_k are loaded one pass ahead (the destination rows, shared
      // by most of the warp's edges, were also requested into L1 during E1a)
      uint4 ngj = __ldg(g4 + oj), nhj = __ldg(h4 + oj), ngk = __ldg(g4 + ok), nhk = __ldg(h4 + ok);
      if (!wait_warp(Q_DONE2A + b, (i >> 1) & 1)) return false;
      tc::fence_after();
      uint8_t* Mb = sQP;
      float s_acc = 0.f;
      // u and v eight columns per TMEM load, the next pair requested before this one is used
      const uint32_t ub = lane_base + 256 * b + f0;
      uint32_t ru[8], rv[8];
      tc::ld8(ub, ru);
      tc::ld8(ub + 128, rv);
#pragma unroll
      for (int p = 0; p < FPT / 8; ++p) {
        const int f8 = f0 + 8 * p;
        const uint4 vgj = ngj, vhj = nhj, vgk = ngk, vhk = nhk;
        if (p + 1 < FPT / 8) {
          ngj = __ldg(g4 + oj + p + 1);
          nhj = __ldg(h4 + oj + p + 1);
          ngk = __ldg(g4 + ok + p + 1);
          nhk = __ldg(h4 + ok + p + 1);
        }
        tc::ld_wait(ru, rv);
        uint32_t cu[8], cv[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          cu[k] = ru[k];
          cv[k] = rv[k];
        }
        if (p + 1 < FPT / 8) {
          tc::ld8(ub + 8 * (p + 1), ru);
          tc::ld8(ub + 128 + 8 * (p + 1), rv);
        }
        const uint32_t a_gj[4] = {vgj.x, vgj.y, vgj.z, vgj.w};
        const uint32_t a_hj[4] = {vhj.x, vhj.y, vhj.z, vhj.w};
        const uint32_t a_gk[4] = {vgk.x, vgk.y, vgk.z, vgk.w};
        const uint32_t a_hk[4] = {vhk.x, vhk.y, vhk.z, vhk.w};
        const float4 ca = *(const float4*)(sc2 + f8);
        const float4 cb = *(const float4*)(sc2 + f8 + 4);
        const float cc[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
        uint32_t w[4];
#pragma unroll
        for (int p2 = 0; p2 < 4; ++p2) {
          float m2[2];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int ii = 2 * p2 + hh;
            const float U = __uint_as_float(cu[ii]) + cc[ii];
            const float Wv = fc * U;
            const float Wp = fmaf(dfc, U, fc * __uint_as_float(cv[ii]));
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
      BwEpi* P = EP(b);
      P->spart[part][e_me] = s_acc;
      if (part != 0) {
        __syncwarp();
        if (lane == 0) mbar_arrive1(&bars[Q_SPART + 4 * b + q4]);
      }
      // rows s < n16 of the 0/1 matrix, 16 bytes (slot s, edges 8m..8m+7) per store; its single
      // buffer is free: MMA3 of tile i-1 was issued before MMA2a of tile i, whose completion this
      // warp waited for
      const int ns = M->nslots;
      const int n16 = ns > 0 ? (ns + 15) & ~15 : 16;
      uint8_t* S = sS;
      for (int k = 32 * ew + lane; k < n16 * 16; k += 32 * NEPI) {
        const int s = k >> 4, m = k & 15;
        const int4 sa = *(const int4*)(M->slot + 8 * m);
        const int4 sb = *(const int4*)(M->slot + 8 * m + 4);
        uint4 wv;
        wv.x = (sa.x == s ? 0x3F80u : 0u) | (sa.y == s ? 0x3F800000u : 0u);
        wv.y = (sa.z == s ? 0x3F80u : 0u) | (sa.w == s ? 0x3F800000u : 0u);
        wv.z = (sb.x == s ? 0x3F80u : 0u) | (sb.y == s ? 0x3F800000u : 0u);
        wv.w = (sb.z == s ? 0x3F80u : 0u) | (sb.w == s ? 0x3F800000u : 0u);
        *(uint4*)(S + kmaj(s, 8 * m, TM)) = wv;
      }
      arrive_warp(Q_FULL_M + b);
      return true;
    };
    // FS of tile i (part-0 warps): s_e = sum of the four feature quarters' partials, then
    // s_e u_e summed per destination row over this warp's 32 edges by a segmented inclusive scan
    // (fixed order: deterministic); the last edge of each row segment records the partial
    auto FS = [&](int i) -> bool {
      const int b = i & 1;
      if (!wait_warp(Q_SPART + 4 * b + q4, (i >> 1) & 1)) return false;
      const BwMeta* M = MB(i % NMETA);
      BwEpi* P = EP(b);
      const float s = ((P->spart[0][e_me] + P->spart[1][e_me]) + P->spart[2][e_me]) +
                      P->spart[3][e_me];
      float px = s * M->ux[e_me], py = s * M->uy[e_me], pz = s * M->uz[e_me];
      const int sl = M->slot[e_me];  // -1 past the tile's last edge
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float ox = __shfl_up_sync(FULL, px, off);
        const float oy = __shfl_up_sync(FULL, py, off);
        const float oz = __shfl_up_sync(FULL, pz, off);
        const int osl = __shfl_up_sync(FULL, sl, off);
        if (lane >= off && osl == sl) {
          px += ox;
          py += oy;
          pz += oz;
        }
      }
      const int nsl = __shfl_down_sync(FULL, sl, 1);
      const int sl0 = __shfl_sync(FULL, sl, 0);  // the quarter's first row segment
      if (sl >= 0 && (lane == 31 || nsl != sl)) {
        float* f = P->fseg[q4][sl - sl0];
        f[0] = px;
        f[1] = py;
        f[2] = pz;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive1(&bars[Q_FORCE + b]);
      return true;
    };
    // FP of tile i (the part-1 warp of lane quarter 0): the forces of the rows completed in the
    // tile, ten rows x three components per pass; the row still open at the tile's end is carried.
    // The values being accumulated into are requested before the wait for the partial sums.
    auto FP = [&](int i) -> bool {
      const int b = i & 1;
      const BwMeta* M = MB(i % NMETA);
      const int ns = M->nslots, c = lane % 3;
      float oldc = 0.f, old0 = 0.f;
      if (accumulate) {
        if (fcarry_row >= 0 && lane < 3) oldc = forces[(size_t)fcarry_row * 3 + lane];
        if (lane < 30 && lane / 3 < ns) old0 = forces[(size_t)M->slot_row[lane / 3] * 3 + c];
      }
      if (!wait_warp(Q_FORCE + b, (i >> 1) & 1)) return false;
      if (ns == 0) return true;
      const BwEpi* P = EP(b);
      if (fcarry_row >= 0 && M->slot_row[0] != fcarry_row) {  // the carried row is complete
        if (lane < 3) forces[(size_t)fcarry_row * 3 + lane] = oldc - fcarry;
        fcarry_row = -1;
      }
#pragma unroll 1
      for (int s0 = 0; s0 < ns; s0 += 10) {
        const int s = s0 + lane / 3;
        const bool act = lane < 30 && s < ns;
        float fv = 0.f, old = s0 == 0 ? old0 : 0.f;
        int row = -1;
        if (act) {
          row = M->slot_row[s];
          const int qa = M->slot_start[s] >> 5, qb = (M->slot_start[s + 1] - 1) >> 5;
          for (int q = qa; q <= qb; ++q) fv += P->fseg[q][s - M->slot[32 * q]][c];
          if (accumulate && s0 > 0 && s != ns - 1) old = forces[(size_t)row * 3 + c];
        }
        const float cin = __shfl_sync(FULL, fcarry, c);
        if (act && s == 0 && row == fcarry_row) fv += cin;
        if (act && s != ns - 1) forces[(size_t)row * 3 + c] = old - fv;
        if (ns - 1 < s0 + 10) {  // this pass holds the tile's last row: carry it
          const float v = __shfl_sync(FULL, fv, 3 * (ns - 1 - s0) + c);
          if (lane < 3) fcarry = v;
        }
      }
      fcarry_row = M->slot_row[ns - 1];
      return true;
    };
    // DR of tile i: grad_h rows (part-0 warps, feature e_me), written once a row is complete (the
    // tile's last slot may continue into the next tile: it is carried); the force warp runs FP
    auto DR = [&](int i) -> bool {
      const int b = i & 1;
      if (part == 0) {
        if (!wait_warp(Q_DONE3 + b, (i >> 1) & 1)) return false;
        tc::fence_after();
        const BwMeta* M = MB(i % NMETA);
        const int ns = M->nslots;
        if (ns > 0 && carry_row >= 0 && M->slot_row[0] != carry_row) {
          emit(carry_row, carry);
          carry_row = -1;
        }
#pragma unroll 1
        for (int s0 = 0; s0 < ns; s0 += 4) {
          uint32_t v4[4];
          tc::ld4(lane_base + 256 * b + s0, v4);
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
                emit(row, v);
              }
            }
          }
        }
      }
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive1(&bars[Q_FREE_T + b]);
      // the force warp reads no TMEM: it releases the tile first, then sums its forces
      if (part == 1 && q4 == 0 && !FP(i)) return false;
      return true;
    };
    // the weight images (c2 is read here) have landed
    bool ok = wait_warp(Q_W, 0);
    if (ok && ntiles > 0) ok = E1a(0) && E1b(0);
    for (int i = 0; ok && i < ntiles; ++i) {
      ok = E2(i);
      if (ok && i + 1 < ntiles) ok = E1a(i + 1);
      if (ok && part == 0) ok = FS(i);
      if (ok && i + 1 < ntiles) ok = E1b(i + 1);
      if (ok) ok = DR(i);
    }
    if (ok && part == 0) {
      if (carry_row >= 0) emit(carry_row, carry);
      zero_rows_bwd(grad_h, forces, accumulate, next_row, r_end, e_me);
    }
    if (ok && part == 1 && q4 == 0 && fcarry_row >= 0 && lane < 3) put_force(fcarry_row, lane, fcarry);
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
  // a Gaussian operand wider than the shared-memory plan allows: the lock-step kernel
  if (!bw_fits(K1))
    return tc_cfconv_bwd_sequential(ctx, block, N, E, pos, row_ptr, col_idx, h, g, grad_h, forces,
                                    accumulate, s);
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
  static_assert(!bw_fits(80) && bw_fits(64) && bw_fits(48) && bw_fits(32), "shared memory plan");
  if (K1 == 64) return go(k_cfconv_bwd_ws<64>, 64);
  if (K1 == 48) return go(k_cfconv_bwd_ws<48>, 48);
  if (K1 == 32) return go(k_cfconv_bwd_ws<32>, 32);
  return MP_ERR_INVALID_ARG;
}

}  // namespace mp
