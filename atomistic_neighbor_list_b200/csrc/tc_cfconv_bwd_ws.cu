// Warp-specialised tensor-core cfconv backward (bf16 path, F = 128) with two epilogue groups that
// work on alternating tiles: grad_h and the block's force contribution in one pass over the
// symmetric CSR, with the arithmetic of the tile description in tc_cfconv_bwd.cu (FlashSchNet
// page, technical summary s.2.3: the backward reduces by source; every output row is written once,
// no atomics; the filter is recomputed rather than stored).
//
// Per tile the work splits into a special-function-heavy phase (E1: sigmoid and softplus of the
// first filter layer, three MUFU operations per edge and feature) and a load- and FP32-heavy phase
// (E2: the filter and its d-derivative, the gathered rows g_j, h_j, g_k, h_k, the messages and
// the pair products). Two epilogue groups take alternate tiles, so one group's E1 can run while
// the other group's E2 does, on the same SM sub-partitions.
//
// Roles of one persistent CTA per SM (20 warps, five per SM sub-partition, 96 registers each; the
// registers are allocated per four warps, so a 21st warp would cost the whole CTA 16 registers
// per thread):
//   prep (warps 0-2)        up to four tiles ahead (the metadata ring): per edge the row, distance,
//                           envelope and its derivative, unit vector; the row segments ("slots")
//   group g (8 warps each:  tiles i = g, g + 2, ...; two warps per TMEM lane quarter, 64 features
//   3-10 and 11-18)         each; per tile:
//                             G    the Gaussian operand e and its d-derivative e' from the stored
//                                  distances (a two-multiplication recurrence over eight centres)
//                             E1a  Q = sigmoid(z1) t stored; P = ssp(z1) packed into the z1
//                                  TMEM columns E1a has already read
//                             E1b  P stored once MMA2b has consumed Q
//                             E2   W = f_c (u + c2), W' = f_c' (u + c2) + f_c v; msg = g_j W for
//                                  the segment-sum MMA; per-edge s_kj = sum_f (g_k h_j + g_j h_k) W'
//                                  in two sweeps; the 0/1 matrix
//                             FS   (feature-half 0 warps) s_kj u_kj summed per row segment by a
//                                  segmented shuffle scan over the warp's 32 edges
//                             DR   (feature-half 0 warps) grad_h rows, written once
//                             FP   (one warp) forces of the rows completed in the tile
//                           The row still open at a tile's end is carried to the next tile (the
//                           other group) through a token in shared memory, in tile order.
//   MMA (warp 19)           one thread: z1 = e A1ext, t = e' A1; v = Q A2, u = P A2; the segment
//                           sums; it polls the hand-off barriers and issues whichever MMA is
//                           ready, in tile order within each of its four streams
// TMEM: 512 columns, 256 per group (z1 | t, then u | v, then the segment sums). Every wait is
// bounded (the context's wait budget); a warp that gives up votes so within the warp, sets the
// CTA's abort flag, and every role then runs out its own bounded waits; the MMA thread waits (full
// budget) for everything it issued before the CTA frees TMEM.
#include "tc_common.cuh"

namespace mp {
namespace {
using namespace tcc;

constexpr int NGRP = 2;                // epilogue groups
constexpr int GW = 8;                  // warps per group: 2 per TMEM lane quarter
constexpr int FPT = FT / 2;            // features per epilogue thread (64)
constexpr int BW_PREP_WARPS = 3, PREP_T = 32 * BW_PREP_WARPS, BW_EPI_WARP0 = BW_PREP_WARPS,
              BW_MMA_WARP = BW_EPI_WARP0 + NGRP * GW;
constexpr int BW_THREADS = 32 * (BW_MMA_WARP + 1);  // 20 warps: five per sub-partition
constexpr int EPT = (TM + PREP_T - 1) / PREP_T;     // edges per prep thread in the per-edge phase
constexpr int SMB = 128;               // destination rows per tile
constexpr int NMETA = 4;               // tile-metadata ring
constexpr unsigned FULL = 0xffffffffu;

struct BwMeta {  // written by prep
  int src[TM];
  int dst[TM];
  float dist[TM], fc[TM], dfc[TM], ux[TM], uy[TM], uz[TM];  // dist < 0: the edge adds nothing
  int slot[TM];
  int slot_row[SMB];
  int slot_start[SMB + 4];
  int nslots, ne, pad0, pad1;
};
struct BwEpi {  // per-group epilogue scratch
  float spart[TM];         // per-edge partial dot products of feature half 1
  float fseg[4][32][4];    // per lane quarter and row segment in it: partial force (x, y, z, -)
};
struct DrTok {   // grad_h state handed from one tile's drain to the next one's
  float carry[FT];
  int carry_row, next_row, pad0, pad1;
};
struct FpTok {   // force state handed from one tile's force pass to the next one's
  float fcarry[4];
  int fcarry_row, pad0, pad1, pad2;
};
__host__ __device__ constexpr uint32_t ee_bytes(int K1) { return (uint32_t)(2 * TM * K1 * 2); }
struct BwSmem {
  uint32_t w1, w2, c2, ee, qp0, s, meta0, epi0, tok, rp, misc, bars, total;
};
__host__ __device__ constexpr BwSmem bw_layout(int K1) {
  // W1, W2, c2 | e, e' | Q/P/msg^T per group | 0/1 matrix | metadata ring | per-group scratch |
  // tokens x2 | prep | misc | mbarriers
  BwSmem L{};
  uint32_t o = 0;
  L.w1 = o;    o += FT * K1 * 2;
  L.w2 = o;    o += FT * K2 * 2;
  L.c2 = o;    o += FT * 4;
  L.ee = o;    o += ee_bytes(K1);
  L.qp0 = o;   o += NGRP * TM * K2 * 2;
  L.s = o;     o += SMB * TM * 2;
  L.meta0 = o; o += NMETA * (uint32_t)sizeof(BwMeta);
  L.epi0 = o;  o += NGRP * (uint32_t)sizeof(BwEpi);
  L.tok = o;   o += 2 * (uint32_t)sizeof(DrTok) + 2 * (uint32_t)sizeof(FpTok);
  L.rp = o;    o += 2 * TM * 4 + 64 + 3 * TM * 4 + TM * 4 + 64;
  L.misc = o;  o += 64;
  L.bars = o;  o += 512;
  L.total = o;
  return L;
}
constexpr int BW_SMEM_LIMIT = 227 * 1024;
__host__ __device__ constexpr bool bw_fits(int K1) {
  return bw_layout(K1).total + 1024 <= BW_SMEM_LIMIT;
}

// mbarriers; the per-group ones at index + g
enum {
  B_FULL_A = 0,    // + slot: prep -> group: the tile's metadata written (one arrival per prep thread)
  B_FULL_E = 4,    // group -> MMA1: the tile's Gaussian operand written (one arrival per warp)
  B_EE_FREE = 5,   // MMA1 complete: the e, e' buffer may be rewritten
  B_DONE1 = 6,     // + g: MMA1 of the group's tile complete
  B_FULL_Q = 8,    // + g: Q written (one arrival per group warp)
  B_DONE2B = 10,   // + g
  B_FULL_P = 12,   // + g: P written
  B_DONE2A = 14,   // + g
  B_FULL_M = 16,   // + g: msg^T and the 0/1 matrix written
  B_DONE3 = 18,    // + g
  B_S_FREE = 20,   // MMA3 complete: the 0/1 matrix may be rewritten
  B_SPART = 21,    // + 4 g + lane quarter: feature half 1's partials written
  B_FORCE = 29,    // + g: per-row force partials of every lane quarter written (4 arrivals)
  B_TOK_DR = 31,   // the drain token of the tile written (4 arrivals)
  B_TOK_FP = 32,   // the force token of the tile written
  B_MFREE = 33,    // + slot: a group is done with the tile's metadata (one arrival per warp)
  B_W = 37,        // weight images landed
  B_FIN = 38,      // completion of everything the MMA thread issued
  B_NBARS = 39
};
static_assert(B_NBARS * 8 + 8 <= 512, "barrier area");

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
    int accumulate, const uint8_t* __restrict__ img, Radial rp, int* status,
    unsigned long long wait_ns) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr BwSmem L = bw_layout(K1);
  uint8_t* sW1 = sm + L.w1;
  uint8_t* sW2 = sm + L.w2;
  float* sc2 = (float*)(sm + L.c2);
  uint8_t* sEE = sm + L.ee;  // e [TM][K1], then e' [TM][K1]
  uint8_t* sS = sm + L.s;    // the 0/1 segment matrix of one tile at a time
  auto QPB = [&](int g) { return sm + L.qp0 + (uint32_t)g * (TM * K2 * 2); };
  auto MB = [&](int k) { return (BwMeta*)(sm + L.meta0) + k; };
  auto EP = [&](int g) { return (BwEpi*)(sm + L.epi0) + g; };
  DrTok* s_dtok = (DrTok*)(sm + L.tok);              // [2], by tile parity
  FpTok* s_ftok = (FpTok*)(s_dtok + 2);              // [2]
  int* s_rp = (int*)(sm + L.rp);               // prep: row window (TM + 1), next row at [TM + 1]
  int* s_pdst = s_rp + TM + 4;                 // prep: dst of each edge of the tile
  float* s_wpos = (float*)(s_pdst + TM + 12);  // prep: positions of the row window
  unsigned* s_bal = (unsigned*)(s_wpos + 3 * TM);  // prep: row-segment starts per 32-edge group
  int* s_misc = (int*)(sm + L.misc);  // [0..3] prep warp totals, [8] r_begin, [9] r_end, [10] abort
  uint64_t* bars = (uint64_t*)(sm + L.bars);
  uint32_t* s_tmem = (uint32_t*)(bars + B_NBARS);

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
    for (int k = 0; k < NMETA; ++k) tc::mbar_init(&bars[B_FULL_A + k], PREP_T);
    tc::mbar_init(&bars[B_FULL_E], GW);
    tc::mbar_init(&bars[B_EE_FREE], 1);
    tc::mbar_init(&bars[B_S_FREE], 1);
    for (int g = 0; g < NGRP; ++g) {
      tc::mbar_init(&bars[B_DONE1 + g], 1);
      tc::mbar_init(&bars[B_FULL_Q + g], GW);
      tc::mbar_init(&bars[B_DONE2B + g], 1);
      tc::mbar_init(&bars[B_FULL_P + g], GW);
      tc::mbar_init(&bars[B_DONE2A + g], 1);
      tc::mbar_init(&bars[B_FULL_M + g], GW);
      tc::mbar_init(&bars[B_DONE3 + g], 1);
      tc::mbar_init(&bars[B_FORCE + g], 4);
      for (int q = 0; q < 4; ++q) tc::mbar_init(&bars[B_SPART + 4 * g + q], 1);
    }
    tc::mbar_init(&bars[B_TOK_DR], 4);
    tc::mbar_init(&bars[B_TOK_FP], 1);
    for (int k = 0; k < NMETA; ++k) tc::mbar_init(&bars[B_MFREE + k], GW);
    tc::mbar_init(&bars[B_W], 1);
    tc::mbar_init(&bars[B_FIN], 1);
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
  auto wait_warp = [&](int idx, uint32_t parity) -> bool {  // the outcome is uniform in the warp
    return !__any_sync(FULL, !wait_bar(idx, parity));
  };
  const uint32_t id12 = tc::idesc(TM, FT, 1, false, false);

  if (warp < BW_PREP_WARPS) {
    // =============================================================== prep role (PREP_T threads)
    const int t = tid;
    const float pi_rc = 3.14159265358979f / rp.r_c;
    int r_lo = r_begin;
    for (int it = 0; it < ntiles; ++it) {
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
      // the metadata slot is free once the group that had tile it - NMETA is done with it
      const bool free_ok =
          it < NMETA || wait_bar(B_MFREE + (it % NMETA), ((it / NMETA) - 1) & 1);
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
              __sincosf(pi_rc * dd, &sn, &cs);  // argument in [0, pi): special-function unit
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
        M->dist[e] = d;  // < 0: the edge contributes nothing (padding or a rejected index)
        M->fc[e] = fc;
        M->dfc[e] = dfc;
        M->ux[e] = ux;
        M->uy[e] = uy;
        M->uz[e] = uz;
        s_pdst[e] = my_dst;
      }
      bar_sync(1, PREP_T);
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
      bar_sync(1, PREP_T);
      r_lo = s_rp[TM + 1];
      mbar_arrive1(&bars[B_FULL_A + (it % NMETA)]);
    }
  } else if (warp == BW_MMA_WARP) {
    // =============================================================== every MMA (one thread)
    // Four in-order streams: MMA1 of every tile; per group, MMA2b then MMA2a of its tiles; MMA3 of
    // every tile. The thread polls the barrier each stream waits for next and issues whatever is
    // ready, so one group's late hand-off does not hold up the other group's MMAs.
    if (lane == 0) {
      const uint32_t sW1_a = tc::smem_u32(sW1), sW2_a = tc::smem_u32(sW2);
      const uint32_t ea = tc::smem_u32(sEE), sa = tc::smem_u32(sS);
      bool ok = wait_bar(B_W, 0);
      int n1 = 0, n3 = 0;
      int n2[NGRP] = {0, 1}, st2[NGRP] = {0, 0};  // next tile of the group; 0: MMA2b next, 1: MMA2a
      uint64_t t_last = tc::global_ns();
      while (ok && n3 < ntiles) {
        bool prog = false;
        // the group arrives after its previous tile, TMEM reads included: its columns are free
        if (n1 < ntiles && tc::mbar_test(&bars[B_FULL_E], n1 & 1)) {
          // z1 = e A1ext -> columns 0..127, t = e' A1 -> 128..255 of the group's TMEM
          tc::fence_after();
          const uint32_t d = tmem + 256 * (n1 & 1);
          for (int ks = 0; ks < K1 / 16; ++ks)
            tc::mma(d, tc::sdesc(ea + ks * 256, 128, K1 * 16),
                    tc::sdesc(sW1_a + ks * 256, 128, K1 * 16), id12, ks > 0);
          for (int ks = 0; ks < K1 / 16; ++ks)
            tc::mma(d + 128, tc::sdesc(ea + TM * K1 * 2 + ks * 256, 128, K1 * 16),
                    tc::sdesc(sW1_a + ks * 256, 128, K1 * 16), id12, ks > 0);
          tc::commit(&bars[B_DONE1 + (n1 & 1)]);
          tc::commit(&bars[B_EE_FREE]);
          ++n1;
          prog = true;
        }
#pragma unroll
        for (int g = 0; g < NGRP; ++g) {
          const int k = n2[g];
          if (k >= n1) continue;  // its MMA1 has not been issued yet
          const uint32_t par = (k >> 1) & 1;
          if (tc::mbar_test(&bars[(st2[g] == 0 ? B_FULL_Q : B_FULL_P) + g], par)) {
            // MMA2b: v = Q A2 -> columns 128..255; MMA2a: u = P A2 -> columns 0..127
            tc::fence_after();
            const uint32_t qa = tc::smem_u32(QPB(g));
            const uint32_t d = tmem + 256 * g + (st2[g] == 0 ? 128 : 0);
            for (int ks = 0; ks < K2 / 16; ++ks)
              tc::mma(d, tc::sdesc(qa + ks * 256, 128, K2 * 16),
                      tc::sdesc(sW2_a + ks * 256, 128, K2 * 16), id12, ks > 0);
            if (st2[g] == 0) {
              tc::commit(&bars[B_DONE2B + g]);
              st2[g] = 1;
            } else {
              tc::commit(&bars[B_DONE2A + g]);
              st2[g] = 0;
              n2[g] += NGRP;
            }
            prog = true;
          }
        }
        if (n3 < n1 && tc::mbar_test(&bars[B_FULL_M + (n3 & 1)], (n3 >> 1) & 1)) {
          // segment sums of g_j W: D^T[F x slots] = msg^T (MN-major) . S^T, N = slots to 16
          tc::fence_after();
          const int g = n3 & 1;
          const int ns = MB(n3 % NMETA)->nslots;
          const int n16 = ns > 0 ? (ns + 15) & ~15 : 16;
          const uint32_t id3 = tc::idesc(TM, n16, 1, true, false);
          const uint32_t qa = tc::smem_u32(QPB(g));
          for (int ks = 0; ks < TM / 16; ++ks)
            tc::mma(tmem + 256 * g, tc::sdesc(qa + ks * 256, 128, 2048),
                    tc::sdesc(sa + ks * 256, 128, TM * 16), id3, ks > 0);
          tc::commit(&bars[B_DONE3 + g]);
          tc::commit(&bars[B_S_FREE]);
          ++n3;
          prog = true;
        }
        const uint64_t now = tc::global_ns();
        if (prog) {
          t_last = now;
        } else {
          if (*abort_flag) break;
          if (now - t_last >= wait_ns) ok = false;
          else __nanosleep(40);
        }
      }
      if (!ok) *abort_flag = 1;
      // everything issued has completed before the CTA frees TMEM (full budget, whatever wait_ns)
      tc::commit(&bars[B_FIN]);
      tc::mbar_wait(&bars[B_FIN], 0, WAIT_LIMIT);
    }
  } else {
    // =============================================================== two epilogue groups
    const int g = (warp - BW_EPI_WARP0) / GW;   // group: tiles g, g + 2, ...
    const int ew = (warp - BW_EPI_WARP0) % GW;  // warp within the group
    const int q4 = warp & 3, part = ew >> 2;    // TMEM lane quarter (warp % 4), feature half
    const int f0 = FPT * part;
    const int e_me = 32 * q4 + lane;            // edge = TMEM lane (drain: feature)
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16) + 256 * g;
    const bool fp_warp = part == 1 && q4 == 0;  // the group's force pass
    uint8_t* QP = QPB(g);
    BwEpi* EPg = EP(g);
    float carry = 0.f;
    int carry_row = -1, next_row = r_begin;
    float fcarry = 0.f;  // lanes 0-2 of the force warp: the carried force component
    int fcarry_row = -1;
    float s_acc = 0.f;   // this edge's pair-product partial over the thread's features (E2 -> FS)
    // this warp's operand writes made visible to the tensor core, then one arrival for the warp
    auto arrive_warp = [&](int idx) {
      tc::fence_proxy_async();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive1(&bars[idx]);
    };
    auto emit = [&](int row, float v) {  // drain threads: feature f = e_me
      if (row != next_row) zero_rows_bwd(grad_h, forces, accumulate, next_row, row, e_me);
      grad_h[(size_t)row * FT + e_me] = v;
      next_row = row + 1;
    };
    auto put_force = [&](int row, int c, float fv) {  // force = -dE/dr, summed over the blocks
      float* fp = forces + (size_t)row * 3 + c;
      *fp = (accumulate ? *fp : 0.f) - fv;
    };
    // G of tile i: the tile's Gaussian operand e (bias column R = 1) and its d-derivative e' from
    // the distances the prep stored, eight centres per item (4 items per thread at K1 = 64).
    // Gaussians on a scaled distance x = (d - mu_k) sqrt(gamma log2 e): e_k = 2^(-x^2) and
    // e'_k = -2 gamma (d - mu_k) e_k = (-2 gamma / sqrt(gamma log2 e)) x e_k. Within a chunk of
    // eight centres, x_{k+1} = x_k - dx gives e_{k+1} = e_k r_k with r_k = 2^(2 x_k dx - dx^2) and
    // r_{k+1} = r_k 2^(-2 dx^2): two ex2 per chunk, then multiplications (the relative error grows
    // by a few ulp per step, far below the bf16 rounding of the operand; where e_k0 underflows to 0
    // the whole chunk is below 2^-70, and r stays within 2^+-64 for |x| <= 80).
    const float xs = sqrtf(rp.gamma * LOG2E), dmu_x = rp.dmu * xs, cdx = -2.f * rp.gamma / xs;
    const float rstep = tc::ex2f(-2.f * dmu_x * dmu_x), cdmu = cdx * dmu_x;
    // chunks that hold a Gaussian or the bias column (R + 1 columns); the rest of K1 is zero
    const int nchunk = min(K1 / 8, rp.R / 8 + 1);
    auto G = [&](int i) -> bool {
      if (!wait_warp(B_FULL_A + (i % NMETA), (i / NMETA) & 1)) return false;
      // the single operand buffer: MMA1 of the previous tile (the other group's) has read it
      if (i > 0 && !wait_warp(B_EE_FREE, (i - 1) & 1)) return false;
      const BwMeta* M = MB(i % NMETA);
#pragma unroll 1
      for (int item = 32 * ew + lane; item < TM * (K1 / 8); item += 32 * GW) {
        const int e = item & (TM - 1), k0 = 8 * (item >> 7);
        uint4 wv = make_uint4(0, 0, 0, 0), wdv = make_uint4(0, 0, 0, 0);
        const float d = M->dist[e];
        if (k0 < 8 * nchunk && d >= 0.f) {
          const bool full = k0 + 8 <= rp.R;  // no bias or padding column in this chunk
          const float xk0 = fmaf(-(float)k0, dmu_x, (d - rp.mu_min) * xs);
          float ek = tc::ex2f(-(xk0 * xk0));
          float rk = tc::ex2f(dmu_x * fmaf(2.f, xk0, -dmu_x));
          float cxk = cdx * xk0;  // cdx x_k, stepped by -cdx dx
          uint32_t w[4], wd[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float v[2], vd[2];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int k = k0 + 2 * q + hh;
              v[hh] = ek;
              vd[hh] = cxk * ek;
              if (!full) {
                v[hh] = k < rp.R ? ek : (k == rp.R ? 1.f : 0.f);
                vd[hh] = k < rp.R ? vd[hh] : 0.f;
              }
              ek *= rk;
              rk *= rstep;
              cxk -= cdmu;
            }
            w[q] = tc::pack_bf16(v[0], v[1]);
            wd[q] = tc::pack_bf16(vd[0], vd[1]);
          }
          wv = make_uint4(w[0], w[1], w[2], w[3]);
          wdv = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        }
        *(uint4*)(sEE + kmaj(e, k0, K1)) = wv;
        *(uint4*)(sEE + TM * K1 * 2 + kmaj(e, k0, K1)) = wdv;
      }
      arrive_warp(B_FULL_E);
      return true;
    };
    // E1a of tile i: Q = sigmoid(z1) t -> QP; P = ssp(z1) parked in TMEM
    auto E1a = [&](int i) -> bool {
      const uint32_t par = (i >> 1) & 1;
      if (!wait_warp(B_DONE1 + g, par)) return false;
      tc::fence_after();
      {  // this tile's destination rows of g and h (this thread's 128 bytes of each) into L1;
         // the metadata is complete: the prep wrote it before MMA1 of this tile was issued
        const size_t ok = (size_t)MB(i % NMETA)->dst[e_me] * FT + f0;
        tc::prefetch_l1(gin + ok);
        tc::prefetch_l1(hin + ok);
      }
      const uint32_t zb = lane_base + f0;
      // the group's operand buffer holds msg^T of its previous tile until that segment sum is done
      if (i >= NGRP && !wait_warp(B_DONE3 + g, ((i - NGRP) >> 1) & 1)) return false;
      // eight columns of z1 and of t per pass, the next pass's requested before this one is used
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
        uint32_t wq[4], wp[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float qo[2], po[2];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const float z = __uint_as_float(cz[2 * q + hh]);
            const float tn = tc::ex2f(-fabsf(z) * LOG2E);                    // e^-|z|
            const float sg = fmaf(0.5f, tc::tanhf_approx(0.5f * z), 0.5f);  // sigmoid(z)
            qo[hh] = sg * __uint_as_float(ct[2 * q + hh]);
            // ssp(z) = max(z, 0) + ln((1 + e^-|z|) / 2)
            po[hh] = fmaf(LN2, tc::lg2f(fmaf(tn, 0.5f, 0.5f)), fmaxf(z, 0.f));
          }
          wq[q] = tc::pack_bf16(qo[0], qo[1]);
          wp[q] = tc::pack_bf16(po[0], po[1]);
        }
        *(uint4*)(QP + kmaj(e_me, f0 + 8 * c, K2)) = make_uint4(wq[0], wq[1], wq[2], wq[3]);
        // P parked in this lane's z1 columns f0 + 4c .. f0 + 4c + 3, already read (passes <= c)
        tc::st4(zb + 4 * c, wp);
      }
      tc::st_wait();
      arrive_warp(B_FULL_Q + g);
      return true;
    };
    // E1b of tile i: P (parked in TMEM by E1a) -> QP once MMA2b has read Q
    auto E1b = [&](int i) -> bool {
      uint32_t pk[32];
      tc::ld32(lane_base + f0, pk);
      tc::ld_wait();
      if (!wait_warp(B_DONE2B + g, (i >> 1) & 1)) return false;
#pragma unroll
      for (int c = 0; c < FPT / 8; ++c)
        *(uint4*)(QP + kmaj(e_me, f0 + 8 * c, K2)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      arrive_warp(B_FULL_P + g);
      return true;
    };
    // E2 of tile i in two sweeps over this thread's 64 features, eight per pass. The thread's
    // part of a source row is one 128-byte line; read a pass at a time it would be fetched from
    // L2 again at every pass (the lines of a group's edges outgrow L1), so each sweep holds its
    // whole line in registers: sweep A holds g_j (loaded before the MMA wait) and forms the
    // messages g_j W and the g_j h_k part of s; its passes free the registers into which h_j is
    // loaded for sweep B, which forms the g_k h_j part (u, v and W' read and formed again). The
    // destination rows (shared by the edges of a row, in L1 since E1a) are loaded a pass ahead.
    auto E2 = [&](int i) -> bool {
      const BwMeta* M = MB(i % NMETA);
      const float fc = M->fc[e_me], dfc = M->dfc[e_me];
      // row offsets in 16-byte units (N * F / 8 < 2^31)
      const uint4* gj4 = (const uint4*)gin + (uint32_t)M->src[e_me] * (FT / 8) + f0 / 8;
      const uint4* hj4 = (const uint4*)hin + (uint32_t)M->src[e_me] * (FT / 8) + f0 / 8;
      const uint4* gk4 = (const uint4*)gin + (uint32_t)M->dst[e_me] * (FT / 8) + f0 / 8;
      const uint4* hk4 = (const uint4*)hin + (uint32_t)M->dst[e_me] * (FT / 8) + f0 / 8;
      uint4 row[FPT / 8];
#pragma unroll
      for (int p = 0; p < FPT / 8; ++p) row[p] = __ldg(gj4 + p);
      uint4 ngk = __ldg(gk4), nhk = __ldg(hk4);
      if (!wait_warp(B_DONE2A + g, (i >> 1) & 1)) return false;
      tc::fence_after();
      float sa = 0.f, sb = 0.f;
      const uint32_t ub = lane_base + f0;
      // u, v eight columns per TMEM load, the next pass's requested before this one is used (a
      // load waited for at once costs its whole latency, several hundred cycles while the tensor
      // core works on the other group's tile)
      uint32_t ru[8], rv[8];
      tc::ld8(ub, ru);
      tc::ld8(ub + 128, rv);
      // ---- sweep A: msg = g_j W -> QP (MN-major), sa += g_j h_k W'
#pragma unroll
      for (int p = 0; p < FPT / 8; ++p) {
        const int f8 = f0 + 8 * p;
        const uint4 vgj = row[p], vhk = nhk;
        row[p] = __ldg(hj4 + p);
        if (p + 1 < FPT / 8) nhk = __ldg(hk4 + p + 1);
        tc::ld_wait(ru, rv);
        uint32_t cu[8], cv[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          cu[k] = ru[k];
          cv[k] = rv[k];
        }
        {  // the next pass (sweep B starts over at column 0)
          const int pn = p + 1 < FPT / 8 ? p + 1 : 0;
          tc::ld8(ub + 8 * pn, ru);
          tc::ld8(ub + 128 + 8 * pn, rv);
        }
        const uint32_t a_gj[4] = {vgj.x, vgj.y, vgj.z, vgj.w};
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
            const float xhk = hh ? bf_hi(a_hk[p2]) : bf_lo(a_hk[p2]);
            m2[hh] = xgj * Wv;
            sa = fmaf(xgj * xhk, Wp, sa);
          }
          w[p2] = tc::pack_bf16(m2[0], m2[1]);
        }
        *(uint4*)(QP + (f8 >> 3) * 2048 + (e_me >> 3) * 128 + (e_me & 7) * 16) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
      // ---- sweep B: sb += g_k h_j W'
      ngk = __ldg(gk4);
#pragma unroll
      for (int p = 0; p < FPT / 8; ++p) {
        const int f8 = f0 + 8 * p;
        const uint4 vhj = row[p], vgk = ngk;
        if (p + 1 < FPT / 8) ngk = __ldg(gk4 + p + 1);
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
        const uint32_t a_hj[4] = {vhj.x, vhj.y, vhj.z, vhj.w};
        const uint32_t a_gk[4] = {vgk.x, vgk.y, vgk.z, vgk.w};
        const float4 ca = *(const float4*)(sc2 + f8);
        const float4 cb = *(const float4*)(sc2 + f8 + 4);
        const float cc[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
#pragma unroll
        for (int p2 = 0; p2 < 4; ++p2) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int ii = 2 * p2 + hh;
            const float U = __uint_as_float(cu[ii]) + cc[ii];
            const float Wp = fmaf(dfc, U, fc * __uint_as_float(cv[ii]));
            const float xhj = hh ? bf_hi(a_hj[p2]) : bf_lo(a_hj[p2]);
            const float xgk = hh ? bf_hi(a_gk[p2]) : bf_lo(a_gk[p2]);
            sb = fmaf(xgk * xhj, Wp, sb);
          }
        }
      }
      s_acc = sa + sb;
      if (part != 0) {
        EPg->spart[e_me] = s_acc;
        __syncwarp();
        if (lane == 0) mbar_arrive1(&bars[B_SPART + 4 * g + q4]);
      }
      // rows s < n16 of the 0/1 matrix, 16 bytes (slot s, edges 8m..8m+7) per store, once the
      // segment-sum MMA of the previous tile (the other group's) has read the single buffer
      if (i > 0 && !wait_warp(B_S_FREE, (i - 1) & 1)) return false;
      const int ns = M->nslots;
      const int n16 = ns > 0 ? (ns + 15) & ~15 : 16;
      for (int k = 32 * ew + lane; k < n16 * 16; k += 32 * GW) {
        const int s = k >> 4, m = k & 15;
        const int4 sa = *(const int4*)(M->slot + 8 * m);
        const int4 sb = *(const int4*)(M->slot + 8 * m + 4);
        uint4 wv;
        wv.x = (sa.x == s ? 0x3F80u : 0u) | (sa.y == s ? 0x3F800000u : 0u);
        wv.y = (sa.z == s ? 0x3F80u : 0u) | (sa.w == s ? 0x3F800000u : 0u);
        wv.z = (sb.x == s ? 0x3F80u : 0u) | (sb.y == s ? 0x3F800000u : 0u);
        wv.w = (sb.z == s ? 0x3F80u : 0u) | (sb.w == s ? 0x3F800000u : 0u);
        *(uint4*)(sS + kmaj(s, 8 * m, TM)) = wv;
      }
      arrive_warp(B_FULL_M + g);
      return true;
    };
    // FS of tile i (feature-half 0 warps): s_e = both halves' partials, then s_e u_e summed per
    // destination row over this warp's 32 edges by a segmented inclusive scan (fixed order:
    // deterministic); the last edge of each row segment records the partial
    auto FS = [&](int i) -> bool {
      if (!wait_warp(B_SPART + 4 * g + q4, (i >> 1) & 1)) return false;
      const BwMeta* M = MB(i % NMETA);
      const float s = s_acc + EPg->spart[e_me];
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
        float* f = EPg->fseg[q4][sl - sl0];
        f[0] = px;
        f[1] = py;
        f[2] = pz;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive1(&bars[B_FORCE + g]);
      return true;
    };
    // FP of tile i (the force warp): the forces of the rows completed in the tile, ten rows x three
    // components per pass; the row still open at the tile's end is carried through the token
    auto FP = [&](int i) -> bool {
      if (i > 0) {
        if (!wait_warp(B_TOK_FP, (i - 1) & 1)) return false;
        const FpTok* tk = &s_ftok[(i - 1) & 1];
        fcarry = lane < 3 ? tk->fcarry[lane] : 0.f;
        fcarry_row = tk->fcarry_row;
      }
      const BwMeta* M = MB(i % NMETA);
      const int ns = M->nslots, c = lane % 3;
      float oldc = 0.f, old0 = 0.f;
      if (accumulate) {
        if (fcarry_row >= 0 && lane < 3) oldc = forces[(size_t)fcarry_row * 3 + lane];
        if (lane < 30 && lane / 3 < ns) old0 = forces[(size_t)M->slot_row[lane / 3] * 3 + c];
      }
      if (!wait_warp(B_FORCE + g, (i >> 1) & 1)) return false;
      if (ns > 0) {
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
            for (int q = qa; q <= qb; ++q) fv += EPg->fseg[q][s - M->slot[32 * q]][c];
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
      }
      FpTok* to = &s_ftok[i & 1];
      if (lane < 3) to->fcarry[lane] = fcarry;
      if (lane == 0) to->fcarry_row = fcarry_row;
      __syncwarp();
      if (lane == 0) mbar_arrive1(&bars[B_TOK_FP]);
      return true;
    };
    // DR of tile i (feature-half 0 warps, feature e_me): grad_h rows written once complete; the
    // tile's last slot may continue into the next tile: it is carried through the token
    auto DR = [&](int i) -> bool {
      if (!wait_warp(B_DONE3 + g, (i >> 1) & 1)) return false;
      tc::fence_after();
      if (i > 0) {
        if (!wait_warp(B_TOK_DR, (i - 1) & 1)) return false;
        const DrTok* tk = &s_dtok[(i - 1) & 1];
        carry = tk->carry[e_me];
        carry_row = tk->carry_row;
        next_row = tk->next_row;
      }
      const BwMeta* M = MB(i % NMETA);
      const int ns = M->nslots;
      if (ns > 0 && carry_row >= 0 && M->slot_row[0] != carry_row) {
        emit(carry_row, carry);
        carry_row = -1;
      }
#pragma unroll 1
      for (int s0 = 0; s0 < ns; s0 += 4) {
        uint32_t v4[4];
        tc::ld4(lane_base + s0, v4);
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
      DrTok* to = &s_dtok[i & 1];
      to->carry[e_me] = carry;
      if (q4 == 0 && lane == 0) {
        to->carry_row = carry_row;
        to->next_row = next_row;
      }
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive1(&bars[B_TOK_DR]);
      return true;
    };
    // the weight images (c2 is read here) have landed
    bool ok = wait_warp(B_W, 0);
    int last_done = -1;
    for (int i = g; ok && i < ntiles; i += NGRP) {
      ok = G(i) && E1a(i) && E1b(i) && E2(i);
      if (ok && part == 0) ok = FS(i) && DR(i);
      if (ok && fp_warp) ok = FP(i);
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive1(&bars[B_MFREE + (i % NMETA)]);
      last_done = i;
    }
    if (ok) {
      if (ntiles == 0) {
        if (g == 0 && part == 0) zero_rows_bwd(grad_h, forces, accumulate, r_begin, r_end, e_me);
      } else if (last_done == ntiles - 1) {  // this group had the last tile: flush the carries
        if (part == 0) {
          if (carry_row >= 0) emit(carry_row, carry);
          zero_rows_bwd(grad_h, forces, accumulate, next_row, r_end, e_me);
        }
        if (fp_warp && fcarry_row >= 0 && lane < 3) put_force(fcarry_row, lane, fcarry);
      }
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
                  forces, (int)accumulate, img, radial_of(ctx), ctx->status_d,
                  (unsigned long long)ctx->wait_ns);
  };
  static_assert(bw_fits(80) && bw_fits(64) && bw_fits(48) && bw_fits(32), "shared memory plan");
  if (K1 == 80) return go(k_cfconv_bwd_ws<80>, 80);
  if (K1 == 64) return go(k_cfconv_bwd_ws<64>, 64);
  if (K1 == 48) return go(k_cfconv_bwd_ws<48>, 48);
  if (K1 == 32) return go(k_cfconv_bwd_ws<32>, 32);
  return MP_ERR_INVALID_ARG;
}

}  // namespace mp
