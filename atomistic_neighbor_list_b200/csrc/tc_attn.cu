// Tensor-core neighbor attention (bf16 path, F = 128, 16 heads x 8), over a padded neighbor list
// whose width K is a multiple of 128 (E2Former-V2 page s.3.2: parallel over destination atoms,
// neighbors streamed tile by tile, online softmax per head, padded slots skipped; s.3.1 for the
// logits). Per pair (i, j):
//   W_ij  = f_c(d) (ssp(e A1 + c1) A2 + c2)              the filter of the cfconv
//   l_ijh = q_ih . k_jh / sqrt(8) + e P_h + p_h          the radial bias rides in MMA1 as 16 more
//                                                         B rows (bias p_h on the constant column)
//   out_ih = sum_j softmax_j(l_ijh) (x_j (.) W_ij)[head h]
// A tile is 128 slots of one atom. Roles of one persistent CTA per SM (22 warps):
//   prep (warps 0-3)       slots, distances, envelope, Gaussian operand, the atom's q row; the x_j
//                          rows of the previous tile copied into a bank-permuted buffer
//   epilogue (warps 4-19)  four warps per TMEM lane quarter (= 32 slots), 32 features = 4 heads
//                          each: E2(i), E1(i+1), DR(i):
//                            E1  h' = f_c ssp(z1) -> MMA2; the 4 heads' radial bias kept
//                            E2  the 4 heads' logits from q and the gathered k_j; the tile's
//                                per-head maximum (shuffles, then the 4 warps of the feature
//                                quarter through an mbarrier); p = e^(l - m) as the B operand of
//                                the weighted-sum MMA; v = x_j (.) W as its A operand
//                            DR  (one warp per lane quarter, thread = feature) the tile's sums
//                                merged into the atom's running (m, z, acc); the row written
//                                once at the atom's last tile
//   MMA1 (warp 20)         [z1 | bias] = e [W1 | P]  (N = 144)
//   MMA2/3 (warp 21)       u = h' A2; D[f][h] = sum over the tile's slots of v p (N = 16)
// Every wait is bounded; a warp that gives up votes so within the warp.
#include "tc_common.cuh"

namespace mp {
namespace {
using namespace tcc;

constexpr int NEPI = 16;
constexpr int FPT = FT * 4 / NEPI;  // 32 features = 4 heads of 8 per epilogue thread
constexpr int AH = 16, AD = 8;      // heads, head width
constexpr int PREP_WARPS = 4, EPI_WARP0 = 4, MMA1_WARP = EPI_WARP0 + NEPI, MMA23_WARP = MMA1_WARP + 1;
constexpr int AT_THREADS = 32 * (MMA23_WARP + 1);  // 22 warps
constexpr int NMETA = 4;
constexpr int N1 = FT + AH;  // MMA1 output columns: z1 and the radial bias
constexpr unsigned FULL = 0xffffffffu;

struct AtMeta {
  int src[TM];
  float fc[TM];
  int ok[TM];
  float q[FT];  // the atom's query row, scaled by 1/sqrt(AD)
  int atom, first, last, pad;
};
struct AtRed {  // per-tile softmax partials (double-buffered)
  float wmax[4][4][4];  // [feature quarter][lane quarter][head in quarter]
  float wsum[4][4][4];
  float mh[AH];         // the tile's per-head maximum
};
struct AtSmem {
  uint32_t w1, w2, c2, a0, p, h0, x, meta0, red0, misc, bars, total;
};
__host__ __device__ constexpr AtSmem at_layout(int K1, int NC) {
  // W1 | P (144 rows) | W2 | c2 | Gaussian operand x2 | p operand | h' / v^T x2 | x_j rows |
  // metadata x4 | softmax partials x2 | misc | mbarriers
  AtSmem L{};
  uint32_t o = 0;
  L.w1 = o;    o += N1 * K1 * 2;
  L.w2 = o;    o += FT * K2 * 2;
  L.c2 = o;    o += 1024;
  L.a0 = o;    o += 2 * TM * K1 * 2;
  L.p = o;     o += AH * TM * 2 * NC;
  L.h0 = o;    o += 2 * TM * K2 * 2;
  L.x = o;     o += TM * FT * 2;
  L.meta0 = o; o += NMETA * (uint32_t)sizeof(AtMeta);
  L.red0 = o;  o += 2 * (uint32_t)sizeof(AtRed);
  L.misc = o;  o += 64;
  L.bars = o;  o += 512;
  L.total = o;
  return L;
}
__host__ __device__ constexpr bool at_fits(int K1, int NC) {
  return at_layout(K1, NC).total + 1024 <= 227 * 1024;
}
__device__ __forceinline__ uint32_t xoff(int r, int c) {  // staged x_j rows (bank-permuted)
  return (uint32_t)(r * (FT * 2) + ((c ^ (r & 7)) << 4));
}

enum {
  B_FULL_A = 0, B_DONE1 = 2, B_FULL_H = 4, B_DONE2 = 6, B_FULL_M = 8, B_DONE3 = 10, B_FREE_T = 12,
  B_W = 14, B_XFULL = 15, B_XFREE = 16, B_FIN1 = 17, B_FIN2 = 18,
  B_WMAX = 20,  // 20 + 2 * feature quarter + b: the quarter's 4 warps wrote their maxima
  N_BARS = 28
};

// NC = 1: the attention of the scalar values; NC = 9: each value also coupled with the solid
// harmonics l <= 2 of r_j - r_i (one weighted-sum MMA per harmonic, p scaled by S_lm(r_ij)), out
// [N][9][F] (E2Former-V2 page s.3.1: direction only through the value path).
template <int K1, int NC>
__global__ void __launch_bounds__(AT_THREADS, 1) k_attn_tc(
    int N, int K, const float* __restrict__ pos, const int* __restrict__ nbr,
    const unsigned char* __restrict__ mask, const __nv_bfloat16* __restrict__ x,
    const float* __restrict__ q, const __half* __restrict__ kx, __nv_bfloat16* __restrict__ out,
    const uint8_t* __restrict__ img, const uint8_t* __restrict__ pimg, Radial rp, float qscale,
    int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr AtSmem L = at_layout(K1, NC);
  uint8_t* sW1 = sm + L.w1;  // rows 0..127 W1 (bias c1 on column R), rows 128..143 P (bias p)
  uint8_t* sW2 = sm + L.w2;
  float* sc2 = (float*)(sm + L.c2);
  uint8_t* sP = sm + L.p;    // softmax weights p, [16 heads][128 slots] K-major
  uint8_t* sX = sm + L.x;
  auto AB = [&](int b) { return sm + L.a0 + (uint32_t)b * (TM * K1 * 2); };
  auto HB = [&](int b) { return sm + L.h0 + (uint32_t)b * (TM * K2 * 2); };
  auto MB = [&](int k) { return (AtMeta*)(sm + L.meta0) + k; };
  auto RB = [&](int b) { return (AtRed*)(sm + L.red0) + b; };
  int* s_misc = (int*)(sm + L.misc);  // [10] abort
  uint64_t* bars = (uint64_t*)(sm + L.bars);
  uint32_t* s_tmem = (uint32_t*)(bars + N_BARS);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  // this CTA's atoms; an atom's K / 128 tiles stay in one CTA (its running softmax state)
  const int a_begin = (int)((long long)N * cta / G), a_end = (int)((long long)N * (cta + 1) / G);
  const int TPA = K / TM;
  const int ntiles = (a_end - a_begin) * TPA;
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
      tc::mbar_init(&bars[B_DONE3 + b], 1);
      tc::mbar_init(&bars[B_FREE_T + b], NEPI);
    }
    tc::mbar_init(&bars[B_W], 1);
    tc::mbar_init(&bars[B_XFULL], 128);
    tc::mbar_init(&bars[B_XFREE], NEPI);
    tc::mbar_init(&bars[B_FIN1], 1);
    tc::mbar_init(&bars[B_FIN2], 1);
    for (int k = 0; k < 8; ++k) tc::mbar_init(&bars[B_WMAX + k], 4);
    const ImgLayout IL = img_layout(K1);
    tc::mbar_expect_tx(&bars[B_W], FT * K1 * 2 + AH * K1 * 2 + FT * K2 * 2 + FT * 4);
    tc::bulk_g2s(sW1, img + IL.w1, FT * K1 * 2, &bars[B_W]);
    tc::bulk_g2s(sW1 + FT * K1 * 2, pimg, AH * K1 * 2, &bars[B_W]);
    tc::bulk_g2s(sW2, img + IL.w2, FT * K2 * 2, &bars[B_W]);
    tc::bulk_g2s(sc2, img + IL.c2, FT * 4, &bars[B_W]);
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
  auto wait_warp = [&](int idx, uint32_t parity) -> bool {  // uniform within the warp
    return !__any_sync(FULL, !wait_bar(idx, parity));
  };

  if (warp < PREP_WARPS) {
    // =============================================================== prep role (128 threads)
    const int t = tid;
    const float xs = sqrtf(rp.gamma * LOG2E), dmu_x = rp.dmu * xs;
    const float rstep = tc::ex2f(-2.f * dmu_x * dmu_x), pi_rc = 3.14159265358979f / rp.r_c;
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
      const int a = a_begin + it / TPA;
      const long long s = (long long)a * K + (long long)(it % TPA) * TM + t;
      // loads that need no buffer go first: they overlap the wait below
      int j = nbr[s];
      bool ok = mask[s] != 0;
      if (ok && (unsigned)j >= (unsigned)N) {
        raise_status(status, kStatusBounds);
        ok = false;
      }
      if (!ok) j = 0;
      const float pjx = pos[3 * j], pjy = pos[3 * j + 1], pjz = pos[3 * j + 2];
      const float pix = pos[3 * a], piy = pos[3 * a + 1], piz = pos[3 * a + 2];
      const float qv = q[(size_t)a * FT + t] * qscale;
      // Gaussian operand buffer b is free once MMA1 of tile it-2 completed (and with it the
      // metadata slot of tile it-4: its drain preceded that MMA1)
      const bool free_ok = it < 2 || wait_bar(B_DONE1 + b, ((it - 2) >> 1) & 1);
      if (bar_sync_or(1, 128, !free_ok || *abort_flag)) {
        live = false;
        break;
      }
      // the x_j rows of the previous tile first: they are needed one tile sooner than this one
      if (it > 0 && !gather(it - 1)) {
        live = false;
        break;
      }
      AtMeta* M = MB(it % NMETA);
      float d = 0.f, fc = 0.f;
      if (ok) {
        const float dx = pix - pjx, dy = piy - pjy, dz = piz - pjz;
        d = sqrtf(dx * dx + dy * dy + dz * dz);
        if (d < rp.r_c) fc = 0.5f * (__cosf(pi_rc * d) + 1.f);  // argument in [0, pi)
      }
      M->src[t] = j;
      M->fc[t] = fc;
      M->ok[t] = ok ? 1 : 0;
      M->q[t] = qv;
      if (t == 0) {
        M->atom = a;
        M->first = (it % TPA) == 0;
        M->last = (it % TPA) == TPA - 1;
      }
      // Gaussian operand row (bf16), bias column R = 1; zero for a padded slot. e_k = 2^(-x_k^2)
      // on the scaled distance, by the two-ex2-per-eight-centres recurrence of the cfconv
      // forward (tc_cfconv_ws.cu)
      const float xk00 = (d - rp.mu_min) * xs;
      uint8_t* A = AB(b);
#pragma unroll
      for (int k0 = 0; k0 < K1; k0 += 8) {
        const float xk0 = fmaf(-(float)k0, dmu_x, xk00);
        float ek = tc::ex2f(-(xk0 * xk0));
        float rk = tc::ex2f(dmu_x * fmaf(2.f, xk0, -dmu_x));
        uint32_t w[4];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          float v[2];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int k = k0 + 2 * qq + hh;
            float val = ek;
            if (k >= K1 - 16) val = k < rp.R ? val : (k == rp.R ? 1.f : 0.f);
            v[hh] = ok ? val : 0.f;
            ek *= rk;
            rk *= rstep;
          }
          w[qq] = tc::pack_bf16(v[0], v[1]);
        }
        *(uint4*)(A + kmaj(t, k0, K1)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      tc::fence_proxy_async();
      bar_sync(1, 128);
      mbar_arrive1(&bars[B_FULL_A + b]);
    }
    if (live) gather(ntiles - 1);
    tc::cp_async_wait_all();  // nothing in flight when the CTA exits
  } else if (warp == MMA1_WARP) {
    // =============================================================== MMA1 (lane 0 issues)
    bool ok = wait_warp(B_W, 0);
    const uint32_t sW1_a = tc::smem_u32(sW1);
    const uint32_t id1 = tc::idesc(TM, N1, 1, false, false);
    for (int n = 0; ok && n < ntiles; ++n) {
      if (__any_sync(FULL, *abort_flag != 0)) break;
      const int b = n & 1;
      ok = wait_warp(B_FULL_A + b, (n >> 1) & 1) &&
           (n < 2 || wait_warp(B_FREE_T + b, ((n - 2) >> 1) & 1));
      if (!ok) break;
      tc::fence_after();
      if (lane == 0) {
        const uint32_t sA_a = tc::smem_u32(AB(b));
        for (int ks = 0; ks < K1 / 16; ++ks)
          tc::mma(tmem + 256 * b, tc::sdesc(sA_a + ks * 256, 128, K1 * 16),
                  tc::sdesc(sW1_a + ks * 256, 128, K1 * 16), id1, ks > 0);
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
      const uint32_t sW2_a = tc::smem_u32(sW2), sP_a = tc::smem_u32(sP);
      const uint32_t id2 = tc::idesc(TM, FT, 1, false, false);
      const uint32_t id3 = tc::idesc(TM, AH, 1, true, false);
      for (int i = 0; ok && i < ntiles && !*abort_flag; ++i) {
        const int b = i & 1;
        const uint32_t par = (i >> 1) & 1;
        if (!(ok = wait_bar(B_FULL_H + b, par))) break;
        tc::fence_after();
        const uint32_t sH_a = tc::smem_u32(HB(b));
        for (int ks = 0; ks < K2 / 16; ++ks)
          tc::mma(tmem + 256 * b, tc::sdesc(sH_a + ks * 256, 128, K2 * 16),
                  tc::sdesc(sW2_a + ks * 256, 128, K2 * 16), id2, ks > 0);
        tc::commit(&bars[B_DONE2 + b]);
        if (!(ok = wait_bar(B_FULL_M + b, par))) break;
        tc::fence_after();
        // D^T[F x 16 heads] = v^T (MN-major) . p^T (K-major): each feature's own head column is
        // the tile's softmax-weighted sum for it; one such product per harmonic
        for (int m = 0; m < NC; ++m)
          for (int ks = 0; ks < TM / 16; ++ks)
            tc::mma(tmem + 256 * b + 16 * m, tc::sdesc(sH_a + ks * 256, 128, 2048),
                    tc::sdesc(sP_a + m * (AH * TM * 2) + ks * 256, 128, TM * 16), id3, ks > 0);
        tc::commit(&bars[B_DONE3 + b]);
      }
      if (!ok) *abort_flag = 1;
      tc::commit(&bars[B_FIN2]);
      tc::mbar_wait(&bars[B_FIN2], 0, WAIT_LIMIT);
    }
  } else {
    // =============================================================== epilogue (16 warps)
    const int ew = warp - EPI_WARP0;          // 0..15
    const int q4 = warp & 3, part = ew >> 2;  // TMEM lane quarter, feature quarter
    const int f0 = FPT * part, h0 = 4 * part; // this thread's 32 features = heads h0..h0+3
    const int e_me = 32 * q4 + lane;          // slot = TMEM lane (drain: feature)
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
    float bias[4] = {0.f, 0.f, 0.f, 0.f};     // this slot's radial logit bias, E1(i) -> E2(i)
    float m_run = -INFINITY, z_run = 0.f, acc_run[NC];    // drain: the atom's running softmax
#pragma unroll
    for (int m = 0; m < NC; ++m) acc_run[m] = 0.f;
    auto arrive_warp = [&](int idx) {
      tc::fence_proxy_async();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive1(&bars[idx]);
    };
    // E1 of tile i: h' = f_c ssp(z1) -> H[b]; the 4 heads' radial bias kept for E2
    auto E1 = [&](int i) -> bool {
      const int b = i & 1;
      if (!wait_warp(B_DONE1 + b, (i >> 1) & 1)) return false;
      tc::fence_after();
      const float fc = MB(i % NMETA)->fc[e_me];
      uint8_t* H = HB(b);
      uint32_t r[32], rb[4];
      tc::ld32(lane_base + 256 * b + f0, r);
      tc::ld4(lane_base + 256 * b + FT + h0, rb);
      tc::ld_wait();
#pragma unroll
      for (int k = 0; k < 4; ++k) bias[k] = __uint_as_float(rb[k]);
#pragma unroll
      for (int g8 = 0; g8 < 4; ++g8) {
        uint32_t w[4];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const int k = 8 * g8 + 2 * qq;
          w[qq] = ssp_scaled_bf16x2(__uint_as_float(r[k]), __uint_as_float(r[k + 1]), fc, fc * LN2);
        }
        *(uint4*)(H + kmaj(e_me, f0 + 8 * g8, K2)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      arrive_warp(B_FULL_H + b);
      return true;
    };
    // E2 of tile i: logits, the tile's softmax weights p (B operand of MMA3), v = x_j (.) W
    auto E2 = [&](int i) -> bool {
      const int b = i & 1;
      const AtMeta* M = MB(i % NMETA);
      AtRed* R = RB(b);
      const bool ok = M->ok[e_me] != 0;
      const float fc = M->fc[e_me];
      // k_j of the 4 heads (fp16, 8 per 16-byte load), requested before the waits
      const uint4* kr = (const uint4*)(kx + (size_t)M->src[e_me] * FT + f0);
      uint4 kv[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) kv[c] = __ldg(kr + c);
      if (!wait_warp(B_XFULL, i & 1)) return false;
      uint4 xv[FPT / 8];
#pragma unroll
      for (int qq = 0; qq < FPT / 8; ++qq) xv[qq] = *(const uint4*)(sX + xoff(e_me, f0 / 8 + qq));
      __syncwarp();
      if (lane == 0) mbar_arrive1(&bars[B_XFREE]);
      // logits l_h = q_h . k_h (q pre-scaled by 1/sqrt(8)) + radial bias; -inf on a padded slot
      float l[4];
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) {
        const float4 qa = *(const float4*)(M->q + f0 + 8 * hh);
        const float4 qb = *(const float4*)(M->q + f0 + 8 * hh + 4);
        const uint32_t kw[4] = {kv[hh].x, kv[hh].y, kv[hh].z, kv[hh].w};
        float2 k2[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) k2[c] = __half22float2(*(const __half2*)&kw[c]);
        float s = qa.x * k2[0].x;
        s = fmaf(qa.y, k2[0].y, s);
        s = fmaf(qa.z, k2[1].x, s);
        s = fmaf(qa.w, k2[1].y, s);
        s = fmaf(qb.x, k2[2].x, s);
        s = fmaf(qb.y, k2[2].y, s);
        s = fmaf(qb.z, k2[3].x, s);
        s = fmaf(qb.w, k2[3].y, s);
        l[hh] = ok ? s + bias[hh] : -INFINITY;
      }
      // the tile's maximum per head: over the warp, then over the 4 warps of this feature quarter
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) {
        float m = l[hh];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
        if (lane == 0) R->wmax[part][q4][hh] = m;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive1(&bars[B_WMAX + 2 * part + b]);
      if (!wait_warp(B_WMAX + 2 * part + b, (i >> 1) & 1)) return false;
      float mh[4], pb[4];
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) {
        mh[hh] = fmaxf(fmaxf(R->wmax[part][0][hh], R->wmax[part][1][hh]),
                       fmaxf(R->wmax[part][2][hh], R->wmax[part][3][hh]));
        // p = e^(l - m), rounded to bf16 (the MMA operand); the sum below uses the rounded values
        const float p = (l[hh] == -INFINITY) ? 0.f : tc::ex2f((l[hh] - mh[hh]) * LOG2E);
        pb[hh] = __bfloat162float(__float2bfloat16_rn(p));
      }
      if (q4 == 0 && lane < 4)
        R->mh[h0 + lane] = lane == 0 ? mh[0] : lane == 1 ? mh[1] : lane == 2 ? mh[2] : mh[3];
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) {
        float z = pb[hh];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(FULL, z, off);
        if (lane == 0) R->wsum[part][q4][hh] = z;
      }
      if (!wait_warp(B_DONE2 + b, (i >> 1) & 1)) return false;
      tc::fence_after();
      // the p operand has one buffer: MMA3 of tile i-1 was issued before MMA2 of tile i, whose
      // completion this warp just saw
      if constexpr (NC == 1) {
#pragma unroll
        for (int hh = 0; hh < 4; ++hh)
          *(__nv_bfloat16*)(sP + kmaj(h0 + hh, e_me, TM)) = __float2bfloat16_rn(pb[hh]);
      } else {  // one operand per harmonic: p S_lm(r_j - r_i) (p is 0 on a padded slot)
        float S[9] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (ok) {
          const int j = M->src[e_me], a = M->atom;
          solid_harmonics9(pos[3 * j] - pos[3 * a], pos[3 * j + 1] - pos[3 * a + 1],
                           pos[3 * j + 2] - pos[3 * a + 2], S);
        }
#pragma unroll
        for (int m = 0; m < NC; ++m)
#pragma unroll
          for (int hh = 0; hh < 4; ++hh)
            *(__nv_bfloat16*)(sP + m * (AH * TM * 2) + kmaj(h0 + hh, e_me, TM)) =
                __float2bfloat16_rn(pb[hh] * S[m]);
      }
      uint8_t* H = HB(b);
      uint32_t r[32];
      tc::ld32(lane_base + 256 * b + f0, r);
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
        for (int qq = 0; qq < 4; ++qq) {
          const int k = 8 * g8 + 2 * qq;
          const float W0 = fmaf(fc, cc[2 * qq], __uint_as_float(r[k]));
          const float W1 = fmaf(fc, cc[2 * qq + 1], __uint_as_float(r[k + 1]));
          w[qq] = tc::pack_bf16(W0 * bf_lo(xw[qq]), W1 * bf_hi(xw[qq]));
        }
        *(uint4*)(H + (f8 >> 3) * 2048 + (e_me >> 3) * 128 + (e_me & 7) * 16) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
      arrive_warp(B_FULL_M + b);
      return true;
    };
    // DR of tile i (part-0 warps, thread = feature e_me of head e_me / 8): the tile's weighted sum
    // merged into the atom's running softmax; the row is written once, at the atom's last tile
    auto DR = [&](int i) -> bool {
      const int b = i & 1;
      if (part == 0) {
        if (!wait_warp(B_DONE3 + b, (i >> 1) & 1)) return false;
        tc::fence_after();
        const AtMeta* M = MB(i % NMETA);
        const AtRed* R = RB(b);
        const int hs = lane >> 3, hf = 4 * q4 + hs;
        float acc_t[NC];
#pragma unroll
        for (int m = 0; m < NC; ++m) {  // heads 4 q4 .. 4 q4 + 3 of this warp's features
          uint32_t v4[4];
          tc::ld4(lane_base + 256 * b + 16 * m + 4 * q4, v4);
          tc::ld_wait();
          acc_t[m] = __uint_as_float(hs == 0 ? v4[0] : hs == 1 ? v4[1] : hs == 2 ? v4[2] : v4[3]);
        }
        const float m_t = R->mh[hf];
        const float z_t = ((R->wsum[hf >> 2][0][hf & 3] + R->wsum[hf >> 2][1][hf & 3]) +
                           R->wsum[hf >> 2][2][hf & 3]) + R->wsum[hf >> 2][3][hf & 3];
        if (M->first) {
          m_run = -INFINITY;
          z_run = 0.f;
#pragma unroll
          for (int m = 0; m < NC; ++m) acc_run[m] = 0.f;
        }
        if (m_t != -INFINITY) {  // a tile with no valid slot adds nothing
          if (m_run == -INFINITY) {
            m_run = m_t;
            z_run = z_t;
#pragma unroll
            for (int m = 0; m < NC; ++m) acc_run[m] = acc_t[m];
          } else {
            const float mn = fmaxf(m_run, m_t);
            const float s1 = tc::ex2f((m_run - mn) * LOG2E), s2 = tc::ex2f((m_t - mn) * LOG2E);
#pragma unroll
            for (int m = 0; m < NC; ++m) acc_run[m] = fmaf(acc_run[m], s1, acc_t[m] * s2);
            z_run = fmaf(z_run, s1, z_t * s2);
            m_run = mn;
          }
        }
        if (M->last) {
          const float iz = z_run > 0.f ? 1.f / z_run : 0.f;
#pragma unroll
          for (int m = 0; m < NC; ++m)
            out[((size_t)M->atom * NC + m) * FT + e_me] =
                __float2bfloat16_rn(NC == 1 ? (z_run > 0.f ? acc_run[m] / z_run : 0.f)
                                            : acc_run[m] * iz);
        }
      }
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive1(&bars[B_FREE_T + b]);
      return true;
    };
    // the weight images (c2 is read here) have landed
    bool ok = wait_warp(B_W, 0);
    if (ok) ok = E1(0);
    for (int i = 0; ok && i < ntiles; ++i) {
      ok = E2(i);
      if (ok && i + 1 < ntiles) ok = E1(i + 1);
      if (ok) ok = DR(i);
    }
  }
  tc::fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag) raise_status(status, kStatusTimeout);
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

}  // namespace

bool tc_attn_supported(const mp_ctx* ctx, int K) {
  const mp_config& c = ctx->cfg;
  return tc_supported(ctx) && ctx->tc_attn_p && ctx->tc_qk && c.n_heads == AH && c.head_dim == AD &&
         K % TM == 0 && k1_of(c.n_rbf) <= 64 && at_fits(k1_of(c.n_rbf), 1);  // built for 32-64
}

template <int NC>
int tc_attn_launch(mp_ctx* ctx, int N, int K, const float* pos, const int* nbr,
                   const unsigned char* mask, const void* x, void* out, cudaStream_t s) {
  const int K1 = k1_of(ctx->cfg.n_rbf);
  const uint8_t* img = (const uint8_t*)ctx->tc_weights;  // the filter of block 0
  int grid = ctx->num_sms;
  if (N < grid) grid = N > 0 ? N : 1;
  const float qscale = 1.f / sqrtf((float)AD);
  auto go = [&](auto kern, int k1) {
    const size_t smem = at_layout(k1, NC).total + 1024;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return launch(ctx, NC == 1 ? K_ATTN_TC : K_ATTN_EQ_TC, kern, dim3(grid), dim3(AT_THREADS),
                  smem, s, N, K, pos, nbr, mask, (const __nv_bfloat16*)x, (const float*)ctx->q,
                  (const __half*)ctx->k, (__nv_bfloat16*)out, img, (const uint8_t*)ctx->tc_attn_p,
                  radial_of(ctx), qscale, ctx->status_d);
  };
  if (K1 == 64) return go(k_attn_tc<64, NC>, 64);
  if (K1 == 48) return go(k_attn_tc<48, NC>, 48);
  if (K1 == 32) return go(k_attn_tc<32, NC>, 32);
  return MP_ERR_INVALID_ARG;
}

int tc_attn_fwd(mp_ctx* ctx, int N, int K, const float* pos, const int* nbr,
                const unsigned char* mask, const void* x, void* out, cudaStream_t s) {
  return tc_attn_launch<1>(ctx, N, K, pos, nbr, mask, x, out, s);
}

bool tc_attn_eq_supported(const mp_ctx* ctx, int K) {
  return tc_attn_supported(ctx, K) && at_fits(k1_of(ctx->cfg.n_rbf), 9);
}

int tc_attn_eq_fwd(mp_ctx* ctx, int N, int K, const float* pos, const int* nbr,
                   const unsigned char* mask, const void* x, void* out, cudaStream_t s) {
  return tc_attn_launch<9>(ctx, N, K, pos, nbr, mask, x, out, s);
}

}  // namespace mp
