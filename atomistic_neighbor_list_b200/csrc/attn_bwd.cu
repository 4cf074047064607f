// Backward of the neighbor attention aggregation (E2Former-V2 page, section 3.2: the fused kernel
// per destination atom; its backward is the reverse-mode derivative of the same quantities).
// Given g = dL/dout it returns dL/dx and dL/dr (the negative forces when L is an energy).
//
// Per destination i, head h, valid slot s with source j (v = x_j (.) W(d_ij), alpha the softmax):
//   dalpha = sum_{c in h} g_i[c] v[c],   dl = alpha (dalpha - D_ih),  D_ih = sum_s alpha dalpha
//   dL/dq_i += dl k_j / sqrt(D)          dL/dk_j += dl q_i / sqrt(D)
//   dL/dx_j += alpha g_i (.) W           dL/dd = sum_h (alpha beta_h + dl b'_h)
//   beta_h = sum_{c in h} g_i[c] x_j[c] W'(d)[c],   b'_h = sum_k e_k'(d) P_kh
//   dL/dr_i += dL/dd (r_i - r_j)/d,      dL/dr_j -= the same.
// No atomics on the data: a destination pass (one CTA per row i) produces the row-side terms and
// the softmax statistics (max, sum, D) of each row; a source pass (one CTA per atom j) walks the
// transposed list -- the (i, slot) entries that read j, in ascending order -- recomputes each
// entry's filter and logit exactly as the destination pass did, and produces the source-side
// terms. The filter and its distance derivative are evaluated once per entry in each pass.
#include <cmath>

#include "mp_internal.cuh"
#include "tc_api.cuh"

namespace mp {
namespace {

constexpr int AB = 16;  // entries per batch

template <int F>
struct AbSmem {
  // rows of AB entries, read as float4 (one load serves four entries' FMAs)
  __align__(16) float rbf[kMaxR][AB];
  __align__(16) float drbf[kMaxR][AB];
  __align__(16) float h1[F][AB];
  __align__(16) float h1p[F][AB];
  int src[AB], dst[AB], ok[AB];
  float d[AB], fc[AB], dfc[AB], u[AB][3];
  float spart[AB][32];  // per entry and head: alpha beta + dl b' (source pass)
  float st[AB][3 * 32];  // per entry: its row's softmax statistics (source pass)
  float red[3][F / 32];
};

// Filter W and dW/dd of the batch's entries for feature f (every thread of the CTA calls it;
// s.d / s.fc / s.dfc / s.ok set for t < nb). Identical arithmetic in both passes.
template <int F>
__device__ __forceinline__ void filter_batch(AbSmem<F>& s, int nb, const float* __restrict__ A1,
                                             const float* __restrict__ A2, float c1f, float c2f,
                                             const Radial& rp, float (&W)[AB], float (&Wp)[AB]) {
  const int f = threadIdx.x;
  for (int idx = f; idx < rp.R * AB; idx += F) {
    const int k = idx / AB, t = idx % AB;
    const float dd = s.d[t] - (rp.mu_min + k * rp.dmu);
    const float e = expf(-rp.gamma * dd * dd);
    s.rbf[k][t] = e;
    s.drbf[k][t] = -2.f * rp.gamma * dd * e;
  }
  __syncthreads();
  float z[AB], tz[AB];
#pragma unroll
  for (int t = 0; t < AB; ++t) {
    z[t] = c1f;
    tz[t] = 0.f;
  }
  for (int k = 0; k < rp.R; ++k) {
    const float a = __ldg(A1 + k * F + f);
#pragma unroll
    for (int t4 = 0; t4 < AB; t4 += 4) {
      const float4 e = *(const float4*)&s.rbf[k][t4];
      const float4 de = *(const float4*)&s.drbf[k][t4];
      z[t4] = fmaf(e.x, a, z[t4]);
      z[t4 + 1] = fmaf(e.y, a, z[t4 + 1]);
      z[t4 + 2] = fmaf(e.z, a, z[t4 + 2]);
      z[t4 + 3] = fmaf(e.w, a, z[t4 + 3]);
      tz[t4] = fmaf(de.x, a, tz[t4]);
      tz[t4 + 1] = fmaf(de.y, a, tz[t4 + 1]);
      tz[t4 + 2] = fmaf(de.z, a, tz[t4 + 2]);
      tz[t4 + 3] = fmaf(de.w, a, tz[t4 + 3]);
    }
  }
  // thread f's row of AB values as float4 stores (the lanes of a warp conflict on these 64-byte
  // rows, but each row is written once per batch and read 4 x F times)
#pragma unroll
  for (int t4 = 0; t4 < AB; t4 += 4) {
    *(float4*)&s.h1[f][t4] = make_float4(ssp_f(z[t4]), ssp_f(z[t4 + 1]), ssp_f(z[t4 + 2]),
                                         ssp_f(z[t4 + 3]));
    *(float4*)&s.h1p[f][t4] =
        make_float4(sigmoid_f(z[t4]) * tz[t4], sigmoid_f(z[t4 + 1]) * tz[t4 + 1],
                    sigmoid_f(z[t4 + 2]) * tz[t4 + 2], sigmoid_f(z[t4 + 3]) * tz[t4 + 3]);
  }
  __syncthreads();
  float u[AB], up[AB];
#pragma unroll
  for (int t = 0; t < AB; ++t) {
    u[t] = c2f;
    up[t] = 0.f;
  }
  for (int g = 0; g < F; ++g) {
    const float a = __ldg(A2 + g * F + f);
#pragma unroll
    for (int t4 = 0; t4 < AB; t4 += 4) {
      const float4 h = *(const float4*)&s.h1[g][t4];
      const float4 hp = *(const float4*)&s.h1p[g][t4];
      u[t4] = fmaf(h.x, a, u[t4]);
      u[t4 + 1] = fmaf(h.y, a, u[t4 + 1]);
      u[t4 + 2] = fmaf(h.z, a, u[t4 + 2]);
      u[t4 + 3] = fmaf(h.w, a, u[t4 + 3]);
      up[t4] = fmaf(hp.x, a, up[t4]);
      up[t4 + 1] = fmaf(hp.y, a, up[t4 + 1]);
      up[t4 + 2] = fmaf(hp.z, a, up[t4 + 2]);
      up[t4 + 3] = fmaf(hp.w, a, up[t4 + 3]);
    }
  }
#pragma unroll
  for (int t = 0; t < AB; ++t) {
    W[t] = s.fc[t] * u[t];
    Wp[t] = fmaf(s.dfc[t], u[t], s.fc[t] * up[t]);
  }
}

// Sum over the D lanes of one head (D divides 32; the lanes of a head are adjacent).
__device__ __forceinline__ float head_sum(float v, int D) {
  for (int o = 1; o < D; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// The entry's geometry: distance, envelope and its derivative, unit vector (r_i - r_j) / d
// (zero at d = 0, where the pair contributes no position gradient).
__device__ __forceinline__ void entry_geometry(const float* __restrict__ pos, int i, int j,
                                               float r_c, float* d, float* fc, float* dfc,
                                               float* u) {
  const float dx = pos[3 * i] - pos[3 * j], dy = pos[3 * i + 1] - pos[3 * j + 1],
              dz = pos[3 * i + 2] - pos[3 * j + 2];
  const float dd = sqrtf(dx * dx + dy * dy + dz * dz);
  const float inv = dd > 0.f ? 1.f / dd : 0.f;
  *d = dd;
  *fc = cutoff_f(dd, r_c);
  *dfc = cutoff_grad_f(dd, r_c);
  u[0] = dx * inv;
  u[1] = dy * inv;
  u[2] = dz * inv;
}

// Logit of head h at this thread's channel: q_i . k_j / sqrt(D) (q pre-scaled) + radial bias.
__device__ __forceinline__ float logit_part(float qi, float kj, const float (*rbf)[AB], int t,
                                            const float* __restrict__ sP, int R, int H, int head,
                                            int c, int D) {
  float part = qi * kj;
  for (int k = c; k < R; k += D) part = fmaf(rbf[k][t], sP[k * H + head], part);
  return part;
}

__device__ __forceinline__ float bias_grad_part(const float (*drbf)[AB], int t,
                                                const float* __restrict__ sP, int R, int H,
                                                int head, int c, int D) {
  float part = 0.f;
  for (int k = c; k < R; k += D) part = fmaf(drbf[k][t], sP[k * H + head], part);
  return part;
}

// ------------------------------------------------------------------------------ destination pass
// One CTA (F threads, thread f = channel f of head f / D) per destination row. Dynamic shared
// memory per slot: logit, dalpha, beta, b' ([K][H] each), the unit vector [K][3] and the source
// [K]; the filter weights are read through L1 (they stay resident: every CTA reads the same).
template <typename T, int F>
__global__ void __launch_bounds__(F) k_attn_bwd_dst(
    int N, int K, const float* __restrict__ pos, const int* __restrict__ nbr,
    const unsigned char* __restrict__ mask, const T* __restrict__ x, const float* __restrict__ g,
    const float* __restrict__ q, const float* __restrict__ kx, FilterW fw, Radial rp,
    const float* __restrict__ P, const float* __restrict__ pb, int H, int D,
    float* __restrict__ gq, float* __restrict__ grad_pos, float* __restrict__ stats, int* status) {
  extern __shared__ float dsm[];
  const float* sP = P;
  float* sl = dsm;
  float* sda = sl + K * H;
  float* sbeta = sda + K * H;
  float* sbp = sbeta + K * H;
  float* su = sbp + K * H;
  int* ssrc = (int*)(su + 3 * K);
  __shared__ AbSmem<F> s;

  const int f = threadIdx.x, lane = f & 31, warp = f >> 5;
  const int head = f / D, c = f % D;
  const float c1f = fw.c1[f], c2f = fw.c2[f];
  const float inv_sqrt_d = rsqrtf((float)D);

  for (int i = blockIdx.x; i < N; i += gridDim.x) {
    const float qi = q[(size_t)i * F + f] * inv_sqrt_d;
    const float gi = g[(size_t)i * F + f];
    for (int s0 = 0; s0 < K; s0 += AB) {
      const int nb = min(AB, K - s0);
      if (f < AB) {
        const int t = f;
        int j = 0, ok = 0;
        float d = 0.f, fc = 0.f, dfc = 0.f, u[3] = {0.f, 0.f, 0.f};
        if (t < nb) {
          const size_t slot = (size_t)i * K + s0 + t;
          j = nbr[slot];
          ok = mask[slot] != 0;
          if (ok && (unsigned)j >= (unsigned)N) {
            raise_status(status, kStatusBounds);
            ok = 0;
          }
          if (ok) entry_geometry(pos, i, j, rp.r_c, &d, &fc, &dfc, u);
          else j = 0;
          ssrc[s0 + t] = ok ? j : -1;
          su[3 * (s0 + t)] = u[0];
          su[3 * (s0 + t) + 1] = u[1];
          su[3 * (s0 + t) + 2] = u[2];
        }
        s.src[t] = j;
        s.ok[t] = ok;
        s.d[t] = d;
        s.fc[t] = fc;
        s.dfc[t] = dfc;
      }
      __syncthreads();
      float W[AB], Wp[AB];
      filter_batch<F>(s, nb, fw.A1, fw.A2, c1f, c2f, rp, W, Wp);
      // the batch's row gathers issued together (s.src is 0 for empty entries: always in range)
      float xr[AB], kr[AB];
#pragma unroll
      for (int t = 0; t < AB; ++t) {
        xr[t] = ldf(x + (size_t)s.src[t] * F + f);
        kr[t] = kx[(size_t)s.src[t] * F + f];
      }
#pragma unroll
      for (int t = 0; t < AB; ++t) {
        if (t < nb && s.ok[t]) {  // uniform across the CTA
          const float xj = xr[t];
          const float l = head_sum(logit_part(qi, kr[t], s.rbf, t, sP, rp.R, H, head, c, D), D) +
                          pb[head];
          const float da = head_sum(gi * xj * W[t], D);
          const float be = head_sum(gi * xj * Wp[t], D);
          const float bp = head_sum(bias_grad_part(s.drbf, t, sP, rp.R, H, head, c, D), D);
          if (c == 0) {
            const int o = (s0 + t) * H + head;
            sl[o] = l;
            sda[o] = da;
            sbeta[o] = be;
            sbp[o] = bp;
          }
        }
      }
      __syncthreads();
    }
    // softmax statistics of head `head` over the valid slots (lanes c stride the slots)
    float m = -INFINITY;
    for (int sl0 = c; sl0 < K; sl0 += D)
      if (ssrc[sl0] >= 0) m = fmaxf(m, sl[sl0 * H + head]);
    for (int o = 1; o < D; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float z = 0.f;
    for (int sl0 = c; sl0 < K; sl0 += D)
      if (ssrc[sl0] >= 0) z += expf(sl[sl0 * H + head] - m);
    z = head_sum(z, D);
    const float iz = z > 0.f ? 1.f / z : 0.f;
    float Dh = 0.f;
    for (int sl0 = c; sl0 < K; sl0 += D)
      if (ssrc[sl0] >= 0) Dh += expf(sl[sl0 * H + head] - m) * iz * sda[sl0 * H + head];
    Dh = head_sum(Dh, D);
    if (c == 0) {
      stats[(size_t)i * 3 * H + head] = m;
      stats[(size_t)i * 3 * H + H + head] = z;
      stats[(size_t)i * 3 * H + 2 * H + head] = Dh;
    }
    // dL/dq_i: every valid slot's dl times k_j
    float acc = 0.f;
    for (int b0 = 0; b0 < K; b0 += 8) {  // eight independent gathers in flight
      float kv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = b0 + u < K ? ssrc[b0 + u] : -1;
        kv[u] = j >= 0 ? kx[(size_t)j * F + f] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int sl0 = b0 + u;
        if (sl0 < K && ssrc[sl0] >= 0) {  // uniform
          const int o = sl0 * H + head;
          const float a = expf(sl[o] - m) * iz;
          acc = fmaf(a * (sda[o] - Dh), kv[u], acc);
        }
      }
    }
    gq[(size_t)i * F + f] = acc * inv_sqrt_d;
    // dL/dr_i: each slot's dL/dd summed over the heads (thread f takes slots f, f + F, ...)
    __syncthreads();  // every head's statistics are needed below: publish them through smem
    if (c == 0) {
      s.spart[0][head] = m;
      s.spart[1][head] = iz;
      s.spart[2][head] = Dh;
    }
    __syncthreads();
    float gp[3] = {0.f, 0.f, 0.f};
    for (int sl0 = f; sl0 < K; sl0 += F) {
      if (ssrc[sl0] < 0) continue;
      float sd = 0.f;
      for (int h = 0; h < H; ++h) {
        const int o = sl0 * H + h;
        const float a = expf(sl[o] - s.spart[0][h]) * s.spart[1][h];
        sd = fmaf(a, sbeta[o], sd);
        sd = fmaf(a * (sda[o] - s.spart[2][h]), sbp[o], sd);
      }
      gp[0] = fmaf(sd, su[3 * sl0], gp[0]);
      gp[1] = fmaf(sd, su[3 * sl0 + 1], gp[1]);
      gp[2] = fmaf(sd, su[3 * sl0 + 2], gp[2]);
    }
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      float v = gp[a];
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) s.red[a][warp] = v;
    }
    __syncthreads();
    if (f < 3) {
      float v = 0.f;
      for (int w = 0; w < F / 32; ++w) v += s.red[f][w];
      grad_pos[3 * i + f] = v;
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------------------ source pass
// One CTA per source atom j over its transposed entries key = i * K + slot (ascending). Writes
// dL/dx_j (value path; the projections are added afterwards), dL/dk_j, and adds the source-side
// position gradient to grad_pos[j].
template <typename T, int F>
__global__ void __launch_bounds__(F) k_attn_bwd_src(
    int N, int K, const float* __restrict__ pos, const int* __restrict__ rev_ptr,
    const int* __restrict__ rev, const T* __restrict__ x, const float* __restrict__ g,
    const float* __restrict__ q, const float* __restrict__ kx, FilterW fw, Radial rp,
    const float* __restrict__ P, const float* __restrict__ pb, int H, int D,
    const float* __restrict__ stats, float* __restrict__ grad_x, float* __restrict__ gk,
    float* __restrict__ grad_pos, int* status) {
  const float* sP = P;
  __shared__ AbSmem<F> s;

  const int f = threadIdx.x, lane = f & 31, warp = f >> 5;
  const int head = f / D, c = f % D;
  const float c1f = fw.c1[f], c2f = fw.c2[f];
  const float inv_sqrt_d = rsqrtf((float)D);

  for (int j = blockIdx.x; j < N; j += gridDim.x) {
    const int r0 = rev_ptr[j], r1 = rev_ptr[j + 1];
    const float xj = ldf(x + (size_t)j * F + f);
    const float kj = kx[(size_t)j * F + f];
    float acc_k = 0.f, acc_x = 0.f;
    float gp[3] = {0.f, 0.f, 0.f};
    for (int e0 = r0; e0 < r1; e0 += AB) {
      const int nb = min(AB, r1 - e0);
      if (f < AB) {
        const int t = f;
        int i = 0, ok = 0;
        float d = 0.f, fc = 0.f, dfc = 0.f, u[3] = {0.f, 0.f, 0.f};
        if (t < nb) {
          i = rev[e0 + t] / K;
          ok = (unsigned)i < (unsigned)N;
          if (ok) {
            entry_geometry(pos, i, j, rp.r_c, &d, &fc, &dfc, u);
          } else {
            raise_status(status, kStatusBounds);
            i = 0;
          }
        }
        if (ok)
          for (int k = 0; k < 3 * H; ++k) s.st[t][k] = stats[(size_t)i * 3 * H + k];
        s.dst[t] = i;
        s.ok[t] = ok;
        s.d[t] = d;
        s.fc[t] = fc;
        s.dfc[t] = dfc;
        s.u[t][0] = u[0];
        s.u[t][1] = u[1];
        s.u[t][2] = u[2];
      }
      __syncthreads();
      float W[AB], Wp[AB];
      filter_batch<F>(s, nb, fw.A1, fw.A2, c1f, c2f, rp, W, Wp);
      float qr[AB], gr[AB];  // the batch's row gathers issued together (s.dst is 0 when empty)
#pragma unroll
      for (int t = 0; t < AB; ++t) {
        qr[t] = q[(size_t)s.dst[t] * F + f];
        gr[t] = g[(size_t)s.dst[t] * F + f];
      }
#pragma unroll
      for (int t = 0; t < AB; ++t) {
        if (t < nb && s.ok[t]) {  // uniform across the CTA
          const float qi = qr[t] * inv_sqrt_d;
          const float gi = gr[t];
          const float* st = s.st[t];
          const float l = head_sum(logit_part(qi, kj, s.rbf, t, sP, rp.R, H, head, c, D), D) +
                          pb[head];
          const float z = st[H + head];
          const float a = z > 0.f ? expf(l - st[head]) * (1.f / z) : 0.f;
          const float da = head_sum(gi * xj * W[t], D);
          const float be = head_sum(gi * xj * Wp[t], D);
          const float bp = head_sum(bias_grad_part(s.drbf, t, sP, rp.R, H, head, c, D), D);
          const float dl = a * (da - st[2 * H + head]);
          acc_k = fmaf(dl, qi, acc_k);
          acc_x = fmaf(a * gi, W[t], acc_x);
          if (c == 0) s.spart[t][head] = fmaf(a, be, dl * bp);
        } else if (t < nb && c == 0) {
          s.spart[t][head] = 0.f;
        }
      }
      __syncthreads();
      if (f < nb) {  // this entry's dL/dd over the heads, times -(r_i - r_j)/d
        float sd = 0.f;
        for (int h = 0; h < H; ++h) sd += s.spart[f][h];
        gp[0] = fmaf(-sd, s.u[f][0], gp[0]);
        gp[1] = fmaf(-sd, s.u[f][1], gp[1]);
        gp[2] = fmaf(-sd, s.u[f][2], gp[2]);
      }
      __syncthreads();
    }
    grad_x[(size_t)j * F + f] = acc_x;
    gk[(size_t)j * F + f] = acc_k;
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      float v = gp[a];
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) s.red[a][warp] = v;
    }
    __syncthreads();
    if (f < 3) {
      float v = 0.f;
      for (int w = 0; w < F / 32; ++w) v += s.red[f][w];
      grad_pos[3 * j + f] += v;  // the destination pass wrote the row-side part
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------------------ transposed list
__global__ void k_rev_count(int N, int K, const int* __restrict__ nbr,
                            const unsigned char* __restrict__ mask, int* __restrict__ cnt) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (long long)N * K) return;
  const int j = nbr[e];
  if (mask[e] != 0 && (unsigned)j < (unsigned)N) atomicAdd(&cnt[j + 1], 1);
}

__global__ void k_rev_fill(int N, int K, const int* __restrict__ nbr,
                           const unsigned char* __restrict__ mask, const int* __restrict__ rev_ptr,
                           int* __restrict__ cursor, int* __restrict__ tmp) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (long long)N * K) return;
  const int j = nbr[e];
  if (mask[e] != 0 && (unsigned)j < (unsigned)N)
    tmp[rev_ptr[j] + atomicAdd(&cursor[j], 1)] = (int)e;  // e = i * K + slot
}

// each atom's entries in ascending key order: an entry goes to its rank within the atom's run
__global__ void k_rev_sort(int N, const int* __restrict__ rev_ptr, const int* __restrict__ tmp,
                           int* __restrict__ rev) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int j = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; j < N; j += warps) {
    const int a = rev_ptr[j], b = rev_ptr[j + 1];
    for (int c = a + lane; c < b; c += 32) {
      const int key = tmp[c];
      int r = 0;
      for (int o = a; o < b; ++o) r += tmp[o] < key ? 1 : 0;
      rev[a + r] = key;
    }
  }
}

template <typename T, int F>
int run_attn_bwd(mp_ctx* c, int N, int K, const float* pos, const int* nbr,
                 const unsigned char* mask, const void* x, const float* g, float* grad_x,
                 float* grad_pos, const int* rev_ptr, const int* rev, cudaStream_t s) {
  const int H = c->cfg.n_heads, D = c->cfg.head_dim;
  const size_t smem_dst = (4 * (size_t)K * H + 3 * (size_t)K) * 4 + (size_t)K * 4;
  auto kd = k_attn_bwd_dst<T, F>;
  auto ks = k_attn_bwd_src<T, F>;
  int optin = 0;
  cudaFuncAttributes fa;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, c->device) !=
          cudaSuccess ||
      cudaFuncGetAttributes(&fa, kd) != cudaSuccess)
    return MP_ERR_CUDA;
  if (fa.sharedSizeBytes + smem_dst > (size_t)optin) return MP_ERR_CAPACITY;
  if (cudaFuncSetAttribute(kd, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_dst) !=
      cudaSuccess) {
    cudaGetLastError();
    return MP_ERR_CAPACITY;  // K too large for the per-slot arrays on chip
  }
  // as many resident CTAs as fit, every SM busy (rows and sources are independent work items)
  int occ_d = 1, occ_s = 1;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_d, kd, F, smem_dst);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_s, ks, F, 0);
  const long long cap_d = (long long)c->num_sms * (occ_d > 0 ? occ_d : 1);
  const long long cap_s = (long long)c->num_sms * (occ_s > 0 ? occ_s : 1);
  const int grid_d = (int)(N < cap_d ? N : cap_d), grid_s = (int)(N < cap_s ? N : cap_s);
  float* gq = c->g_x;     // [N][F] scratch: dL/dq
  float* gk = c->grad_h;  // [N][F] scratch: dL/dk
  // destination pass: on the tensor cores where the bf16 kernel covers the shape
  int rc = tc_attn_bwd_supported(c, K)
               ? tc_attn_bwd_dst(c, N, K, pos, nbr, mask, x, g, gq, grad_pos, s)
               : launch(c, K_ATTN_BWD, kd, dim3(grid_d), dim3(F), smem_dst, s, N, K, pos, nbr,
                        mask, (const T*)x, g, (const float*)c->q, (const float*)c->k,
                        filter_of(c, 0), radial_of(c), (const float*)c->P, (const float*)c->p, H,
                        D, gq, grad_pos, c->attn_stats, c->status_d);
  if (rc == MP_OK && tc_attn_bwd_supported(c, K))
    rc = tc_attn_bwd_src(c, N, K, pos, rev_ptr, rev, x, g, grad_x, gk, grad_pos, s);
  else if (rc == MP_OK)
    rc = launch(c, K_ATTN_BWD_SRC, ks, dim3(grid_s), dim3(F), 0, s, N, K, pos, rev_ptr, rev,
                (const T*)x, g, (const float*)c->q, (const float*)c->k, filter_of(c, 0),
                radial_of(c), (const float*)c->P, (const float*)c->p, H, D,
                (const float*)c->attn_stats, grad_x, gk, grad_pos, c->status_d);
  // dL/dx += dL/dq Wq^T + dL/dk Wk^T
  if (rc == MP_OK)
    rc = launch_dense(c, N, F, F, gq, false, c->WqT, nullptr, true, grad_x, false, s);
  if (rc == MP_OK)
    rc = launch_dense(c, N, F, F, gk, false, c->WkT, nullptr, true, grad_x, false, s);
  return rc;
}

}  // namespace
}  // namespace mp

using namespace mp;

extern "C" int mp_attn_bwd(mp_ctx* c, int N, int K, const float* pos, const int* nbr,
                           const unsigned char* mask, const void* x, const float* g_out,
                           float* grad_x, float* grad_pos, void* stream) {
  if (!c || N < 0 || K < 1 ||
      (N > 0 && (!pos || !nbr || !mask || !x || !g_out || !grad_x || !grad_pos)))
    return MP_ERR_INVALID_ARG;
  if (c->cfg.n_heads < 1 || c->cfg.n_heads > 32 || c->cfg.head_dim < 1 ||
      32 % c->cfg.head_dim != 0 || c->cfg.n_heads * c->cfg.head_dim != c->cfg.F || !c->WqT)
    return MP_ERR_INVALID_ARG;
  if (N > c->cfg.max_atoms) return MP_ERR_CAPACITY;
  if ((long long)N * K > 0x7fffffffLL) return MP_ERR_CAPACITY;
  if (N == 0) return MP_OK;
  cudaStream_t s = (cudaStream_t)stream;
  const int F = c->cfg.F;
  const bool bf = c->cfg.dtype == MP_BF16;
  int rc = attn_project(c, N, x, s);
  if (rc != MP_OK) return rc;
  // the transposed list: for each source j, the (row, slot) entries reading it, ascending
  const long long NK = (long long)N * K;
  const int nb = scan_blocks(N) > 0 ? scan_blocks(N) : 1;
  const size_t bytes = 4 * ((size_t)(N + 1) + (size_t)N + 2 * (size_t)NK) + 8 * (size_t)nb + 16;
  char* buf = nullptr;
  if (scratch_alloc((void**)&buf, bytes, s) != cudaSuccess) return MP_ERR_CUDA;
  int* rev_ptr = (int*)buf;
  int* cursor = rev_ptr + N + 1;
  int* tmp = cursor + N;
  int* rev = tmp + NK;
  long long* bsum = (long long*)(((uintptr_t)(rev + NK) + 15) & ~(uintptr_t)15);
  int* overflow = (int*)(bsum + nb);
  cudaMemsetAsync(rev_ptr, 0, 4 * ((size_t)N + 1 + (size_t)N), s);
  cudaMemsetAsync(overflow, 0, 4, s);
  const int eb = (int)((NK + 255) / 256);
  rc = launch(c, K_ATTN_REV, k_rev_count, dim3(eb), dim3(256), 0, s, N, K, nbr, mask, rev_ptr);
  if (rc == MP_OK) {
    launch_scan(N, rev_ptr, bsum, overflow, s);
    rc = launch(c, K_ATTN_REV, k_rev_fill, dim3(eb), dim3(256), 0, s, N, K, nbr, mask,
                (const int*)rev_ptr, cursor, tmp);
  }
  if (rc == MP_OK)
    rc = launch(c, K_ATTN_REV, k_rev_sort, dim3(c->num_sms * 8), dim3(256), 0, s, N,
                (const int*)rev_ptr, (const int*)tmp, rev);
  if (rc == MP_OK) {
    if (F == 64)
      rc = bf ? run_attn_bwd<__nv_bfloat16, 64>(c, N, K, pos, nbr, mask, x, g_out, grad_x,
                                                grad_pos, rev_ptr, rev, s)
              : run_attn_bwd<float, 64>(c, N, K, pos, nbr, mask, x, g_out, grad_x, grad_pos,
                                        rev_ptr, rev, s);
    else if (F == 128)
      rc = bf ? run_attn_bwd<__nv_bfloat16, 128>(c, N, K, pos, nbr, mask, x, g_out, grad_x,
                                                 grad_pos, rev_ptr, rev, s)
              : run_attn_bwd<float, 128>(c, N, K, pos, nbr, mask, x, g_out, grad_x, grad_pos,
                                         rev_ptr, rev, s);
    else
      rc = MP_ERR_INVALID_ARG;
  }
  scratch_free(buf, s);
  return rc;
}
