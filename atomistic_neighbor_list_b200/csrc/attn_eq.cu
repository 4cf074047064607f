// Neighbor attention with an equivariant value path (E2Former-V2 page, section 3.1: direction
// enters only through the values, the attention weights stay scalar). Per destination i, head h,
// valid slot j:
//   out_i[lm, c] = sum_j alpha_ij,h(c) (x_j (.) W(d_ij))[c] S_lm(r_j - r_i),   l <= 2,
// with the softmax weights of the scalar attention and S the regular solid harmonics |r|^l Y_lm
// (real, orthonormal on the sphere, m = -l..l). The page's node-centric form couples each source
// with the harmonics of its own position and the destination afterwards; that needs moments up to
// |r|^2 of absolute positions, whose cancellation costs digits in fp32, so here S is evaluated per
// edge on chip from the edge vector the distance already needs -- the same sum, streamed, with no
// edge tensor in memory and one online softmax (running maximum and normaliser) per head.
#include "mp_internal.cuh"
#include "tc_api.cuh"

namespace mp {
namespace {

constexpr int QB = 16;  // slots per batch
constexpr int NSH = 9;  // solid harmonics l <= 2

template <typename T, int F>
__global__ void __launch_bounds__(F) k_attn_eq_simt(
    int N, int K, const float* __restrict__ pos, const int* __restrict__ nbr,
    const unsigned char* __restrict__ mask, const T* __restrict__ x, const float* __restrict__ q,
    const float* __restrict__ kx, T* __restrict__ out, FilterW fw, Radial rp,
    const float* __restrict__ P, const float* __restrict__ pb, int H, int D, int* status) {
  __shared__ float s_rbf[kMaxR][QB];
  __shared__ float s_h1[F][QB + 1];
  __shared__ float s_sh[NSH][QB];
  __shared__ int s_src[QB], s_ok[QB];
  __shared__ float s_d[QB], s_fc[QB];

  const int f = threadIdx.x;
  const int head = f / D, c = f % D;
  const float c1f = fw.c1[f], c2f = fw.c2[f];
  const float inv_sqrt_d = rsqrtf((float)D);

  for (int i = blockIdx.x; i < N; i += gridDim.x) {
    const float qi = q[(size_t)i * F + f] * inv_sqrt_d;
    float mu = -INFINITY, z = 0.f, acc[NSH];
#pragma unroll
    for (int m = 0; m < NSH; ++m) acc[m] = 0.f;
    for (int s0 = 0; s0 < K; s0 += QB) {
      const int nb = min(QB, K - s0);
      if (f < QB) {
        const int t = f;
        int j = 0, ok = 0;
        float d = 0.f, fc = 0.f, S[NSH] = {};
        if (t < nb) {
          const size_t slot = (size_t)i * K + s0 + t;
          j = nbr[slot];
          ok = mask[slot] != 0;
          if (ok && (unsigned)j >= (unsigned)N) {
            raise_status(status, kStatusBounds);
            ok = 0;
          }
          if (ok) {
            const float rx = pos[3 * j] - pos[3 * i], ry = pos[3 * j + 1] - pos[3 * i + 1],
                        rz = pos[3 * j + 2] - pos[3 * i + 2];
            d = sqrtf(rx * rx + ry * ry + rz * rz);
            fc = cutoff_f(d, rp.r_c);
            solid_harmonics9(rx, ry, rz, S);
          } else {
            j = 0;
          }
        }
        s_src[t] = j;
        s_ok[t] = ok;
        s_d[t] = d;
        s_fc[t] = fc;
#pragma unroll
        for (int m = 0; m < NSH; ++m) s_sh[m][t] = S[m];
      }
      __syncthreads();
      for (int idx = f; idx < rp.R * QB; idx += F) {
        const int k = idx / QB, t = idx % QB;
        const float dd = s_d[t] - (rp.mu_min + k * rp.dmu);
        s_rbf[k][t] = expf(-rp.gamma * dd * dd);
      }
      __syncthreads();
      float zz[QB];
#pragma unroll
      for (int t = 0; t < QB; ++t) zz[t] = c1f;
      for (int k = 0; k < rp.R; ++k) {
        const float a = __ldg(fw.A1 + k * F + f);
#pragma unroll
        for (int t = 0; t < QB; ++t) zz[t] = fmaf(s_rbf[k][t], a, zz[t]);
      }
#pragma unroll
      for (int t = 0; t < QB; ++t) s_h1[f][t] = ssp_f(zz[t]);
      __syncthreads();
      float u[QB];
#pragma unroll
      for (int t = 0; t < QB; ++t) u[t] = c2f;
      for (int g = 0; g < F; ++g) {
        const float a = __ldg(fw.A2 + g * F + f);
#pragma unroll
        for (int t = 0; t < QB; ++t) u[t] = fmaf(s_h1[g][t], a, u[t]);
      }
      float xr[QB], kr[QB];  // the batch's row gathers issued together (s_src is 0 when empty)
#pragma unroll
      for (int t = 0; t < QB; ++t) {
        xr[t] = ldf(x + (size_t)s_src[t] * F + f);
        kr[t] = kx[(size_t)s_src[t] * F + f];
      }
#pragma unroll
      for (int t = 0; t < QB; ++t) {
        if (t < nb && s_ok[t]) {  // uniform across the CTA
          float part = qi * kr[t];
          for (int k = c; k < rp.R; k += D) part = fmaf(s_rbf[k][t], __ldg(P + k * H + head), part);
          for (int o = 1; o < D; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
          const float l = part + pb[head];
          const float v = xr[t] * s_fc[t] * u[t];
          const float mnew = fmaxf(mu, l);
          const float scale = expf(mu - mnew);  // 0 on the first valid neighbor
          const float w = expf(l - mnew) * v;
#pragma unroll
          for (int m = 0; m < NSH; ++m) acc[m] = fmaf(acc[m], scale, w * s_sh[m][t]);
          z = fmaf(z, scale, expf(l - mnew));
          mu = mnew;
        }
      }
      __syncthreads();
    }
    const float iz = z > 0.f ? 1.f / z : 0.f;
#pragma unroll
    for (int m = 0; m < NSH; ++m) stf(out + ((size_t)i * NSH + m) * F + f, acc[m] * iz);
  }
}

template <typename T, int F>
int run_attn_eq(mp_ctx* c, int N, int K, const float* pos, const int* nbr,
                const unsigned char* mask, const void* x, void* out, cudaStream_t s) {
  auto kern = k_attn_eq_simt<T, F>;
  int occ = 1;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, F, 0);
  const long long cap = (long long)c->num_sms * (occ > 0 ? occ : 1);
  const int grid = (int)(N < cap ? N : cap);
  return launch(c, K_ATTN_EQ, kern, dim3(grid), dim3(F), 0, s, N, K, pos, nbr, mask,
                (const T*)x, (const float*)c->q, (const float*)c->k, (T*)out, filter_of(c, 0),
                radial_of(c), (const float*)c->P, (const float*)c->p, c->cfg.n_heads,
                c->cfg.head_dim, c->status_d);
}

}  // namespace
}  // namespace mp

using namespace mp;

extern "C" int mp_attn_eq_fwd(mp_ctx* c, int N, int K, const float* pos, const int* nbr,
                              const unsigned char* mask, const void* x, void* out,
                              void* stream) {
  if (!c || N < 0 || K < 1 || (N > 0 && (!pos || !nbr || !mask || !x || !out)))
    return MP_ERR_INVALID_ARG;
  if (c->cfg.n_heads < 1 || c->cfg.head_dim < 1 || 32 % c->cfg.head_dim != 0 ||
      c->cfg.n_heads * c->cfg.head_dim != c->cfg.F)
    return MP_ERR_INVALID_ARG;
  if (N > c->cfg.max_atoms) return MP_ERR_CAPACITY;
  if (N == 0) return MP_OK;
  cudaStream_t s = (cudaStream_t)stream;
  const int F = c->cfg.F;
  const bool bf = c->cfg.dtype == MP_BF16;
  const bool tc = tc_attn_eq_supported(c, K) && ((uintptr_t)x & 15) == 0;
  int rc = attn_project(c, N, x, s, tc);
  if (rc != MP_OK) return rc;
  if (tc) return tc_attn_eq_fwd(c, N, K, pos, nbr, mask, x, out, s);
  if (F == 64)
    return bf ? run_attn_eq<__nv_bfloat16, 64>(c, N, K, pos, nbr, mask, x, out, s)
              : run_attn_eq<float, 64>(c, N, K, pos, nbr, mask, x, out, s);
  if (F == 128)
    return bf ? run_attn_eq<__nv_bfloat16, 128>(c, N, K, pos, nbr, mask, x, out, s)
              : run_attn_eq<float, 128>(c, N, K, pos, nbr, mask, x, out, s);
  return MP_ERR_INVALID_ARG;
}
