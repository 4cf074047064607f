// SIMT (CUDA-core, fp32 math) kernels: atomwise layers, readout, fused cfconv forward and backward,
// neighbor attention with an online softmax, and the device CSR check.
//
// The fused cfconv follows the FlashSchNet page (technical summary s.2.1-2.3): per destination-row
// range, edges are streamed in CSR order; distance, Gaussian basis and cosine envelope are computed
// on chip and never stored (s.2.1); the filter MLP, the gather of x_j and the filter product run in
// the same kernel with no edge tensor in memory (s.2.2); the reduction into the destination row is
// a register accumulation written once per row, no atomics (s.2.3). One thread owns one feature
// column, so the gather of x_j rows and the row writes are coalesced and the segment sum is a plain
// in-register sum. These kernels are the fp32 path and the cross-check of the tensor-core path.
#include "mp_internal.cuh"

namespace mp {

constexpr int EB = 16;     // edges per batch
constexpr int ROWS = 16;   // destination rows per CTA work item (at most; small systems take fewer)

FilterW filter_of(const mp_ctx* ctx, int b) {
  return FilterW{ctx->A1[b], ctx->c1[b], ctx->A2[b], ctx->c2[b]};
}

Radial radial_of(const mp_ctx* ctx) {
  Radial r;
  r.R = ctx->cfg.n_rbf;
  r.gamma = ctx->cfg.gamma;
  r.mu_min = ctx->cfg.mu_min;
  r.dmu = (ctx->cfg.mu_max - ctx->cfg.mu_min) / (float)(ctx->cfg.n_rbf - 1);
  r.r_c = ctx->cfg.r_c;
  return r;
}

// Destination rows per CTA work item of the fp32 cfconv kernels: up to ROWS, fewer when that would
// leave SMs idle (a 512-atom system in 16-row items is 32 CTAs of F threads on 148 SMs).
static int rows_for(const mp_ctx* ctx, int N, int ctas_per_sm) {
  const long long slots = (long long)ctx->num_sms * ctas_per_sm;
  const long long r = (N + slots - 1) / slots;
  return (int)(r < 1 ? 1 : (r > ROWS ? ROWS : r));
}

static int grid_for(const mp_ctx* ctx, long long items, int per_cta_items, int ctas_per_sm) {
  long long need = (items + per_cta_items - 1) / per_cta_items;
  long long cap = (long long)ctx->num_sms * ctas_per_sm;
  if (need < 1) need = 1;
  return (int)(need < cap ? need : cap);
}

// ------------------------------------------------------------------------------------ embedding
// x[i][f] = emb[types[i]][f], four features per thread (16-byte loads and stores; F / 4 = 2^q4)
__global__ void k_embed(int N, int F, int n_types, const int* __restrict__ types,
                        const float* __restrict__ emb, float* __restrict__ x, int* status) {
  const int q4 = F == 128 ? 5 : 4;
  const long long total = (long long)N << q4;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int i = (int)(idx >> q4), f4 = (int)(idx & ((1 << q4) - 1));
    int t = __ldg(types + i);
    if ((unsigned)t >= (unsigned)n_types) {
      raise_status(status, kStatusBounds);
      t = 0;
    }
    reinterpret_cast<float4*>(x)[idx] = __ldg(reinterpret_cast<const float4*>(emb) + ((size_t)t << q4) + f4);
  }
}

int launch_embed(mp_ctx* ctx, int N, const int* types, cudaStream_t s) {
  int F = ctx->cfg.F;
  int grid = grid_for(ctx, (long long)N * F / 4, 256, 8);
  return launch(ctx, K_EMBED, k_embed, dim3(grid), dim3(256), 0, s, N, F, ctx->cfg.n_types, types,
                (const float*)ctx->emb, ctx->x_res, ctx->status_d);
}

// ------------------------------------------------------------------------------------ dense
// out[i][o] = sum_k in[i][k] W[k][o] + b[o]  (+ out[i][o] if residual). One thread per output column,
// DR rows per CTA staged in shared memory.
constexpr int DR = 32;

template <typename TI, typename TO>
__global__ void k_dense(int N, int Fin, int Fout, const TI* __restrict__ in,
                        const float* __restrict__ W, const float* __restrict__ b, int residual,
                        TO* out) {
  __shared__ float s_in[DR][128 + 1];
  const int o = threadIdx.x;
  for (int r0 = blockIdx.x * DR; r0 < N; r0 += gridDim.x * DR) {
    const int nr = min(DR, N - r0);
    for (int idx = threadIdx.x; idx < nr * Fin; idx += blockDim.x) {
      int r = idx / Fin, k = idx % Fin;
      s_in[r][k] = ldf(in + (size_t)(r0 + r) * Fin + k);
    }
    __syncthreads();
    if (o < Fout) {
      float acc[DR];
      const float bias = b ? b[o] : 0.f;
#pragma unroll
      for (int r = 0; r < DR; ++r) acc[r] = bias;
      for (int k = 0; k < Fin; ++k) {
        const float w = __ldg(W + (size_t)k * Fout + o);
#pragma unroll
        for (int r = 0; r < DR; ++r) acc[r] = fmaf(s_in[r][k], w, acc[r]);
      }
#pragma unroll
      for (int r = 0; r < DR; ++r) {
        if (r < nr) {
          TO* dst = out + (size_t)(r0 + r) * Fout + o;
          float v = acc[r];
          if (residual) v += ldf((const TO*)dst);
          stf(dst, v);
        }
      }
    }
    __syncthreads();
  }
}

int launch_dense(mp_ctx* ctx, int N, int Fin, int Fout, const void* in, bool in_bf16,
                 const float* W, const float* b, bool residual, void* out, bool out_bf16,
                 cudaStream_t s) {
  if (Fin > 128 || Fout > 128) return MP_ERR_INVALID_ARG;
  int grid = grid_for(ctx, N, DR, 8);
  dim3 blk(Fout < 32 ? 32 : Fout);
  typedef __nv_bfloat16 bf;
  if (!in_bf16 && !out_bf16)
    return launch(ctx, K_DENSE, k_dense<float, float>, dim3(grid), blk, 0, s, N, Fin, Fout,
                  (const float*)in, W, b, (int)residual, (float*)out);
  if (in_bf16 && !out_bf16)
    return launch(ctx, K_DENSE, k_dense<bf, float>, dim3(grid), blk, 0, s, N, Fin, Fout,
                  (const bf*)in, W, b, (int)residual, (float*)out);
  if (!in_bf16 && out_bf16)
    return launch(ctx, K_DENSE, k_dense<float, bf>, dim3(grid), blk, 0, s, N, Fin, Fout,
                  (const float*)in, W, b, (int)residual, (bf*)out);
  return launch(ctx, K_DENSE, k_dense<bf, bf>, dim3(grid), blk, 0, s, N, Fin, Fout, (const bf*)in,
                W, b, (int)residual, (bf*)out);
}

// ------------------------------------------------------------------------------------ readout
// e_i = sum_k ssp(a_ik) B2_k + d2, one warp per atom.
__global__ void k_readout_energy(int N, int Fh, const float* __restrict__ a,
                                 const float* __restrict__ B2, const float* __restrict__ d2,
                                 float* __restrict__ e_atom) {
  const int lane = threadIdx.x & 31;
  long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (; warp < N; warp += nwarps) {
    float s = 0.f;
    for (int k = lane; k < Fh; k += 32) s = fmaf(ssp_f(a[warp * Fh + k]), B2[k], s);
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) e_atom[warp] = s + d2[0];
  }
}

int launch_readout(mp_ctx* ctx, int N, cudaStream_t s) {
  int grid = grid_for(ctx, N, 8, 16);
  return launch(ctx, K_READOUT_E, k_readout_energy, dim3(grid), dim3(256), 0, s, N,
                ctx->cfg.F / 2, (const float*)ctx->a, (const float*)ctx->B2,
                (const float*)ctx->d2, ctx->e_atom);
}

// u_ik = sigmoid(a_ik) B2_k  (de_i/da_ik)
__global__ void k_readout_bwd(int N, int Fh, const float* __restrict__ a,
                              const float* __restrict__ B2, float* __restrict__ u) {
  long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)N * Fh;
  for (; idx < total; idx += (long long)gridDim.x * blockDim.x)
    u[idx] = sigmoid_f(a[idx]) * B2[idx % Fh];
}

int launch_readout_bwd(mp_ctx* ctx, int N, cudaStream_t s) {
  int Fh = ctx->cfg.F / 2;
  int grid = grid_for(ctx, (long long)N * Fh, 256, 8);
  return launch(ctx, K_READOUT_BWD, k_readout_bwd, dim3(grid), dim3(256), 0, s, N, Fh,
                (const float*)ctx->a, (const float*)ctx->B2, ctx->u_ro);
}

// energy[g] = sum_{i in graph g} e_i: one CTA per graph, fixed-order tree sum (deterministic).
// Per-graph energy: a fixed-order sum in two launches. CTA (c, g) sums chunks c, c + C, c + 2C, ...
// of GS_CHUNK atoms of graph g (thread t the atoms chunk + t, + 256, ..., then a fixed tree) into
// part[g C + c]; then thread g sums part[g C .. g C + C) in order. The order depends only on N,
// the graph ranges and C, so the result is the same every run (one CTA per graph was a serial
// chain of loads: 91 us at 100,000 atoms).
constexpr int GS_CHUNK = 1024;

__global__ void k_graph_partial(int N, const int* __restrict__ graph_ptr, int n_graphs, int C,
                                const float* __restrict__ e_atom, float* __restrict__ part,
                                int* status) {
  __shared__ float s_part[256];
  const int g = blockIdx.y, c = blockIdx.x;
  const int lo = graph_ptr ? graph_ptr[g] : 0, hi = graph_ptr ? graph_ptr[g + 1] : N;
  const bool ok = lo >= 0 && hi <= N && hi >= lo;
  if (!ok && c == 0 && threadIdx.x == 0) raise_status(status, kStatusBounds);
  float s = 0.f;
  if (ok)
    for (int base = lo + c * GS_CHUNK; base < hi; base += C * GS_CHUNK)
#pragma unroll
      for (int k = 0; k < GS_CHUNK / 256; ++k) {
        const int i = base + 256 * k + (int)threadIdx.x;
        if (i < hi) s += e_atom[i];
      }
  s_part[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) s_part[threadIdx.x] += s_part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) part[(size_t)g * C + c] = s_part[0];
}

__global__ void k_graph_total(int n_graphs, int C, const float* __restrict__ part,
                              float* __restrict__ energy) {
  const int g = blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= n_graphs) return;
  float e = 0.f;
  for (int c = 0; c < C; ++c) e += part[(size_t)g * C + c];
  energy[g] = e;
}

int launch_graph_sum(mp_ctx* ctx, int N, const int* graph_ptr, int n_graphs, float* energy,
                     cudaStream_t s) {
  // C chunks per graph: C n_graphs <= N / GS_CHUNK + n_graphs, the size of ctx->gsum_part
  long long per = ((long long)N + (long long)n_graphs * GS_CHUNK - 1) / ((long long)n_graphs * GS_CHUNK);
  const int C = per < 1 ? 1 : (int)per;
  int rc = launch(ctx, K_GRAPH_SUM, k_graph_partial, dim3(C, n_graphs), dim3(256), 0, s, N,
                  graph_ptr, n_graphs, C, (const float*)ctx->e_atom, ctx->gsum_part,
                  ctx->status_d);
  if (rc != MP_OK) return rc;
  return launch(ctx, K_GRAPH_SUM, k_graph_total, dim3((n_graphs + 127) / 128), dim3(128), 0, s,
                n_graphs, C, (const float*)ctx->gsum_part, energy);
}

// ------------------------------------------------------------------------------------ cfconv fwd
// Shared layout per CTA: A1 [R][F], A2 [F][F] (dynamic), plus per-batch edge data.
template <typename T, int F>
__global__ void __launch_bounds__(F) k_cfconv_fwd_simt(
    int N, long long E, const float* __restrict__ pos, const int* __restrict__ row_ptr,
    const int* __restrict__ col_idx, const T* __restrict__ x, T* __restrict__ out, FilterW fw,
    Radial rp, int* status, int rows) {
  extern __shared__ float dsm[];
  float* sA1 = dsm;                 // [R][F]
  float* sA2 = dsm + rp.R * F;      // [F][F]
  __shared__ float s_rbf[kMaxR][EB];
  __shared__ float s_h1[F][EB + 1];
  __shared__ int s_src[EB], s_dst[EB];
  __shared__ float s_d[EB], s_fc[EB];

  const int f = threadIdx.x;
  for (int i = f; i < rp.R * F; i += F) sA1[i] = fw.A1[i];
  for (int i = f; i < F * F; i += F) sA2[i] = fw.A2[i];
  const float c1f = fw.c1[f], c2f = fw.c2[f];
  __syncthreads();

  for (int r0 = blockIdx.x * rows; r0 < N; r0 += gridDim.x * rows) {
    const int r1 = min(r0 + rows, N);
    const long long e_beg = clamp_off(row_ptr[r0], E);
    long long e_end = clamp_off(row_ptr[r1], E);
    if (e_end < e_beg) e_end = e_beg;
    int cur = r0;
    float acc = 0.f;
    for (long long eb = e_beg; eb < e_end; eb += EB) {
      const int nb = (int)min((long long)EB, e_end - eb);
      if (f < EB) {
        const int t = f;
        if (t < nb) {
          const long long e = eb + t;
          int r = r0;
          while (r + 1 < r1 && row_ptr[r + 1] <= e) ++r;
          int j = col_idx[e];
          float fc = 0.f, d = 0.f;
          if ((unsigned)j < (unsigned)N) {
            const float dx = pos[3 * r] - pos[3 * j], dy = pos[3 * r + 1] - pos[3 * j + 1],
                        dz = pos[3 * r + 2] - pos[3 * j + 2];
            d = sqrtf(dx * dx + dy * dy + dz * dz);
            fc = cutoff_f(d, rp.r_c);
          } else {
            raise_status(status, kStatusBounds);
            j = r;
          }
          s_src[t] = j;
          s_dst[t] = r;
          s_d[t] = d;
          s_fc[t] = fc;
        } else {
          s_src[t] = 0;
          s_dst[t] = -1;
          s_d[t] = 0.f;
          s_fc[t] = 0.f;
        }
      }
      __syncthreads();
      for (int idx = f; idx < rp.R * EB; idx += F) {
        const int k = idx / EB, t = idx % EB;
        const float dd = s_d[t] - (rp.mu_min + k * rp.dmu);
        s_rbf[k][t] = expf(-rp.gamma * dd * dd);
      }
      __syncthreads();
      float z[EB];
#pragma unroll
      for (int t = 0; t < EB; ++t) z[t] = c1f;
      for (int k = 0; k < rp.R; ++k) {
        const float a = sA1[k * F + f];
#pragma unroll
        for (int t = 0; t < EB; ++t) z[t] = fmaf(s_rbf[k][t], a, z[t]);
      }
#pragma unroll
      for (int t = 0; t < EB; ++t) s_h1[f][t] = ssp_f(z[t]);
      __syncthreads();
      float u[EB];
#pragma unroll
      for (int t = 0; t < EB; ++t) u[t] = c2f;
      for (int g = 0; g < F; ++g) {
        const float a = sA2[g * F + f];
#pragma unroll
        for (int t = 0; t < EB; ++t) u[t] = fmaf(s_h1[g][t], a, u[t]);
      }
#pragma unroll
      for (int t = 0; t < EB; ++t) {
        if (t < nb) {
          const int dst = s_dst[t];
          if (dst != cur) {
            stf(out + (size_t)cur * F + f, acc);
            for (int rr = cur + 1; rr < dst; ++rr) stf(out + (size_t)rr * F + f, 0.f);
            cur = dst;
            acc = 0.f;
          }
          acc = fmaf(s_fc[t] * u[t], ldf(x + (size_t)s_src[t] * F + f), acc);
        }
      }
      __syncthreads();
    }
    stf(out + (size_t)cur * F + f, acc);
    for (int rr = cur + 1; rr < r1; ++rr) stf(out + (size_t)rr * F + f, 0.f);
  }
}

template <typename T, int F>
static int run_fwd(mp_ctx* ctx, int block, int N, long long E, const float* pos, const int* rp,
                   const int* ci, const void* x, void* out, cudaStream_t s) {
  const int R = ctx->cfg.n_rbf;
  size_t smem = (size_t)(R * F + F * F) * sizeof(float);
  auto kern = k_cfconv_fwd_simt<T, F>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const int per_sm = F == 64 ? 4 : 2;  // CTAs one SM holds (shared memory)
  const int rows = rows_for(ctx, N, per_sm);
  int grid = grid_for(ctx, N, rows, per_sm);
  return launch(ctx, K_CFCONV_FWD_SIMT, kern, dim3(grid), dim3(F), smem, s, N, E, pos, rp, ci,
                (const T*)x, (T*)out, filter_of(ctx, block), radial_of(ctx), ctx->status_d, rows);
}

int launch_cfconv_fwd_simt(mp_ctx* ctx, int block, int N, long long E, const float* pos,
                           const int* rp, const int* ci, const void* x, void* out,
                           cudaStream_t s) {
  const bool bf = ctx->cfg.dtype == MP_BF16;
  if (ctx->cfg.F == 64)
    return bf ? run_fwd<__nv_bfloat16, 64>(ctx, block, N, E, pos, rp, ci, x, out, s)
              : run_fwd<float, 64>(ctx, block, N, E, pos, rp, ci, x, out, s);
  return bf ? run_fwd<__nv_bfloat16, 128>(ctx, block, N, E, pos, rp, ci, x, out, s)
            : run_fwd<float, 128>(ctx, block, N, E, pos, rp, ci, x, out, s);
}

// ------------------------------------------------------------------------------------ cfconv bwd
// For each destination row k of the symmetric CSR and edge j in row k:
//   grad_h[k] += g_j (.) W(d_kj)                                  (source-grouped reduce, s.2.3)
//   s_kj = sum_f (g_k h_j + g_j h_k)_f dW_f/dd(d_kj)
//   forces[k] -= s_kj (r_k - r_j) / d_kj
// dW/dd is carried forward from de/dd through both filter layers (forward-mode in d), so no
// edge-sized tensor is stored: the filter is recomputed.
template <typename T, int F>
__global__ void __launch_bounds__(F) k_cfconv_bwd_simt(
    int N, long long E, const float* __restrict__ pos, const int* __restrict__ row_ptr,
    const int* __restrict__ col_idx, const T* __restrict__ h, const T* __restrict__ g,
    float* __restrict__ grad_h, float* __restrict__ forces, int accumulate, FilterW fw, Radial rp,
    int* status, int rows) {
  extern __shared__ float dsm[];
  float* sA1 = dsm;
  float* sA2 = dsm + rp.R * F;
  __shared__ float s_e[kMaxR][EB], s_de[kMaxR][EB];
  __shared__ float s_h1[F][EB + 1], s_s1[F][EB + 1];
  __shared__ int s_src[EB], s_dst[EB];
  __shared__ float s_d[EB], s_fc[EB], s_dfc[EB], s_u[EB][3];
  __shared__ float s_part[F / 32][EB];
  __shared__ float s_s[EB];

  const int f = threadIdx.x, lane = f & 31, warp = f >> 5;
  for (int i = f; i < rp.R * F; i += F) sA1[i] = fw.A1[i];
  for (int i = f; i < F * F; i += F) sA2[i] = fw.A2[i];
  const float c1f = fw.c1[f], c2f = fw.c2[f];
  __syncthreads();

  for (int r0 = blockIdx.x * rows; r0 < N; r0 += gridDim.x * rows) {
    const int r1 = min(r0 + rows, N);
    const long long e_beg = clamp_off(row_ptr[r0], E);
    long long e_end = clamp_off(row_ptr[r1], E);
    if (e_end < e_beg) e_end = e_beg;
    int cur = r0;
    float acc = 0.f, fx = 0.f, fy = 0.f, fz = 0.f;
    for (long long eb = e_beg; eb < e_end; eb += EB) {
      const int nb = (int)min((long long)EB, e_end - eb);
      if (f < EB) {
        const int t = f;
        int j = 0, r = -1;
        float d = 0.f, fc = 0.f, dfc = 0.f, ux = 0.f, uy = 0.f, uz = 0.f;
        if (t < nb) {
          const long long e = eb + t;
          r = r0;
          while (r + 1 < r1 && row_ptr[r + 1] <= e) ++r;
          j = col_idx[e];
          if ((unsigned)j < (unsigned)N) {
            const float dx = pos[3 * r] - pos[3 * j], dy = pos[3 * r + 1] - pos[3 * j + 1],
                        dz = pos[3 * r + 2] - pos[3 * j + 2];
            d = sqrtf(dx * dx + dy * dy + dz * dz);
            fc = cutoff_f(d, rp.r_c);
            dfc = cutoff_grad_f(d, rp.r_c);
            if (d > 0.f) {
              const float inv = 1.f / d;
              ux = dx * inv;
              uy = dy * inv;
              uz = dz * inv;
            }
          } else {
            raise_status(status, kStatusBounds);
            j = r;
          }
        }
        s_src[t] = j;
        s_dst[t] = r;
        s_d[t] = d;
        s_fc[t] = fc;
        s_dfc[t] = dfc;
        s_u[t][0] = ux;
        s_u[t][1] = uy;
        s_u[t][2] = uz;
      }
      __syncthreads();
      for (int idx = f; idx < rp.R * EB; idx += F) {
        const int k = idx / EB, t = idx % EB;
        const float dd = s_d[t] - (rp.mu_min + k * rp.dmu);
        const float e = expf(-rp.gamma * dd * dd);
        s_e[k][t] = e;
        s_de[k][t] = -2.f * rp.gamma * dd * e;
      }
      __syncthreads();
      float z[EB], tz[EB];
#pragma unroll
      for (int t = 0; t < EB; ++t) {
        z[t] = c1f;
        tz[t] = 0.f;
      }
      for (int k = 0; k < rp.R; ++k) {
        const float a = sA1[k * F + f];
#pragma unroll
        for (int t = 0; t < EB; ++t) {
          z[t] = fmaf(s_e[k][t], a, z[t]);
          tz[t] = fmaf(s_de[k][t], a, tz[t]);
        }
      }
#pragma unroll
      for (int t = 0; t < EB; ++t) {
        s_h1[f][t] = ssp_f(z[t]);
        s_s1[f][t] = sigmoid_f(z[t]) * tz[t];
      }
      __syncthreads();
      float u[EB], v[EB];
#pragma unroll
      for (int t = 0; t < EB; ++t) {
        u[t] = c2f;
        v[t] = 0.f;
      }
      for (int gg = 0; gg < F; ++gg) {
        const float a = sA2[gg * F + f];
#pragma unroll
        for (int t = 0; t < EB; ++t) {
          u[t] = fmaf(s_h1[gg][t], a, u[t]);
          v[t] = fmaf(s_s1[gg][t], a, v[t]);
        }
      }
      // per-edge products; p = (g_k h_j + g_j h_k) dW/dd reduced over the F threads
      float gh[EB];
#pragma unroll
      for (int t = 0; t < EB; ++t) {
        float p = 0.f;
        gh[t] = 0.f;
        if (t < nb) {
          const int j = s_src[t], k = s_dst[t];
          const float gj = ldf(g + (size_t)j * F + f), hj = ldf(h + (size_t)j * F + f);
          const float gk = ldf(g + (size_t)k * F + f), hk = ldf(h + (size_t)k * F + f);
          const float W = s_fc[t] * u[t];
          const float Wp = s_dfc[t] * u[t] + s_fc[t] * v[t];
          gh[t] = gj * W;
          p = (gk * hj + gj * hk) * Wp;
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
        if (lane == 0) s_part[warp][t] = p;
      }
      __syncthreads();
      if (f < EB) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < F / 32; ++w) sum += s_part[w][f];
        s_s[f] = sum;
      }
      __syncthreads();
#pragma unroll
      for (int t = 0; t < EB; ++t) {
        if (t < nb) {
          const int dst = s_dst[t];
          if (dst != cur) {
            grad_h[(size_t)cur * F + f] = acc;
            if (f < 3) {
              const float fv = f == 0 ? fx : (f == 1 ? fy : fz);
              float* fp = forces + (size_t)cur * 3 + f;
              *fp = (accumulate ? *fp : 0.f) - fv;
            }
            for (int rr = cur + 1; rr < dst; ++rr) {
              grad_h[(size_t)rr * F + f] = 0.f;
              if (f < 3 && !accumulate) forces[(size_t)rr * 3 + f] = 0.f;
            }
            cur = dst;
            acc = 0.f;
            fx = fy = fz = 0.f;
          }
          acc += gh[t];
          const float sv = s_s[t];
          fx = fmaf(sv, s_u[t][0], fx);
          fy = fmaf(sv, s_u[t][1], fy);
          fz = fmaf(sv, s_u[t][2], fz);
        }
      }
      __syncthreads();
    }
    grad_h[(size_t)cur * F + f] = acc;
    if (f < 3) {
      const float fv = f == 0 ? fx : (f == 1 ? fy : fz);
      float* fp = forces + (size_t)cur * 3 + f;
      *fp = (accumulate ? *fp : 0.f) - fv;
    }
    for (int rr = cur + 1; rr < r1; ++rr) {
      grad_h[(size_t)rr * F + f] = 0.f;
      if (f < 3 && !accumulate) forces[(size_t)rr * 3 + f] = 0.f;
    }
  }
}

template <typename T, int F>
static int run_bwd(mp_ctx* ctx, int block, int N, long long E, const float* pos, const int* rp,
                   const int* ci, const void* h, const void* g, float* grad_h, float* forces,
                   bool acc, cudaStream_t s) {
  const int R = ctx->cfg.n_rbf;
  size_t smem = (size_t)(R * F + F * F) * sizeof(float);
  auto kern = k_cfconv_bwd_simt<T, F>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const int per_sm = F == 64 ? 3 : 1;  // CTAs one SM holds (shared memory)
  const int rows = rows_for(ctx, N, per_sm);
  int grid = grid_for(ctx, N, rows, per_sm);
  return launch(ctx, K_CFCONV_BWD_SIMT, kern, dim3(grid), dim3(F), smem, s, N, E, pos, rp, ci,
                (const T*)h, (const T*)g, grad_h, forces, (int)acc, filter_of(ctx, block),
                radial_of(ctx), ctx->status_d, rows);
}

int launch_cfconv_bwd_simt(mp_ctx* ctx, int block, int N, long long E, const float* pos,
                           const int* rp, const int* ci, const void* h, const void* g,
                           float* grad_h, float* forces, bool acc, cudaStream_t s) {
  const bool bf = ctx->cfg.dtype == MP_BF16;
  if (ctx->cfg.F == 64)
    return bf ? run_bwd<__nv_bfloat16, 64>(ctx, block, N, E, pos, rp, ci, h, g, grad_h, forces,
                                           acc, s)
              : run_bwd<float, 64>(ctx, block, N, E, pos, rp, ci, h, g, grad_h, forces, acc, s);
  return bf ? run_bwd<__nv_bfloat16, 128>(ctx, block, N, E, pos, rp, ci, h, g, grad_h, forces,
                                          acc, s)
            : run_bwd<float, 128>(ctx, block, N, E, pos, rp, ci, h, g, grad_h, forces, acc, s);
}

// ------------------------------------------------------------------------------------ attention
// E2Former-V2 page s.3.2: parallel over destination atoms, neighbors streamed in batches, online
// softmax with a running maximum mu and normaliser z per head, each neighbor's key and value
// computed once, padded slots skipped. One CTA per destination row (grid-stride), one thread per
// channel f (head f / D).
template <typename T, int F>
__global__ void __launch_bounds__(F) k_attn_simt(
    int N, int K, const float* __restrict__ pos, const int* __restrict__ nbr,
    const unsigned char* __restrict__ mask, const T* __restrict__ x, const float* __restrict__ q,
    const float* __restrict__ kx, T* __restrict__ out, FilterW fw, Radial rp,
    const float* __restrict__ P, const float* __restrict__ pb, int H, int D, int* status) {
  extern __shared__ float dsm[];
  float* sA1 = dsm;
  float* sA2 = dsm + rp.R * F;
  float* sP = sA2 + F * F;  // [R][H]
  __shared__ float s_rbf[kMaxR][EB];
  __shared__ float s_h1[F][EB + 1];
  __shared__ int s_src[EB], s_ok[EB];
  __shared__ float s_d[EB], s_fc[EB];

  const int f = threadIdx.x;
  const int head = f / D, c = f % D;
  for (int i = f; i < rp.R * F; i += F) sA1[i] = fw.A1[i];
  for (int i = f; i < F * F; i += F) sA2[i] = fw.A2[i];
  for (int i = f; i < rp.R * H; i += F) sP[i] = P[i];
  const float c1f = fw.c1[f], c2f = fw.c2[f];
  const float inv_sqrt_d = rsqrtf((float)D);
  __syncthreads();

  for (int i = blockIdx.x; i < N; i += gridDim.x) {
    const float qi = q[(size_t)i * F + f] * inv_sqrt_d;
    float mu = -INFINITY, z = 0.f, acc = 0.f;
    for (int s0 = 0; s0 < K; s0 += EB) {
      const int nb = min(EB, K - s0);
      if (f < EB) {
        const int t = f;
        int j = 0, ok = 0;
        float d = 0.f, fc = 0.f;
        if (t < nb) {
          const size_t slot = (size_t)i * K + s0 + t;
          j = nbr[slot];
          ok = mask[slot] != 0;
          if (ok && (unsigned)j >= (unsigned)N) {
            raise_status(status, kStatusBounds);
            ok = 0;
          }
          if (ok) {
            const float dx = pos[3 * i] - pos[3 * j], dy = pos[3 * i + 1] - pos[3 * j + 1],
                        dz = pos[3 * i + 2] - pos[3 * j + 2];
            d = sqrtf(dx * dx + dy * dy + dz * dz);
            fc = cutoff_f(d, rp.r_c);
          } else {
            j = 0;
          }
        }
        s_src[t] = j;
        s_ok[t] = ok;
        s_d[t] = d;
        s_fc[t] = fc;
      }
      __syncthreads();
      for (int idx = f; idx < rp.R * EB; idx += F) {
        const int k = idx / EB, t = idx % EB;
        const float dd = s_d[t] - (rp.mu_min + k * rp.dmu);
        s_rbf[k][t] = expf(-rp.gamma * dd * dd);
      }
      __syncthreads();
      float zz[EB];
#pragma unroll
      for (int t = 0; t < EB; ++t) zz[t] = c1f;
      for (int k = 0; k < rp.R; ++k) {
        const float a = sA1[k * F + f];
#pragma unroll
        for (int t = 0; t < EB; ++t) zz[t] = fmaf(s_rbf[k][t], a, zz[t]);
      }
#pragma unroll
      for (int t = 0; t < EB; ++t) s_h1[f][t] = ssp_f(zz[t]);
      __syncthreads();
      float u[EB];
#pragma unroll
      for (int t = 0; t < EB; ++t) u[t] = c2f;
      for (int g = 0; g < F; ++g) {
        const float a = sA2[g * F + f];
#pragma unroll
        for (int t = 0; t < EB; ++t) u[t] = fmaf(s_h1[g][t], a, u[t]);
      }
#pragma unroll
      for (int t = 0; t < EB; ++t) {
        if (t < nb && s_ok[t]) {  // uniform across the CTA
          const int j = s_src[t];
          // logit partial: this channel's q.k term plus a share of the radial bias
          float part = qi * kx[(size_t)j * F + f];
          for (int k = c; k < rp.R; k += D) part = fmaf(s_rbf[k][t], sP[k * H + head], part);
          for (int o = 1; o < D; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
          const float l = part + pb[head];
          const float v = ldf(x + (size_t)j * F + f) * s_fc[t] * u[t];
          const float mnew = fmaxf(mu, l);
          const float scale = expf(mu - mnew);  // 0 on the first valid neighbor
          const float w = expf(l - mnew);
          acc = fmaf(acc, scale, w * v);
          z = fmaf(z, scale, w);
          mu = mnew;
        }
      }
      __syncthreads();
    }
    stf(out + (size_t)i * F + f, z > 0.f ? acc / z : 0.f);
  }
}

template <typename T, int F>
static int run_attn(mp_ctx* ctx, int N, int K, const float* pos, const int* nbr,
                    const unsigned char* mask, const void* x, void* out, cudaStream_t s) {
  const int R = ctx->cfg.n_rbf, H = ctx->cfg.n_heads;
  size_t smem = (size_t)(R * F + F * F + R * H) * sizeof(float);
  auto kern = k_attn_simt<T, F>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  int grid = grid_for(ctx, N, 1, 2);
  return launch(ctx, K_ATTN_SIMT, kern, dim3(grid), dim3(F), smem, s, N, K, pos, nbr, mask,
                (const T*)x, (const float*)ctx->q, (const float*)ctx->k, (T*)out,
                filter_of(ctx, 0), radial_of(ctx), (const float*)ctx->P, (const float*)ctx->p,
                H, ctx->cfg.head_dim, ctx->status_d);
}

int launch_attn_simt(mp_ctx* ctx, int N, int K, const float* pos, const int* nbr,
                     const unsigned char* mask, const void* x, void* out, cudaStream_t s) {
  const bool bf = ctx->cfg.dtype == MP_BF16;
  if (ctx->cfg.F == 64)
    return bf ? run_attn<__nv_bfloat16, 64>(ctx, N, K, pos, nbr, mask, x, out, s)
              : run_attn<float, 64>(ctx, N, K, pos, nbr, mask, x, out, s);
  return bf ? run_attn<__nv_bfloat16, 128>(ctx, N, K, pos, nbr, mask, x, out, s)
            : run_attn<float, 128>(ctx, N, K, pos, nbr, mask, x, out, s);
}

// ------------------------------------------------------------------------------------ CSR check
// Bits: 1 = malformed (row_ptr ends/monotonicity, column range, edge leaving its graph),
// 2 = unsorted row or self edge, 4 = asymmetric. One thread per row; every read is bounds-checked.
__device__ __forceinline__ int graph_lo_hi(const int* gp, int G, int N, int i, int* lo, int* hi) {
  if (!gp) {
    *lo = 0;
    *hi = N;
    return 1;
  }
  int a = 0, b = G;  // largest g with gp[g] <= i
  while (b - a > 1) {
    int mid = (a + b) >> 1;
    if (gp[mid] <= i) a = mid; else b = mid;
  }
  *lo = gp[a];
  *hi = gp[a + 1];
  return 1;
}

__global__ void k_validate_csr(int N, long long E, const int* __restrict__ row_ptr,
                               const int* __restrict__ col_idx, const int* __restrict__ gp, int G,
                               int need_sym, int* __restrict__ bits) {
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  if (tid == 0) {
    if (row_ptr[0] != 0 || (long long)row_ptr[N] != E) atomicOr(bits, 1);
    if (gp) {
      if (gp[0] != 0 || gp[G] != N) atomicOr(bits, 1);
      for (int g = 0; g < G; ++g)
        if (gp[g + 1] < gp[g]) atomicOr(bits, 1);
    }
  }
  for (int i = tid; i < N; i += gridDim.x * blockDim.x) {
    const long long a = row_ptr[i], b = row_ptr[i + 1];
    if (a < 0 || b < a || b > E) {
      atomicOr(bits, 1);
      continue;
    }
    int lo = 0, hi = N;
    graph_lo_hi(gp, G, N, i, &lo, &hi);
    int prev = -1;
    for (long long e = a; e < b; ++e) {
      const int j = col_idx[e];
      if (j < 0 || j >= N || j < lo || j >= hi) {
        atomicOr(bits, 1);
        break;
      }
      if (j <= prev || j == i) atomicOr(bits, 2);
      prev = j;
      if (need_sym) {
        long long ja = row_ptr[j], jb = row_ptr[j + 1];
        if (ja < 0 || jb < ja || jb > E) {
          atomicOr(bits, 1);
          break;
        }
        bool found = false;
        while (ja < jb) {  // binary search for i in row j
          long long mid = (ja + jb) >> 1;
          const int v = col_idx[mid];
          if (v == i) {
            found = true;
            break;
          }
          if (v < i) ja = mid + 1; else jb = mid;
        }
        if (!found) atomicOr(bits, 4);
      }
    }
  }
}

int launch_validate_csr(mp_ctx* ctx, int N, long long E, const int* row_ptr, const int* col_idx,
                        const int* graph_ptr, int n_graphs, bool need_sym, cudaStream_t s) {
  cudaMemsetAsync(ctx->status_d, 0, sizeof(int), s);
  int grid = grid_for(ctx, N > 0 ? N : 1, 256, 8);
  int rc = launch(ctx, K_VALIDATE, k_validate_csr, dim3(grid), dim3(256), 0, s, N, E, row_ptr,
                  col_idx, graph_ptr, n_graphs, (int)need_sym, ctx->status_d);
  if (rc != MP_OK) return rc;
  cudaMemcpyAsync(ctx->status_h, ctx->status_d, sizeof(int), cudaMemcpyDeviceToHost, s);
  cudaMemsetAsync(ctx->status_d, 0, sizeof(int), s);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MP_ERR_CUDA;
  const int bits = *ctx->status_h;
  if (bits & 1) return MP_ERR_BAD_CSR;
  if (bits & 2) return MP_ERR_CSR_UNSORTED;
  if (bits & 4) return MP_ERR_CSR_NOT_SYMMETRIC;
  return MP_OK;
}

}  // namespace mp
