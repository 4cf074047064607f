// Tensor-core (tcgen05 / TMEM) atomwise layers for the bf16 path: out = act(in . W + b) over 128-row
// tiles, with the weight matrix held in shared memory as a packed bf16 operand and fp32 accumulation
// in TMEM. The update network and the readout run in 16-bit on the tensor cores like the filter
// (FlashSchNet page, technical summary s.2.4: W16A16 for the filter, update and readout networks;
// energy accumulation in fp32).
//
// Epilogue modes (thread = row = TMEM lane):
//   STORE     out[r] = acc + b              (bf16 or fp32)
//   RESIDUAL  out[r] += acc + b             (fp32, in place)
//   READOUT   a = acc + d1 (F/2 wide): e_atom[r] = sum_k ssp(a_k) B2_k + d2 and
//             u[r][k] = sigmoid(a_k) B2_k = de_r/da_k, in one pass
#include "tc_common.cuh"

namespace mp {
namespace {
using namespace tcc;

constexpr int DT = 128;  // rows per tile
constexpr int DTHREADS = 128;

enum { MODE_STORE = 0, MODE_RESIDUAL = 1, MODE_READOUT = 2, MODE_STORE_F16 = 3 };

// Row r of a bf16 or fp32 [*][Kin] input, as bf16, into row `lane` of a K-major operand tile (all
// loads of a half issued before use); zeros for rows past the end.
__device__ __forceinline__ void load_a_row(uint8_t* sA, const void* in, bool in_bf16, int Kin, int r,
                                           bool valid, int lane) {
  if (in_bf16) {
    const uint4* src = (const uint4*)((const __nv_bfloat16*)in + (size_t)r * Kin);
    uint4 v[16];
#pragma unroll
    for (int c = 0; c < 16; ++c)
      v[c] = (valid && c < Kin / 8) ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int c = 0; c < 16; ++c)
      if (c < Kin / 8) *(uint4*)(sA + kmaj(lane, 8 * c, Kin)) = v[c];
  } else {
    const float4* src = (const float4*)((const float*)in + (size_t)r * Kin);
#pragma unroll
    for (int hb = 0; hb < 2; ++hb) {
      if (hb * 64 >= Kin) break;
      float4 v[16];
#pragma unroll
      for (int c = 0; c < 16; ++c)
        v[c] = valid ? __ldg(src + hb * 16 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *(uint4*)(sA + kmaj(lane, hb * 64 + 8 * c, Kin)) =
            make_uint4(tc::pack_bf16(v[2 * c].x, v[2 * c].y), tc::pack_bf16(v[2 * c].z, v[2 * c].w),
                       tc::pack_bf16(v[2 * c + 1].x, v[2 * c + 1].y),
                       tc::pack_bf16(v[2 * c + 1].z, v[2 * c + 1].w));
    }
  }
}

// Columns [half Kin/2, (half + 1) Kin/2) of row r, the same way: two threads per row share a tile.
__device__ __forceinline__ void load_a_half(uint8_t* sA, const void* in, bool in_bf16, int Kin, int r,
                                            bool valid, int lane, int half) {
  const int k0 = half * (Kin / 2), kn = Kin / 2;  // 32 or 64 columns
  if (in_bf16) {
    const uint4* src = (const uint4*)((const __nv_bfloat16*)in + (size_t)r * Kin + k0);
    uint4 v[8];
#pragma unroll
    for (int c = 0; c < 8; ++c)
      v[c] = (valid && c < kn / 8) ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int c = 0; c < 8; ++c)
      if (c < kn / 8) *(uint4*)(sA + kmaj(lane, k0 + 8 * c, Kin)) = v[c];
  } else {
    const float4* src = (const float4*)((const float*)in + (size_t)r * Kin + k0);
    float4 v[16];
#pragma unroll
    for (int c = 0; c < 16; ++c)
      v[c] = (valid && c < kn / 4) ? __ldg(src + c) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int c = 0; c < 8; ++c)
      if (c < kn / 8)
        *(uint4*)(sA + kmaj(lane, k0 + 8 * c, Kin)) =
            make_uint4(tc::pack_bf16(v[2 * c].x, v[2 * c].y), tc::pack_bf16(v[2 * c].z, v[2 * c].w),
                       tc::pack_bf16(v[2 * c + 1].x, v[2 * c + 1].y),
                       tc::pack_bf16(v[2 * c + 1].z, v[2 * c + 1].w));
  }
}

// The readout epilogue for one row: a = acc + d1 over `ncol` columns starting at col; u = dE/da =
// sigmoid(a) B2 stored, and sum ssp(a) B2 returned.
__device__ __forceinline__ float readout_cols(const float* v, int col, const float* B2, float* u) {
  float e_acc = 0.f;
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    float4 o;
    float* po = &o.x;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float z = v[i + q], b2 = B2[col + i + q];
      const float t = tc::ex2f(-fabsf(z) * LOG2E);
      const float ssp = fmaf(LN2, tc::lg2f(fmaf(t, 0.5f, 0.5f)), fmaxf(z, 0.f));
      e_acc = fmaf(ssp, b2, e_acc);
      const float sg = z >= 0.f ? 1.f / (1.f + t) : t / (1.f + t);
      po[q] = sg * b2;
    }
    *(float4*)(u + i) = o;
  }
  return e_acc;
}

struct DenseArgs {
  int N, Kin, Nout;
  const void* in;
  int in_bf16;
  const uint8_t* wimg;  // [Nout][Kin] bf16 K-major core-matrix layout
  const float* bias;    // [Nout] or null
  void* out;
  int out_bf16;
  int mode;
  const float* B2;      // readout: [Nout]
  const float* d2;      // readout: [1]
  float* e_atom;        // readout: [N]
};

__global__ void __launch_bounds__(DTHREADS) k_dense_tc(DenseArgs a, int* status) {
  // CTA = (row tile, 64-column slice of the output)
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sB = sm;                          // 64 x Kin bf16 (this CTA's output columns)
  uint8_t* sA = sm + 64 * 128 * 2;           // 128 x Kin bf16
  __shared__ uint64_t mbar_w, mbar;
  __shared__ uint32_t tslot;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int Kin = a.Kin, nsplit = a.Nout / 64;
  const int tile = blockIdx.x / nsplit, n0 = (blockIdx.x % nsplit) * 64;
  if (warp == 0) tc::tmem_alloc(&tslot, 64);
  if (tid == 0) {
    tc::mbar_init(&mbar_w, 1);
    tc::mbar_init(&mbar, 1);
    const uint32_t wbytes = 64 * Kin * 2;
    tc::mbar_expect_tx(&mbar_w, wbytes);
    tc::bulk_g2s(sB, a.wimg + (size_t)n0 * Kin * 2, wbytes, &mbar_w);
  }
  const int r = tile * DT + tid;
  const bool valid = r < a.N;
  load_a_row(sA, a.in, a.in_bf16 != 0, Kin, r, valid, tid);
  tc::fence_proxy_async();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = tslot;
  int bad = 0;
  if (tid == 0) {
    if (!tc::mbar_wait(&mbar_w, 0, WAIT_LIMIT)) {
      bad = 1;
    } else {
      const uint32_t sa = tc::smem_u32(sA), sb = tc::smem_u32(sB);
      const uint32_t id = tc::idesc(DT, 64, 1, false, false);
      for (int ks = 0; ks < Kin / 16; ++ks)
        tc::mma(tmem, tc::sdesc(sa + ks * 256, 128, Kin * 16), tc::sdesc(sb + ks * 256, 128, Kin * 16),
                id, ks > 0);
      tc::commit(&mbar);
    }
  }
  if (__syncthreads_or(bad)) {
    if (tid == 0) raise_status(status, kStatusTimeout);
  } else {
    bad = tc::mbar_wait(&mbar, 0, WAIT_LIMIT) ? 0 : 1;
    tc::fence_after();
    if (__syncthreads_or(bad)) {
      if (tid == 0) {
        raise_status(status, kStatusTimeout);
        tc::mbar_wait(&mbar, 0, WAIT_LIMIT);
      }
    } else {
      // ---- epilogue: thread = row = TMEM lane, 64 columns
      const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
      float e_acc = 0.f;
#pragma unroll
      for (int c0 = 0; c0 < 64; c0 += 32) {
        uint32_t rr[32];
        tc::ld32(lane_base + c0, rr);
        tc::ld_wait();
        if (valid) {
          const int col = n0 + c0;
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(rr[i]) + (a.bias ? a.bias[col + i] : 0.f);
          if (a.mode == MODE_READOUT) {
            e_acc += readout_cols(v, col, a.B2, (float*)a.out + (size_t)r * a.Nout + col);
          } else if (a.mode == MODE_STORE_F16) {  // fp16 rows (10-bit mantissa)
            uint4* o = (uint4*)((__half*)a.out + (size_t)r * a.Nout + col);
            auto h2 = [](float lo, float hi) {
              const __half2 h = __floats2half2_rn(lo, hi);
              return *(const uint32_t*)&h;
            };
#pragma unroll
            for (int i = 0; i < 32; i += 8)
              o[i / 8] = make_uint4(h2(v[i], v[i + 1]), h2(v[i + 2], v[i + 3]),
                                    h2(v[i + 4], v[i + 5]), h2(v[i + 6], v[i + 7]));
          } else if (a.out_bf16) {
            uint4* o = (uint4*)((__nv_bfloat16*)a.out + (size_t)r * a.Nout + col);
#pragma unroll
            for (int i = 0; i < 32; i += 8)
              o[i / 8] = make_uint4(tc::pack_bf16(v[i], v[i + 1]), tc::pack_bf16(v[i + 2], v[i + 3]),
                                    tc::pack_bf16(v[i + 4], v[i + 5]), tc::pack_bf16(v[i + 6], v[i + 7]));
          } else {
            float4* o = (float4*)((float*)a.out + (size_t)r * a.Nout + col);
            float4 old[8];
            if (a.mode == MODE_RESIDUAL) {
#pragma unroll
              for (int i = 0; i < 8; ++i) old[i] = o[i];
            }
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              float4 w = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
              if (a.mode == MODE_RESIDUAL) {
                w.x += old[i / 4].x;
                w.y += old[i / 4].y;
                w.z += old[i / 4].z;
                w.w += old[i / 4].w;
              }
              o[i / 4] = w;
            }
          }
        }
      }
      if (a.mode == MODE_READOUT && valid) a.e_atom[r] = e_acc + a.d2[0];
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 64);
}

// Two atomwise layers in one pass over a 128-row tile (two threads per row = TMEM lane, one per
// half of the columns):
//   y   = in1 . W1 + b1            (128 columns, fp32): out1 = y (STORE) or out1 += y (RESIDUAL)
//   out2 = out1_row . W2 + b2      (the updated fp32 row, as bf16, is the second MMA's operand):
//          STORE -> bf16 [N][128], or READOUT (W2 = B1, 64 columns) -> u [N][64] and e_atom
// The pairs it serves (residual update then the next block's input layer, the last residual then
// the readout, and their transposes in the backward) each depend only on the row itself.
struct Dense2Args {
  int N, K1;
  const void* in1;
  int in1_bf16;
  const uint8_t* w1;  // [128][K1]
  const float* b1;
  float* out1;        // fp32 [N][128]
  int mode1;
  const uint8_t* w2;  // [N2][128]
  const float* b2;
  int N2;
  void* out2;
  int mode2;
  const float* B2;
  const float* d2;
  float* e_atom;
};

constexpr int D2THREADS = 256;

__global__ void __launch_bounds__(D2THREADS) k_dense2_tc(Dense2Args a, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sW1 = sm;                     // 128 x K1
  uint8_t* sW2 = sm + 128 * 128 * 2;     // N2 x 128
  uint8_t* sA1 = sm + 2 * 128 * 128 * 2; // 128 x K1
  uint8_t* sA2 = sm + 3 * 128 * 128 * 2; // 128 x 128
  __shared__ uint64_t mbar_w, mbar1, mbar2;
  __shared__ uint32_t tslot;
  __shared__ float s_e[2][DT];  // readout: the two halves' partial energies of each row
  const int tid = threadIdx.x, warp = tid >> 5;
  const int lrow = tid & (DT - 1), half = tid >> 7;  // row of the tile, half of the columns
  const int K1 = a.K1, N2 = a.N2;
  if (warp == 0) tc::tmem_alloc(&tslot, 256);
  if (tid == 0) {
    tc::mbar_init(&mbar_w, 1);
    tc::mbar_init(&mbar1, 1);
    tc::mbar_init(&mbar2, 1);
    tc::mbar_expect_tx(&mbar_w, 128 * K1 * 2 + N2 * 128 * 2);
    tc::bulk_g2s(sW1, a.w1, 128 * K1 * 2, &mbar_w);
    tc::bulk_g2s(sW2, a.w2, N2 * 128 * 2, &mbar_w);
  }
  const int r = blockIdx.x * DT + lrow;
  const bool valid = r < a.N;
  load_a_half(sA1, a.in1, a.in1_bf16 != 0, K1, r, valid, lrow, half);
  tc::fence_proxy_async();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = tslot;
  const uint32_t lane_base = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
  int bad = 0;
  bool issued1 = false, issued2 = false;  // thread 0: MMAs it has issued
  if (tid == 0) {
    if (!tc::mbar_wait(&mbar_w, 0, WAIT_LIMIT)) {
      bad = 1;
    } else {
      issued1 = true;
      const uint32_t sa = tc::smem_u32(sA1), sb = tc::smem_u32(sW1);
      const uint32_t id = tc::idesc(DT, 128, 1, false, false);
      for (int ks = 0; ks < K1 / 16; ++ks)
        tc::mma(tmem, tc::sdesc(sa + ks * 256, 128, K1 * 16), tc::sdesc(sb + ks * 256, 128, K1 * 16),
                id, ks > 0);
      tc::commit(&mbar1);
    }
  }
  // the residual this thread's 64 columns add to, requested before the wait for the first MMA
  float4 old[16];
  const bool resid = a.mode1 == MODE_RESIDUAL && valid;
#pragma unroll
  for (int i = 0; i < 16; ++i)
    old[i] = resid ? ((const float4*)(a.out1 + (size_t)r * 128 + 64 * half))[i]
                   : make_float4(0.f, 0.f, 0.f, 0.f);
  bool ok = !__syncthreads_or(bad);
  if (ok) {
    ok = !__syncthreads_or(tc::mbar_wait(&mbar1, 0, WAIT_LIMIT) ? 0 : 1);
    tc::fence_after();
  }
  if (ok) {
    // ---- first layer's epilogue: the updated row, kept in fp32 and staged as bf16
#pragma unroll
    for (int hc = 0; hc < 2; ++hc) {
      const int c0 = 64 * half + 32 * hc;
      uint32_t rr[32];
      tc::ld32(lane_base + c0, rr);
      tc::ld_wait();
      float v[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(rr[i]) + (a.b1 ? a.b1[c0 + i] : 0.f);
      if (valid) {
        float4* o = (float4*)(a.out1 + (size_t)r * 128 + c0);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          v[4 * i] += old[8 * hc + i].x;
          v[4 * i + 1] += old[8 * hc + i].y;
          v[4 * i + 2] += old[8 * hc + i].z;
          v[4 * i + 3] += old[8 * hc + i].w;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      }
#pragma unroll
      for (int i = 0; i < 32; i += 8)
        *(uint4*)(sA2 + kmaj(lrow, c0 + i, 128)) =
            valid ? make_uint4(tc::pack_bf16(v[i], v[i + 1]), tc::pack_bf16(v[i + 2], v[i + 3]),
                               tc::pack_bf16(v[i + 4], v[i + 5]), tc::pack_bf16(v[i + 6], v[i + 7]))
                  : make_uint4(0, 0, 0, 0);
    }
    tc::fence_proxy_async();
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (tid == 0) {
      issued2 = true;
      const uint32_t sa = tc::smem_u32(sA2), sb = tc::smem_u32(sW2);
      const uint32_t id = tc::idesc(DT, N2, 1, false, false);
      for (int ks = 0; ks < 128 / 16; ++ks)
        tc::mma(tmem + 128, tc::sdesc(sa + ks * 256, 128, 128 * 16),
                tc::sdesc(sb + ks * 256, 128, 128 * 16), id, ks > 0);
      tc::commit(&mbar2);
    }
    ok = !__syncthreads_or(tc::mbar_wait(&mbar2, 0, WAIT_LIMIT) ? 0 : 1);
    tc::fence_after();
  }
  if (ok) {
    // ---- second layer's epilogue
    float e_acc = 0.f;
#pragma unroll 1
    for (int c0 = half * (N2 / 2); c0 < (half + 1) * (N2 / 2); c0 += 32) {
      uint32_t rr[32];
      tc::ld32(lane_base + 128 + c0, rr);
      tc::ld_wait();
      if (valid) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(rr[i]) + (a.b2 ? a.b2[c0 + i] : 0.f);
        if (a.mode2 == MODE_READOUT) {
          e_acc += readout_cols(v, c0, a.B2, (float*)a.out2 + (size_t)r * N2 + c0);
        } else {
          uint4* o = (uint4*)((__nv_bfloat16*)a.out2 + (size_t)r * N2 + c0);
#pragma unroll
          for (int i = 0; i < 32; i += 8)
            o[i / 8] = make_uint4(tc::pack_bf16(v[i], v[i + 1]), tc::pack_bf16(v[i + 2], v[i + 3]),
                                  tc::pack_bf16(v[i + 4], v[i + 5]), tc::pack_bf16(v[i + 6], v[i + 7]));
        }
      }
    }
    if (a.mode2 == MODE_READOUT) {  // the two halves' sums, added in a fixed order
      s_e[half][lrow] = e_acc;
      __syncthreads();
      if (half == 0 && valid) a.e_atom[r] = (s_e[0][lrow] + s_e[1][lrow]) + a.d2[0];
    }
  } else if (tid == 0) {
    raise_status(status, kStatusTimeout);
    // nothing this thread issued may still run when TMEM is freed: the second barrier's first
    // phase completes once everything issued before its commit has completed
    if (issued1 && !issued2) tc::commit(&mbar2);
    if (issued1) tc::mbar_wait(&mbar2, 0, WAIT_LIMIT);
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 256);
}

}  // namespace

// Packed dense weight images in ctx->tc_dense: per block W_in, W_out, W_out^T, W_in^T (each
// [128][128]), then B1 ([64][128]) and B1^T ([128][64]), then the attention's Wq and Wk.
size_t tc_dense_bytes(int B) { return (size_t)(4 * B + 3) * 128 * 128 * 2; }

int tc_dense_pack(const float* W, int rows, int cols, bool transpose, uint8_t* dst) {
  // B operand [Nout][Kin]: element (n, k) = transpose ? W[n][k] : W[k][n], W row-major [rows][cols]
  const int Nout = transpose ? rows : cols, Kin = transpose ? cols : rows;
  for (int n = 0; n < Nout; ++n)
    for (int k = 0; k < Kin; ++k) {
      const float v = transpose ? W[(size_t)n * cols + k] : W[(size_t)k * cols + n];
      uint32_t u;
      memcpy(&u, &v, 4);
      const uint16_t bits = (uint16_t)(u >> 16);  // values are bf16-rounded already
      memcpy(dst + kmaj(n, k, Kin), &bits, 2);
    }
  return MP_OK;
}

int attn_project(mp_ctx* ctx, int N, const void* x, cudaStream_t s, bool k_f16) {
  const int F = ctx->cfg.F, B = ctx->cfg.n_blocks;
  const bool bf = ctx->cfg.dtype == MP_BF16;
  if (ctx->tc_qk && ((uintptr_t)x & 15) == 0) {  // bf16 rows x bf16 weights, fp32 accumulation
    int rc = tc_dense(ctx, N, F, F, x, true, ctx->tc_dense_img + tc_dense_off(6, 0, B), nullptr,
                      ctx->q, false, TC_DENSE_STORE, s);
    if (rc != MP_OK) return rc;
    return tc_dense(ctx, N, F, F, x, true, ctx->tc_dense_img + tc_dense_off(7, 0, B), nullptr,
                    ctx->k, false, k_f16 ? TC_DENSE_STORE_F16 : TC_DENSE_STORE, s);
  }
  if (k_f16) return MP_ERR_INVALID_ARG;  // the fp16 keys come from the tensor-core projection
  int rc = launch_dense(ctx, N, F, F, x, bf, ctx->Wq, nullptr, false, ctx->q, false, s);
  if (rc != MP_OK) return rc;
  return launch_dense(ctx, N, F, F, x, bf, ctx->Wk, nullptr, false, ctx->k, false, s);
}

int tc_dense(mp_ctx* ctx, int N, int Kin, int Nout, const void* in, bool in_bf16, const uint8_t* wimg,
             const float* bias, void* out, bool out_bf16, int mode, cudaStream_t s) {
  DenseArgs a;
  a.N = N;
  a.Kin = Kin;
  a.Nout = Nout;
  a.in = in;
  a.in_bf16 = in_bf16;
  a.wimg = wimg;
  a.bias = bias;
  a.out = out;
  a.out_bf16 = out_bf16;
  a.mode = mode;
  a.B2 = ctx->B2;
  a.d2 = ctx->d2;
  a.e_atom = ctx->e_atom;
  if (Nout % 64 != 0 || (Kin != 64 && Kin != 128) || (mode == MODE_READOUT && Nout != 64))
    return MP_ERR_INVALID_ARG;
  const size_t smem = 64 * 128 * 2 + 128 * 128 * 2 + 1024;
  cudaFuncSetAttribute(k_dense_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const int ntiles = (N + DT - 1) / DT;
  const int grid = (ntiles > 0 ? ntiles : 1) * (Nout / 64);
  return launch(ctx, K_DENSE_TC, k_dense_tc, dim3(grid), dim3(DTHREADS), smem, s, a, ctx->status_d);
}

int tc_dense2(mp_ctx* ctx, int N, int K1, const void* in1, bool in1_bf16, const uint8_t* w1,
              const float* b1, float* out1, int mode1, const uint8_t* w2, const float* b2, int N2,
              void* out2, int mode2, cudaStream_t s) {
  if ((K1 != 64 && K1 != 128) || (mode1 != MODE_STORE && mode1 != MODE_RESIDUAL) ||
      !(mode2 == MODE_STORE && N2 == 128) && !(mode2 == MODE_READOUT && N2 == 64))
    return MP_ERR_INVALID_ARG;
  Dense2Args a;
  a.N = N;
  a.K1 = K1;
  a.in1 = in1;
  a.in1_bf16 = in1_bf16;
  a.w1 = w1;
  a.b1 = b1;
  a.out1 = out1;
  a.mode1 = mode1;
  a.w2 = w2;
  a.b2 = b2;
  a.N2 = N2;
  a.out2 = out2;
  a.mode2 = mode2;
  a.B2 = ctx->B2;
  a.d2 = ctx->d2;
  a.e_atom = ctx->e_atom;
  const size_t smem = 4 * 128 * 128 * 2 + 1024;
  cudaFuncSetAttribute(k_dense2_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const int ntiles = (N + DT - 1) / DT;
  return launch(ctx, K_DENSE_TC, k_dense2_tc, dim3(ntiles > 0 ? ntiles : 1), dim3(D2THREADS), smem,
                s, a, ctx->status_d);
}

}  // namespace mp
