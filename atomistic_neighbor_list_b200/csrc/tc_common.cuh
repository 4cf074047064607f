// Shared constants and helpers of the tensor-core cfconv kernels (forward and backward).
#pragma once

#include "tc_api.cuh"
#include "tc_ptx.cuh"

namespace mp {
namespace tcc {

constexpr int TM = 128;            // edges per tile
constexpr int FT = 128;            // channels on this path
constexpr int K2 = 128;            // second filter layer K
constexpr uint32_t WAIT_LIMIT = 1u << 22;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

__host__ __device__ constexpr int k1_of(int R) { return ((R + 1) + 15) / 16 * 16; }

// Byte offset of element (r, k) in a K-major no-swizzle operand whose K extent is kext.
__host__ __device__ constexpr uint32_t kmaj(int r, int k, int kext) {
  return (uint32_t)((r >> 3) * (kext * 16) + (k >> 3) * 128 + (r & 7) * 16 + (k & 7) * 2);
}

// Per-block packed weights: W1 [F][K1] (B operand of MMA1: W1[f][k] = A1[k][f], W1[f][R] = c1[f]),
// W2 [F][128] (B operand of MMA2: W2[f][g] = A2[g][f]), c2 fp32 [F].
struct ImgLayout {
  size_t w1, w2, c2, bytes;
};
__host__ __device__ inline ImgLayout img_layout(int K1) {
  ImgLayout L;
  L.w1 = 0;
  L.w2 = (size_t)FT * K1 * 2;
  L.c2 = L.w2 + (size_t)FT * K2 * 2;
  L.bytes = (L.c2 + FT * 4 + 1023) / 1024 * 1024;
  return L;
}

__device__ __forceinline__ float ssp_scaled(float z, float fc, float fcln2) {
  // f_c * (max(z,0) + ln(1 + e^-|z|) - ln 2) = f_c max(z,0) + f_c ln2 log2((1 + e^-|z|) / 2)
  const float t = tc::ex2f(-fabsf(z) * LOG2E);
  const float l = tc::lg2f(fmaf(t, 0.5f, 0.5f));
  return fmaf(fcln2, l, fc * fmaxf(z, 0.f));
}

// The same for two values, e^-|z| of both from one fp16-pair exponential: t <= 1 in fp16 is good
// to 2^-11 relative (its argument rounded to fp16 adds at most about 2.6e-4 to t), below the bf16
// rounding of the result that feeds the next MMA; returned packed as bf16 (lo = z0).
__device__ __forceinline__ uint32_t ssp_scaled_bf16x2(float z0, float z1, float fc, float fcln2) {
  const uint32_t th = tc::ex2h2(tc::pack_f16(-fabsf(z0) * LOG2E, -fabsf(z1) * LOG2E));
  const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&th));
  const float l0 = tc::lg2f(fmaf(t.x, 0.5f, 0.5f)), l1 = tc::lg2f(fmaf(t.y, 0.5f, 0.5f));
  return tc::pack_bf16(fmaf(fcln2, l0, fc * fmaxf(z0, 0.f)), fmaf(fcln2, l1, fc * fmaxf(z1, 0.f)));
}

// Named barrier over n threads; the _or form also returns the OR of pred over them.
__device__ __forceinline__ void bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ bool bar_sync_or(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n.reg .pred p, q;\nsetp.ne.b32 p, %1, 0;\nbar.red.or.pred q, %2, %3, p;\n"
      "selp.b32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void mbar_arrive1(uint64_t* m) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_u32(m)) : "memory");
}

__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// largest r in [lo, hi) with row_ptr[r] <= e   (row_ptr nondecreasing; row_ptr[lo] <= e)
__device__ __forceinline__ int row_of(const int* __restrict__ row_ptr, int lo, int hi, long long e) {
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((long long)row_ptr[mid] <= e) lo = mid; else hi = mid;
  }
  return lo;
}

// first r in [0, N] with row_ptr[r] >= v
__device__ __forceinline__ int lower_row(const int* __restrict__ row_ptr, int N, long long v) {
  int lo = 0, hi = N + 1;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if ((long long)row_ptr[mid] < v) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// The same search by a whole warp (all 32 lanes call it): each round probes 32 rows at once, so
// it takes ceil(log33(N + 1)) + 1 dependent loads instead of log2(N + 1). Result on every lane.
__device__ __forceinline__ int warp_lower_row(const int* __restrict__ row_ptr, int N, long long v) {
  const int lane = threadIdx.x & 31;
  int lo = 0, hi = N + 1;  // the answer lies in [lo, hi); row_ptr[N] >= v for every v <= E
  while (hi - lo > 32) {
    const int len = hi - lo;
    const int r = lo + (int)(((long long)len * (lane + 1)) / 33);
    const unsigned hit = __ballot_sync(0xffffffffu, (long long)row_ptr[r] >= v);
    if (hit == 0u) {
      lo = lo + (int)(((long long)len * 32) / 33) + 1;
    } else {
      const int l = __ffs(hit) - 1;
      hi = lo + (int)(((long long)len * (l + 1)) / 33) + 1;
      if (l > 0) lo = lo + (int)(((long long)len * l) / 33) + 1;
    }
  }
  const int r = lo + lane;
  const unsigned hit = __ballot_sync(0xffffffffu, r < hi && (long long)row_ptr[r] >= v);
  return hit ? lo + __ffs(hit) - 1 : hi;
}


}  // namespace tcc
}  // namespace mp
