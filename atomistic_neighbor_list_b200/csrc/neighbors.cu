// Neighbor lists by the exact rule (j != i, same graph, d2 < r_c^2 with d2 evaluated in float64 as
// (dx*dx + dy*dy) + dz*dz, each operation individually rounded to nearest, no fused multiply-add).
//
// One warp owns one destination row and scans the candidate sources of its graph in ascending order,
// 32 at a time; a ballot compacts the hits in order, so rows come out sorted by source without a
// sort and the result is bit-identical to any implementation of the same rule. (The Tessera page
// reuses a neighbor topology across steps and builds it by a spatial search; this brute-force scan
// is the construction used to feed the message-passing kernels and their tests.)
#include "mp_internal.cuh"

namespace mp {

__device__ __forceinline__ double d2_exact(const float* __restrict__ pos, int i, int j) {
  const double dx = __dsub_rn((double)pos[3 * j], (double)pos[3 * i]);
  const double dy = __dsub_rn((double)pos[3 * j + 1], (double)pos[3 * i + 1]);
  const double dz = __dsub_rn((double)pos[3 * j + 2], (double)pos[3 * i + 2]);
  return __dadd_rn(__dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy)), __dmul_rn(dz, dz));
}

__device__ __forceinline__ void graph_range(const int* gp, int G, int N, int i, int* lo,
                                            int* hi) {
  if (!gp) {
    *lo = 0;
    *hi = N;
    return;
  }
  int a = 0, b = G;
  while (b - a > 1) {
    const int mid = (a + b) >> 1;
    if (gp[mid] <= i) a = mid; else b = mid;
  }
  int l = gp[a], h = gp[a + 1];
  *lo = l < 0 ? 0 : l;
  *hi = h > N ? N : h;
}

// pass 1: counts[i] = number of neighbors of row i (written to row_ptr[i+1])
__global__ void k_nbr_count(int N, const float* __restrict__ pos, const int* __restrict__ gp,
                            int G, double rc2, int* __restrict__ row_ptr) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < N; i += warps) {
    int lo, hi;
    graph_range(gp, G, N, i, &lo, &hi);
    int cnt = 0;
    for (int j0 = lo; j0 < hi; j0 += 32) {
      const int j = j0 + lane;
      const bool hit = j < hi && j != i && d2_exact(pos, i, j) < rc2;
      cnt += __popc(__ballot_sync(0xffffffffu, hit));
    }
    if (lane == 0) row_ptr[i + 1] = cnt;
  }
}

// in-place inclusive scan of row_ptr[1..N] by one CTA; row_ptr[0] = 0; overflow past INT_MAX flags
__global__ void k_scan_rows(int N, int* __restrict__ row_ptr, int* __restrict__ overflow) {
  __shared__ long long s_warp[32];
  __shared__ long long s_carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    row_ptr[0] = 0;
    s_carry = 0;
  }
  __syncthreads();
  for (int base = 0; base < N; base += blockDim.x) {
    const int i = base + tid;
    long long v = i < N ? row_ptr[i + 1] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long t = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += t;
    }
    if (lane == 31) s_warp[warp] = v;
    __syncthreads();
    if (warp == 0) {
      long long w = lane < (int)(blockDim.x >> 5) ? s_warp[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long t = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += t;
      }
      s_warp[lane] = w;
    }
    __syncthreads();
    const long long total = v + (warp ? s_warp[warp - 1] : 0) + s_carry;
    if (i < N) {
      if (total > 0x7fffffffLL) *overflow = 1;
      row_ptr[i + 1] = (int)(total > 0x7fffffffLL ? 0x7fffffffLL : total);
    }
    __syncthreads();
    if (tid == blockDim.x - 1) s_carry = total;
    __syncthreads();
  }
}

// pass 2: write the sources of each row in ascending order
__global__ void k_nbr_fill(int N, const float* __restrict__ pos, const int* __restrict__ gp, int G,
                           double rc2, const int* __restrict__ row_ptr, int* __restrict__ col_idx,
                           long long capacity) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < N; i += warps) {
    int lo, hi;
    graph_range(gp, G, N, i, &lo, &hi);
    long long out = row_ptr[i];
    for (int j0 = lo; j0 < hi; j0 += 32) {
      const int j = j0 + lane;
      const bool hit = j < hi && j != i && d2_exact(pos, i, j) < rc2;
      const unsigned b = __ballot_sync(0xffffffffu, hit);
      const long long slot = out + __popc(b & ((1u << lane) - 1u));
      if (hit && slot < capacity) col_idx[slot] = j;
      out += __popc(b);
    }
  }
}

// Padded list: candidates of a row staged in shared memory; if more than K, keep those whose rank
// by (d2, j) is below K; kept entries are written in ascending j (their staging order).
constexpr int kPadCap = 1024;   // candidates per row
constexpr int kPadWarps = 4;

__global__ void __launch_bounds__(kPadWarps * 32) k_nbr_padded(
    int N, const float* __restrict__ pos, const int* __restrict__ gp, int G, double rc2, int K,
    int* __restrict__ nbr, unsigned char* __restrict__ mask, int* __restrict__ overflow) {
  __shared__ int s_j[kPadWarps][kPadCap];
  __shared__ double s_d2[kPadWarps][kPadCap];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  int* sj = s_j[wib];
  double* sd = s_d2[wib];
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < N; i += warps) {
    int lo, hi;
    graph_range(gp, G, N, i, &lo, &hi);
    int cnt = 0;
    for (int j0 = lo; j0 < hi; j0 += 32) {
      const int j = j0 + lane;
      double d2 = 0.0;
      bool hit = false;
      if (j < hi && j != i) {
        d2 = d2_exact(pos, i, j);
        hit = d2 < rc2;
      }
      const unsigned b = __ballot_sync(0xffffffffu, hit);
      const int slot = cnt + __popc(b & ((1u << lane) - 1u));
      if (hit && slot < kPadCap) {
        sj[slot] = j;
        sd[slot] = d2;
      }
      cnt += __popc(b);
    }
    __syncwarp();
    int* row_n = nbr + (size_t)i * K;
    unsigned char* row_m = mask + (size_t)i * K;
    if (cnt > kPadCap) {
      if (lane == 0) *overflow = 1;
      for (int s = lane; s < K; s += 32) {
        row_n[s] = -1;
        row_m[s] = 0;
      }
      __syncwarp();
      continue;
    }
    int kept = 0;
    if (cnt <= K) {
      for (int s = lane; s < cnt; s += 32) {
        row_n[s] = sj[s];
        row_m[s] = 1;
      }
      kept = cnt;
    } else {
      for (int c0 = 0; c0 < cnt; c0 += 32) {
        const int c = c0 + lane;
        bool keep = false;
        int jc = 0;
        if (c < cnt) {
          jc = sj[c];
          const double dc = sd[c];
          int rank = 0;
          for (int o = 0; o < cnt; ++o) {
            const double dd = sd[o];
            rank += (dd < dc || (dd == dc && sj[o] < jc)) ? 1 : 0;
          }
          keep = rank < K;
        }
        const unsigned b = __ballot_sync(0xffffffffu, keep);
        const int slot = kept + __popc(b & ((1u << lane) - 1u));
        if (keep) {
          row_n[slot] = jc;
          row_m[slot] = 1;
        }
        kept += __popc(b);
      }
    }
    for (int s = kept + lane; s < K; s += 32) {
      row_n[s] = -1;
      row_m[s] = 0;
    }
    __syncwarp();
  }
}

static int sm_count() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

}  // namespace mp

using namespace mp;

extern "C" int mp_neighbor_csr(int N, const float* pos, const int* graph_ptr, int n_graphs,
                               float r_c, int* row_ptr, int* col_idx, long long capacity,
                               long long* n_edges, void* stream) {
  if (N < 0 || !row_ptr || !n_edges || (N > 0 && !pos) || !(r_c > 0.f) || capacity < 0 ||
      (capacity > 0 && !col_idx) || (graph_ptr && n_graphs < 1))
    return MP_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  const double rcd = (double)r_c;
  const double rc2 = rcd * rcd;  // exact for the cutoffs in use; one rounded multiply on the host
  int* flag = nullptr;
  if (cudaMallocAsync(&flag, sizeof(int), s) != cudaSuccess) return MP_ERR_CUDA;
  cudaMemsetAsync(flag, 0, sizeof(int), s);
  const int G = graph_ptr ? n_graphs : 1;
  const int grid = sm_count() * 8;
  if (N > 0) k_nbr_count<<<grid, 256, 0, s>>>(N, pos, graph_ptr, G, rc2, row_ptr);
  k_scan_rows<<<1, 1024, 0, s>>>(N, row_ptr, flag);
  int hflag = 0, total = 0;
  cudaMemcpyAsync(&total, row_ptr + N, sizeof(int), cudaMemcpyDeviceToHost, s);
  cudaMemcpyAsync(&hflag, flag, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (cudaStreamSynchronize(s) != cudaSuccess || cudaGetLastError() != cudaSuccess) {
    cudaFreeAsync(flag, s);
    return MP_ERR_CUDA;
  }
  *n_edges = total;
  if (hflag || total > capacity) {
    cudaFreeAsync(flag, s);
    return MP_ERR_CAPACITY;
  }
  if (N > 0 && total > 0)
    k_nbr_fill<<<grid, 256, 0, s>>>(N, pos, graph_ptr, G, rc2, row_ptr, col_idx, capacity);
  cudaFreeAsync(flag, s);
  return cudaGetLastError() == cudaSuccess ? MP_OK : MP_ERR_CUDA;
}

extern "C" int mp_neighbor_padded(int N, const float* pos, const int* graph_ptr, int n_graphs,
                                  float r_c, int K, int* nbr, unsigned char* mask, void* stream) {
  if (N < 0 || K < 1 || (N > 0 && (!pos || !nbr || !mask)) || !(r_c > 0.f) ||
      (graph_ptr && n_graphs < 1))
    return MP_ERR_INVALID_ARG;
  if (N == 0) return MP_OK;
  cudaStream_t s = (cudaStream_t)stream;
  const double rcd = (double)r_c;
  const double rc2 = rcd * rcd;  // exact for the cutoffs in use; one rounded multiply on the host
  int* flag = nullptr;
  if (cudaMallocAsync(&flag, sizeof(int), s) != cudaSuccess) return MP_ERR_CUDA;
  cudaMemsetAsync(flag, 0, sizeof(int), s);
  const int G = graph_ptr ? n_graphs : 1;
  k_nbr_padded<<<sm_count() * 4, kPadWarps * 32, 0, s>>>(N, pos, graph_ptr, G, rc2, K, nbr, mask,
                                                          flag);
  int hflag = 0;
  cudaMemcpyAsync(&hflag, flag, sizeof(int), cudaMemcpyDeviceToHost, s);
  const bool ok = cudaStreamSynchronize(s) == cudaSuccess && cudaGetLastError() == cudaSuccess;
  cudaFreeAsync(flag, s);
  if (!ok) return MP_ERR_CUDA;
  return hflag ? MP_ERR_CAPACITY : MP_OK;
}
