// Neighbor lists by the exact rule (j != i, same graph, d2 < r_c^2 with d2 evaluated in float64 as
// (dx*dx + dy*dy) + dz*dz, each operation individually rounded to nearest, no fused multiply-add).
//
// Construction by a cell list (Tessera page, neighbor search: spatial boxes narrow the candidates,
// an exact distance test decides): every graph gets its own grid of cells at least r_c wide on each
// axis over its bounding box, atoms are counting-sorted into cells, and a row's candidates are the
// atoms of the 3 x 3 x 3 cells around its own. The exact test above then decides each candidate, so
// the cells only prune (a coarser grid gives the same list). Rows are written in ascending source
// order: the hits of a row are staged in shared memory and each is stored at its rank. A row with
// more hits than the staging holds is filled by an ordered scan over its whole graph instead.
// The result is bit-identical to any implementation of the same rule.
#include <cmath>
#include <mutex>

#include "mp_internal.cuh"

namespace mp {
namespace {

__device__ __forceinline__ double d2_exact(float xi, float yi, float zi, float xj, float yj,
                                           float zj) {
  const double dx = __dsub_rn((double)xj, (double)xi);
  const double dy = __dsub_rn((double)yj, (double)yi);
  const double dz = __dsub_rn((double)zj, (double)zi);
  return __dadd_rn(__dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy)), __dmul_rn(dz, dz));
}

// graph of atom i: g with gp[g] <= i < gp[g+1], or -1 when no graph holds i
__device__ __forceinline__ int graph_of(const int* __restrict__ gp, int G, int i) {
  if (!gp) return 0;
  int a = 0, b = G;  // gp[a] <= i < gp[b] if i is held at all
  if (i < gp[0] || i >= gp[G]) return -1;
  while (b - a > 1) {
    const int mid = (a + b) >> 1;
    if (gp[mid] <= i) a = mid; else b = mid;
  }
  return a;
}

__device__ __forceinline__ void graph_bounds(const int* __restrict__ gp, int G, int N, int g,
                                             int* lo, int* hi) {
  int l = gp ? gp[g] : 0, h = gp ? gp[g + 1] : N;
  l = l < 0 ? 0 : (l > N ? N : l);
  h = h < l ? l : (h > N ? N : h);
  *lo = l;
  *hi = h;
}

// ------------------------------------------------------------------------------------ scans
// In place: a[1..n] holds counts; afterwards a[0..n] holds their prefix sums (a[0] = 0). Three
// launches: per-block local scans of 4096 elements, one scan of the block totals (64-bit, with an
// overflow flag past INT_MAX), then the block offsets added.
constexpr int kScanThreads = 1024, kScanPer = 4 * kScanThreads;

__global__ void __launch_bounds__(kScanThreads) k_scan_local(long long n, int* __restrict__ a,
                                                             long long* __restrict__ bsum) {
  __shared__ long long s_w[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long e0 = (long long)blockIdx.x * kScanPer + 4LL * tid;
  long long v[4], run = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    run += (e0 + k < n) ? (long long)a[e0 + k + 1] : 0LL;
    v[k] = run;
  }
  long long t = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long u = __shfl_up_sync(0xffffffffu, t, o);
    if (lane >= o) t += u;
  }
  if (lane == 31) s_w[warp] = t;
  __syncthreads();
  if (warp == 0) {
    long long w = s_w[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long u = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += u;
    }
    s_w[lane] = w;
  }
  __syncthreads();
  const long long excl = t - run + (warp ? s_w[warp - 1] : 0LL);
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (e0 + k < n) a[e0 + k + 1] = (int)(excl + v[k]);  // exact whenever the total fits
  if (tid == kScanThreads - 1) bsum[blockIdx.x] = excl + v[3];
}

__global__ void __launch_bounds__(kScanThreads) k_scan_totals(int nb, long long* __restrict__ bsum,
                                                              int* __restrict__ overflow) {
  __shared__ long long s_w[32];
  __shared__ long long s_carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) s_carry = 0;
  __syncthreads();
  for (int base = 0; base < nb; base += kScanThreads) {
    const int b = base + tid;
    const long long x = b < nb ? bsum[b] : 0LL;
    long long t = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long u = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += u;
    }
    if (lane == 31) s_w[warp] = t;
    __syncthreads();
    if (warp == 0) {
      long long w = s_w[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long u = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += u;
      }
      s_w[lane] = w;
    }
    __syncthreads();
    const long long incl = t + (warp ? s_w[warp - 1] : 0LL) + s_carry;
    if (b < nb) bsum[b] = incl - x;  // exclusive offset of block b
    if (b < nb && incl > 0x7fffffffLL) *overflow = 1;
    __syncthreads();
    if (tid == kScanThreads - 1) s_carry = incl;
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kScanThreads) k_scan_add(long long n, int* __restrict__ a,
                                                           const long long* __restrict__ bsum) {
  const long long e0 = (long long)blockIdx.x * kScanPer + 4LL * threadIdx.x;
  const int off = (int)bsum[blockIdx.x];
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (e0 + k < n) a[e0 + k + 1] += off;
  if (blockIdx.x == 0 && threadIdx.x == 0) a[0] = 0;
}

}  // namespace

int scan_blocks(long long n) { return (int)((n + kScanPer - 1) / kScanPer); }

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_pool_mu;
cudaMemPool_t g_pool[kMaxDevices] = {};
}  // namespace

cudaError_t scratch_alloc(void** p, size_t bytes, cudaStream_t s) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaMallocAsync(p, bytes, s);
  cudaMemPool_t pool;
  {
    std::lock_guard<std::mutex> lock(g_pool_mu);
    if (!g_pool[dev]) {
      cudaMemPoolProps props{};
      props.allocType = cudaMemAllocationTypePinned;
      props.location.type = cudaMemLocationTypeDevice;
      props.location.id = dev;
      if ((err = cudaMemPoolCreate(&g_pool[dev], &props)) != cudaSuccess) {
        g_pool[dev] = nullptr;
        return err;
      }
      uint64_t keep = ~0ull;  // never return memory to the device on synchronisation
      cudaMemPoolSetAttribute(g_pool[dev], cudaMemPoolAttrReleaseThreshold, &keep);
    }
    pool = g_pool[dev];
  }
  return cudaMallocFromPoolAsync(p, bytes, pool, s);
}

void scratch_free(void* p, cudaStream_t s) {
  if (p) cudaFreeAsync(p, s);
}

// bsum: scan_blocks(n) (at least 1) long longs of scratch
void launch_scan(long long n, int* a, long long* bsum, int* overflow, cudaStream_t s) {
  if (n <= 0) {
    cudaMemsetAsync(a, 0, sizeof(int), s);
    return;
  }
  const int nb = scan_blocks(n);
  k_scan_local<<<nb, kScanThreads, 0, s>>>(n, a, bsum);
  k_scan_totals<<<1, kScanThreads, 0, s>>>(nb, bsum, overflow);
  k_scan_add<<<nb, kScanThreads, 0, s>>>(n, a, bsum);
}

namespace {

// ------------------------------------------------------------------------------------ cells
struct CellGrid {
  double lo[3];     // bounding-box corner of the graph
  double scale[3];  // cells per Angstrom on each axis (0 when the axis has one cell)
  int dim[3];
  int pad;
};

// A graph of n atoms gets at most 2n + 8 cells (then cells only coarsen): the sum over graphs
// bounds the cell arrays before the grids are known, so no synchronisation is needed.
__host__ __device__ inline long long cell_cap(long long n) { return 2 * n + 8; }

__global__ void __launch_bounds__(256) k_cell_grid(int N, const float* __restrict__ pos,
                                                   const int* __restrict__ gp, int G, float side_min,
                                                   CellGrid* __restrict__ grids,
                                                   int* __restrict__ ncell) {
  __shared__ float s_mn[3][8], s_mx[3][8];
  const int g = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int lo, hi;
  graph_bounds(gp, G, N, g, &lo, &hi);
  float mn[3] = {INFINITY, INFINITY, INFINITY}, mx[3] = {-INFINITY, -INFINITY, -INFINITY};
  for (int i = lo + tid; i < hi; i += blockDim.x)
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      const float x = pos[3 * i + a];
      mn[a] = fminf(mn[a], x);
      mx[a] = fmaxf(mx[a], x);
    }
#pragma unroll
  for (int a = 0; a < 3; ++a) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mn[a] = fminf(mn[a], __shfl_xor_sync(0xffffffffu, mn[a], o));
      mx[a] = fmaxf(mx[a], __shfl_xor_sync(0xffffffffu, mx[a], o));
    }
    if (lane == 0) {
      s_mn[a][warp] = mn[a];
      s_mx[a][warp] = mx[a];
    }
  }
  __syncthreads();
  if (tid != 0) return;
  CellGrid cg;
  double ext[3];
  for (int a = 0; a < 3; ++a) {
    float m0 = s_mn[a][0], m1 = s_mx[a][0];
    for (int w = 1; w < 8; ++w) {
      m0 = fminf(m0, s_mn[a][w]);
      m1 = fmaxf(m1, s_mx[a][w]);
    }
    const bool any = hi > lo && m0 <= m1;  // false also when a coordinate is NaN throughout
    cg.lo[a] = any ? (double)m0 : 0.0;
    ext[a] = any ? (double)m1 - (double)m0 : 0.0;
    // floor(ext / side_min) cells keep each cell at least side_min wide; 1024 per axis at most
    const double q = ext[a] / (double)side_min;
    cg.dim[a] = q >= 2.0 ? (q >= 1024.0 ? 1024 : (int)q) : 1;
  }
  const long long cap = cell_cap(hi - lo);
  while ((long long)cg.dim[0] * cg.dim[1] * cg.dim[2] > cap) {
    const int a = (cg.dim[0] >= cg.dim[1] && cg.dim[0] >= cg.dim[2]) ? 0
                  : (cg.dim[1] >= cg.dim[2] ? 1 : 2);
    cg.dim[a] = cg.dim[a] / 2 > 1 ? cg.dim[a] / 2 : 1;
  }
  for (int a = 0; a < 3; ++a) cg.scale[a] = cg.dim[a] > 1 ? (double)cg.dim[a] / ext[a] : 0.0;
  cg.pad = 0;
  grids[g] = cg;
  ncell[g + 1] = cg.dim[0] * cg.dim[1] * cg.dim[2];
}

__device__ __forceinline__ int cell_coord(float x, double lo, double scale, int dim) {
  const double u = ((double)x - lo) * scale;  // the subtraction is exact in float64
  int c = u >= 0.0 ? (int)fmin(u, (double)(dim - 1)) : 0;  // NaN compares false: cell 0
  return c;
}

// cellinfo[i] = (cx, cy, cz, g), cell id of i counted in cnt[id + 1]; atoms outside every graph
// get g = -1 and no cell
__global__ void k_cell_assign(int N, const float* __restrict__ pos, const int* __restrict__ gp,
                              int G, const CellGrid* __restrict__ grids,
                              const int* __restrict__ cell_off, long long cmax, int* bad,
                              int4* __restrict__ cellinfo, int* __restrict__ cell_id,
                              int* __restrict__ cnt) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  int g = graph_of(gp, G, i);
  if (g >= 0 && (cell_off[g] < 0 || (long long)cell_off[g + 1] > cmax)) {
    *bad = 1;  // overlapping graph ranges: more cells than the bound; this atom gets none
    g = -1;
  }
  if (g < 0) {
    cellinfo[i] = make_int4(0, 0, 0, -1);
    cell_id[i] = -1;
    return;
  }
  const CellGrid& cg = grids[g];
  const int cx = cell_coord(pos[3 * i], cg.lo[0], cg.scale[0], cg.dim[0]);
  const int cy = cell_coord(pos[3 * i + 1], cg.lo[1], cg.scale[1], cg.dim[1]);
  const int cz = cell_coord(pos[3 * i + 2], cg.lo[2], cg.scale[2], cg.dim[2]);
  const int id = cell_off[g] + (cz * cg.dim[1] + cy) * cg.dim[0] + cx;
  cellinfo[i] = make_int4(cx, cy, cz, g);
  cell_id[i] = id;
  // one atomic per cell and warp: atoms in spatial order share cells within a warp
  const unsigned peers = __match_any_sync(__activemask(), id);
  if ((int)(threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&cnt[id + 1], __popc(peers));
}

// counting-sort placement: cpos[slot] = (x, y, z, i as int bits); order inside a cell is free
__global__ void k_cell_place(int N, const float* __restrict__ pos, const int* __restrict__ cell_id,
                             const int* __restrict__ cell_start, int* __restrict__ cursor,
                             float4* __restrict__ cpos) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  const int id = cell_id[i];
  if (id < 0) return;
  // one atomic per cell and warp; each lane then takes its rank among the warp's atoms of the cell
  const unsigned peers = __match_any_sync(__activemask(), id);
  const int lane = threadIdx.x & 31, leader = __ffs(peers) - 1;
  int base = 0;
  if (lane == leader) base = atomicAdd(&cursor[id], __popc(peers));
  base = __shfl_sync(peers, base, leader);
  const int slot = cell_start[id] + base + __popc(peers & ((1u << lane) - 1u));
  cpos[slot] = make_float4(pos[3 * i], pos[3 * i + 1], pos[3 * i + 2], __int_as_float(i));
}

// The candidate runs of a row: for each (dy, dz) in range, the cells x-1 .. x+1 of that line are
// consecutive ids, so one contiguous run of cpos. Calls f(begin, end) for each run.
template <typename F>
__device__ __forceinline__ void for_each_run(const int4 ci, const CellGrid& cg, int base,
                                             const int* __restrict__ cell_start, F&& f) {
  const int x0 = ci.x > 0 ? ci.x - 1 : 0, x1 = ci.x + 1 < cg.dim[0] ? ci.x + 1 : cg.dim[0] - 1;
  for (int z = ci.z - 1; z <= ci.z + 1; ++z) {
    if (z < 0 || z >= cg.dim[2]) continue;
    for (int y = ci.y - 1; y <= ci.y + 1; ++y) {
      if (y < 0 || y >= cg.dim[1]) continue;
      const int line = base + (z * cg.dim[1] + y) * cg.dim[0];
      f(cell_start[line + x0], cell_start[line + x1 + 1]);
    }
  }
}

// pass 1: row_ptr[i + 1] = number of neighbors of row i (one warp per row)
__global__ void __launch_bounds__(256) k_cell_count(
    int N, const float* __restrict__ pos, const int4* __restrict__ cellinfo,
    const CellGrid* __restrict__ grids, const int* __restrict__ cell_off,
    const int* __restrict__ cell_start, const float4* __restrict__ cpos, double rc2,
    int* __restrict__ row_ptr) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < N; i += warps) {
    const int4 ci = cellinfo[i];
    int cnt = 0;
    if (ci.w >= 0) {
      const float xi = pos[3 * i], yi = pos[3 * i + 1], zi = pos[3 * i + 2];
      for_each_run(ci, grids[ci.w], cell_off[ci.w], cell_start, [&](int b, int e) {
        for (int k = b + lane; k < e; k += 32) {
          const float4 q = cpos[k];
          cnt += (__float_as_int(q.w) != i && d2_exact(xi, yi, zi, q.x, q.y, q.z) < rc2) ? 1 : 0;
        }
      });
    }
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (lane == 0) row_ptr[i + 1] = cnt;
  }
}

__device__ __forceinline__ unsigned lanemask_lt() {
  return (1u << (threadIdx.x & 31)) - 1u;
}

// pass 2: the sources of each row in ascending order (one warp per row)
constexpr int kFillWarps = 8, kFillCap = 1024;

__global__ void __launch_bounds__(kFillWarps * 32) k_cell_fill(
    int N, const float* __restrict__ pos, const int* __restrict__ gp, int G,
    const int4* __restrict__ cellinfo, const CellGrid* __restrict__ grids,
    const int* __restrict__ cell_off, const int* __restrict__ cell_start,
    const float4* __restrict__ cpos, double rc2, const int* __restrict__ row_ptr,
    int* __restrict__ col_idx, long long capacity) {
  __shared__ int s_j[kFillWarps][kFillCap];
  const int lane = threadIdx.x & 31;
  int* sj = s_j[threadIdx.x >> 5];
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < N; i += warps) {
    const long long start = row_ptr[i];
    const int cnt = row_ptr[i + 1] - row_ptr[i];
    const int4 ci = cellinfo[i];
    if (cnt <= 0 || ci.w < 0) continue;
    const long long stop = start + cnt < capacity ? start + cnt : capacity;
    const float xi = pos[3 * i], yi = pos[3 * i + 1], zi = pos[3 * i + 2];
    if (cnt <= kFillCap) {
      int n = 0;
      for_each_run(ci, grids[ci.w], cell_off[ci.w], cell_start, [&](int b, int e) {
        for (int k0 = b; k0 < e; k0 += 32) {
          const int k = k0 + lane;
          bool hit = false;
          int j = 0;
          if (k < e) {
            const float4 q = cpos[k];
            j = __float_as_int(q.w);
            hit = j != i && d2_exact(xi, yi, zi, q.x, q.y, q.z) < rc2;
          }
          const unsigned m = __ballot_sync(0xffffffffu, hit);
          const int slot = n + __popc(m & lanemask_lt());
          if (hit && slot < kFillCap) sj[slot] = j;
          n += __popc(m);
        }
      });
      __syncwarp();
      const int m = n < cnt ? n : cnt;  // equal for any input: the same test as pass 1
      for (int c = lane; c < m; c += 32) {
        const int jc = sj[c];
        int r = 0;
        for (int o = 0; o < m; ++o) r += sj[o] < jc ? 1 : 0;
        if (start + r < stop) col_idx[start + r] = jc;
      }
      __syncwarp();
    } else {  // more hits than the staging holds: ordered scan over the row's graph
      int lo, hi;
      graph_bounds(gp, G, N, ci.w, &lo, &hi);
      long long out = start;
      for (int j0 = lo; j0 < hi; j0 += 32) {
        const int j = j0 + lane;
        const bool hit = j < hi && j != i &&
                         d2_exact(xi, yi, zi, pos[3 * j], pos[3 * j + 1], pos[3 * j + 2]) < rc2;
        const unsigned m = __ballot_sync(0xffffffffu, hit);
        const long long slot = out + __popc(m & lanemask_lt());
        if (hit && slot < stop) col_idx[slot] = j;
        out += __popc(m);
      }
    }
  }
}

// Bitonic sorting network over P (a power of two) staged entries of one warp, ascending by
// (d2, j) or by j alone; every lane takes P / 64 compare-exchanges per stage.
__device__ __forceinline__ void warp_bitonic(int* __restrict__ sj, double* __restrict__ sd, int P,
                                             bool by_dist) {
  const int lane = threadIdx.x & 31;
  for (int k = 2; k <= P; k <<= 1) {
    for (int h = k >> 1; h > 0; h >>= 1) {
      for (int i = lane; i < P; i += 32) {
        const int l = i ^ h;
        if (l > i) {
          const int ji = sj[i], jl = sj[l];
          bool gt;
          if (by_dist) {
            const double di = sd[i], dl = sd[l];
            gt = di > dl || (di == dl && ji > jl);
          } else {
            gt = ji > jl;
          }
          if (gt == ((i & k) == 0)) {  // out of order for this block's direction
            sj[i] = jl;
            sj[l] = ji;
            if (by_dist) {
              const double t = sd[i];
              sd[i] = sd[l];
              sd[l] = t;
            }
          }
        }
      }
      __syncwarp();
    }
  }
}

// Padded list: the hits of a row staged as (j, d2); with more than K, keep those whose rank by
// (d2, j) is below K (a sorting network by (d2, j)); kept entries are written in ascending j (a
// sorting network by j). A row with more than 1024 hits raises the overflow flag and is written
// empty.
constexpr int kPadCap = 1024, kPadWarps = 4;

__global__ void __launch_bounds__(kPadWarps * 32) k_cell_padded(
    int N, const float* __restrict__ pos, const int4* __restrict__ cellinfo,
    const CellGrid* __restrict__ grids, const int* __restrict__ cell_off,
    const int* __restrict__ cell_start, const float4* __restrict__ cpos, double rc2, int K,
    int* __restrict__ nbr, unsigned char* __restrict__ mask, int* __restrict__ overflow) {
  __shared__ int s_j[kPadWarps][kPadCap];
  __shared__ double s_d2[kPadWarps][kPadCap];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  int* sj = s_j[wib];
  double* sd = s_d2[wib];
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < N; i += warps) {
    const int4 ci = cellinfo[i];
    int n = 0;
    if (ci.w >= 0) {
      const float xi = pos[3 * i], yi = pos[3 * i + 1], zi = pos[3 * i + 2];
      for_each_run(ci, grids[ci.w], cell_off[ci.w], cell_start, [&](int b, int e) {
        for (int k0 = b; k0 < e; k0 += 32) {
          const int k = k0 + lane;
          bool hit = false;
          int j = 0;
          double d2 = 0.0;
          if (k < e) {
            const float4 q = cpos[k];
            j = __float_as_int(q.w);
            d2 = d2_exact(xi, yi, zi, q.x, q.y, q.z);
            hit = j != i && d2 < rc2;
          }
          const unsigned m = __ballot_sync(0xffffffffu, hit);
          const int slot = n + __popc(m & lanemask_lt());
          if (hit && slot < kPadCap) {
            sj[slot] = j;
            sd[slot] = d2;
          }
          n += __popc(m);
        }
      });
    }
    __syncwarp();
    int* row_n = nbr + (size_t)i * K;
    unsigned char* row_m = mask + (size_t)i * K;
    if (n > kPadCap) {
      if (lane == 0) *overflow = 1;
      n = 0;
    }
    // sorting network over the staged hits, padded to a power of two with entries that sort last
    int P = 1;
    while (P < n) P <<= 1;
    for (int c = n + lane; c < P; c += 32) {
      sj[c] = 0x7fffffff;
      sd[c] = INFINITY;
    }
    __syncwarp();
    int kept = n;
    if (n > K) {  // the K nearest by (d2, j) come first; the rest are dropped
      warp_bitonic(sj, sd, P, true);
      for (int c = K + lane; c < P; c += 32) sj[c] = 0x7fffffff;
      __syncwarp();
      kept = K;
      P = 1;
      while (P < K) P <<= 1;
    }
    warp_bitonic(sj, sd, P, false);  // the kept entries by ascending j
    for (int c = lane; c < kept; c += 32) {
      row_n[c] = sj[c];
      row_m[c] = 1;
    }
    for (int s = kept + lane; s < K; s += 32) {
      row_n[s] = -1;
      row_m[s] = 0;
    }
    __syncwarp();
  }
}

// The atoms of each cell in ascending index order, cells in their grid order: perm[k] is the
// atom at position k (one warp per cell; an atom's place is its rank among the cell's atoms).
__global__ void k_cell_order(long long cmax, const int* __restrict__ cell_start,
                             const float4* __restrict__ cpos, int* __restrict__ perm) {
  const int lane = threadIdx.x & 31;
  const long long warps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long c = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; c < cmax;
       c += warps) {
    const int a = cell_start[c], b = cell_start[c + 1];
    for (int k = a + lane; k < b; k += 32) {
      const int me = __float_as_int(cpos[k].w);
      int r = 0;
      for (int o = a; o < b; ++o) r += __float_as_int(cpos[o].w) < me ? 1 : 0;
      perm[a + r] = me;
    }
  }
}

int sm_count() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// Device scratch of one build: the grids, the cell arrays and the per-atom cell records.
struct Cells {
  void* buf = nullptr;
  CellGrid* grids;
  int *cell_off, *cell_start, *cursor, *cell_id, *flag, *bad;
  int4* cellinfo;
  float4* cpos;
  long long* bsum;
  long long cmax;
};

size_t align16(size_t b) { return (b + 15) / 16 * 16; }

// every atom's cell record; the cell arrays bounded by the per-graph caps (no synchronisation)
__global__ void k_check_cells(int G, const int* __restrict__ cell_off, long long cmax,
                              int* __restrict__ bad) {
  if (threadIdx.x == 0 && blockIdx.x == 0 && (long long)cell_off[G] > cmax) *bad = 1;
}

int build_cells(Cells& c, int N, const float* pos, const int* gp, int G, float r_c,
                cudaStream_t s) {
  c.cmax = 2LL * N + 8LL * G;
  if (c.cmax + 1 > 0x7fffffffLL) return MP_ERR_CAPACITY;
  long long nb = scan_blocks(N);
  if (scan_blocks(c.cmax) > nb) nb = scan_blocks(c.cmax);
  if (scan_blocks(G) > nb) nb = scan_blocks(G);
  if (nb < 1) nb = 1;
  const size_t sz_grid = align16(sizeof(CellGrid) * (size_t)G),
               sz_off = align16(4 * (size_t)(G + 1)), sz_start = align16(4 * (size_t)(c.cmax + 1)),
               sz_cur = align16(4 * (size_t)c.cmax), sz_info = align16(16 * (size_t)N),
               sz_id = align16(4 * (size_t)N), sz_cpos = align16(16 * (size_t)N),
               sz_bsum = align16(8 * (size_t)nb), sz_flag = 16;
  const size_t total =
      sz_grid + sz_off + sz_start + sz_cur + sz_info + sz_id + sz_cpos + sz_bsum + sz_flag;
  if (scratch_alloc(&c.buf, total, s) != cudaSuccess) return MP_ERR_CUDA;
  char* p = (char*)c.buf;
  c.grids = (CellGrid*)p, p += sz_grid;
  c.cell_off = (int*)p, p += sz_off;
  c.cell_start = (int*)p, p += sz_start;
  c.cursor = (int*)p, p += sz_cur;
  c.cellinfo = (int4*)p, p += sz_info;
  c.cell_id = (int*)p, p += sz_id;
  c.cpos = (float4*)p, p += sz_cpos;
  c.bsum = (long long*)p, p += sz_bsum;
  c.flag = (int*)p;
  c.bad = c.flag + 1;
  cudaMemsetAsync(c.cell_start, 0, sz_start + sz_cur, s);  // cell counts and cursors
  cudaMemsetAsync(c.flag, 0, sz_flag, s);
  const float side_min = r_c * (1.0f + 1.0f / 1024.0f);
  k_cell_grid<<<G, 256, 0, s>>>(N, pos, gp, G, side_min, c.grids, c.cell_off);
  launch_scan(G, c.cell_off, c.bsum, c.flag, s);
  k_check_cells<<<1, 32, 0, s>>>(G, c.cell_off, c.cmax, c.bad);
  if (N > 0) {
    k_cell_assign<<<(N + 255) / 256, 256, 0, s>>>(N, pos, gp, G, c.grids, c.cell_off, c.cmax,
                                                  c.bad, c.cellinfo, c.cell_id, c.cell_start);
  }
  launch_scan(c.cmax, c.cell_start, c.bsum, c.flag, s);
  if (N > 0)
    k_cell_place<<<(N + 255) / 256, 256, 0, s>>>(N, pos, c.cell_id, c.cell_start, c.cursor,
                                                 c.cpos);
  return cudaGetLastError() == cudaSuccess ? MP_OK : MP_ERR_CUDA;
}

}  // namespace
}  // namespace mp

using namespace mp;

extern "C" int mp_neighbor_csr(int N, const float* pos, const int* graph_ptr, int n_graphs,
                               float r_c, int* row_ptr, int* col_idx, long long capacity,
                               long long* n_edges, void* stream) {
  if (N < 0 || !row_ptr || !n_edges || (N > 0 && !pos) || !(r_c > 0.f) || !std::isfinite(r_c) ||
      capacity < 0 || (capacity > 0 && !col_idx) || (graph_ptr && n_graphs < 1))
    return MP_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  const double rcd = (double)r_c;
  const double rc2 = rcd * rcd;  // exact for the cutoffs in use; one rounded multiply on the host
  const int G = graph_ptr ? n_graphs : 1;
  Cells c;
  int rc = build_cells(c, N, pos, graph_ptr, G, r_c, s);
  if (rc != MP_OK) {
    if (c.buf) scratch_free(c.buf, s);
    return rc;
  }
  const int grid = sm_count() * 8;
  if (N > 0)
    k_cell_count<<<grid, 256, 0, s>>>(N, pos, c.cellinfo, c.grids, c.cell_off, c.cell_start,
                                      c.cpos, rc2, row_ptr);
  launch_scan(N, row_ptr, c.bsum, c.flag, s);
  int host[3] = {0, 0, 0};  // E, overflow, bad input
  cudaMemcpyAsync(&host[0], row_ptr + N, sizeof(int), cudaMemcpyDeviceToHost, s);
  cudaMemcpyAsync(&host[1], c.flag, 2 * sizeof(int), cudaMemcpyDeviceToHost, s);
  if (cudaStreamSynchronize(s) != cudaSuccess || cudaGetLastError() != cudaSuccess) {
    scratch_free(c.buf, s);
    return MP_ERR_CUDA;
  }
  *n_edges = host[0];
  rc = host[2] ? MP_ERR_INVALID_ARG : (host[1] || host[0] > capacity) ? MP_ERR_CAPACITY : MP_OK;
  if (rc == MP_OK && N > 0 && host[0] > 0)
    k_cell_fill<<<sm_count() * 4, kFillWarps * 32, 0, s>>>(N, pos, graph_ptr, G, c.cellinfo,
                                                           c.grids, c.cell_off, c.cell_start,
                                                           c.cpos, rc2, row_ptr, col_idx, capacity);
  scratch_free(c.buf, s);
  if (rc != MP_OK) return rc;
  return cudaGetLastError() == cudaSuccess ? MP_OK : MP_ERR_CUDA;
}

extern "C" int mp_neighbor_padded(int N, const float* pos, const int* graph_ptr, int n_graphs,
                                  float r_c, int K, int* nbr, unsigned char* mask, void* stream) {
  if (N < 0 || K < 1 || (N > 0 && (!pos || !nbr || !mask)) || !(r_c > 0.f) ||
      !std::isfinite(r_c) || (graph_ptr && n_graphs < 1))
    return MP_ERR_INVALID_ARG;
  if (N == 0) return MP_OK;
  cudaStream_t s = (cudaStream_t)stream;
  const double rcd = (double)r_c;
  const double rc2 = rcd * rcd;  // exact for the cutoffs in use; one rounded multiply on the host
  const int G = graph_ptr ? n_graphs : 1;
  Cells c;
  int rc = build_cells(c, N, pos, graph_ptr, G, r_c, s);
  if (rc == MP_OK)
    k_cell_padded<<<sm_count() * 4, kPadWarps * 32, 0, s>>>(N, pos, c.cellinfo, c.grids,
                                                            c.cell_off, c.cell_start, c.cpos, rc2,
                                                            K, nbr, mask, c.flag);
  int host[2] = {0, 0};
  if (rc == MP_OK) cudaMemcpyAsync(host, c.flag, 2 * sizeof(int), cudaMemcpyDeviceToHost, s);
  const bool ok = cudaStreamSynchronize(s) == cudaSuccess && cudaGetLastError() == cudaSuccess;
  if (c.buf) scratch_free(c.buf, s);
  if (rc != MP_OK) return rc;
  if (!ok) return MP_ERR_CUDA;
  return host[1] ? MP_ERR_INVALID_ARG : host[0] ? MP_ERR_CAPACITY : MP_OK;
}

extern "C" int mp_spatial_order(int N, const float* pos, const int* graph_ptr, int n_graphs,
                                float cell, int* perm, void* stream) {
  if (N < 0 || (N > 0 && (!pos || !perm)) || !(cell > 0.f) || !std::isfinite(cell) ||
      (graph_ptr && n_graphs < 1))
    return MP_ERR_INVALID_ARG;
  if (N == 0) return MP_OK;
  cudaStream_t s = (cudaStream_t)stream;
  const int G = graph_ptr ? n_graphs : 1;
  Cells c;
  int rc = build_cells(c, N, pos, graph_ptr, G, cell, s);
  if (rc == MP_OK) {
    cudaMemsetAsync(perm, 0xff, sizeof(int) * (size_t)N, s);  // atoms outside every graph: -1
    k_cell_order<<<sm_count() * 8, 256, 0, s>>>(c.cmax, c.cell_start, c.cpos, perm);
    if (cudaGetLastError() != cudaSuccess) rc = MP_ERR_CUDA;
  }
  int host[2] = {0, 0};
  if (rc == MP_OK) cudaMemcpyAsync(host, c.flag, 2 * sizeof(int), cudaMemcpyDeviceToHost, s);
  const bool ok = cudaStreamSynchronize(s) == cudaSuccess && cudaGetLastError() == cudaSuccess;
  if (c.buf) scratch_free(c.buf, s);
  if (rc != MP_OK) return rc;
  if (!ok) return MP_ERR_CUDA;
  return host[1] ? MP_ERR_INVALID_ARG : MP_OK;
}
