// Undirected-pair plan of a symmetric neighbor list, and the fixed-order sum of the pair
// kernel's partial rows.
//
// The filter W(d_ij) depends on the pair's distance only, so W_ij = W_ji: evaluated once per
// pair {i, j} it serves both messages, x_j (.) W to row i and x_i (.) W to row j (the symmetric
// list of the FlashSchNet page, 2.3; the filter-MLP stage, 2.4, is then run on half the edges).
// Without atomics the two messages of a tile must land in accumulators that cover their rows, so
// the pairs are grouped by blocks of 128 atoms: a tile holds 128 pairs (i, j), i < j, of one block
// pair (I, J) = (i / 128, j / 128), I <= J, sorted by i then j. The pair kernel keeps m_I (the rows
// of block I) and m_J (block J) in TMEM and writes each as an fp32 partial block when its run of
// tiles ends; k_pair_sum adds, per block of rows, its partials in a fixed order.
//
// The plan (rebuilt with the neighbor list; distances are not part of it):
//   k_pair_blocks  per block R: its upper pairs (i in R, j > i) sorted by (J, i, j) in shared
//                  memory, their segments (one per block pair), and the blocks J < R below it
//   k_pair_scan    tile offsets of the blocks
//   k_pair_tiles   the tiles: 128 pair slots each (padding i = j = -1), and their block pair
//   k_pair_flags   for the kernel's split of the tiles over G CTAs: which tile starts an
//                  accumulator run, which ends one, and the partial slot each run writes
//   k_pair_sumlist per block of rows, the partial slots it sums, in a fixed order
#include <climits>

#include "mp_internal.cuh"

namespace mp {
namespace {

constexpr int PB_THREADS = 512;
constexpr int SUM_ROWS = 8;  // rows per k_pair_sum CTA (a multiple of 4)

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *(const uint32_t*)&h;
}

// Block-wide exclusive scan of one int per thread (blockDim.x a multiple of 32, at most 1024).
__device__ int block_excl_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[w] = x;
  __syncthreads();
  if (w == 0) {
    int t = lane < nw ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < nw) s_warp[lane] = t;  // inclusive warp totals
  }
  __syncthreads();
  const int before = (w > 0 ? s_warp[w - 1] : 0) + x - v;
  if (total) *total = s_warp[nw - 1];
  __syncthreads();
  return before;
}

// Per block R of 128 rows: the upper pairs, their block-pair segments and the lower blocks.
// Output regions of block R start at row_ptr[128 R] in pairs / segs / low: each holds fewer
// entries than block R has edges, so the regions of different blocks never overlap.
__global__ void __launch_bounds__(PB_THREADS) k_pair_blocks(
    int N, int NB, const int* __restrict__ row_ptr, const int* __restrict__ col_idx, int kcap,
    int2* __restrict__ pairs, int4* __restrict__ segs, int* __restrict__ low,
    int* __restrict__ nseg, int* __restrict__ ntile, int* __restrict__ nlow,
    int* __restrict__ pbase_out, int* status) {
  extern __shared__ __align__(16) uint32_t psm[];
  uint32_t* keys = psm;                        // [kcap]
  uint32_t* bitmap = psm + kcap;               // [NB / 32 + 1]
  __shared__ int s_rp[129], s_warp[32], s_cnt;
  __shared__ int s_seg_start[1024];
  const int R = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
  const int r0 = R * 128, r1 = min(r0 + 128, N);
  const int nbw = NB / 32 + 1;
  for (int k = tid; k <= r1 - r0; k += nt) s_rp[k] = row_ptr[r0 + k];
  for (int k = tid; k < nbw; k += nt) bitmap[k] = 0u;
  if (tid == 0) s_cnt = 0;
  __syncthreads();
  const int e0 = s_rp[0], e1 = s_rp[r1 - r0];
  if (tid == 0) pbase_out[R] = e0;
  // the upper pairs as keys (J - R, i - r0, j mod 128); the lower blocks as bits
  for (int e = e0 + tid; e < e1; e += nt) {
    int lo = 0, hi = r1 - r0;  // s_rp[lo] <= e < s_rp[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_rp[mid] <= e) lo = mid; else hi = mid;
    }
    const int i = r0 + lo, j = col_idx[e];
    if ((unsigned)j >= (unsigned)N) {
      raise_status(status, kStatusBounds);
      continue;
    }
    if (j > i) {
      const int slot = atomicAdd(&s_cnt, 1);  // positions only: the keys are sorted below
      if (slot < kcap)
        keys[slot] = ((uint32_t)((j >> 7) - R) << 14) | ((uint32_t)lo << 7) | (uint32_t)(j & 127);
    } else if ((j >> 7) < R) {
      atomicOr(&bitmap[(j >> 7) >> 5], 1u << ((j >> 7) & 31));
    }
  }
  __syncthreads();
  const int cnt = s_cnt;
  if (cnt > kcap) {  // more pairs than shared memory holds
    if (tid == 0) raise_status(status, kStatusCapacity);
    if (tid == 0) { nseg[R] = 0; ntile[R] = 0; nlow[R] = 0; }
    return;
  }
  // bitonic sort of the keys (padded to a power of two with the largest key)
  int n2 = 1;
  while (n2 < cnt) n2 <<= 1;
  for (int k = cnt + tid; k < n2; k += nt) keys[k] = 0xffffffffu;
  __syncthreads();
  for (int k = 2; k <= n2; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int a = tid; a < n2; a += nt) {
        const int b = a ^ jj;
        if (b > a) {
          const uint32_t ka = keys[a], kb = keys[b];
          const bool up = (a & k) == 0;
          if ((ka > kb) == up) {
            keys[a] = kb;
            keys[b] = ka;
          }
        }
      }
      __syncthreads();
    }
  }
  const int pbase = e0;
  for (int k = tid; k < cnt; k += nt) {
    const uint32_t key = keys[k];
    const int J = R + (int)(key >> 14);
    pairs[pbase + k] = make_int2(r0 + (int)((key >> 7) & 127), (J << 7) | (int)(key & 127));
  }
  // segments: one per run of equal J, found in order (contiguous key ranges per thread)
  const int per = (cnt + nt - 1) / nt;
  const int k0 = min(cnt, tid * per), k1 = min(cnt, k0 + per);
  int starts = 0;
  for (int k = k0; k < k1; ++k) starts += (k == 0 || (keys[k] >> 14) != (keys[k - 1] >> 14));
  int ns = 0;
  int off = block_excl_scan(starts, s_warp, &ns);
  for (int k = k0; k < k1; ++k)
    if (k == 0 || (keys[k] >> 14) != (keys[k - 1] >> 14)) {
      if (off < 1024) s_seg_start[off] = k;
      ++off;
    }
  __syncthreads();
  if (ns > 1024) {  // more block pairs than the segment table holds
    if (tid == 0) { raise_status(status, kStatusCapacity); nseg[R] = 0; ntile[R] = 0; nlow[R] = 0; }
    return;
  }
  if (tid == 0) {
    int tf = 0;
    for (int s = 0; s < ns; ++s) {
      const int a = s_seg_start[s], b = s + 1 < ns ? s_seg_start[s + 1] : cnt;
      segs[pbase + s] = make_int4(R + (int)(keys[a] >> 14), pbase + a, b - a, tf);
      tf += (b - a + 127) / 128;
    }
    nseg[R] = ns;
    ntile[R] = tf;
  }
  // the lower blocks in increasing order (contiguous word ranges per thread)
  const int wper = (nbw + nt - 1) / nt;
  const int w0 = min(nbw, tid * wper), w1 = min(nbw, w0 + wper);
  int bits = 0;
  for (int w = w0; w < w1; ++w) bits += __popc(bitmap[w]);
  int nl = 0;
  int lo_off = block_excl_scan(bits, s_warp, &nl);
  for (int w = w0; w < w1; ++w) {
    uint32_t m = bitmap[w];
    while (m) {
      const int b = __ffs(m) - 1;
      m &= m - 1;
      low[pbase + lo_off++] = w * 32 + b;
    }
  }
  if (tid == 0) nlow[R] = nl;
}

// toff[0..NB] = exclusive prefix of ntile (one CTA); toff[NB] = number of tiles
__global__ void __launch_bounds__(1024) k_pair_scan(int NB, const int* __restrict__ ntile,
                                                     int* __restrict__ toff) {
  __shared__ int s_warp[32];
  int base = 0;
  for (int c = 0; c < NB; c += blockDim.x) {
    const int k = c + threadIdx.x;
    const int v = k < NB ? ntile[k] : 0;
    int tot = 0;
    const int ex = block_excl_scan(v, s_warp, &tot);
    if (k < NB) toff[k] = base + ex;
    base += tot;
  }
  if (threadIdx.x == 0) toff[NB] = base;
}

// The tiles of block R: pair slots (i, j) padded to 128 per tile, and the tile's block pair.
__global__ void __launch_bounds__(128) k_pair_tiles(
    const int* __restrict__ pbase_of, const int2* __restrict__ pairs,
    const int4* __restrict__ segs, const int* __restrict__ nseg, const int* __restrict__ ntile,
    const int* __restrict__ toff, int2* __restrict__ tpairs, PairTile* __restrict__ tiles) {
  const int R = blockIdx.x;
  const int pbase = pbase_of[R], ns = nseg[R], nt = ntile[R], t0 = toff[R];
  int s = 0;  // the segment holding local tile lt (every thread follows it)
  for (int lt = 0; lt < nt; ++lt) {
    while (s + 1 < ns && segs[pbase + s + 1].w <= lt) ++s;
    const int4 sg = segs[pbase + s];
    const int k = lt - sg.w, start = sg.y + 128 * k, count = min(128, sg.z - 128 * k);
    const int p = threadIdx.x;
    tpairs[(size_t)(t0 + lt) * 128 + p] = p < count ? pairs[start + p] : make_int2(-1, -1);
    if (p == 0) {
      PairTile T{};
      T.I = R;
      T.J = sg.x;
      T.count = count;
      tiles[t0 + lt] = T;
    }
  }
}

// Runs of the pair kernel's split of T tiles over G CTAs (CTA c takes [T c / G, T (c + 1) / G)):
// accumulate flags, flushes and their partial slots, numbered in tile order. One CTA.
__global__ void __launch_bounds__(1024) k_pair_flags(int G, const int* __restrict__ toff, int NB,
                                                     PairTile* __restrict__ tiles,
                                                     int* __restrict__ nslots) {
  __shared__ int s_warp[32];
  const int T = toff[NB];
  auto start = [&](int c) { return (int)(((long long)T * c) / G); };
  int base = 0;
  for (int c0 = 0; c0 < T; c0 += blockDim.x) {
    const int t = c0 + threadIdx.x;
    int nf = 0, flags = 0;
    if (t < T) {
      int c = (int)(((long long)t * G) / T);
      while (c + 1 <= G && start(c + 1) <= t) ++c;
      while (c > 0 && start(c) > t) --c;
      const bool first = start(c) == t, last = start(c + 1) == t + 1;
      const PairTile me = tiles[t];
      const bool diag = me.I == me.J;
      const bool newI = first || tiles[t - 1].I != me.I;
      const bool newBP = newI || tiles[t - 1].J != me.J;
      const bool endI = last || tiles[t + 1].I != me.I;
      const bool endBP = endI || tiles[t + 1].J != me.J;
      const bool fI = endI, fJ = !diag && endBP;
      flags = (newI ? 0 : kPairAccI) | (newBP ? 0 : kPairAccJ) | (diag ? kPairDiag : 0) |
              (fI ? kPairFlushI : 0) | (fJ ? kPairFlushJ : 0);
      nf = (int)fI + (int)fJ;
    }
    int tot = 0;
    const int ex = block_excl_scan(nf, s_warp, &tot);
    if (t < T) {
      tiles[t].flags = flags;
      tiles[t].slotI = (flags & kPairFlushI) ? base + ex : -1;
      tiles[t].slotJ = (flags & kPairFlushJ) ? base + ex + ((flags & kPairFlushI) ? 1 : 0) : -1;
    }
    base += tot;
  }
  if (threadIdx.x == 0) *nslots = base;
}

// The partial slots that block R's rows receive, in the order they are summed: first those of
// the runs ending in R's own tiles (the I side, tile order), then those of the tiles of each block
// pair (I', R), I' < R, in increasing I' (the J side). count: slots per block; fill: the list at
// sum_ptr[R] (the same walk, with a prefix of the counts). One thread per block.
template <bool FILL>
__global__ void k_pair_sumlist(int NB, const int* __restrict__ pbase_of,
                               const int* __restrict__ toff, const PairTile* __restrict__ tiles,
                               const int4* __restrict__ segs, const int* __restrict__ nseg,
                               const int* __restrict__ low, const int* __restrict__ nlow,
                               int* __restrict__ sum_cnt, const int* __restrict__ sum_ptr,
                               int* __restrict__ sum_slots) {
  const int R = blockIdx.x * blockDim.x + threadIdx.x;
  if (R >= NB) return;
  int n = 0, o = FILL ? sum_ptr[R] : 0;
  auto put = [&](int slot) {
    if (FILL) sum_slots[o + n] = slot;
    ++n;
  };
  for (int t = toff[R]; t < toff[R + 1]; ++t)
    if (tiles[t].slotI >= 0) put(tiles[t].slotI);
  const int lb = pbase_of[R], nl = nlow[R];
  for (int l = 0; l < nl; ++l) {
    const int Ip = low[lb + l];
    const int pb = pbase_of[Ip], ns = nseg[Ip];
    int lo = 0, hi = ns;  // the segment of block pair (Ip, R): segments are sorted by J
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (segs[pb + mid].x < R) lo = mid + 1; else hi = mid;
    }
    if (lo >= ns || segs[pb + lo].x != R) continue;  // not reached on a symmetric list
    const int4 sg = segs[pb + lo];
    const int tb = toff[Ip] + sg.w, te = tb + (sg.z + 127) / 128;
    for (int t = tb; t < te; ++t)
      if (tiles[t].slotJ >= 0) put(tiles[t].slotJ);
  }
  if (!FILL) sum_cnt[R] = n;
}

// out rows of block R, SUM_ROWS per CTA: the sum of the partial blocks on R's list, in list
// order, each row read only where the block's row mask has it; rows without pairs get 0. Thread =
// (row r0 + (t >> 5) + 4 m, features 4 (t & 31) .. + 3): 16-byte loads, many partials in flight.
__global__ void __launch_bounds__(128) k_pair_sum(int N, const int* __restrict__ sum_ptr,
                                                  const int* __restrict__ sum_slots,
                                                  const float* __restrict__ part,
                                                  const uint32_t* __restrict__ pmask,
                                                  __nv_bfloat16* __restrict__ out) {
  constexpr int RPT = SUM_ROWS / 4;  // rows per thread
  const int R = blockIdx.x / (128 / SUM_ROWS), rg = blockIdx.x % (128 / SUM_ROWS);
  const int lr0 = rg * SUM_ROWS, fq = threadIdx.x & 31, rs = threadIdx.x >> 5;
  if (R * 128 + lr0 >= N) return;
  float4 acc[RPT];
#pragma unroll
  for (int m = 0; m < RPT; ++m) acc[m] = make_float4(0.f, 0.f, 0.f, 0.f);
  const int s0 = sum_ptr[R], s1 = sum_ptr[R + 1];
  __shared__ int s_slot[128];
  __shared__ uint32_t s_rows[128];
  for (int c0 = s0; c0 < s1; c0 += 128) {  // the list in chunks: slots and masks loaded at once
    const int m = min(128, s1 - c0);
    if ((int)threadIdx.x < m) {
      const int slot = sum_slots[c0 + threadIdx.x];
      s_slot[threadIdx.x] = slot;
      s_rows[threadIdx.x] = __ldg(pmask + (size_t)slot * 4 + (lr0 >> 5)) >> (lr0 & 31);
    }
    __syncthreads();
#pragma unroll 4
    for (int q = 0; q < m; ++q) {
      const uint32_t rows = s_rows[q];
      const float4* p = (const float4*)(part + ((size_t)s_slot[q] * 128 + lr0 + rs) * kPairF) + fq;
#pragma unroll
      for (int k = 0; k < RPT; ++k) {
        if ((rows >> (rs + 4 * k)) & 1u) {
          const float4 v = __ldg(p + k * 4 * (kPairF / 4));
          acc[k].x += v.x;
          acc[k].y += v.y;
          acc[k].z += v.z;
          acc[k].w += v.w;
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int k = 0; k < RPT; ++k) {
    const int r = R * 128 + lr0 + rs + 4 * k;
    if (r < N)
      *(uint2*)(out + (size_t)r * kPairF + 4 * fq) =
          make_uint2(pack_bf16x2(acc[k].x, acc[k].y), pack_bf16x2(acc[k].z, acc[k].w));
  }
}

}  // namespace

// Shared memory of k_pair_blocks for a key capacity.
static size_t pair_blocks_smem(int kcap, int NB) { return (size_t)kcap * 4 + (NB / 32 + 1) * 4; }

// Grow-only device buffer.
static int ensure(void** p, size_t* have, size_t need) {
  if (need <= *have) return MP_OK;
  cudaFree(*p);
  *p = nullptr;
  *have = 0;
  if (cudaMalloc(p, need) != cudaSuccess) return MP_ERR_CUDA;
  *have = need;
  return MP_OK;
}

// The status bits a plan kernel raised (bounds, capacity), read once and cleared.
static int plan_status(mp_ctx* ctx) {
  int st = 0;
  if (cudaMemcpy(&st, ctx->status_d, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return MP_ERR_CUDA;
  if (!(st & (kStatusCapacity | kStatusBounds))) return MP_OK;
  const int clear = st & ~(kStatusCapacity | kStatusBounds);
  cudaMemcpy(ctx->status_d, &clear, 4, cudaMemcpyHostToDevice);
  return (st & kStatusBounds) ? MP_ERR_DEVICE_BOUNDS : MP_ERR_CAPACITY;
}

int pair_plan_build(mp_ctx* ctx, int N, long long E, const int* row_ptr, const int* col_idx,
                    cudaStream_t s) {
  PairPlan& P = ctx->pair;
  P.valid = false;
  if (N < 0 || E < 0 || E > INT32_MAX) return MP_ERR_INVALID_ARG;
  if (ctx->ef_graph) {  // a recorded energy/forces graph may hold the previous plan's buffers
    cudaGraphExecDestroy(ctx->ef_graph);
    ctx->ef_graph = nullptr;
  }
  const int NB = (N + 127) / 128;
  if (NB > (1 << 16)) return MP_ERR_CAPACITY;  // the lower-block bitmap of k_pair_blocks
  // phase 1: per block, arrays indexed by the list's offsets (pairs, segments, lower blocks)
  const size_t sz[] = {(size_t)(E + 1) * 8, (size_t)(E + 1) * 16, (size_t)(E + 1) * 4,
                       (size_t)(NB + 2) * 4, (size_t)(NB + 2) * 4, (size_t)(NB + 2) * 4,
                       (size_t)(NB + 2) * 4, (size_t)(NB + 2) * 4, 16};
  size_t need = 0;
  for (size_t v : sz) need += align_up_sz(v);
  int rc = ensure(&P.ws, &P.ws_bytes, need);
  if (rc != MP_OK) return rc;
  char* b = (char*)P.ws;
  int k = 0;
  auto take = [&]() {
    char* p = b;
    b += align_up_sz(sz[k++]);
    return (void*)p;
  };
  P.pairs = (int2*)take();
  P.segs = (int4*)take();
  P.low = (int*)take();
  P.pbase = (int*)take();
  P.nseg = (int*)take();
  P.ntile = (int*)take();
  P.nlow = (int*)take();
  P.toff = (int*)take();
  P.counts = (int*)take();
  P.N = N;
  P.E = E;
  P.NB = NB;
  P.G = ctx->num_sms;
  P.list_row_ptr = row_ptr;
  P.list_col_idx = col_idx;
  // a block's upper pairs are sorted in shared memory: at most 32 Ki of them (128 KB; a power of
  // two, the bitonic sort's padded length)
  const int kcap = 32 * 1024;
  const size_t smem = pair_blocks_smem(kcap, NB);
  cudaFuncSetAttribute(k_pair_blocks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaMemsetAsync(P.counts, 0, 16, s);
  cudaMemsetAsync(P.toff, 0, 4, s);
  if (NB > 0) {
    rc = launch(ctx, K_PAIR_PLAN, k_pair_blocks, dim3(NB), dim3(PB_THREADS), smem, s, N, NB,
                row_ptr, col_idx, kcap, P.pairs, P.segs, P.low, P.nseg, P.ntile, P.nlow, P.pbase,
                ctx->status_d);
    if (rc == MP_OK)
      rc = launch(ctx, K_PAIR_PLAN, k_pair_scan, dim3(1), dim3(1024), 0, s, NB,
                  (const int*)P.ntile, P.toff);
    if (rc != MP_OK) return rc;
  }
  int T = 0;
  cudaMemcpyAsync(&T, P.toff + NB, 4, cudaMemcpyDeviceToHost, s);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MP_ERR_CUDA;
  if ((rc = plan_status(ctx)) != MP_OK) return rc;
  // phase 2: the tiles (now counted) and the runs of the kernel's split over the SMs
  // (tiles, their pair slots, and the summing lists: at most two slots per tile)
  const size_t tsz = align_up_sz((size_t)(T + 1) * 128 * 8) +
                     align_up_sz((size_t)(T + 1) * sizeof(PairTile)) +
                     align_up_sz((size_t)(2 * T + 1) * 4) + 2 * align_up_sz((size_t)(NB + 2) * 4);
  if ((rc = ensure(&P.tws, &P.tws_bytes, tsz)) != MP_OK) return rc;
  P.tpairs = (int2*)P.tws;
  P.tiles = (PairTile*)((char*)P.tws + align_up_sz((size_t)(T + 1) * 128 * 8));
  P.sum_slots = (int*)((char*)P.tiles + align_up_sz((size_t)(T + 1) * sizeof(PairTile)));
  P.sum_cnt = (int*)((char*)P.sum_slots + align_up_sz((size_t)(2 * T + 1) * 4));
  P.sum_ptr = (int*)((char*)P.sum_cnt + align_up_sz((size_t)(NB + 2) * 4));
  P.T = T;
  if (T > 0) {
    rc = launch(ctx, K_PAIR_PLAN, k_pair_tiles, dim3(NB), dim3(128), 0, s, (const int*)P.pbase,
                (const int2*)P.pairs, (const int4*)P.segs, (const int*)P.nseg,
                (const int*)P.ntile, (const int*)P.toff, P.tpairs, P.tiles);
    if (rc == MP_OK)
      rc = launch(ctx, K_PAIR_PLAN, k_pair_flags, dim3(1), dim3(1024), 0, s, P.G,
                  (const int*)P.toff, NB, P.tiles, P.counts);
    const dim3 lg((NB + 127) / 128), lb(128);
    if (rc == MP_OK)
      rc = launch(ctx, K_PAIR_PLAN, k_pair_sumlist<false>, lg, lb, 0, s, NB, (const int*)P.pbase,
                  (const int*)P.toff, (const PairTile*)P.tiles, (const int4*)P.segs,
                  (const int*)P.nseg, (const int*)P.low, (const int*)P.nlow, P.sum_cnt,
                  (const int*)nullptr, (int*)nullptr);
    if (rc == MP_OK)
      rc = launch(ctx, K_PAIR_PLAN, k_pair_scan, dim3(1), dim3(1024), 0, s, NB,
                  (const int*)P.sum_cnt, P.sum_ptr);
    if (rc == MP_OK)
      rc = launch(ctx, K_PAIR_PLAN, k_pair_sumlist<true>, lg, lb, 0, s, NB, (const int*)P.pbase,
                  (const int*)P.toff, (const PairTile*)P.tiles, (const int4*)P.segs,
                  (const int*)P.nseg, (const int*)P.low, (const int*)P.nlow, (int*)nullptr,
                  (const int*)P.sum_ptr, P.sum_slots);
    if (rc != MP_OK) return rc;
  } else {
    cudaMemsetAsync(P.sum_ptr, 0, (size_t)(NB + 1) * 4, s);
  }
  int nslots = 0;
  cudaMemcpyAsync(&nslots, P.counts, 4, cudaMemcpyDeviceToHost, s);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MP_ERR_CUDA;
  P.nslots = nslots;
  // one 64 KiB fp32 block of partial rows per run of tiles, and its 128-bit row mask
  const size_t pb = align_up_sz((size_t)(nslots > 0 ? nslots : 1) * 128 * kPairF * 4);
  if ((rc = ensure((void**)&P.part, &P.part_bytes, pb + (size_t)(nslots + 1) * 16)) != MP_OK)
    return rc;
  P.pmask = (uint32_t*)((char*)P.part + pb);
  P.valid = true;
  return MP_OK;
}

int pair_sum_launch(mp_ctx* ctx, int N, void* out, cudaStream_t s) {
  const PairPlan& P = ctx->pair;
  if (P.NB == 0) return MP_OK;
  return launch(ctx, K_PAIR_SUM, k_pair_sum, dim3(P.NB * (128 / SUM_ROWS)), dim3(128), 0, s, N,
                (const int*)P.sum_ptr, (const int*)P.sum_slots, (const float*)P.part,
                (const uint32_t*)P.pmask, (__nv_bfloat16*)out);
}

void pair_plan_free(mp_ctx* ctx) {
  cudaFree(ctx->pair.ws);
  cudaFree(ctx->pair.tws);
  cudaFree(ctx->pair.part);
  ctx->pair = PairPlan{};
}

}  // namespace mp
