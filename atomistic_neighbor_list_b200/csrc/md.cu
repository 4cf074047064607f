// Velocity-Verlet molecular dynamics with the model's forces (FlashSchNet page, s.3: MD steps of
// replicated systems; Tessera page: the neighbor topology is reused across steps). One step:
//   v += (dt/2) F/m;  r += dt v;  (E, F) = energy and forces at r;  v += (dt/2) F/m.
// The list passed in (or built) may hold pairs up to r_c + skin; each step first cuts it to the
// pairs within r_c at the step's positions (three small kernels), so the force kernels see only
// pairs whose envelope is non-zero. The whole step (the integration kernels, the cut and the
// energy/forces launches) is recorded once per call as a CUDA graph and replayed n_steps times.
#include <cmath>

#include "mp_internal.cuh"

namespace mp {

// The list cut to r_c, in scratch from the library's pool: offsets [N + 1], sources [cap].
struct CutList {
  int* rp = nullptr;
  int* ci = nullptr;
  long long cap = 0;
  void* buf = nullptr;
  int alloc(int N, long long cap, cudaStream_t s);
  void release(cudaStream_t s);
};

namespace {

// v += (dt/2) F im; r += dt v   (im: 1/m per atom, or null for unit masses)
__global__ void k_kick_drift(int N, float* __restrict__ pos, float* __restrict__ vel,
                             const float* __restrict__ forces, const float* __restrict__ im,
                             float dt) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  const float h = 0.5f * dt * (im ? im[i] : 1.f);
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    const float v = fmaf(h, forces[3 * i + c], vel[3 * i + c]);
    vel[3 * i + c] = v;
    pos[3 * i + c] = fmaf(dt, v, pos[3 * i + c]);
  }
}

// v += (dt/2) F im
__global__ void k_kick(int N, float* __restrict__ vel, const float* __restrict__ forces,
                       const float* __restrict__ im, float dt) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  const float h = 0.5f * dt * (im ? im[i] : 1.f);
#pragma unroll
  for (int c = 0; c < 3; ++c) vel[3 * i + c] = fmaf(h, forces[3 * i + c], vel[3 * i + c]);
}

// kinetic[g] = sum over the atoms of graph g of |v|^2 / (2 im), fixed-order reduction per graph
__global__ void k_kinetic(int N, const int* __restrict__ graph_ptr, int n_graphs,
                          const float* __restrict__ vel, const float* __restrict__ im,
                          float* __restrict__ kinetic, int* status) {
  __shared__ float s_part[256];
  for (int g = blockIdx.x; g < n_graphs; g += gridDim.x) {
    const int lo = graph_ptr ? graph_ptr[g] : 0, hi = graph_ptr ? graph_ptr[g + 1] : N;
    if (lo < 0 || hi > N || hi < lo) {
      if (threadIdx.x == 0) {
        raise_status(status, kStatusBounds);
        kinetic[g] = 0.f;
      }
      continue;
    }
    float s = 0.f;
    for (int i = lo + threadIdx.x; i < hi; i += blockDim.x) {
      const float vx = vel[3 * i], vy = vel[3 * i + 1], vz = vel[3 * i + 2];
      s += 0.5f * (vx * vx + vy * vy + vz * vz) / (im ? im[i] : 1.f);
    }
    s_part[threadIdx.x] = s;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
      if (threadIdx.x < w) s_part[threadIdx.x] += s_part[threadIdx.x + w];
      __syncthreads();
    }
    if (threadIdx.x == 0) kinetic[g] = s_part[0];
    __syncthreads();
  }
}

// flag = 1 when some atom has moved more than sqrt(lim2) from its reference position
__global__ void k_displaced(int N, const float* __restrict__ pos, const float* __restrict__ ref,
                            float lim2, int* __restrict__ flag) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  const float dx = pos[3 * i] - ref[3 * i], dy = pos[3 * i + 1] - ref[3 * i + 1],
              dz = pos[3 * i + 2] - ref[3 * i + 2];
  if (dx * dx + dy * dy + dz * dz > lim2) *flag = 1;
}

// ---- the list at r_c from a list built at r_c + skin, once per step. A pair is kept when
// d^2 < r_c^2 with d^2 = dx dx + dy dy + dz dz, each product and sum rounded on its own (no
// contraction), so (i, j) and (j, i) get the same decision and the list stays symmetric. A dropped
// pair has f_c = f_c' = 0 at the step's positions: energy and forces are those of the full list.
// An index outside [0, N) is kept, for the force kernels to report.
__device__ __forceinline__ bool within_cut(const float* __restrict__ pos, float xi, float yi,
                                           float zi, int j, int N, float rc2) {
  if ((unsigned)j >= (unsigned)N) return true;
  const float dx = pos[3 * j] - xi, dy = pos[3 * j + 1] - yi, dz = pos[3 * j + 2] - zi;
  const float d2 = __fadd_rn(__fadd_rn(__fmul_rn(dx, dx), __fmul_rn(dy, dy)), __fmul_rn(dz, dz));
  return d2 < rc2;
}

// one warp per row: rp_c[i + 1] = the number of kept edges of row i
__global__ void k_cut_count(int N, const float* __restrict__ pos, const int* __restrict__ row_ptr,
                            const int* __restrict__ col_idx, float rc2, int* __restrict__ rp_c) {
  const int i = (int)((blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5),
            lane = threadIdx.x & 31;
  if (i >= N) return;
  const int lo = row_ptr[i], hi = row_ptr[i + 1];
  const float xi = pos[3 * i], yi = pos[3 * i + 1], zi = pos[3 * i + 2];
  int n = 0;
  for (int e0 = lo; e0 < hi; e0 += 32) {
    const int e = e0 + lane;
    const bool keep = e < hi && within_cut(pos, xi, yi, zi, col_idx[e], N, rc2);
    n += __popc(__ballot_sync(0xffffffffu, keep));
  }
  if (lane == 0) rp_c[i + 1] = n;
}

// rp_c[1..N] counts -> rp_c[0..N] offsets, one CTA: a serial run per thread over a contiguous
// chunk, then a scan of the run totals
constexpr int kCutScanT = 1024;
__global__ void __launch_bounds__(kCutScanT) k_cut_scan(int N, int* __restrict__ rp_c) {
  __shared__ int s_w[32];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int per = (N + kCutScanT - 1) / kCutScanT;
  const int lo = min(N, t * per), hi = min(N, lo + per);
  int run = 0;
  for (int k = lo; k < hi; ++k) run += rp_c[k + 1];
  int x = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += u;
  }
  if (lane == 31) s_w[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = s_w[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += u;
    }
    s_w[lane] = w;
  }
  __syncthreads();
  int off = x - run + (warp ? s_w[warp - 1] : 0);
  for (int k = lo; k < hi; ++k) {
    off += rp_c[k + 1];
    rp_c[k + 1] = off;
  }
  if (t == 0) rp_c[0] = 0;
}

// one warp per row: the kept sources of row i, in the list's order, from rp_c[i]
__global__ void k_cut_fill(int N, const float* __restrict__ pos, const int* __restrict__ row_ptr,
                           const int* __restrict__ col_idx, float rc2,
                           const int* __restrict__ rp_c, long long cap, int* __restrict__ ci_c) {
  const int i = (int)((blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5),
            lane = threadIdx.x & 31;
  if (i >= N) return;
  const int lo = row_ptr[i], hi = row_ptr[i + 1];
  const float xi = pos[3 * i], yi = pos[3 * i + 1], zi = pos[3 * i + 2];
  long long out = rp_c[i];
  for (int e0 = lo; e0 < hi; e0 += 32) {
    const int e = e0 + lane;
    const int j = e < hi ? col_idx[e] : 0;
    const bool keep = e < hi && within_cut(pos, xi, yi, zi, j, N, rc2);
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    const long long o = out + __popc(bal & ((1u << lane) - 1u));
    if (keep && o < cap) ci_c[o] = j;
    out += __popc(bal);
  }
}

}  // namespace

int CutList::alloc(int N, long long cap, cudaStream_t s) {
  const size_t rp_bytes = ((size_t)N + 1) * 4, ci_bytes = (size_t)(cap > 0 ? cap : 1) * 4;
  const size_t rp_pad = (rp_bytes + 255) / 256 * 256;
  if (scratch_alloc(&buf, rp_pad + ci_bytes, s) != cudaSuccess) {
    buf = nullptr;
    return MP_ERR_CUDA;
  }
  rp = (int*)buf;
  ci = (int*)((char*)buf + rp_pad);
  this->cap = cap;
  return MP_OK;
}

void CutList::release(cudaStream_t s) {
  if (buf) scratch_free(buf, s);
  buf = nullptr;
  rp = ci = nullptr;
}

int cut_launches(mp_ctx* c, int N, const float* pos, const int* row_ptr, const int* col_idx,
                 const CutList& L, cudaStream_t s) {
  if (N <= 0) return MP_OK;
  const float rc2 = c->cfg.r_c * c->cfg.r_c;
  const int blocks = (int)(((long long)N * 32 + 255) / 256);
  int rc = launch(c, K_MD_CUT, k_cut_count, dim3(blocks), dim3(256), 0, s, N, pos, row_ptr,
                  col_idx, rc2, L.rp);
  if (rc == MP_OK)
    rc = launch(c, K_MD_CUT, k_cut_scan, dim3(1), dim3(kCutScanT), 0, s, N, L.rp);
  if (rc == MP_OK)
    rc = launch(c, K_MD_CUT, k_cut_fill, dim3(blocks), dim3(256), 0, s, N, pos, row_ptr, col_idx,
                rc2, (const int*)L.rp, L.cap, L.ci);
  return rc;
}

// energy and forces at pos with the list cut to r_c first (E is then an upper bound of the edge
// count the force kernels read from the cut list's offsets)
int cut_energy_forces(mp_ctx* c, int N, long long E, const float* pos, const int* types,
                      const int* row_ptr, const int* col_idx, const CutList& L,
                      const int* graph_ptr, int n_graphs, float* energy, float* forces,
                      cudaStream_t s) {
  int rc = cut_launches(c, N, pos, row_ptr, col_idx, L, s);
  if (rc == MP_OK)
    rc = energy_forces_launches(c, N, E, pos, types, L.rp, L.ci, graph_ptr, n_graphs, energy,
                                forces, s);
  return rc;
}

int md_step_launches(mp_ctx* c, int N, long long E, float* pos, float* vel, float* forces,
                     const float* inv_mass, float dt, const int* types, const int* row_ptr,
                     const int* col_idx, const CutList& L, const int* graph_ptr, int n_graphs,
                     float* energy, cudaStream_t s) {
  const int blocks = (N + 255) / 256;
  int rc = launch(c, K_MD, k_kick_drift, dim3(blocks), dim3(256), 0, s, N, pos, vel,
                  (const float*)forces, inv_mass, dt);
  if (rc == MP_OK)
    rc = cut_energy_forces(c, N, E, pos, types, row_ptr, col_idx, L, graph_ptr, n_graphs, energy,
                           forces, s);
  if (rc == MP_OK)
    rc = launch(c, K_MD, k_kick, dim3(blocks), dim3(256), 0, s, N, vel, (const float*)forces,
                inv_mass, dt);
  return rc;
}

int md_kinetic(mp_ctx* c, int N, const int* graph_ptr, int n_graphs, const float* vel,
               const float* inv_mass, float* kinetic, cudaStream_t s) {
  const int grid = n_graphs < 4 * c->num_sms ? n_graphs : 4 * c->num_sms;
  return launch(c, K_MD, k_kinetic, dim3(grid), dim3(256), 0, s, N, graph_ptr, n_graphs, vel,
                inv_mass, kinetic, c->status_d);
}

// One recorded step, replayed: capture succeeds on a non-default stream that is not already
// capturing; otherwise ex stays null and the caller launches the step's kernels itself.
struct StepGraph {
  cudaGraphExec_t ex = nullptr;
  long long per_step = 0;
  ~StepGraph() { reset(); }
  void reset() {
    if (ex) cudaGraphExecDestroy(ex);  // a pending launch completes first
    ex = nullptr;
  }
};

bool can_record(mp_ctx* c, cudaStream_t s) {
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  return c->graphs && !c->graphs_broken && !c->profiling && s != nullptr &&
         cudaStreamIsCapturing(s, &cap) == cudaSuccess && cap == cudaStreamCaptureStatusNone;
}

void record_step(mp_ctx* c, StepGraph& sg, int N, long long E, float* pos, float* vel,
                 float* forces, const float* inv_mass, float dt, const int* types,
                 const int* row_ptr, const int* col_idx, const CutList& L, const int* graph_ptr,
                 int n_graphs, float* energy, cudaStream_t s) {
  sg.reset();
  if (!can_record(c, s)) return;
  const long long l0 = c->launches;
  cudaGraph_t g = nullptr;
  int rc = cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal) == cudaSuccess ? MP_OK
                                                                                    : MP_ERR_CUDA;
  if (rc == MP_OK) {
    rc = md_step_launches(c, N, E, pos, vel, forces, inv_mass, dt, types, row_ptr, col_idx, L,
                          graph_ptr, n_graphs, energy, s);
    if (cudaStreamEndCapture(s, &g) != cudaSuccess && rc == MP_OK) rc = MP_ERR_CUDA;
  }
  if (rc == MP_OK && (!g || cudaGraphInstantiate(&sg.ex, g, 0) != cudaSuccess)) rc = MP_ERR_CUDA;
  if (g) cudaGraphDestroy(g);
  sg.per_step = c->launches - l0;
  c->launches = l0;
  if (rc != MP_OK) {  // plain launches from now on for this context
    cudaGetLastError();
    c->graphs_broken = true;
    sg.ex = nullptr;
  }
}

int run_steps(mp_ctx* c, StepGraph& sg, int n, int N, long long E, float* pos, float* vel,
              float* forces, const float* inv_mass, float dt, const int* types, const int* row_ptr,
              const int* col_idx, const CutList& L, const int* graph_ptr, int n_graphs,
              float* energy, cudaStream_t s) {
  int rc = MP_OK;
  for (int st = 0; st < n && rc == MP_OK; ++st) {
    if (sg.ex) {
      rc = cudaGraphLaunch(sg.ex, s) == cudaSuccess ? MP_OK : MP_ERR_CUDA;
      c->launches += sg.per_step;
    } else {
      rc = md_step_launches(c, N, E, pos, vel, forces, inv_mass, dt, types, row_ptr, col_idx, L,
                            graph_ptr, n_graphs, energy, s);
    }
  }
  return rc;
}

}  // namespace mp

extern "C" int mp_md_verlet(mp_ctx* c, int N, long long E, float* pos, float* vel, float* forces,
                            const float* inv_mass, float dt, int n_steps, const int* types,
                            const int* row_ptr, const int* col_idx, const int* graph_ptr,
                            int n_graphs, float* energy, float* kinetic, void* stream) {
  using namespace mp;
  if (!c || N < 0 || E < 0 || n_steps < 0 || !row_ptr || !energy || n_graphs < 1 ||
      (N > 0 && (!pos || !vel || !forces || !types)) || (E > 0 && !col_idx) ||
      (!graph_ptr && n_graphs != 1) || !std::isfinite(dt))
    return MP_ERR_INVALID_ARG;
  if (N > c->cfg.max_atoms || E > c->cfg.max_edges || n_graphs > c->cfg.max_graphs)
    return MP_ERR_CAPACITY;
  cudaStream_t s = (cudaStream_t)stream;
  if (c->cfg.validate) {
    const int rc = launch_validate_csr(c, N, E, row_ptr, col_idx, graph_ptr, n_graphs, true, s);
    if (rc != MP_OK) return rc;
  }
  if (N == 0 || n_steps == 0) {  // no atoms: energies are zero; no steps: kinetic only
    int rc = MP_OK;
    if (N == 0 && n_steps > 0)
      rc = energy_forces_launches(c, 0, E, pos, types, row_ptr, col_idx, graph_ptr, n_graphs,
                                  energy, forces, s);
    if (rc == MP_OK && kinetic)
      rc = md_kinetic(c, N, graph_ptr, n_graphs, vel, inv_mass, kinetic, s);
    return rc;
  }
  CutList L;
  int rc = L.alloc(N, E, s);
  {
    StepGraph sg;  // released before the cut list's memory
    if (rc == MP_OK)
      record_step(c, sg, N, E, pos, vel, forces, inv_mass, dt, types, row_ptr, col_idx, L,
                  graph_ptr, n_graphs, energy, s);
    if (rc == MP_OK)
      rc = run_steps(c, sg, n_steps, N, E, pos, vel, forces, inv_mass, dt, types, row_ptr, col_idx,
                     L, graph_ptr, n_graphs, energy, s);
  }
  L.release(s);
  if (rc == MP_OK && kinetic) rc = md_kinetic(c, N, graph_ptr, n_graphs, vel, inv_mass, kinetic, s);
  return rc;
}

extern "C" int mp_md_run(mp_ctx* c, int N, float* pos, float* vel, float* forces,
                         const float* inv_mass, float dt, int n_steps, const int* types,
                         const int* graph_ptr, int n_graphs, float skin, int rebuild_every,
                         float max_disp, int check_every, int* row_ptr, int* col_idx,
                         long long capacity, long long* n_edges, float* energy, float* kinetic,
                         int* n_builds, void* stream) {
  using namespace mp;
  if (!c || N < 0 || n_steps < 0 || !row_ptr || !energy || n_graphs < 1 || !n_edges ||
      (N > 0 && (!pos || !vel || !forces || !types)) || (capacity > 0 && !col_idx) ||
      capacity < 0 || (!graph_ptr && n_graphs != 1) || !std::isfinite(dt) ||
      !std::isfinite(skin) || skin < 0.f || !std::isfinite(max_disp) || rebuild_every < 0 ||
      check_every < 1)
    return MP_ERR_INVALID_ARG;
  if (N > c->cfg.max_atoms || n_graphs > c->cfg.max_graphs) return MP_ERR_CAPACITY;
  cudaStream_t s = (cudaStream_t)stream;
  const float r_list = c->cfg.r_c + skin;
  long long E = 0;
  int builds = 0;
  CutList L;  // the list cut to r_c at each step's positions
  if (L.alloc(N, capacity < c->cfg.max_edges ? capacity : c->cfg.max_edges, s) != MP_OK)
    return MP_ERR_CUDA;
  StepGraph sg;
  // the list at the current positions, the reference positions, and energy/forces with it
  // The forces at the current positions came from the old list; they are those of an exact r_c
  // list as long as no atom has moved skin / 2 since that list was built (a pair now within r_c
  // was then within r_c + skin). Only otherwise are they evaluated again with the new list.
  const float half_skin = 0.5f * skin * 0.999f;
  auto build = [&]() -> int {
    bool fresh_forces = builds == 0;
    if (!fresh_forces) {  // read back by the synchronisation inside the list build
      cudaMemsetAsync(c->md_flag, 0, sizeof(int), s);
      int rc0 = launch(c, K_MD, k_displaced, dim3((N + 255) / 256), dim3(256), 0, s, N,
                       (const float*)pos, (const float*)c->md_ref, half_skin * half_skin,
                       c->md_flag);
      if (rc0 != MP_OK) return rc0;
      cudaMemcpyAsync(c->md_flag_h, c->md_flag, sizeof(int), cudaMemcpyDeviceToHost, s);
    }
    int rc = mp_neighbor_csr(N, pos, graph_ptr, n_graphs, r_list, row_ptr, col_idx, capacity, &E,
                             stream);
    *n_edges = E;
    if (rc != MP_OK) return rc;
    if (E > c->cfg.max_edges) return MP_ERR_CAPACITY;
    ++builds;
    if (!fresh_forces && *c->md_flag_h != 0) fresh_forces = true;
    if (N > 0 && cudaMemcpyAsync(c->md_ref, pos, sizeof(float) * 3 * (size_t)N,
                                 cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return MP_ERR_CUDA;
    if (fresh_forces) {
      rc = cut_energy_forces(c, N, E, pos, types, row_ptr, col_idx, L, graph_ptr, n_graphs, energy,
                             forces, s);
    }
    if (rc == MP_OK && N > 0)
      record_step(c, sg, N, E, pos, vel, forces, inv_mass, dt, types, row_ptr, col_idx, L,
                  graph_ptr, n_graphs, energy, s);
    return rc;
  };
  int rc = build();
  const float lim2 = max_disp * max_disp;
  int done = 0, since = 0;
  while (rc == MP_OK && N > 0 && done < n_steps) {
    int chunk = n_steps - done < check_every ? n_steps - done : check_every;
    if (rebuild_every > 0 && rebuild_every - since < chunk) chunk = rebuild_every - since;
    rc = run_steps(c, sg, chunk, N, E, pos, vel, forces, inv_mass, dt, types, row_ptr, col_idx, L,
                   graph_ptr, n_graphs, energy, s);
    done += chunk;
    since += chunk;
    if (rc != MP_OK || done == n_steps) break;
    bool rebuild = rebuild_every > 0 && since >= rebuild_every;
    if (!rebuild && max_disp > 0.f) {  // early rebuild: one flag read per check
      cudaMemsetAsync(c->md_flag, 0, sizeof(int), s);
      rc = launch(c, K_MD, k_displaced, dim3((N + 255) / 256), dim3(256), 0, s, N,
                  (const float*)pos, (const float*)c->md_ref, lim2, c->md_flag);
      if (rc != MP_OK) break;
      cudaMemcpyAsync(c->md_flag_h, c->md_flag, sizeof(int), cudaMemcpyDeviceToHost, s);
      if (cudaStreamSynchronize(s) != cudaSuccess) {
        rc = MP_ERR_CUDA;
        break;
      }
      rebuild = *c->md_flag_h != 0;
    }
    if (rebuild) {
      rc = build();
      since = 0;
    }
  }
  sg.reset();
  L.release(s);
  if (n_builds) *n_builds = builds;
  if (rc == MP_OK && kinetic) rc = md_kinetic(c, N, graph_ptr, n_graphs, vel, inv_mass, kinetic, s);
  return rc;
}
