// Internal declarations of libmp: context layout, kernel launch/profiling helper, device helpers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "../../include/mp.h"

namespace mp {

constexpr int kMaxR = 64;   // radial functions supported by the kernels

// Device-status bits raised by kernels (read and cleared by mp_status_sync).
enum : int { kStatusBounds = 1, kStatusCapacity = 2, kStatusTimeout = 4 };

// Radial-basis and envelope parameters of the model.
struct Radial {
  int R;
  float gamma, mu_min, dmu, r_c;
};

// Filter-MLP weights of one block (device, fp32 values; bf16-rounded under MP_BF16).
struct FilterW {
  const float* A1;  // [R][F]
  const float* c1;  // [F]
  const float* A2;  // [F][F]
  const float* c2;  // [F]
};

// Kernel identities for launch counting and per-kernel timing.
enum KernelId : int {
  K_EMBED = 0, K_DENSE, K_READOUT_E, K_READOUT_BWD, K_GRAPH_SUM, K_CFCONV_FWD_SIMT,
  K_CFCONV_BWD_SIMT, K_ATTN_SIMT, K_VALIDATE, K_CFCONV_FWD_TC, K_CFCONV_BWD_TC, K_ATTN_TC,
  K_DENSE_TC, K_MD, K_ATTN_BWD, K_ATTN_BWD_SRC, K_ATTN_REV, K_ATTN_EQ,
  K_ATTN_BWD_TC, K_ATTN_BWD_SRC_TC, K_ATTN_EQ_TC, K_MD_CUT, K_PAIR_PLAN, K_CFCONV_PAIR_TC,
  K_PAIR_SUM, K_NUM
};
const char* kernel_name(int id);

// One tile of the undirected-pair cfconv (pairs.cu, tc_cfconv_pair.cu): 128 pair slots of the
// block pair (I, J) of 128-atom blocks, and how the kernel's accumulators m_I, m_J treat it.
enum : int {
  kPairAccI = 1,     // add to m_I (0: this tile starts a run of m_I)
  kPairAccJ = 2,     // add to m_J (0: this tile starts a run of m_J)
  kPairDiag = 4,     // I == J: both messages go to m_I
  kPairFlushI = 8,   // the run of m_I ends here: written to partial slotI
  kPairFlushJ = 16   // the run of m_J ends here: written to partial slotJ
};
struct PairTile {
  int I, J, count, flags, slotI, slotJ, pad0, pad1;
};
constexpr int kPairF = 128;  // features of the pair path (the tensor-core configuration)

// The plan of one symmetric neighbor list (pairs.cu); device arrays in one allocation.
struct PairPlan {
  bool valid = false;
  int N = 0, NB = 0, G = 0, T = 0, nslots = 0;
  long long E = 0;
  const int* list_row_ptr = nullptr;  // the list the plan was built from (mp_energy_forces uses
  const int* list_col_idx = nullptr;  // the pair forward for calls on these same buffers)
  void* ws = nullptr;      // per-block arrays (sized by E and the number of blocks)
  size_t ws_bytes = 0;
  void* tws = nullptr;     // the tiles (sized by their count)
  size_t tws_bytes = 0;
  float* part = nullptr;  // [nslots][128 rows][128 features] fp32 partial rows
  uint32_t* pmask = nullptr;  // [nslots][4]: the rows each partial block holds (the rest unset)
  size_t part_bytes = 0;
  int2* pairs = nullptr;  // per block, at pbase[R]: its upper pairs sorted by (J, i, j)
  int4* segs = nullptr;   // per block, at pbase[R]: (J, first pair, pairs, first local tile)
  int* low = nullptr;     // per block, at pbase[R]: the blocks J < R that hold neighbors
  int *pbase = nullptr, *nseg = nullptr, *ntile = nullptr, *nlow = nullptr, *toff = nullptr;
  int2* tpairs = nullptr; // [T][128] pair slots (i, j), (-1, -1) on padding
  PairTile* tiles = nullptr;
  int *sum_cnt = nullptr, *sum_ptr = nullptr, *sum_slots = nullptr;  // summing lists per block
  int* counts = nullptr;
};

}  // namespace mp

struct mp_ctx {
  mp_config cfg;
  int device = 0;
  int num_sms = 148;
  // weights (device, fp32; values bf16-rounded under MP_BF16)
  float* emb = nullptr;
  float *A1[MP_MAX_BLOCKS] = {}, *c1[MP_MAX_BLOCKS] = {}, *A2[MP_MAX_BLOCKS] = {},
        *c2[MP_MAX_BLOCKS] = {};
  float *W_in[MP_MAX_BLOCKS] = {}, *b_in[MP_MAX_BLOCKS] = {}, *W_out[MP_MAX_BLOCKS] = {},
        *b_out[MP_MAX_BLOCKS] = {};
  float *W_inT[MP_MAX_BLOCKS] = {}, *W_outT[MP_MAX_BLOCKS] = {};
  float *B1 = nullptr, *d1 = nullptr, *B2 = nullptr, *d2 = nullptr, *B1T = nullptr;
  float *Wq = nullptr, *Wk = nullptr, *P = nullptr, *p = nullptr;
  // packed 16-bit operand images for the tensor-core kernels (see tc_*.cu)
  void* tc_weights = nullptr;
  size_t tc_weights_bytes = 0;
  uint8_t* tc_dense_img = nullptr;        // packed bf16 atomwise weights (tc_dense.cu)
  bool tc_qk = false;                     // tc_dense_img also holds the attention's Wq, Wk
  uint8_t* tc_attn_p = nullptr;           // attention: [16 heads][K1] bf16 P^T with p on column R
  // workspace, sized from max_atoms
  float* x_res = nullptr;                 // [N][F] fp32 residual stream
  void* h[MP_MAX_BLOCKS] = {};            // [N][F] storage dtype: block inputs to the cfconv
  void* m = nullptr;                      // [N][F] storage dtype: cfconv output
  float* a = nullptr;                     // [N][F/2] readout pre-activation
  float* u_ro = nullptr;                  // [N][F/2] readout backward
  float* e_atom = nullptr;                // [N]
  float* gsum_part = nullptr;             // per-graph energy partials: N / 1024 + max_graphs
  float* g_x = nullptr;                   // [N][F] dE/dx
  void* g_m = nullptr;                    // [N][F] storage dtype: dE/dm
  float* grad_h = nullptr;                // [N][F] dE/dh
  float* q = nullptr;                     // [N][F] attention queries
  float* k = nullptr;                     // [N][F] attention keys
  float* md_ref = nullptr;                // [N][3] positions at the last neighbor-list build
  float* attn_stats = nullptr;            // [N][3H] attention backward: row max, sum, g . out
  float *WqT = nullptr, *WkT = nullptr;   // [F][F] transposed attention projections
  int* status_d = nullptr;                // device status bits (then the MD displacement flag)
  int* status_h = nullptr;                // pinned host copy
  int* md_flag = nullptr;                 // status_d + 1: an atom moved past the rebuild limit
  int* md_flag_h = nullptr;               // status_h + 1
  long long launches = 0;
  // budget of every bounded device wait in the tensor-core kernels (ns of global time)
  unsigned long long wait_ns = 2000000000ull;
  // CUDA graph of the last energy/forces call, replayed when a call repeats its arguments
  bool graphs = true, graphs_broken = false;
  cudaGraphExec_t ef_graph = nullptr;
  long long ef_launches = 0;
  struct EfKey {
    int N, n_graphs;
    long long E;
    const void *pos, *types, *row_ptr, *col_idx, *graph_ptr;
    void *energy, *forces, *stream;
  } ef_key{};
  // undirected-pair plan of the last list given to mp_pair_plan
  mp::PairPlan pair;
  // profiling
  bool profiling = false;
  std::vector<cudaEvent_t> ev_pool;
  std::vector<int> rec_kernel;            // kernel id per recorded pair
  size_t rec_used = 0;
  double prof_ms[mp::K_NUM] = {};
  long long prof_n[mp::K_NUM] = {};
  std::vector<int> prof_order;            // kernels seen, in first-seen order
};

namespace mp {

// Launch a kernel, counting it and (when profiling) bracketing it with an event pair.
template <typename Kern, typename... Args>
inline int launch(mp_ctx* ctx, int kid, Kern kernel, dim3 grid, dim3 block, size_t smem,
                  cudaStream_t s, Args... args) {
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  if (ctx && ctx->profiling && ctx->rec_used + 2 <= ctx->ev_pool.size()) {
    e0 = ctx->ev_pool[ctx->rec_used];
    e1 = ctx->ev_pool[ctx->rec_used + 1];
    ctx->rec_used += 2;
    ctx->rec_kernel.push_back(kid);
    cudaEventRecord(e0, s);
  }
  kernel<<<grid, block, smem, s>>>(args...);
  cudaError_t err = cudaGetLastError();
  if (e1) cudaEventRecord(e1, s);
  if (ctx) ctx->launches++;
  return err == cudaSuccess ? MP_OK : MP_ERR_CUDA;
}

// ---------------------------------------------------------------------------------------------
// Device helpers shared by the kernels.
template <typename T>
__device__ __forceinline__ float ldf(const T* p);
template <>
__device__ __forceinline__ float ldf<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename T>
__device__ __forceinline__ void stf(T* p, float v);
template <>
__device__ __forceinline__ void stf<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void stf<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

// Shifted softplus ln(e^x/2 + 1/2) = max(x,0) + ln(1 + e^-|x|) - ln 2.
__device__ __forceinline__ float ssp_f(float x) {
  return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))) - 0.693147180559945309f;
}
__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + expf(-x)); }

// Cosine envelope and its derivative; exactly 0 at and beyond the cutoff.
__device__ __forceinline__ float cutoff_f(float d, float rc) {
  return d < rc ? 0.5f * (cospif(d / rc) + 1.f) : 0.f;
}
__device__ __forceinline__ float cutoff_grad_f(float d, float rc) {
  return d < rc ? -0.5f * 3.14159265358979f / rc * sinpif(d / rc) : 0.f;
}

// The nine regular solid harmonics |r|^l Y_lm(r/|r|), l <= 2, of r = (x, y, z), Y the real
// spherical harmonics orthonormal on the sphere, in the order (0,0), (1,-1), (1,0), (1,1), (2,-2),
// (2,-1), (2,0), (2,1), (2,2) (E2Former-V2 page s.3.1: the geometry of the value path).
__device__ __forceinline__ void solid_harmonics9(float x, float y, float z, float* S) {
  const float c0 = 0.28209479177387814f;   // 1 / (2 sqrt(pi))
  const float c1 = 0.48860251190291992f;   // sqrt(3 / (4 pi))
  const float c2 = 1.09254843059207907f;   // sqrt(15 / pi) / 2
  const float c20 = 0.31539156525252005f;  // sqrt(5 / pi) / 4
  const float c22 = 0.54627421529603953f;  // sqrt(15 / pi) / 4
  S[0] = c0;
  S[1] = c1 * y;
  S[2] = c1 * z;
  S[3] = c1 * x;
  S[4] = c2 * x * y;
  S[5] = c2 * y * z;
  S[6] = c20 * (2.f * z * z - x * x - y * y);
  S[7] = c2 * x * z;
  S[8] = c22 * (x * x - y * y);
}

__device__ __forceinline__ void raise_status(int* status, int bit) {
  if (status) atomicOr(status, bit);
}

// Clamp a CSR offset read from device memory into [0, E].
__device__ __forceinline__ long long clamp_off(long long v, long long E) {
  return v < 0 ? 0 : (v > E ? E : v);
}

// ---------------------------------------------------------------------------------------------
// Host-side launchers implemented in the .cu files.
int launch_embed(mp_ctx*, int N, const int* types, cudaStream_t);
int launch_dense(mp_ctx*, int N, int Fin, int Fout, const void* in, bool in_bf16, const float* W,
                 const float* b, bool residual, void* out, bool out_bf16, cudaStream_t);
int launch_readout(mp_ctx*, int N, cudaStream_t);
int launch_readout_bwd(mp_ctx*, int N, cudaStream_t);
int launch_graph_sum(mp_ctx*, int N, const int* graph_ptr, int n_graphs, float* energy,
                     cudaStream_t);
int launch_cfconv_fwd_simt(mp_ctx*, int block, int N, long long E, const float* pos,
                           const int* row_ptr, const int* col_idx, const void* x, void* out,
                           cudaStream_t);
int launch_cfconv_bwd_simt(mp_ctx*, int block, int N, long long E, const float* pos,
                           const int* row_ptr, const int* col_idx, const void* h, const void* g,
                           float* grad_h, float* forces, bool accumulate, cudaStream_t);
int launch_attn_simt(mp_ctx*, int N, int K, const float* pos, const int* nbr,
                     const unsigned char* mask, const void* x, void* out, cudaStream_t);
int launch_validate_csr(mp_ctx*, int N, long long E, const int* row_ptr, const int* col_idx,
                        const int* graph_ptr, int n_graphs, bool need_sym, cudaStream_t);
// Stream-ordered scratch of the context-free calls (neighbor lists, the attention backward's
// transposed list) from a memory pool of the library's own per device that keeps its memory
// between calls (the default pool returns memory at each synchronisation, and mapping it again
// costs more than the kernels it serves). The pool holds at most the largest scratch used.
cudaError_t scratch_alloc(void** p, size_t bytes, cudaStream_t s);
void scratch_free(void* p, cudaStream_t s);
// In place on the stream: a[1..n] counts -> a[0..n] prefix sums (a[0] = 0); *overflow = 1 when the
// total passes INT_MAX. bsum: scan_blocks(n) (at least 1) long longs of scratch (neighbors.cu).
int scan_blocks(long long n);
void launch_scan(long long n, int* a, long long* bsum, int* overflow, cudaStream_t s);
// The kernel sequence of one energy + forces evaluation (mp_api.cu), without validation or graphs.
int energy_forces_launches(mp_ctx*, int N, long long E, const float* pos, const int* types,
                           const int* row_ptr, const int* col_idx, const int* graph_ptr,
                           int n_graphs, float* energy, float* forces, cudaStream_t);

// Undirected-pair cfconv (pairs.cu, tc_cfconv_pair.cu): build the plan of a symmetric list
// (synchronises the stream), the pair kernel, and the fixed-order sum of its partial rows.
int pair_plan_build(mp_ctx*, int N, long long E, const int* row_ptr, const int* col_idx,
                    cudaStream_t);
int pair_sum_launch(mp_ctx*, int N, void* out, cudaStream_t);
int tc_cfconv_fwd_pairs(mp_ctx*, int block, int N, const float* pos, const void* x, void* out,
                        cudaStream_t);
void pair_plan_free(mp_ctx*);
inline size_t align_up_sz(size_t v) { return (v + 255) / 256 * 256; }

FilterW filter_of(const mp_ctx* ctx, int block);
Radial radial_of(const mp_ctx* ctx);

}  // namespace mp
