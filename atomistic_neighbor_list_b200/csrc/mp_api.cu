// C-ABI entry points of libmp (declared in include/mp.h): context creation, argument checks, the
// energy/forces pipeline, and kernel timing. All numerical work happens in the kernels of simt.cu,
// tc_cfconv.cu and neighbors.cu; this file only validates, orders launches and owns memory.
#include <cmath>
#include <cstring>
#include <vector>

#include "mp_internal.cuh"
#include "tc_api.cuh"

namespace mp {

const char* kernel_name(int id) {
  static const char* names[K_NUM] = {
      "embed", "dense", "readout_energy", "readout_bwd", "graph_energy_sum", "cfconv_fwd_simt",
      "cfconv_bwd_simt", "attn_simt", "validate_csr", "cfconv_fwd_tc", "cfconv_bwd_tc",
      "attn_tc", "dense_tc", "md_integrate", "attn_bwd_dst", "attn_bwd_src",
      "attn_transpose", "attn_eq_simt", "attn_bwd_dst_tc",
      "attn_bwd_src_tc", "attn_eq_tc", "md_cutoff_list", "pair_plan", "cfconv_pair_tc",
      "pair_sum"};
  return (id >= 0 && id < K_NUM) ? names[id] : "?";
}

// Round a float to the nearest bfloat16 value (ties to even), returned as float.
static float round_bf16_host(float v) {
  if (std::isnan(v)) return v;
  uint32_t u;
  std::memcpy(&u, &v, 4);
  u = (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;
  float r;
  std::memcpy(&r, &u, 4);
  return r;
}

}  // namespace mp

using namespace mp;

extern "C" const char* mp_strerror(int s) {
  switch (s) {
    case MP_OK: return "ok";
    case MP_ERR_INVALID_ARG: return "invalid argument";
    case MP_ERR_BAD_CSR: return "malformed CSR neighbor list";
    case MP_ERR_CSR_UNSORTED: return "CSR row not strictly ascending or has a self edge";
    case MP_ERR_CSR_NOT_SYMMETRIC: return "CSR neighbor list is not symmetric";
    case MP_ERR_CAPACITY: return "size exceeds the context or output capacity";
    case MP_ERR_CUDA: return "CUDA error";
    case MP_ERR_DEVICE_BOUNDS: return "a kernel met an out-of-range index";
    case MP_ERR_TIMEOUT: return "a bounded device wait ran out";
    case MP_ERR_UNIMPLEMENTED: return "not implemented";
    default: return "unknown status";
  }
}

namespace {

struct HostWeights {
  std::vector<float> data;
  std::vector<size_t> off;
};

// Fetch n floats from a host or device pointer.
bool fetch(const float* src, size_t n, bool on_device, std::vector<float>& out) {
  out.resize(n);
  if (n == 0) return true;
  if (on_device)
    return cudaMemcpy(out.data(), src, n * sizeof(float), cudaMemcpyDeviceToHost) == cudaSuccess;
  std::memcpy(out.data(), src, n * sizeof(float));
  return true;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool cfg_ok(const mp_config* c) {
  if (!c) return false;
  if (c->F != 64 && c->F != 128) return false;
  if (c->n_rbf < 2 || c->n_rbf > kMaxR) return false;
  if (c->n_blocks < 1 || c->n_blocks > MP_MAX_BLOCKS) return false;
  if (c->n_types < 1) return false;
  if (c->n_heads < 0 || c->head_dim < 0) return false;
  if (c->n_heads > 0 && (c->n_heads * c->head_dim != c->F || c->head_dim > 32 ||
                         (c->head_dim & (c->head_dim - 1)) != 0))
    return false;
  if (!(c->r_c > 0.f) || !(c->gamma > 0.f) || !(c->mu_max >= c->mu_min)) return false;
  if (c->dtype != MP_FP32 && c->dtype != MP_BF16) return false;
  if (c->max_atoms < 0 || c->max_edges < 0 || c->max_graphs < 1) return false;
  return true;
}

void free_ctx(mp_ctx* c) {
  if (!c) return;
  cudaDeviceSynchronize();
  cudaFree(c->emb);  // one allocation holds every weight array
  cudaFree(c->tc_weights);
  cudaFree(c->tc_dense_img);
  cudaFree(c->tc_attn_p);
  if (c->ef_graph) cudaGraphExecDestroy(c->ef_graph);
  pair_plan_free(c);
  cudaFree(c->x_res);  // one allocation holds the whole workspace
  cudaFree(c->status_d);
  if (c->status_h) cudaFreeHost(c->status_h);
  for (auto e : c->ev_pool) cudaEventDestroy(e);
  delete c;
}

}  // namespace

extern "C" int mp_init(mp_ctx** out_ctx, const mp_config* cfg, const mp_weights* w, void* stream) {
  if (!out_ctx || !cfg_ok(cfg) || !w) return MP_ERR_INVALID_ARG;
  *out_ctx = nullptr;
  cudaStream_t s = (cudaStream_t)stream;
  mp_ctx* c = new mp_ctx();
  c->cfg = *cfg;
  cudaGetDevice(&c->device);
  cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device);
  const int F = cfg->F, R = cfg->n_rbf, B = cfg->n_blocks, Fh = F / 2, H = cfg->n_heads;
  const bool bf = cfg->dtype == MP_BF16;
  const bool dev = w->on_device != 0;

  // ---- gather every weight on the host, round under bf16, derive the transposes
  struct Item {
    const float* src;
    size_t n;
    float** dst;
  };
  std::vector<Item> items;
  items.push_back({w->emb, (size_t)cfg->n_types * F, &c->emb});
  for (int b = 0; b < B; ++b) {
    items.push_back({w->A1[b], (size_t)R * F, &c->A1[b]});
    items.push_back({w->c1[b], (size_t)F, &c->c1[b]});
    items.push_back({w->A2[b], (size_t)F * F, &c->A2[b]});
    items.push_back({w->c2[b], (size_t)F, &c->c2[b]});
    items.push_back({w->W_in[b], (size_t)F * F, &c->W_in[b]});
    items.push_back({w->b_in[b], (size_t)F, &c->b_in[b]});
    items.push_back({w->W_out[b], (size_t)F * F, &c->W_out[b]});
    items.push_back({w->b_out[b], (size_t)F, &c->b_out[b]});
  }
  items.push_back({w->B1, (size_t)F * Fh, &c->B1});
  items.push_back({w->d1, (size_t)Fh, &c->d1});
  items.push_back({w->B2, (size_t)Fh, &c->B2});
  items.push_back({w->d2, (size_t)1, &c->d2});
  if (H > 0) {
    items.push_back({w->Wq, (size_t)F * F, &c->Wq});
    items.push_back({w->Wk, (size_t)F * F, &c->Wk});
    items.push_back({w->P, (size_t)R * H, &c->P});
    items.push_back({w->p, (size_t)H, &c->p});
  }
  std::vector<std::vector<float>> host(items.size());
  for (size_t i = 0; i < items.size(); ++i) {
    if (!items[i].src) {
      host[i].assign(items[i].n, 0.f);  // absent weights: zeros (the calls needing them check)
      continue;
    }
    if (!fetch(items[i].src, items[i].n, dev, host[i])) {
      free_ctx(c);
      return MP_ERR_CUDA;
    }
    if (bf)
      for (auto& v : host[i]) v = round_bf16_host(v);
  }
  // transposed copies used by the backward dense layers
  auto transpose = [](const std::vector<float>& a, int rows, int cols) {
    std::vector<float> t((size_t)rows * cols);
    for (int r = 0; r < rows; ++r)
      for (int q = 0; q < cols; ++q) t[(size_t)q * rows + r] = a[(size_t)r * cols + q];
    return t;
  };
  std::vector<std::vector<float>> extra;
  std::vector<float**> extra_dst;
  for (int b = 0; b < B; ++b) {
    const size_t base = 1 + (size_t)b * 8;
    extra.push_back(transpose(host[base + 4], F, F));
    extra_dst.push_back(&c->W_inT[b]);
    extra.push_back(transpose(host[base + 6], F, F));
    extra_dst.push_back(&c->W_outT[b]);
  }
  extra.push_back(transpose(host[1 + (size_t)B * 8], F, Fh));
  extra_dst.push_back(&c->B1T);
  if (H > 0) {  // the attention backward's dL/dx = dL/dq Wq^T + dL/dk Wk^T
    const size_t qi = 1 + (size_t)B * 8 + 4;
    extra.push_back(transpose(host[qi], F, F));
    extra_dst.push_back(&c->WqT);
    extra.push_back(transpose(host[qi + 1], F, F));
    extra_dst.push_back(&c->WkT);
  }

  size_t total = 0;
  for (auto& h : host) total += align_up(h.size() * sizeof(float), 256);
  for (auto& h : extra) total += align_up(h.size() * sizeof(float), 256);
  char* wbuf = nullptr;
  if (cudaMalloc(&wbuf, total) != cudaSuccess) {
    free_ctx(c);
    return MP_ERR_CUDA;
  }
  c->emb = (float*)wbuf;  // first item; the buffer is freed through this pointer
  size_t off = 0;
  for (size_t i = 0; i < items.size(); ++i) {
    *items[i].dst = (float*)(wbuf + off);
    cudaMemcpyAsync(wbuf + off, host[i].data(), host[i].size() * sizeof(float),
                    cudaMemcpyHostToDevice, s);
    off += align_up(host[i].size() * sizeof(float), 256);
  }
  for (size_t i = 0; i < extra.size(); ++i) {
    *extra_dst[i] = (float*)(wbuf + off);
    cudaMemcpyAsync(wbuf + off, extra[i].data(), extra[i].size() * sizeof(float),
                    cudaMemcpyHostToDevice, s);
    off += align_up(extra[i].size() * sizeof(float), 256);
  }

  // ---- workspace, O(max_atoms * F * n_blocks)
  const size_t N = (size_t)(cfg->max_atoms > 0 ? cfg->max_atoms : 1);
  const size_t st = bf ? 2 : 4;
  const size_t nf = N * F;
  size_t sizes[] = {nf * 4,            // x_res
                    nf * st * B,       // h[0..B)
                    nf * st,           // m
                    N * Fh * 4,        // a
                    N * Fh * 4,        // u_ro
                    N * 4,             // e_atom
                    nf * 4,            // g_x
                    nf * st,           // g_m
                    nf * 4,            // grad_h
                    nf * 4, nf * 4,    // q, k
                    N * 3 * 4,         // md_ref
                    N * 3 * (size_t)(H > 0 ? H : 1) * 4,   // attn_stats
                    (N / 1024 + (size_t)cfg->max_graphs + 8) * 4};  // gsum_part
  size_t ws = 0;
  for (size_t v : sizes) ws += align_up(v, 256);
  char* wsb = nullptr;
  if (cudaMalloc(&wsb, ws) != cudaSuccess) {
    free_ctx(c);
    return MP_ERR_CUDA;
  }
  size_t o = 0;
  auto take = [&](size_t bytes) {
    char* p = wsb + o;
    o += align_up(bytes, 256);
    return (void*)p;
  };
  c->x_res = (float*)take(sizes[0]);
  char* hb = (char*)take(sizes[1]);
  for (int b = 0; b < B; ++b) c->h[b] = hb + (size_t)b * nf * st;
  c->m = take(sizes[2]);
  c->a = (float*)take(sizes[3]);
  c->u_ro = (float*)take(sizes[4]);
  c->e_atom = (float*)take(sizes[5]);
  c->g_x = (float*)take(sizes[6]);
  c->g_m = take(sizes[7]);
  c->grad_h = (float*)take(sizes[8]);
  c->q = (float*)take(sizes[9]);
  c->k = (float*)take(sizes[10]);
  c->md_ref = (float*)take(sizes[11]);
  c->attn_stats = (float*)take(sizes[12]);
  c->gsum_part = (float*)take(sizes[13]);
  if (cudaMalloc(&c->status_d, 4 * sizeof(int)) != cudaSuccess ||
      cudaMallocHost(&c->status_h, 4 * sizeof(int)) != cudaSuccess) {
    free_ctx(c);
    return MP_ERR_CUDA;
  }
  c->md_flag = c->status_d + 1;
  c->md_flag_h = c->status_h + 1;
  cudaMemsetAsync(c->status_d, 0, 4 * sizeof(int), s);
  int rc = tc_prepare(c, s);  // packed operand images for the tensor-core kernels
  if (rc != MP_OK || cudaStreamSynchronize(s) != cudaSuccess) {
    free_ctx(c);
    return rc != MP_OK ? rc : MP_ERR_CUDA;
  }
  *out_ctx = c;
  return MP_OK;
}

extern "C" void mp_destroy(mp_ctx* c) { free_ctx(c); }

extern "C" int mp_status_sync(mp_ctx* c, void* stream) {
  if (!c) return MP_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  cudaMemcpyAsync(c->status_h, c->status_d, sizeof(int), cudaMemcpyDeviceToHost, s);
  cudaMemsetAsync(c->status_d, 0, sizeof(int), s);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MP_ERR_CUDA;
  const int bits = *c->status_h;
  if (bits & kStatusBounds) return MP_ERR_DEVICE_BOUNDS;
  if (bits & kStatusCapacity) return MP_ERR_CAPACITY;
  if (bits & kStatusTimeout) return MP_ERR_TIMEOUT;
  return MP_OK;
}

extern "C" long long mp_launch_count(mp_ctx* c) { return c ? c->launches : -1; }

extern "C" int mp_set_wait_budget(mp_ctx* c, long long ns) {
  if (!c || ns < 0) return MP_ERR_INVALID_ARG;
  c->wait_ns = (unsigned long long)ns;
  if (c->ef_graph) {  // the budget is a kernel argument: a recorded graph holds the old one
    cudaGraphExecDestroy(c->ef_graph);
    c->ef_graph = nullptr;
  }
  return MP_OK;
}

extern "C" int mp_shard_graphs(const int* graph_ptr, int n_graphs, int rank, int world, int* g0,
                               int* g1) {
  if (!graph_ptr || n_graphs < 1 || world < 1 || rank < 0 || rank >= world || !g0 || !g1)
    return MP_ERR_INVALID_ARG;
  for (int g = 0; g < n_graphs; ++g)
    if (graph_ptr[g + 1] < graph_ptr[g]) return MP_ERR_INVALID_ARG;
  const long long a_begin = graph_ptr[0], total = (long long)graph_ptr[n_graphs] - a_begin;
  // boundary k: the graph start nearest to the atom target a_begin + total k / world (the later
  // one on a tie); nondecreasing in k, since the starts are
  auto bound = [&](int k) {
    if (k <= 0) return 0;
    if (k >= world) return n_graphs;
    const long long target = a_begin + total * k / world;
    int lo = 0, hi = n_graphs;  // first start at or after the target (graph_ptr[n_graphs] is)
    while (lo < hi) {
      const int mid = (lo + hi) / 2;
      if ((long long)graph_ptr[mid] < target) lo = mid + 1; else hi = mid;
    }
    if (lo > 0 && target - graph_ptr[lo - 1] < (long long)graph_ptr[lo] - target) --lo;
    return lo;
  };
  *g0 = bound(rank);
  *g1 = bound(rank + 1);
  return MP_OK;
}

// ---------------------------------------------------------------------------------------------
extern "C" int mp_cfconv_fwd(mp_ctx* c, int block, int N, long long E, const float* pos,
                             const int* row_ptr, const int* col_idx, const void* x, void* out,
                             void* stream) {
  if (!c || block < 0 || block >= c->cfg.n_blocks || N < 0 || E < 0 || !row_ptr ||
      (N > 0 && (!pos || !x || !out)) || (E > 0 && !col_idx) || (x && x == out) ||
      ((uintptr_t)x & 15) != 0 || ((uintptr_t)out & 15) != 0)
    return MP_ERR_INVALID_ARG;
  if (N > c->cfg.max_atoms || E > c->cfg.max_edges) return MP_ERR_CAPACITY;
  cudaStream_t s = (cudaStream_t)stream;
  if (c->cfg.validate) {
    int rc = launch_validate_csr(c, N, E, row_ptr, col_idx, nullptr, 1, false, s);
    if (rc != MP_OK) return rc;
  }
  if (N == 0) return MP_OK;
  if (tc_supported(c)) return tc_cfconv_fwd(c, block, N, E, pos, row_ptr, col_idx, x, out, s);
  return launch_cfconv_fwd_simt(c, block, N, E, pos, row_ptr, col_idx, x, out, s);
}

extern "C" int mp_pair_plan(mp_ctx* c, int N, long long E, const int* row_ptr,
                            const int* col_idx, void* stream) {
  if (!c || N < 0 || E < 0 || !row_ptr || (E > 0 && !col_idx)) return MP_ERR_INVALID_ARG;
  if (N > c->cfg.max_atoms || E > c->cfg.max_edges) return MP_ERR_CAPACITY;
  cudaStream_t s = (cudaStream_t)stream;
  if (c->cfg.validate) {
    int rc = launch_validate_csr(c, N, E, row_ptr, col_idx, nullptr, 1, true, s);
    if (rc != MP_OK) return rc;
  }
  return pair_plan_build(c, N, E, row_ptr, col_idx, s);
}

extern "C" int mp_cfconv_fwd_pairs(mp_ctx* c, int block, int N, const float* pos, const void* x,
                                   void* out, void* stream) {
  if (!c || block < 0 || block >= c->cfg.n_blocks || N < 0 ||
      (N > 0 && (!pos || !x || !out)) || (x && x == out) || ((uintptr_t)x & 15) != 0 ||
      ((uintptr_t)out & 15) != 0)
    return MP_ERR_INVALID_ARG;
  if (!tc_supported(c)) return MP_ERR_UNIMPLEMENTED;
  if (!c->pair.valid || c->pair.N != N) return MP_ERR_INVALID_ARG;
  if (N == 0) return MP_OK;
  return tc_cfconv_fwd_pairs(c, block, N, pos, x, out, (cudaStream_t)stream);
}

extern "C" int mp_attn_fwd(mp_ctx* c, int N, int K, const float* pos, const int* nbr,
                           const unsigned char* mask, const void* x, void* out, void* stream) {
  if (!c || N < 0 || K < 1 || c->cfg.n_heads < 1 ||
      (N > 0 && (!pos || !nbr || !mask || !x || !out)) || (x && x == out))
    return MP_ERR_INVALID_ARG;
  if (N > c->cfg.max_atoms) return MP_ERR_CAPACITY;
  if (N == 0) return MP_OK;
  cudaStream_t s = (cudaStream_t)stream;
  const bool tc = tc_attn_supported(c, K) && ((uintptr_t)x & 15) == 0;
  int rc = attn_project(c, N, x, s, tc);
  if (rc != MP_OK) return rc;
  if (tc) return tc_attn_fwd(c, N, K, pos, nbr, mask, x, out, s);
  return launch_attn_simt(c, N, K, pos, nbr, mask, x, out, s);
}

// The launches of one energy + forces evaluation (arguments already checked).
int mp::energy_forces_launches(mp_ctx* c, int N, long long E, const float* pos, const int* types,
                                  const int* row_ptr, const int* col_idx, const int* graph_ptr,
                                  int n_graphs, float* energy, float* forces, cudaStream_t s) {
  const int F = c->cfg.F, Fh = F / 2, B = c->cfg.n_blocks;
  const bool bf = c->cfg.dtype == MP_BF16;
  const bool tc = tc_supported(c), tc_bwd = tc_bwd_supported(c);
  int rc = MP_OK;
#define MP_TRY(x)             \
  do {                        \
    rc = (x);                 \
    if (rc != MP_OK) return rc; \
  } while (0)
  if (tc && tc_bwd && N > 0) {
    // bf16 path: every atomwise layer and both cfconv passes on the tensor cores
    // consecutive atomwise layers that depend only on the row run as one launch (tc_dense2)
    auto img = [&](int kind, int b) { return c->tc_dense_img + tc_dense_off(kind, b, B); };
    // the forward cfconv over undirected pairs when the context holds a plan of this very list
    // (mp_pair_plan on these buffers; the caller builds it again whenever the list changes)
    const PairPlan& P = c->pair;
    const bool pairs = P.valid && P.N == N && P.E == E && P.list_row_ptr == row_ptr &&
                       P.list_col_idx == col_idx && P.G == c->num_sms;
    MP_TRY(launch_embed(c, N, types, s));
    MP_TRY(tc_dense(c, N, F, F, c->x_res, false, img(0, 0), c->b_in[0], c->h[0], true,
                    TC_DENSE_STORE, s));
    for (int b = 0; b < B; ++b) {
      MP_TRY(pairs ? tc_cfconv_fwd_pairs(c, b, N, pos, c->h[b], c->m, s)
                   : tc_cfconv_fwd(c, b, N, E, pos, row_ptr, col_idx, c->h[b], c->m, s));
      if (b + 1 < B)  // x += m W_out + b_out, then h of the next block = x W_in + b_in
        MP_TRY(tc_dense2(c, N, F, c->m, true, img(1, b), c->b_out[b], c->x_res, TC_DENSE_RESIDUAL,
                         img(0, b + 1), c->b_in[b + 1], F, c->h[b + 1], TC_DENSE_STORE, s));
      else  // the last residual, then the readout: pre-activation, atomic energies and dE/da
        MP_TRY(tc_dense2(c, N, F, c->m, true, img(1, b), c->b_out[b], c->x_res, TC_DENSE_RESIDUAL,
                         img(4, 0), c->d1, Fh, c->u_ro, TC_DENSE_READOUT, s));
    }
    MP_TRY(launch_graph_sum(c, N, graph_ptr, n_graphs, energy, s));
    // dE/dx = u B1^T, then g_m of the last block = dE/dx W_out^T
    MP_TRY(tc_dense2(c, N, Fh, c->u_ro, false, img(5, 0), nullptr, c->g_x, TC_DENSE_STORE,
                     img(2, B - 1), nullptr, F, c->g_m, TC_DENSE_STORE, s));
    for (int b = B - 1; b >= 0; --b) {
      MP_TRY(tc_cfconv_bwd(c, b, N, E, pos, row_ptr, col_idx, c->h[b], c->g_m, c->grad_h, forces,
                           b != B - 1, s));
      if (b > 0)  // dE/dx += grad_h W_in^T, then g_m of the block before = dE/dx W_out^T
        MP_TRY(tc_dense2(c, N, F, c->grad_h, false, img(3, b), nullptr, c->g_x, TC_DENSE_RESIDUAL,
                         img(2, b - 1), nullptr, F, c->g_m, TC_DENSE_STORE, s));
    }
    return MP_OK;
  }
  if (N > 0) {
    MP_TRY(launch_embed(c, N, types, s));
    for (int b = 0; b < B; ++b) {
      MP_TRY(launch_dense(c, N, F, F, c->x_res, false, c->W_in[b], c->b_in[b], false, c->h[b], bf,
                          s));
      if (tc)
        MP_TRY(tc_cfconv_fwd(c, b, N, E, pos, row_ptr, col_idx, c->h[b], c->m, s));
      else
        MP_TRY(launch_cfconv_fwd_simt(c, b, N, E, pos, row_ptr, col_idx, c->h[b], c->m, s));
      MP_TRY(launch_dense(c, N, F, F, c->m, bf, c->W_out[b], c->b_out[b], true, c->x_res, false,
                          s));
    }
    MP_TRY(launch_dense(c, N, F, Fh, c->x_res, false, c->B1, c->d1, false, c->a, false, s));
    MP_TRY(launch_readout(c, N, s));
  }
  MP_TRY(launch_graph_sum(c, N, graph_ptr, n_graphs, energy, s));
  if (N == 0) return MP_OK;
  // backward: dE/dx from the readout, then the blocks in reverse
  MP_TRY(launch_readout_bwd(c, N, s));
  MP_TRY(launch_dense(c, N, Fh, F, c->u_ro, false, c->B1T, nullptr, false, c->g_x, false, s));
  for (int b = B - 1; b >= 0; --b) {
    MP_TRY(launch_dense(c, N, F, F, c->g_x, false, c->W_outT[b], nullptr, false, c->g_m, bf, s));
    if (tc_bwd)
      MP_TRY(tc_cfconv_bwd(c, b, N, E, pos, row_ptr, col_idx, c->h[b], c->g_m, c->grad_h, forces,
                           b != B - 1, s));
    else
      MP_TRY(launch_cfconv_bwd_simt(c, b, N, E, pos, row_ptr, col_idx, c->h[b], c->g_m,
                                    c->grad_h, forces, b != B - 1, s));
    if (b > 0)
      MP_TRY(launch_dense(c, N, F, F, c->grad_h, false, c->W_inT[b], nullptr, true, c->g_x, false,
                          s));
  }
#undef MP_TRY
  return MP_OK;
}

extern "C" int mp_energy_forces(mp_ctx* c, int N, long long E, const float* pos, const int* types,
                                const int* row_ptr, const int* col_idx, const int* graph_ptr,
                                int n_graphs, float* energy, float* forces, void* stream) {
  if (!c || N < 0 || E < 0 || !row_ptr || !energy || n_graphs < 1 ||
      (N > 0 && (!pos || !types || !forces)) || (E > 0 && !col_idx) ||
      (!graph_ptr && n_graphs != 1))
    return MP_ERR_INVALID_ARG;
  if (N > c->cfg.max_atoms || E > c->cfg.max_edges || n_graphs > c->cfg.max_graphs)
    return MP_ERR_CAPACITY;
  cudaStream_t s = (cudaStream_t)stream;
  if (c->cfg.validate) {  // synchronises the stream to read its verdict: never captured
    int rc = launch_validate_csr(c, N, E, row_ptr, col_idx, graph_ptr, n_graphs, true, s);
    if (rc != MP_OK) return rc;
  }
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  const bool use_graph = c->graphs && !c->graphs_broken && !c->profiling && !c->cfg.validate &&
                         s != nullptr && cudaStreamIsCapturing(s, &cap) == cudaSuccess &&
                         cap == cudaStreamCaptureStatusNone;
  if (!use_graph)
    return energy_forces_launches(c, N, E, pos, types, row_ptr, col_idx, graph_ptr, n_graphs,
                                  energy, forces, s);
  mp_ctx::EfKey key;
  std::memset(&key, 0, sizeof key);  // padding included: the key is compared bytewise
  key.N = N;
  key.n_graphs = n_graphs;
  key.E = E;
  key.pos = pos;
  key.types = types;
  key.row_ptr = row_ptr;
  key.col_idx = col_idx;
  key.graph_ptr = graph_ptr;
  key.energy = energy;
  key.forces = forces;
  key.stream = stream;
  if (c->ef_graph && std::memcmp(&key, &c->ef_key, sizeof key) == 0) {  // a repeat: replay
    if (cudaGraphLaunch(c->ef_graph, s) != cudaSuccess) return MP_ERR_CUDA;
    c->launches += c->ef_launches;
    return MP_OK;
  }
  if (c->ef_graph) {
    cudaGraphExecDestroy(c->ef_graph);
    c->ef_graph = nullptr;
  }
  // capture the launches once; on any failure fall back to plain launches for good
  const long long l0 = c->launches;
  cudaGraph_t g = nullptr;
  int rc = cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal) == cudaSuccess ? MP_OK
                                                                                     : MP_ERR_CUDA;
  if (rc == MP_OK) {
    rc = energy_forces_launches(c, N, E, pos, types, row_ptr, col_idx, graph_ptr, n_graphs, energy,
                                forces, s);
    if (cudaStreamEndCapture(s, &g) != cudaSuccess && rc == MP_OK) rc = MP_ERR_CUDA;
  }
  cudaGraphExec_t ex = nullptr;
  if (rc == MP_OK && (!g || cudaGraphInstantiate(&ex, g, 0) != cudaSuccess)) rc = MP_ERR_CUDA;
  if (g) cudaGraphDestroy(g);
  const long long captured = c->launches - l0;  // kernels recorded into the graph (none ran)
  c->launches = l0;
  if (rc != MP_OK) {
    cudaGetLastError();  // clear a capture error
    c->graphs_broken = true;
    return energy_forces_launches(c, N, E, pos, types, row_ptr, col_idx, graph_ptr, n_graphs,
                                  energy, forces, s);
  }
  c->ef_graph = ex;
  c->ef_key = key;
  c->ef_launches = captured;
  if (cudaGraphLaunch(ex, s) != cudaSuccess) return MP_ERR_CUDA;
  c->launches += c->ef_launches;
  return MP_OK;
}

extern "C" int mp_set_graphs(mp_ctx* c, int on) {
  if (!c) return MP_ERR_INVALID_ARG;
  c->graphs = on != 0;
  if (!c->graphs && c->ef_graph) {
    cudaGraphExecDestroy(c->ef_graph);
    c->ef_graph = nullptr;
  }
  return MP_OK;
}

// ---------------------------------------------------------------------------------------------
extern "C" int mp_profile_begin(mp_ctx* c) {
  if (!c) return MP_ERR_INVALID_ARG;
  if (c->ev_pool.empty()) {
    c->ev_pool.resize(1 << 14);
    for (auto& e : c->ev_pool)
      if (cudaEventCreate(&e) != cudaSuccess) return MP_ERR_CUDA;
  }
  c->rec_used = 0;
  c->rec_kernel.clear();
  for (int i = 0; i < K_NUM; ++i) {
    c->prof_ms[i] = 0;
    c->prof_n[i] = 0;
  }
  c->prof_order.clear();
  c->profiling = true;
  return MP_OK;
}

extern "C" int mp_profile_end(mp_ctx* c, void* stream) {
  if (!c) return MP_ERR_INVALID_ARG;
  c->profiling = false;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MP_ERR_CUDA;
  for (size_t r = 0; r < c->rec_kernel.size(); ++r) {
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, c->ev_pool[2 * r], c->ev_pool[2 * r + 1]) != cudaSuccess)
      return MP_ERR_CUDA;
    const int k = c->rec_kernel[r];
    if (c->prof_n[k] == 0) c->prof_order.push_back(k);
    c->prof_ms[k] += ms;
    c->prof_n[k] += 1;
  }
  return MP_OK;
}

extern "C" int mp_profile_get(mp_ctx* c, int index, const char** name, double* total_ms,
                              long long* launches) {
  if (!c || index < 0 || index >= (int)c->prof_order.size()) return MP_ERR_INVALID_ARG;
  const int k = c->prof_order[index];
  if (name) *name = kernel_name(k);
  if (total_ms) *total_ms = c->prof_ms[k];
  if (launches) *launches = c->prof_n[k];
  return MP_OK;
}
