// mp_attn_fwd_noalloc: the neighbor attention aggregation for callers that cannot allocate device
// memory. It runs the same kernels as mp_attn_fwd (fp32 path) but needs no context: the caller passes
// the configuration, device pointers to the fp32 weights, the inputs and the output, and the query and
// key rows the attention kernel reads live in a fixed-size file-scope device array instead of a
// cudaMalloc'd workspace. Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <mutex>

#include "mp_internal.cuh"

namespace mp {
namespace {

// Layout of the array: [0, 256) status word (device status bits), then q [N][F], then k [N][F].
constexpr size_t kHeaderBytes = 256;
constexpr size_t kScratchBytes = kHeaderBytes + 2 * (size_t)MP_NOALLOC_MAX_NF * sizeof(float);

// One copy per device that loads the library, kept until the process exits.
static __device__ __align__(256) unsigned char g_mp_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_addr[kMaxDevices] = {};

// The array's device address on the current device (host code may not use the symbol itself: on
// the host it names a stand-in, not device memory). Looked up once per device.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MP_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MP_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_mp_noalloc_scratch) != cudaSuccess || !p) return MP_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MP_OK;
}

bool config_ok(const mp_config* c) {
  return c && (c->F == 64 || c->F == 128) && c->n_rbf >= 2 && c->n_rbf <= kMaxR &&
         c->n_heads >= 1 && c->head_dim >= 1 && c->n_heads * c->head_dim == c->F &&
         c->head_dim <= 32 && (c->head_dim & (c->head_dim - 1)) == 0 && c->r_c > 0.f &&
         c->gamma > 0.f && c->mu_max >= c->mu_min && c->dtype == MP_FP32;
}

}  // namespace
}  // namespace mp

using namespace mp;

extern "C" int mp_attn_fwd_noalloc(const mp_config* cfg, const mp_weights* w, int N, int K,
                                   const float* pos, const int* nbr, const unsigned char* mask,
                                   const float* x, float* out, int* status, void* stream) {
  if (!config_ok(cfg) || !w || !w->on_device || !w->Wq || !w->Wk || !w->P || !w->p ||
      !w->A1[0] || !w->c1[0] || !w->A2[0] || !w->c2[0] || N < 0 || K < 1 ||
      (N > 0 && (!pos || !nbr || !mask || !x || !out)) || (x && (const void*)x == (void*)out))
    return MP_ERR_INVALID_ARG;
  if ((long long)N * cfg->F > MP_NOALLOC_MAX_NF) return MP_ERR_CAPACITY;
  cudaStream_t s = (cudaStream_t)stream;
  void* base = nullptr;
  int rc = scratch_address(&base);
  if (rc != MP_OK) return rc;
  int* status_word = (int*)base;
  float* q = (float*)((char*)base + kHeaderBytes);
  float* k = q + (size_t)N * cfg->F;

  // A context on the stack that only points at caller memory and the array (no allocation).
  mp_ctx tmp;
  tmp.cfg = *cfg;
  tmp.cfg.max_atoms = N;
  cudaGetDevice(&tmp.device);
  cudaDeviceGetAttribute(&tmp.num_sms, cudaDevAttrMultiProcessorCount, tmp.device);
  tmp.A1[0] = const_cast<float*>(w->A1[0]);
  tmp.c1[0] = const_cast<float*>(w->c1[0]);
  tmp.A2[0] = const_cast<float*>(w->A2[0]);
  tmp.c2[0] = const_cast<float*>(w->c2[0]);
  tmp.Wq = const_cast<float*>(w->Wq);
  tmp.Wk = const_cast<float*>(w->Wk);
  tmp.P = const_cast<float*>(w->P);
  tmp.p = const_cast<float*>(w->p);
  tmp.q = q;
  tmp.k = k;
  tmp.status_d = status_word;

  // the status word keeps the previous call's bits: it must start at zero
  if (cudaMemsetAsync(status_word, 0, sizeof(int), s) != cudaSuccess) return MP_ERR_CUDA;
  if (N > 0) {
    const int F = cfg->F;
    rc = launch_dense(&tmp, N, F, F, x, false, tmp.Wq, nullptr, false, q, false, s);
    if (rc == MP_OK) rc = launch_dense(&tmp, N, F, F, x, false, tmp.Wk, nullptr, false, k, false, s);
    if (rc == MP_OK) rc = launch_attn_simt(&tmp, N, K, pos, nbr, mask, x, out, s);
    if (rc != MP_OK) return rc;
  }
  if (status &&
      cudaMemcpyAsync(status, status_word, sizeof(int), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return MP_ERR_CUDA;
  return MP_OK;
}
