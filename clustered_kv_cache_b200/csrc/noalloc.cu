// Clustered-codec encode that needs no caller workspace.
//
// kvc_encode_layer with the clustered predictor needs a small device scratch
// (per-centre squared norms and the centres projected by the encoder) that the
// caller passes as `ws`.  Some callers cannot allocate device memory at the
// point where they encode: code running inside a custom allocator or memory
// pool callback, a runtime whose device memory is carved up in advance and
// handed out by someone else, or a plugin host that forbids cudaMalloc on its
// threads.  kvc_encode_layer_cluster_static keeps that scratch in a file-scope
// __device__ array instead, so it allocates nothing.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "simt.h"

namespace kvc {
namespace {

constexpr int kMaxCentres = 256;
constexpr int kCodeDim = 128;
// (norms + projected centres) for K, then the same for V
constexpr size_t kTableFloats = kMaxCentres + (size_t)kMaxCentres * kCodeDim;

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) float g_cluster_scratch[2 * kTableFloats];

// Set-up, once per device: the device address of g_cluster_scratch, looked up
// with that device current.  In host code the symbol's name is only a stand-in
// for that address.  The address belongs to the device's current context, so
// the cache also keeps that context's unique id and repeats the lookup when
// the id changes (after cudaDeviceReset the next call sees a new context).
constexpr int kMaxDevices = 64;
std::mutex g_mu;
struct ScratchSlot {
  float* ptr = nullptr;
  unsigned long long ctx_id = 0;
};
ScratchSlot g_slot[kMaxDevices];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 if unknown).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

cudaError_t scratch_for_current_device(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const unsigned long long id = current_context_id();  // 0 before the runtime has made a context current
  std::lock_guard<std::mutex> lock(g_mu);
  ScratchSlot& slot = g_slot[dev];
  if (!slot.ptr || id == 0 || slot.ctx_id != id) {
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_cluster_scratch)) != cudaSuccess) return e;
    slot.ptr = static_cast<float*>(p);
    slot.ctx_id = current_context_id();  // the lookup made the device's primary context current
  }
  *out = slot.ptr;
  return cudaSuccess;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <typename TS, typename TP>
cudaError_t encode(const kvc_layer_desc* d, const kvc_predictor* p, const void* K, const void* V, const kvc_codes* c,
                   void* Kr, void* Vr, float* scratch, cudaStream_t st) {
  const int C = d->n_heads * d->head_dim, m = p->code_dim, nc = p->n_clusters;
  cudaError_t e;
  for (int which = 0; which < 2; ++which) {
    float* cn = scratch + which * kTableFloats;  // fully rewritten by the prep kernel below
    float* P = cn + kMaxCentres;
    const TS* cent = (const TS*)(which ? p->v_centroids : p->k_centroids);
    const TS* encw = (const TS*)(which ? p->v_enc : p->k_enc);
    ClusterPrepArgs<TS> pa{nc, C, m, cent, encw, cn, P};
    if ((e = launch_cluster_prep(pa, st)) != cudaSuccess) return e;
    ClusterArgs<TS, TP> a{d->n_tokens, C, m, nc, d->bits, d->group, (const TS*)(which ? V : K), cent, encw,
                          (const TS*)(which ? p->v_dec : p->k_dec), cn, P,
                          (uint8_t*)(which ? c->v_codes : c->k_codes),
                          (Pair<TP>*)(which ? c->v_params : c->k_params),
                          (uint8_t*)(which ? c->v_assign : c->k_assign), (TS*)(which ? Vr : Kr)};
    if ((e = launch_cluster(a, true, st)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace
}  // namespace kvc

extern "C" kvc_status kvc_encode_layer_cluster_static(const kvc_layer_desc* d, const kvc_predictor* p, const void* K,
                                                      const void* V, const kvc_codes* c, void* K_rec, void* V_rec,
                                                      void* stream) {
  using namespace kvc;
  if (!d || !p || !c || p->kind != KVC_PRED_CLUSTER) return KVC_ERR_INVALID_ARGUMENT;
  if (d->n_tokens < 0 || d->n_heads < 1) return KVC_ERR_INVALID_ARGUMENT;
  if (d->head_dim != 64 && d->head_dim != 128) return KVC_ERR_UNSUPPORTED;  // as kvc_encode_layer
  // the scratch array holds tables for at most 256 centres of 128 coefficients
  if (p->n_clusters < 1 || p->n_clusters > kMaxCentres || p->code_dim != kCodeDim) return KVC_ERR_UNSUPPORTED;
  if (d->dtype != KVC_F32 && d->dtype != KVC_BF16) return KVC_ERR_UNSUPPORTED;
  if (d->param_dtype != KVC_F32 && d->param_dtype != KVC_F16) return KVC_ERR_UNSUPPORTED;
  if (d->bits != 2 && d->bits != 4 && d->bits != 8) return KVC_ERR_UNSUPPORTED;
  if (d->group <= 0 || kCodeDim % d->group || d->group % 4 || (d->group / 4) & (d->group / 4 - 1) || d->group > 128)
    return KVC_ERR_UNSUPPORTED;
  if (d->n_tokens == 0) return KVC_OK;
  const void* need[] = {K, V, c->k_codes, c->k_params, c->v_codes, c->v_params, c->k_assign, c->v_assign,
                        p->k_centroids, p->k_enc, p->k_dec, p->v_centroids, p->v_enc, p->v_dec};
  for (const void* q : need) {
    if (!q) return KVC_ERR_INVALID_ARGUMENT;
    if (!aligned16(q)) return KVC_ERR_MISALIGNED;
  }
  if ((K_rec && !aligned16(K_rec)) || (V_rec && !aligned16(V_rec))) return KVC_ERR_MISALIGNED;
  float* scratch = nullptr;
  cudaError_t e = scratch_for_current_device(&scratch);
  if (e != cudaSuccess) return record_cuda_error(e);
  cudaStream_t st = (cudaStream_t)stream;
  if (d->dtype == KVC_F32) {
    e = d->param_dtype == KVC_F32 ? encode<float, float>(d, p, K, V, c, K_rec, V_rec, scratch, st)
                                  : encode<float, __half>(d, p, K, V, c, K_rec, V_rec, scratch, st);
  } else {
    e = d->param_dtype == KVC_F32 ? encode<__nv_bfloat16, float>(d, p, K, V, c, K_rec, V_rec, scratch, st)
                                  : encode<__nv_bfloat16, __half>(d, p, K, V, c, K_rec, V_rec, scratch, st);
  }
  return e == cudaSuccess ? KVC_OK : record_cuda_error(e);
}
