// C-ABI entry points of libkvc.so: argument validation, storage sizes,
// workspace carving and dispatch to the CUDA kernels.  See include/kvc.h.
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <type_traits>

#include "common.cuh"
#include "simt.h"
#include "tc.h"

using namespace kvc;

namespace kvc {
static std::atomic<unsigned long long> g_launches{0};
void count_launches(unsigned long long n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

static thread_local char g_last_cuda[256] = "";

kvc_status record_cuda_error(cudaError_t e) {
  snprintf(g_last_cuda, sizeof(g_last_cuda), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return KVC_ERR_CUDA;
}
}  // namespace kvc

namespace {

kvc_status cuda_fail(cudaError_t e) { return record_cuda_error(e); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

int state_size(int dtype) { return dtype == KVC_F32 ? 4 : 2; }
int param_size(int dtype) { return dtype == KVC_F32 ? 4 : 2; }

// A row of n elements held by a warp (n/32 per lane) grouped by `group`.
bool row_layout_ok(int n, int group) {
  if (n % 32 || group <= 0 || n % group) return false;
  const int e = n / 32;
  return group % e == 0 && pow2(group / e) && group / e <= 32;
}

kvc_status check_desc(const kvc_layer_desc* d, const kvc_predictor* p) {
  if (!d || !p) return KVC_ERR_INVALID_ARGUMENT;
  if (d->n_tokens < 0 || d->n_heads < 1) return KVC_ERR_INVALID_ARGUMENT;
  if (d->q_heads < 0 || (d->q_heads > 0 && d->q_heads % d->n_heads)) return KVC_ERR_INVALID_ARGUMENT;
  if (d->head_dim != 64 && d->head_dim != 128) return KVC_ERR_UNSUPPORTED;
  if (d->dtype != KVC_F32 && d->dtype != KVC_BF16) return KVC_ERR_UNSUPPORTED;
  if (d->param_dtype != KVC_F32 && d->param_dtype != KVC_F16) return KVC_ERR_UNSUPPORTED;
  if (d->bits != 2 && d->bits != 4 && d->bits != 8) return KVC_ERR_UNSUPPORTED;
  if (d->residual_codec == KVC_RESIDUAL_H64_EDEN2) {
    // one scale per 64 transformed values, 4 bits per pair (the INT2 rate)
    if (p->kind != KVC_PRED_NONE && p->kind != KVC_PRED_XLAYER_DPLR) return KVC_ERR_UNSUPPORTED;
    if (d->bits != 2 || d->group != 64) return KVC_ERR_UNSUPPORTED;
    if (p->kind == KVC_PRED_XLAYER_DPLR && (p->rank < 0 || p->rank > 128)) return KVC_ERR_UNSUPPORTED;
    return KVC_OK;
  }
  if (d->residual_codec != KVC_RESIDUAL_RTN) return KVC_ERR_UNSUPPORTED;
  switch (p->kind) {
    case KVC_PRED_NONE:
    case KVC_PRED_XLAYER_DPLR:
      if (!row_layout_ok(d->head_dim, d->group)) return KVC_ERR_UNSUPPORTED;
      if (p->kind == KVC_PRED_XLAYER_DPLR && (p->rank < 0 || p->rank > 128)) return KVC_ERR_UNSUPPORTED;
      return KVC_OK;
    case KVC_PRED_TEMPORAL:
      if (!row_layout_ok(d->head_dim, d->group)) return KVC_ERR_UNSUPPORTED;
      if (d->frame_tokens < 1) return KVC_ERR_INVALID_ARGUMENT;
      if (d->anchor_bits != 0 && d->anchor_bits != 2 && d->anchor_bits != 4 && d->anchor_bits != 8)
        return KVC_ERR_UNSUPPORTED;
      return KVC_OK;
    case KVC_PRED_CLUSTER:
      if (p->code_dim != 128 || !row_layout_ok(128, d->group)) return KVC_ERR_UNSUPPORTED;
      if (p->n_clusters < 1 || p->n_clusters > 256) return KVC_ERR_UNSUPPORTED;
      return KVC_OK;
    default:
      return KVC_ERR_UNSUPPORTED;
  }
}

struct Sizes {
  size_t codes, params, assign;
};

Sizes sizes_of(const kvc_layer_desc* d, const kvc_predictor* p) {
  const size_t T = (size_t)d->n_tokens, H = d->n_heads, D = d->head_dim;
  const size_t pair = 2 * (size_t)param_size(d->param_dtype);
  Sizes s{0, 0, 0};
  if (d->residual_codec == KVC_RESIDUAL_H64_EDEN2) {
    s.codes = T * H * D / 4;  // a 4-bit index per pair
    s.params = T * H * (D / 64) * (size_t)param_size(d->param_dtype);
    return s;
  }
  if (p->kind == KVC_PRED_CLUSTER) {
    const size_t m = p->code_dim;
    s.codes = T * m * d->bits / 8;
    s.params = T * (m / d->group) * pair;
    s.assign = T;
  } else if (p->kind == KVC_PRED_TEMPORAL) {
    const size_t F0 = d->anchor_bits == 0 ? 0 : ((size_t)d->frame_tokens < T ? (size_t)d->frame_tokens : T);
    s.codes = F0 * H * D * d->anchor_bits / 8 + (T - F0) * H * D * d->bits / 8;
    s.params = T * H * (D / d->group) * pair;
  } else {
    s.codes = T * H * D * d->bits / 8;
    s.params = T * H * (D / d->group) * pair;
  }
  return s;
}

// Workspace of the CUDA-core path.
size_t simt_workspace(int op, const kvc_layer_desc* d, const kvc_predictor* p) {
  const size_t T = (size_t)d->n_tokens;
  size_t ws = 0;
  if (p->kind == KVC_PRED_XLAYER_DPLR && p->rank > 0) ws += 2 * align256(T * p->rank * sizeof(float));
  if (p->kind == KVC_PRED_CLUSTER && op != KVC_OP_ATTEND)
    ws += 2 * (align256(p->n_clusters * sizeof(float)) + align256((size_t)p->n_clusters * p->code_dim * sizeof(float)));
  if (op == KVC_OP_ATTEND && (p->kind == KVC_PRED_NONE || p->kind == KVC_PRED_XLAYER_DPLR))
    ws += 2 * align256(T * d->n_heads * d->head_dim * state_size(d->dtype));
  return ws;
}

struct Carve {
  char* p;
  size_t left;
  bool ok = true;
  void* take(size_t n) {
    n = align256(n);
    if (n > left) {
      ok = false;
      return nullptr;
    }
    void* r = p;
    p += n;
    left -= n;
    return r;
  }
};

template <typename F>
kvc_status dispatch(const kvc_layer_desc* d, F&& f) {
  cudaError_t e;
  if (d->dtype == KVC_F32) {
    e = d->param_dtype == KVC_F32 ? f((float*)nullptr, (float*)nullptr) : f((float*)nullptr, (__half*)nullptr);
  } else {
    e = d->param_dtype == KVC_F32 ? f((__nv_bfloat16*)nullptr, (float*)nullptr)
                                  : f((__nv_bfloat16*)nullptr, (__half*)nullptr);
  }
  return e == cudaSuccess ? KVC_OK : cuda_fail(e);
}

// ---------------------------------------------------------------- the codec, one layer

template <typename TS, typename TP>
cudaError_t codec_xlayer(const kvc_layer_desc* d, const kvc_predictor* p, bool enc, const void* K, const void* V,
                         const void* Ks, const void* Vs, const kvc_codes* c, void* Kr, void* Vr, Carve& ws,
                         cudaStream_t st) {
  const int64_t T = d->n_tokens;
  const int H = d->n_heads, D = d->head_dim, C = H * D;
  const bool pred = p->kind == KVC_PRED_XLAYER_DPLR;
  const int r = pred ? p->rank : 0;
  float* Zk = r ? (float*)ws.take(T * r * sizeof(float)) : nullptr;
  float* Zv = r ? (float*)ws.take(T * r * sizeof(float)) : nullptr;
  cudaError_t e;
  if (r) {
    LatentArgs<TS> la{T, C, r, (const TS*)Ks, nullptr, (const TS*)p->k_w, Zk};
    if ((e = launch_latent(la, st)) != cudaSuccess) return e;
  }
  const float* cb = d->residual_codec == KVC_RESIDUAL_H64_EDEN2 ? (const float*)p->residual_codebook : nullptr;
  HeadsArgs<TS, TP> hk{T, H, d->bits, d->group, r,
                       pred ? (const TS*)Ks : nullptr, nullptr, pred ? (const TS*)p->k_block : nullptr,
                       Zk, (const TS*)p->k_u, (const TS*)K,
                       (uint8_t*)c->k_codes, (Pair<TP>*)c->k_params, (TS*)Kr, cb};
  if ((e = launch_heads(hk, D, enc, st)) != cudaSuccess) return e;
  if (r) {
    LatentArgs<TS> la{T, C, r, (const TS*)Kr, (const TS*)Vs, (const TS*)p->v_w, Zv};
    if ((e = launch_latent(la, st)) != cudaSuccess) return e;
  }
  HeadsArgs<TS, TP> hv{T, H, d->bits, d->group, r,
                       pred ? (const TS*)Kr : nullptr, pred ? (const TS*)Vs : nullptr,
                       pred ? (const TS*)p->v_block : nullptr, Zv, (const TS*)p->v_u, (const TS*)V,
                       (uint8_t*)c->v_codes, (Pair<TP>*)c->v_params, (TS*)Vr, cb};
  return launch_heads(hv, D, enc, st);
}

template <typename TS, typename TP>
cudaError_t codec_temporal(const kvc_layer_desc* d, const kvc_predictor* p, bool enc, const void* K, const void* V,
                           const void* Ks, const void* Vs, const kvc_codes* c, void* Kr, void* Vr, cudaStream_t st) {
  TemporalArgs<TS, TP> a{d->n_tokens, d->frame_tokens, d->n_heads, d->bits, d->anchor_bits, d->group,
                         (const TS*)K, (const TS*)V, (const TS*)Ks, (const TS*)Vs,
                         (const TS*)p->k_block, (const TS*)p->v_block,
                         (uint8_t*)c->k_codes, (Pair<TP>*)c->k_params, (uint8_t*)c->v_codes,
                         (Pair<TP>*)c->v_params, (TS*)Kr, (TS*)Vr};
  return launch_temporal(a, d->head_dim, enc, st);
}

template <typename TS, typename TP>
cudaError_t codec_cluster(const kvc_layer_desc* d, const kvc_predictor* p, bool enc, const void* K, const void* V,
                          const kvc_codes* c, void* Kr, void* Vr, Carve& ws, cudaStream_t st) {
  const int C = d->n_heads * d->head_dim, m = p->code_dim, nc = p->n_clusters;
  cudaError_t e;
  float* cns[2] = {nullptr, nullptr};
  float* Ps[2] = {nullptr, nullptr};
  if (enc)
    for (int which = 0; which < 2; ++which) {
      cns[which] = (float*)ws.take(nc * sizeof(float));
      Ps[which] = (float*)ws.take((size_t)nc * m * sizeof(float));
    }
  if constexpr (std::is_same<TS, __nv_bfloat16>::value && std::is_same<TP, __half>::value) {
    if (tc_cluster_supported(d, p)) {
      if (enc) {
        // centre norms, then P = C E^T of both tensors on the tensor cores (the same
        // accumulation as the tokens' coefficients) in one launch
        for (int which = 0; which < 2; ++which) {
          ClusterPrepArgs<TS> pa{nc, C, m, (const TS*)(which ? p->v_centroids : p->k_centroids),
                                 (const TS*)(which ? p->v_enc : p->k_enc), cns[which], Ps[which]};
          if ((e = launch_cluster_norms(pa, st)) != cudaSuccess) return e;
        }
        const float* const cnc[2] = {cns[0], cns[1]};
        if ((e = tc_cluster_prepare(d, p, cnc, Ps, st)) != cudaSuccess) return e;
      }
      // K and V share each launch: the token pass of both, then the decode of both
      void* const codes[2] = {c->k_codes, c->v_codes};
      void* const params[2] = {c->k_params, c->v_params};
      void* const assign[2] = {c->k_assign, c->v_assign};
      if (enc) {
        const void* const X[2] = {K, V};
        const float* const cnc[2] = {cns[0], cns[1]};
        if ((e = tc_cluster_encode(d, p, X, cnc, Ps, codes, params, assign, st)) != cudaSuccess) return e;
      }
      // the encode's reconstruction is the decode of what it wrote, so the two agree bit for bit
      const void* const ccodes[2] = {codes[0], codes[1]};
      const void* const cparams[2] = {params[0], params[1]};
      const void* const cassign[2] = {assign[0], assign[1]};
      void* const rec[2] = {Kr, Vr};
      return tc_cluster_decode(d, p, ccodes, cparams, cassign, rec, st);
    }
  }
  for (int which = 0; which < 2; ++which) {
    const TS* cent = (const TS*)(which ? p->v_centroids : p->k_centroids);
    const TS* encw = (const TS*)(which ? p->v_enc : p->k_enc);
    const TS* dec = (const TS*)(which ? p->v_dec : p->k_dec);
    float* cn = cns[which];
    float* P = Ps[which];
    if (enc) {
      ClusterPrepArgs<TS> pa{nc, C, m, cent, encw, cn, P};
      if ((e = launch_cluster_prep(pa, st)) != cudaSuccess) return e;
    }
    ClusterArgs<TS, TP> a{d->n_tokens, C, m, nc, d->bits, d->group, (const TS*)(which ? V : K), cent, encw, dec,
                          cn, P, (uint8_t*)(which ? c->v_codes : c->k_codes),
                          (Pair<TP>*)(which ? c->v_params : c->k_params),
                          (uint8_t*)(which ? c->v_assign : c->k_assign), (TS*)(which ? Vr : Kr)};
    if ((e = launch_cluster(a, enc, st)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

bool codes_ok(const kvc_predictor* p, const kvc_codes* c) {
  if (!c || !c->k_codes || !c->k_params || !c->v_codes || !c->v_params) return false;
  if (p->kind == KVC_PRED_CLUSTER && (!c->k_assign || !c->v_assign)) return false;
  return true;
}

bool codes_aligned(const kvc_predictor* p, const kvc_codes* c) {
  bool a = aligned16(c->k_codes) && aligned16(c->k_params) && aligned16(c->v_codes) && aligned16(c->v_params);
  if (p->kind == KVC_PRED_CLUSTER) a = a && aligned16(c->k_assign) && aligned16(c->v_assign);
  return a;
}

kvc_status check_weights(const kvc_predictor* p) {
  const void* const* need = nullptr;
  const void* xl[] = {p->k_block, p->v_block};
  const void* xr[] = {p->k_w, p->k_u, p->v_w, p->v_u};
  const void* cl[] = {p->k_centroids, p->k_enc, p->k_dec, p->v_centroids, p->v_enc, p->v_dec};
  int n = 0;
  if (p->kind == KVC_PRED_XLAYER_DPLR || p->kind == KVC_PRED_TEMPORAL) {
    need = xl;
    n = 2;
  } else if (p->kind == KVC_PRED_CLUSTER) {
    need = cl;
    n = 6;
  }
  for (int i = 0; i < n; ++i) {
    if (!need[i]) return KVC_ERR_INVALID_ARGUMENT;
    if (!aligned16(need[i])) return KVC_ERR_MISALIGNED;
  }
  if (p->kind == KVC_PRED_XLAYER_DPLR && p->rank > 0) {
    for (const void* w : xr) {
      if (!w) return KVC_ERR_INVALID_ARGUMENT;
      if (!aligned16(w)) return KVC_ERR_MISALIGNED;
    }
  }
  return KVC_OK;
}

kvc_status check_codebook(const kvc_layer_desc* d, const kvc_predictor* p) {
  if (d->residual_codec != KVC_RESIDUAL_H64_EDEN2) return KVC_OK;
  if (!p->residual_codebook) return KVC_ERR_INVALID_ARGUMENT;
  return aligned16(p->residual_codebook) ? KVC_OK : KVC_ERR_MISALIGNED;
}

kvc_status codec_common(const kvc_layer_desc* d, const kvc_predictor* p, bool enc, const void* K, const void* V,
                        const void* Ks, const void* Vs, const kvc_codes* c, void* Kr, void* Vr, void* ws,
                        size_t ws_bytes, void* stream) {
  kvc_status s = check_desc(d, p);
  if (s != KVC_OK) return s;
  if (d->n_tokens == 0) return KVC_OK;  // nothing to code
  if ((s = check_weights(p)) != KVC_OK) return s;
  if ((s = check_codebook(d, p)) != KVC_OK) return s;
  if (!codes_ok(p, c)) return KVC_ERR_INVALID_ARGUMENT;
  if (enc && (!K || !V)) return KVC_ERR_INVALID_ARGUMENT;
  if (p->kind == KVC_PRED_TEMPORAL && d->anchor_bits == 0 && (!Ks || !Vs)) return KVC_ERR_INVALID_ARGUMENT;
  if (!enc && (!Kr || !Vr)) return KVC_ERR_INVALID_ARGUMENT;
  if (p->kind == KVC_PRED_XLAYER_DPLR && (!Ks || !Vs || !Kr)) return KVC_ERR_INVALID_ARGUMENT;
  const void* ptrs[] = {K, V, Ks, Vs, Kr, Vr, ws};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return KVC_ERR_MISALIGNED;
  if (!codes_aligned(p, c)) return KVC_ERR_MISALIGNED;
  const int op = enc ? KVC_OP_ENCODE : KVC_OP_DECODE;
  const size_t need = kvc_workspace_bytes(op, d, p, 0);
  if (ws_bytes < need || (need && !ws)) return KVC_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = (cudaStream_t)stream;
  // tensor-core paths for bf16, D = 128
  if (tc_codec_supported(d, p)) {
    cudaError_t e = tc_codec_layer(d, p, enc, K, V, Ks, Vs, c, Kr, Vr, ws, ws_bytes, st);
    return e == cudaSuccess ? KVC_OK : cuda_fail(e);
  }
  if (tc_temporal_supported(d, p)) {
    cudaError_t e = tc_temporal_layer(d, p, enc, K, V, Ks, Vs, c, Kr, Vr, st);
    return e == cudaSuccess ? KVC_OK : cuda_fail(e);
  }
  if (anchor_supported(d, p)) {
    cudaError_t e = anchor_layer(d, enc, K, V, c, Kr, Vr, st);
    return e == cudaSuccess ? KVC_OK : cuda_fail(e);
  }
  Carve cv{(char*)ws, ws_bytes};
  return dispatch(d, [&](auto* ts, auto* tp) -> cudaError_t {
    using TS = std::remove_pointer_t<decltype(ts)>;
    using TP = std::remove_pointer_t<decltype(tp)>;
    switch (p->kind) {
      case KVC_PRED_TEMPORAL:
        return codec_temporal<TS, TP>(d, p, enc, K, V, Ks, Vs, c, Kr, Vr, st);
      case KVC_PRED_CLUSTER:
        return codec_cluster<TS, TP>(d, p, enc, K, V, c, Kr, Vr, cv, st);
      default:
        return codec_xlayer<TS, TP>(d, p, enc, K, V, Ks, Vs, c, Kr, Vr, cv, st);
    }
  });
}

// Attention over a predicted (or anchor) history: the history is decoded once
// (into the caller's outputs when given, else the workspace), then attended
// with the chunk's own keys; jensen: the debiased scores (tensor cores only).
kvc_status attend_decoded(const kvc_layer_desc* d, const kvc_predictor* p, const void* Q, int64_t n_q,
                          const kvc_codes* codes, const void* K_src, const void* V_src, const void* K_self,
                          const void* V_self, int64_t n_self, float scale, void* O, void* K_rec_opt, void* V_rec_opt,
                          void* ws, size_t ws_bytes, cudaStream_t st, bool jensen) {
  Carve cv{(char*)ws, ws_bytes};
  return dispatch(d, [&](auto* ts, auto* tp) -> cudaError_t {
    using TS = std::remove_pointer_t<decltype(ts)>;
    using TP = std::remove_pointer_t<decltype(tp)>;
    const int H = d->n_heads, D = d->head_dim;
    const size_t bytes = (size_t)d->n_tokens * H * D * sizeof(TS);
    TS* Kh = (TS*)cv.take(bytes);
    TS* Vh = (TS*)cv.take(bytes);
    if (K_rec_opt) Kh = (TS*)K_rec_opt;
    if (V_rec_opt) Vh = (TS*)V_rec_opt;
    if (d->n_tokens > 0) {
      cudaError_t e =
          tc_codec_supported(d, p)  ? tc_codec_layer(d, p, false, nullptr, nullptr, K_src, V_src, codes, Kh, Vh,
                                                     nullptr, 0, st)
          : anchor_supported(d, p) ? anchor_layer(d, false, nullptr, nullptr, codes, Kh, Vh, st)
                                   : codec_xlayer<TS, TP>(d, p, false, nullptr, nullptr, K_src, V_src, codes, Kh, Vh,
                                                          cv, st);
      if (e != cudaSuccess) return e;
    }
    if (tc_flash_supported(d))
      return tc_flash(d, Q, n_q, Kh, Vh, K_self, V_self, n_self, scale, O, jensen ? codes->k_params : nullptr, st);
    if (jensen) return cudaErrorNotSupported;
    AttnArgs<TS> a{n_q, d->n_tokens, n_self, H, d->q_heads > 0 ? d->q_heads : H, scale, (const TS*)Q, Kh, Vh,
                   (const TS*)K_self, (const TS*)V_self, (TS*)O};
    return launch_attention(a, D, st);
  });
}

// A chain of predicted layers: layer i of the call predicts from layer i-1's
// reconstruction (K_src / V_src for i = 0).  One persistent launch on the
// tensor cores where every layer is supported there, else the layers in turn.
kvc_status layers_common(const kvc_layer_desc* d, const kvc_predictor* preds, int n, bool enc,
                         const void* const* K, const void* const* V, const void* K_src, const void* V_src,
                         const kvc_codes* c, void* const* K_rec, void* const* V_rec, void* ws, size_t ws_bytes,
                         void* stream) {
  if (!d || !preds || n < 1 || !c || !K_rec || !V_rec || !K_src || !V_src) return KVC_ERR_INVALID_ARGUMENT;
  if (enc && (!K || !V)) return KVC_ERR_INVALID_ARGUMENT;
  for (int i = 0; i < n; ++i) {
    kvc_status s = check_desc(d, &preds[i]);
    if (s != KVC_OK) return s;
    if (preds[i].kind != KVC_PRED_XLAYER_DPLR) return KVC_ERR_UNSUPPORTED;
    if ((s = check_weights(&preds[i])) != KVC_OK) return s;
    if ((s = check_codebook(d, &preds[i])) != KVC_OK) return s;
    if (!codes_ok(&preds[i], &c[i])) return KVC_ERR_INVALID_ARGUMENT;
    if (!codes_aligned(&preds[i], &c[i])) return KVC_ERR_MISALIGNED;
    if (!K_rec[i] || !V_rec[i] || (enc && (!K[i] || !V[i]))) return KVC_ERR_INVALID_ARGUMENT;
    const void* ptrs[] = {K_rec[i], V_rec[i], enc ? K[i] : nullptr, enc ? V[i] : nullptr};
    for (const void* q : ptrs)
      if (q && !aligned16(q)) return KVC_ERR_MISALIGNED;
    // a layer's reconstruction is the next layer's source: it may not overwrite its own source
    const void* ks = i ? K_rec[i - 1] : K_src;
    const void* vs = i ? V_rec[i - 1] : V_src;
    if (K_rec[i] == ks || V_rec[i] == vs || K_rec[i] == V_rec[i]) return KVC_ERR_INVALID_ARGUMENT;
  }
  if (!aligned16(K_src) || !aligned16(V_src) || (ws && !aligned16(ws))) return KVC_ERR_MISALIGNED;
  const size_t need = kvc_layers_workspace_bytes(enc ? KVC_OP_ENCODE : KVC_OP_DECODE, d, preds, n);
  if (ws_bytes < need || (need && !ws)) return KVC_ERR_WORKSPACE_TOO_SMALL;
  if (d->n_tokens == 0) return KVC_OK;
  cudaStream_t st = (cudaStream_t)stream;
  if (tc_codec_layers_supported(d, preds, n)) {
    cudaError_t e = tc_codec_layers(d, preds, n, enc, K, V, K_src, V_src, c, K_rec, V_rec, ws, ws_bytes, st);
    return e == cudaSuccess ? KVC_OK : cuda_fail(e);
  }
  for (int i = 0; i < n; ++i) {
    const void* ks = i ? K_rec[i - 1] : K_src;
    const void* vs = i ? V_rec[i - 1] : V_src;
    kvc_status s = codec_common(d, &preds[i], enc, enc ? K[i] : nullptr, enc ? V[i] : nullptr, ks, vs, &c[i],
                                K_rec[i], V_rec[i], ws, ws_bytes, stream);
    if (s != KVC_OK) return s;
  }
  return KVC_OK;
}
}  // namespace

extern "C" {

kvc_status kvc_codes_sizes(const kvc_layer_desc* desc, const kvc_predictor* pred, kvc_codes_size* out) {
  if (!out) return KVC_ERR_INVALID_ARGUMENT;
  kvc_status s = check_desc(desc, pred);
  if (s != KVC_OK) return s;
  Sizes z = sizes_of(desc, pred);
  out->codes = z.codes;
  out->params = z.params;
  out->assign = z.assign;
  return KVC_OK;
}

size_t kvc_codes_bytes(const kvc_layer_desc* desc, const kvc_predictor* pred) {
  if (check_desc(desc, pred) != KVC_OK) return 0;
  Sizes z = sizes_of(desc, pred);
  return 2 * (z.codes + z.params + z.assign);
}

size_t kvc_workspace_bytes(int op, const kvc_layer_desc* desc, const kvc_predictor* pred, int64_t n_q) {
  if (check_desc(desc, pred) != KVC_OK) return 0;
  if (op == KVC_OP_REFIT_K || op == KVC_OP_REFIT_V)
    return pred->kind == KVC_PRED_XLAYER_DPLR
               ? refit_workspace(desc->n_tokens, desc->n_heads, desc->head_dim, pred->rank, op == KVC_OP_REFIT_V)
               : 0;
  size_t a = simt_workspace(op, desc, pred);
  size_t b = tc_workspace(op, desc, pred, n_q);
  return a > b ? a : b;
}

kvc_status kvc_encode_layer(const kvc_layer_desc* desc, const kvc_predictor* pred, const void* K, const void* V,
                            const void* K_src, const void* V_src, const kvc_codes* out, void* K_rec, void* V_rec,
                            void* ws, size_t ws_bytes, void* stream) {
  return codec_common(desc, pred, true, K, V, K_src, V_src, out, K_rec, V_rec, ws, ws_bytes, stream);
}

kvc_status kvc_decode_layer(const kvc_layer_desc* desc, const kvc_predictor* pred, const kvc_codes* codes,
                            const void* K_src, const void* V_src, void* K_rec, void* V_rec, void* ws, size_t ws_bytes,
                            void* stream) {
  return codec_common(desc, pred, false, nullptr, nullptr, K_src, V_src, codes, K_rec, V_rec, ws, ws_bytes, stream);
}

size_t kvc_layers_workspace_bytes(int op, const kvc_layer_desc* desc, const kvc_predictor* preds, int n_layers) {
  if (!desc || !preds || n_layers < 1 || (op != KVC_OP_ENCODE && op != KVC_OP_DECODE)) return 0;
  size_t per = 0;
  for (int i = 0; i < n_layers; ++i) {
    if (check_desc(desc, &preds[i]) != KVC_OK) return 0;
    const size_t w = kvc_workspace_bytes(op, desc, &preds[i], 0);
    per = w > per ? w : per;
  }
  const size_t fused = tc_codec_layers_supported(desc, preds, n_layers) ? tc_codec_layers_workspace(desc, n_layers) : 0;
  return fused > per ? fused : per;
}


kvc_status kvc_encode_layers(const kvc_layer_desc* desc, const kvc_predictor* preds, int n_layers,
                             const void* const* K, const void* const* V, const void* K_src, const void* V_src,
                             const kvc_codes* out, void* const* K_rec, void* const* V_rec, void* ws,
                             size_t ws_bytes, void* stream) {
  return layers_common(desc, preds, n_layers, true, K, V, K_src, V_src, out, K_rec, V_rec, ws, ws_bytes, stream);
}

kvc_status kvc_decode_layers(const kvc_layer_desc* desc, const kvc_predictor* preds, int n_layers,
                             const kvc_codes* codes, const void* K_src, const void* V_src, void* const* K_rec,
                             void* const* V_rec, void* ws, size_t ws_bytes, void* stream) {
  return layers_common(desc, preds, n_layers, false, nullptr, nullptr, K_src, V_src, codes, K_rec, V_rec, ws,
                       ws_bytes, stream);
}

kvc_status kvc_attend_compressed(const kvc_layer_desc* d, const kvc_predictor* p, const void* Q, int64_t n_q,
                                 const kvc_codes* codes, const void* K_src, const void* V_src, const void* K_self,
                                 const void* V_self, int64_t n_self, float scale, void* O, void* K_rec_opt,
                                 void* V_rec_opt, void* ws, size_t ws_bytes, void* stream) {
  kvc_status s = check_desc(d, p);
  if (s != KVC_OK) return s;
  if (p->kind == KVC_PRED_TEMPORAL) return KVC_ERR_UNSUPPORTED;
  if ((s = check_weights(p)) != KVC_OK) return s;
  if ((s = check_codebook(d, p)) != KVC_OK) return s;
  if (n_q < 0 || n_self < 0) return KVC_ERR_INVALID_ARGUMENT;
  if (p->kind == KVC_PRED_CLUSTER && n_self != 0) return KVC_ERR_UNSUPPORTED;
  if (p->kind == KVC_PRED_CLUSTER && d->q_heads > 0 && d->q_heads != d->n_heads) return KVC_ERR_UNSUPPORTED;
  if (!codes_ok(p, codes) || (n_q > 0 && (!Q || !O))) return KVC_ERR_INVALID_ARGUMENT;
  if (n_self > 0 && (!K_self || !V_self)) return KVC_ERR_INVALID_ARGUMENT;
  if (p->kind == KVC_PRED_XLAYER_DPLR && (!K_src || !V_src)) return KVC_ERR_INVALID_ARGUMENT;
  if (d->n_tokens + n_self == 0 && n_q > 0) return KVC_ERR_INVALID_ARGUMENT;  // softmax over no keys
  const void* ptrs[] = {Q, K_src, V_src, K_self, V_self, O, K_rec_opt, V_rec_opt, ws};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return KVC_ERR_MISALIGNED;
  if (!codes_aligned(p, codes)) return KVC_ERR_MISALIGNED;
  const size_t need = kvc_workspace_bytes(KVC_OP_ATTEND, d, p, n_q);
  if (ws_bytes < need || (need && !ws)) return KVC_ERR_WORKSPACE_TOO_SMALL;
  if (n_q == 0) return KVC_OK;
  cudaStream_t st = (cudaStream_t)stream;
  // the clustered history's reconstruction, when asked for, is its decode (the
  // attention itself never rebuilds it)
  if (p->kind == KVC_PRED_CLUSTER && (K_rec_opt || V_rec_opt) && d->n_tokens > 0) {
    Carve none{nullptr, 0};
    kvc_status s2 = dispatch(d, [&](auto* ts, auto* tp) -> cudaError_t {
      using TS = std::remove_pointer_t<decltype(ts)>;
      using TP = std::remove_pointer_t<decltype(tp)>;
      return codec_cluster<TS, TP>(d, p, false, nullptr, nullptr, codes, K_rec_opt, V_rec_opt, none, st);
    });
    if (s2 != KVC_OK) return s2;
  }
  if (tc_mixed_supported(d, p)) {
    cudaError_t e = tc_mixed_attend(d, p, Q, n_q, codes, scale, O, ws, ws_bytes, st);
    return e == cudaSuccess ? KVC_OK : cuda_fail(e);
  }
  if (p->kind == KVC_PRED_CLUSTER) {
    return dispatch(d, [&](auto* ts, auto* tp) -> cudaError_t {
      using TS = std::remove_pointer_t<decltype(ts)>;
      using TP = std::remove_pointer_t<decltype(tp)>;
      const int H = d->n_heads, D = d->head_dim;
      MixedArgs<TS, TP> a{n_q, d->n_tokens, H, D, H * D, p->n_clusters, d->bits, d->group, scale,
                          (const TS*)Q, (const TS*)p->k_centroids, (const TS*)p->k_dec, (const TS*)p->v_centroids,
                          (const TS*)p->v_dec, (const uint8_t*)codes->k_codes, (const Pair<TP>*)codes->k_params,
                          (const uint8_t*)codes->k_assign, (const uint8_t*)codes->v_codes,
                          (const Pair<TP>*)codes->v_params, (const uint8_t*)codes->v_assign, (TS*)O};
      return launch_mixed_attention(a, st);
    });
  }
  return attend_decoded(d, p, Q, n_q, codes, K_src, V_src, K_self, V_self, n_self, scale, O, K_rec_opt, V_rec_opt,
                        ws, ws_bytes, st, false);
}

kvc_status kvc_attend_compressed_debiased(const kvc_layer_desc* d, const kvc_predictor* p, const void* Q,
                                          int64_t n_q, const kvc_codes* codes, const void* K_src, const void* V_src,
                                          const void* K_self, const void* V_self, int64_t n_self, float scale,
                                          void* O, void* K_rec_opt, void* V_rec_opt, void* ws, size_t ws_bytes,
                                          void* stream) {
  kvc_status s = check_desc(d, p);
  if (s != KVC_OK) return s;
  // the corrected softmax is written for the tensor-core attention over an
  // INT-coded cross-layer history
  if (!tc_flash_debiased_supported(d, p) || d->n_tokens == 0) return KVC_ERR_UNSUPPORTED;
  if ((s = check_weights(p)) != KVC_OK) return s;
  if (n_q < 0 || n_self < 0) return KVC_ERR_INVALID_ARGUMENT;
  if (!codes_ok(p, codes) || (n_q > 0 && (!Q || !O))) return KVC_ERR_INVALID_ARGUMENT;
  if (n_self > 0 && (!K_self || !V_self)) return KVC_ERR_INVALID_ARGUMENT;
  if (!K_src || !V_src) return KVC_ERR_INVALID_ARGUMENT;
  const void* ptrs[] = {Q, K_src, V_src, K_self, V_self, O, K_rec_opt, V_rec_opt, ws};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return KVC_ERR_MISALIGNED;
  if (!codes_aligned(p, codes)) return KVC_ERR_MISALIGNED;
  const size_t need = kvc_workspace_bytes(KVC_OP_ATTEND, d, p, n_q);
  if (ws_bytes < need || (need && !ws)) return KVC_ERR_WORKSPACE_TOO_SMALL;
  if (n_q == 0) return KVC_OK;
  return attend_decoded(d, p, Q, n_q, codes, K_src, V_src, K_self, V_self, n_self, scale, O, K_rec_opt, V_rec_opt,
                        ws, ws_bytes, (cudaStream_t)stream, true);
}

kvc_status kvc_refit_block_diag(const kvc_layer_desc* d, const kvc_predictor* p, int tensor, const void* X0,
                                const void* X1, const void* Y, float ridge, void* block_out, void* ws,
                                size_t ws_bytes, void* stream) {
  kvc_status s = check_desc(d, p);
  if (s != KVC_OK) return s;
  if (p->kind != KVC_PRED_XLAYER_DPLR) return KVC_ERR_UNSUPPORTED;
  if (tensor != 0 && tensor != 1) return KVC_ERR_INVALID_ARGUMENT;
  if (d->n_tokens < 1 || !(ridge >= 0.f)) return KVC_ERR_INVALID_ARGUMENT;
  if (!X0 || !Y || !block_out || (tensor == 1 && !X1)) return KVC_ERR_INVALID_ARGUMENT;
  const void* w = tensor ? p->v_w : p->k_w;
  const void* u = tensor ? p->v_u : p->k_u;
  if (p->rank > 0 && (!w || !u)) return KVC_ERR_INVALID_ARGUMENT;
  const void* ptrs[] = {X0, tensor ? X1 : nullptr, Y, block_out, ws, p->rank ? w : nullptr, p->rank ? u : nullptr};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return KVC_ERR_MISALIGNED;
  const size_t need = kvc_workspace_bytes(tensor ? KVC_OP_REFIT_V : KVC_OP_REFIT_K, d, p, 0);
  if (ws_bytes < need || !ws) return KVC_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = (cudaStream_t)stream;
  const void* x1 = tensor ? X1 : nullptr;
  cudaError_t e;
  if (d->dtype == KVC_F32)
    e = launch_refit<float>(d->n_tokens, d->n_heads, d->head_dim, p->rank, (const float*)X0, (const float*)x1,
                            (const float*)Y, (const float*)w, (const float*)u, ridge, (float*)block_out, ws, st);
  else
    e = launch_refit<__nv_bfloat16>(d->n_tokens, d->n_heads, d->head_dim, p->rank, (const __nv_bfloat16*)X0,
                                    (const __nv_bfloat16*)x1, (const __nv_bfloat16*)Y, (const __nv_bfloat16*)w,
                                    (const __nv_bfloat16*)u, ridge, (__nv_bfloat16*)block_out, ws, st);
  return e == cudaSuccess ? KVC_OK : cuda_fail(e);
}

kvc_status kvc_pack_codes(const uint8_t* codes, int64_t n, int bits, void* packed, void* stream) {
  if (bits != 2 && bits != 4 && bits != 8) return KVC_ERR_UNSUPPORTED;
  if (n < 0 || (n * bits) % 128) return KVC_ERR_INVALID_ARGUMENT;
  if (n && (!codes || !packed)) return KVC_ERR_INVALID_ARGUMENT;
  if (!aligned16(codes) || !aligned16(packed)) return KVC_ERR_MISALIGNED;
  cudaError_t e = launch_pack(codes, n, bits, packed, (cudaStream_t)stream);
  return e == cudaSuccess ? KVC_OK : cuda_fail(e);
}

kvc_status kvc_unpack_codes(const void* packed, int64_t n, int bits, uint8_t* codes, void* stream) {
  if (bits != 2 && bits != 4 && bits != 8) return KVC_ERR_UNSUPPORTED;
  if (n < 0 || (n * bits) % 128) return KVC_ERR_INVALID_ARGUMENT;
  if (n && (!codes || !packed)) return KVC_ERR_INVALID_ARGUMENT;
  if (!aligned16(codes) || !aligned16(packed)) return KVC_ERR_MISALIGNED;
  cudaError_t e = launch_unpack(packed, n, bits, codes, (cudaStream_t)stream);
  return e == cudaSuccess ? KVC_OK : cuda_fail(e);
}

kvc_status kvc_copy_to_device(void* dst, const void* src, size_t bytes, void* stream) {
  if (bytes == 0) return KVC_OK;
  if (!dst || !src) return KVC_ERR_INVALID_ARGUMENT;
  cudaError_t e = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, (cudaStream_t)stream);
  return e == cudaSuccess ? KVC_OK : cuda_fail(e);
}

kvc_status kvc_copy_to_host(void* dst, const void* src, size_t bytes, void* stream) {
  if (bytes == 0) return KVC_OK;
  if (!dst || !src) return KVC_ERR_INVALID_ARGUMENT;
  cudaError_t e = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  return e == cudaSuccess ? KVC_OK : cuda_fail(e);
}

kvc_status kvc_get_device_error(void* stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e);
  unsigned int v = 0;
  e = tc_read_and_clear_error(&v);
  if (e != cudaSuccess) return cuda_fail(e);
  return v ? KVC_ERR_DEVICE_TIMEOUT : KVC_OK;
}

const char* kvc_status_string(kvc_status s) {
  switch (s) {
    case KVC_OK: return "ok";
    case KVC_ERR_INVALID_ARGUMENT: return "invalid argument";
    case KVC_ERR_UNSUPPORTED: return "unsupported configuration";
    case KVC_ERR_MISALIGNED: return "device pointer not 16-byte aligned";
    case KVC_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case KVC_ERR_CUDA: return "CUDA error";
    case KVC_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

const char* kvc_last_cuda_error(void) { return g_last_cuda; }

uint64_t kvc_launch_counter(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
