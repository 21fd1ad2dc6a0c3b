// Tensor-core (tcgen05 / TMEM / TMA) kernels for bf16, head_dim 128 (internal).
#pragma once

#include "common.cuh"

namespace kvc {

bool tc_codec_supported(const kvc_layer_desc* d, const kvc_predictor* p);
size_t tc_workspace(int op, const kvc_layer_desc* d, const kvc_predictor* p, int64_t n_q);
cudaError_t tc_codec_layer(const kvc_layer_desc* d, const kvc_predictor* p, bool enc, const void* K, const void* V,
                           const void* Ks, const void* Vs, const kvc_codes* c, void* Kr, void* Vr, void* ws,
                           size_t ws_bytes, cudaStream_t st);
// a chain of n predicted layers in one persistent launch (layer i reads layer
// i-1's reconstruction; Ks0 / Vs0 for i = 0); Kr / Vr of every layer required
bool tc_codec_layers_supported(const kvc_layer_desc* d, const kvc_predictor* preds, int n);
size_t tc_codec_layers_workspace(const kvc_layer_desc* d, int n);
cudaError_t tc_codec_layers(const kvc_layer_desc* d, const kvc_predictor* preds, int n, bool enc,
                            const void* const* K, const void* const* V, const void* Ks0, const void* Vs0,
                            const kvc_codes* c, void* const* Kr, void* const* Vr, void* ws, size_t ws_bytes,
                            cudaStream_t st);
bool tc_temporal_supported(const kvc_layer_desc* d, const kvc_predictor* p);
cudaError_t tc_temporal_layer(const kvc_layer_desc* d, const kvc_predictor* p, bool enc, const void* K, const void* V,
                              const void* Ks, const void* Vs, const kvc_codes* c, void* Kr, void* Vr, cudaStream_t st);
// flash attention over a decoded bf16 history [T][H][128] and the chunk's own
// keys; k_params non-null: the debiased variant (the history's K scale pairs)
bool tc_flash_supported(const kvc_layer_desc* d);
bool tc_flash_debiased_supported(const kvc_layer_desc* d, const kvc_predictor* p);
cudaError_t tc_flash(const kvc_layer_desc* d, const void* Q, int64_t n_q, const void* Kh, const void* Vh,
                     const void* K_self, const void* V_self, int64_t n_self, float scale, void* O,
                     const void* k_params, cudaStream_t st);
bool tc_mixed_supported(const kvc_layer_desc* d, const kvc_predictor* p);
size_t tc_mixed_workspace(const kvc_layer_desc* d, int64_t n_q);
cudaError_t tc_mixed_attend(const kvc_layer_desc* d, const kvc_predictor* p, const void* Q, int64_t n_q,
                            const kvc_codes* c, float scale, void* O, void* ws, size_t ws_bytes, cudaStream_t st);
bool tc_cluster_supported(const kvc_layer_desc* d, const kvc_predictor* p);
// P = C E^T of both tensors (K: [0], V: [1]) on the tensor cores, one launch;
// the encode of either tensor reads its P
cudaError_t tc_cluster_prepare(const kvc_layer_desc* d, const kvc_predictor* p, const float* const cnorm[2],
                               float* const P[2], cudaStream_t st);
// The token pass of both tensors (K: [0], V: [1]) in one launch
cudaError_t tc_cluster_encode(const kvc_layer_desc* d, const kvc_predictor* p, const void* const X[2],
                              const float* const cnorm[2], float* const P[2], void* const codes[2],
                              void* const params[2], void* const assign[2], cudaStream_t st);
// x^ = c_a + coef^ W_dec^T for each tensor whose out[w] is given, in one launch
cudaError_t tc_cluster_decode(const kvc_layer_desc* d, const kvc_predictor* p, const void* const codes[2],
                              const void* const params[2], const void* const assign[2], void* const out[2],
                              cudaStream_t st);
// The anchor layer (no predictor; bf16 values, fp16 (scale, zero), 2 or 4 bits,
// groups of 32 or 64): a streaming kernel over both tensors, sharing the
// quantizer arithmetic of the tensor-core epilogues (anchor.cu)
bool anchor_supported(const kvc_layer_desc* d, const kvc_predictor* p);
cudaError_t anchor_layer(const kvc_layer_desc* d, bool enc, const void* K, const void* V, const kvc_codes* c,
                         void* Kr, void* Vr, cudaStream_t st);
// reads the device error word of the current device and resets it to 0
cudaError_t tc_read_and_clear_error(unsigned int* value);
// device address of the error word on the current device (nullptr on failure)
unsigned int* tc_error_word();

}  // namespace kvc
