/*
 * kvc.h - C ABI of libkvc.so, a predict-then-quantize-residual KV-cache codec
 * for autoregressive video diffusion, and attention over the compressed
 * history, written for NVIDIA B200 (sm_100a).
 *
 * What the codec computes (sources by page title and figure / table):
 *  - Every K/V row gets a prediction; only the residual (row - prediction) is
 *    stored, as b-bit codes with one (scale, zero) pair per group of `group`
 *    consecutive channels.  Scale s = (max - min) / (2^b - 1), zero z = min,
 *    code q = clamp(rint((r - z) / s), 0, 2^b - 1); the reconstruction is
 *    round_state(prediction + z + s*q).  ("CORAL-KV: Compact Cross-Layer
 *    Prediction and Residual Coding for Autoregressive Video KV Caches",
 *    Fig. 3 and Fig. 5; "TempoKV: Predictive KV Cache Quantization for
 *    Autoregressive Video Generation", Fig. 2(b), Tables 1-3.)
 *  - Predictions always use reconstructed, never clean, states (closed loop).
 *  - KVC_PRED_NONE: prediction 0 (the anchor: CORAL-KV layer 0, Fig. 8;
 *    TempoKV frame 0, appendix Table 7).
 *  - KVC_PRED_XLAYER_DPLR: K_l from the reconstructed K_{l-1}, V_l from the
 *    reconstructed [K_l, V_{l-1}], each by a per-head block-diagonal map plus
 *    a global rank-r map ("CORAL-KV ...", abstract and Fig. 3).
 *  - KVC_PRED_TEMPORAL: inside one layer, K of frame f from the reconstructed K
 *    of frames f-1 and f-2 at the same spatial position, V of frame f from the
 *    reconstructed K of frame f plus V of frame f-1 ("TempoKV ...", Fig. 2(b)).
 *    Frame 0 is coded with prediction 0 at anchor_bits; at frame 1 the missing
 *    lag-2 frame is zero.
 *  - KVC_PRED_CLUSTER: each token's whole (all heads) K row is predicted by its
 *    nearest centre c_a (ties to the lowest index); the residual is mapped to
 *    code_dim coefficients by an encoder, those are coded, and decoding is
 *    c_a + W_dec * coefficients ("NanoKV: High-Ratio KV Cache Compression for
 *    Autoregressive Video Generation", abstract).
 *
 * Conventions shared by every entry point:
 *  - Tensors are row-major.  K, V, Q, O and reconstructions are [T][H][D].
 *    Weights use the [out][in] convention, y = x * W^T.
 *  - Every pointer is caller-owned device memory unless stated otherwise;
 *    the library keeps no allocation between calls.  All device pointers must
 *    be 16-byte aligned (KVC_ERR_MISALIGNED otherwise).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Calls validate their arguments synchronously, enqueue work on `stream`
 *    and return; nothing is launched when validation fails.
 *  - Kernel launch failures return KVC_ERR_CUDA.  Kernels that wait on
 *    hardware barriers give up after a bounded time and record
 *    KVC_ERR_DEVICE_TIMEOUT in a device word read by kvc_get_device_error().
 */
#ifndef KVC_H
#define KVC_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVC_API __attribute__((visibility("default")))
#else
#define KVC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVC_OK = 0,
  KVC_ERR_INVALID_ARGUMENT = 1, /* NULL where a buffer is required, bad sizes */
  KVC_ERR_UNSUPPORTED = 2,      /* a combination the library does not implement */
  KVC_ERR_MISALIGNED = 3,       /* a device pointer not 16-byte aligned */
  KVC_ERR_WORKSPACE_TOO_SMALL = 4,
  KVC_ERR_CUDA = 5,             /* a CUDA runtime call or launch failed */
  KVC_ERR_DEVICE_TIMEOUT = 6    /* a bounded device-side wait gave up */
} kvc_status;

typedef enum { KVC_F32 = 0, KVC_BF16 = 1, KVC_F16 = 2 } kvc_dtype;

/* Residual codecs (kvc_layer_desc.residual_codec). */
typedef enum {
  KVC_RESIDUAL_RTN = 0,       /* scalar asymmetric group quantizer (the default) */
  KVC_RESIDUAL_H64_EDEN2 = 1  /* H64 Hadamard transform + EDEN-2 pair quantizer */
} kvc_residual_codec;

typedef enum {
  KVC_PRED_NONE = 0,
  KVC_PRED_XLAYER_DPLR = 1,
  KVC_PRED_TEMPORAL = 2,
  KVC_PRED_CLUSTER = 3
} kvc_pred_kind;

/* One layer's history.
 *  n_tokens T >= 0; n_heads H >= 1; head_dim D in {64, 128}.
 *  dtype: KVC_F32 or KVC_BF16; the type of K, V, Q, O, reconstructions and
 *         predictor weights.  Arithmetic accumulates in fp32.
 *  bits in {2, 4, 8}; group divides D (clustered: divides code_dim) and is a
 *         multiple of D/32.
 *  param_dtype: KVC_F16 or KVC_F32; the (scale, zero) storage type.
 *  frame_tokens: tokens per frame (temporal only; token t = f*frame_tokens+s).
 *  anchor_bits: temporal only: bits of frame 0, coded with prediction 0
 *         (2, 4 or 8); or 0 when the call continues a sequence, whose
 *         reconstructed history then arrives in K_src / V_src.
 *  residual_codec: KVC_RESIDUAL_RTN, or KVC_RESIDUAL_H64_EDEN2 ("CORAL-KV ...",
 *         Fig. 5, Fig. 9, Table 9): each group of 64 residual channels is
 *         multiplied by the orthonormal Sylvester Walsh-Hadamard matrix
 *         H64 / 8; its 32 pairs (y_2p, y_2p+1), normalised by
 *         sigma = sqrt(mean y^2), take the 4-bit index of the nearest of 16
 *         points (pred->residual_codebook; ties to the lowest index); one
 *         scale per group, S = |y|^2 / <y, c> (EDEN's unbiased scale, 0 when
 *         y = 0 or <y, c> <= 0), is stored in param_dtype; decoding applies
 *         H64 / 8 to S c.  Requires bits = 2 (4 bits per pair), group = 64 and
 *         KVC_PRED_NONE or KVC_PRED_XLAYER_DPLR; runs on the CUDA cores.
 *  q_heads: attention only: query heads, 0 (= n_heads) or a multiple of
 *         n_heads (grouped-query attention, as in MAGI-1's native GQA,
 *         "CORAL-KV ...", Table 3): query head j attends over the history of
 *         KV head j / (q_heads / n_heads); Q and O are then [n_q][q_heads][D]
 *         while the history, K_self and V_self keep n_heads.  Not for
 *         KVC_PRED_CLUSTER (KVC_ERR_UNSUPPORTED). */
typedef struct {
  int64_t n_tokens;
  int32_t n_heads;
  int32_t head_dim;
  int32_t dtype;
  int32_t bits;
  int32_t group;
  int32_t param_dtype;
  int32_t frame_tokens;
  int32_t anchor_bits;
  int32_t residual_codec;
  int32_t q_heads;
} kvc_layer_desc;

/* Predictor weights (device pointers, dtype of the layer, read only).
 *  XLAYER_DPLR: k_block [H][D][D], k_w [rank][C], k_u [C][rank],
 *               v_block [H][D][2D] over the per-head input [K_l,h | V_{l-1},h],
 *               v_w [rank][2C] over [K_l | V_{l-1}], v_u [C][rank];
 *               C = H*D; rank may be 0 (then k_w, k_u, v_w, v_u may be NULL).
 *  TEMPORAL:    k_block [H][D][2D] over [K_{f-1},h | K_{f-2},h],
 *               v_block [H][D][2D] over [K_f,h | V_{f-1},h].
 *  CLUSTER:     k_centroids [n_clusters][C], k_enc [code_dim][C],
 *               k_dec [C][code_dim], and the same for v; n_clusters <= 256.
 *  residual_codebook: with KVC_RESIDUAL_H64_EDEN2, the 16 two-dimensional
 *               points as fp32 [16][2] (device memory); else ignored. */
typedef struct {
  int32_t kind;
  int32_t rank;
  int32_t n_clusters;
  int32_t code_dim;
  const void *k_block, *k_w, *k_u;
  const void *v_block, *v_w, *v_u;
  const void *k_centroids, *k_enc, *k_dec;
  const void *v_centroids, *v_enc, *v_dec;
  const void* residual_codebook;
} kvc_predictor;

/* Compressed storage of one layer (device pointers, caller-owned).
 *  NONE / XLAYER: k_codes [T][H][D*bits/8] bytes, k_params [T][H][D/group][2]
 *    of (scale, zero) in param_dtype; element j of a row sits at bits
 *    [j*bits, (j+1)*bits) of the row, least significant bit first.
 *  TEMPORAL: as above, except that (unless anchor_bits is 0) the rows of
 *    frame 0 come first at anchor_bits, followed by the rows of all later
 *    frames at bits.
 *  CLUSTER: k_codes [T][code_dim*bits/8], k_params [T][code_dim/group][2],
 *    k_assign [T] uint8 centre index.
 *  H64 / EDEN-2 residuals: k_codes [T][H][D/4] bytes, pair p's index at bits
 *    [4p, 4p+4) of the row, least significant first; k_params [T][H][D/64]
 *    scales in param_dtype (one value per group, no zero-point).
 *  The v_* members hold V the same way.  Sizes: kvc_codes_sizes(). */
typedef struct {
  void *k_codes, *k_params, *v_codes, *v_params;
  void *k_assign, *v_assign;
} kvc_codes;

/* Bytes of each buffer of kvc_codes for one tensor (K; V is the same). */
typedef struct {
  size_t codes;
  size_t params;
  size_t assign;
} kvc_codes_size;

/* Closed-form storage of one tensor's codes, parameters and assignments.
 * Returns KVC_ERR_INVALID_ARGUMENT / KVC_ERR_UNSUPPORTED for bad descriptors.
 * The ratio 16 / (bits + 32/group) of bf16 data to INT-b codes with fp16
 * (scale, zero) pairs is the 5.33x (INT2) / 3.20x (INT4) of "TempoKV ...",
 * Tables 1-3 and appendix Table 8. */
KVC_API kvc_status kvc_codes_sizes(const kvc_layer_desc* desc, const kvc_predictor* pred, kvc_codes_size* out);

/* Total bytes (K and V) of codes + parameters + assignments of one layer;
 * 0 for an invalid descriptor. */
KVC_API size_t kvc_codes_bytes(const kvc_layer_desc* desc, const kvc_predictor* pred);

/* Operation codes of kvc_workspace_bytes. */
enum { KVC_OP_ENCODE = 0, KVC_OP_DECODE = 1, KVC_OP_ATTEND = 2, KVC_OP_REFIT_K = 3, KVC_OP_REFIT_V = 4 };

/* Device workspace (bytes) that `op` needs for this layer; n_q = number of
 * query rows (attend only).  The caller passes a buffer of at least this size
 * as `ws`; its contents are scratch and need no initialisation. */
KVC_API size_t kvc_workspace_bytes(int op, const kvc_layer_desc* desc, const kvc_predictor* pred, int64_t n_q);

/* Encode one layer: prediction, residual, group quantization, packing, and the
 * closed-loop reconstruction.
 *  K, V:         [T][H][D] clean values of this layer (read).
 *  K_src, V_src: XLAYER: reconstructions of layer l-1 [T][H][D] (read).
 *                TEMPORAL with anchor_bits == 0: the reconstructed K of the
 *                two frames before this call, [2][frame_tokens][H][D] (older
 *                first), and the reconstructed V of the frame before,
 *                [frame_tokens][H][D].  Otherwise ignored (may be NULL).
 *  out:          codes / params / assignments (written).
 *  K_rec, V_rec: reconstructions of this layer (written); may be NULL unless
 *                the caller chains them into the next layer, except that
 *                XLAYER needs K_rec (V's prediction reads the reconstructed K).
 *  ws, ws_bytes: workspace of kvc_workspace_bytes(KVC_OP_ENCODE, ...).
 * T = 0 is a no-op.  For temporal layers the whole frame chain of the call
 * runs inside it, in time order. */
KVC_API kvc_status kvc_encode_layer(const kvc_layer_desc* desc, const kvc_predictor* pred, const void* K,
                            const void* V, const void* K_src, const void* V_src, const kvc_codes* out,
                            void* K_rec, void* V_rec, void* ws, size_t ws_bytes, void* stream);

/* Decode one layer: unpack, dequantize, replay the same prediction chain and
 * add; K_rec and V_rec [T][H][D] are required.  K_src / V_src as for encode. */
KVC_API kvc_status kvc_decode_layer(const kvc_layer_desc* desc, const kvc_predictor* pred, const kvc_codes* codes,
                            const void* K_src, const void* V_src, void* K_rec, void* V_rec, void* ws,
                            size_t ws_bytes, void* stream);

/* A chain of n_layers predicted (KVC_PRED_XLAYER_DPLR) layers in one call
 * ("CORAL-KV ...", Fig. 3: layer l predicts from the reconstruction of layer
 * l-1).  Layer i of the call (0-based) predicts from the reconstruction of layer
 * i-1, or from K_src / V_src [T][H][D] for i = 0, and writes its own to
 * K_rec[i] / V_rec[i] [T][H][D] (all required).  Results are identical, byte for
 * byte, to n_layers kvc_encode_layer / kvc_decode_layer calls in order.
 *  desc:          shared by every layer; preds[i], out[i] / codes[i] (arrays of
 *                 n_layers) are layer i's predictor and codes; K[i], V[i] its
 *                 clean values (encode).
 *  K_rec, V_rec:  arrays of n_layers device pointers.  K_rec[i] may be the
 *                 buffer of layer i-2 (two buffers in turn suffice) but not of
 *                 layer i-1 (its source); KVC_ERR_INVALID_ARGUMENT otherwise.
 *  ws, ws_bytes:  kvc_layers_workspace_bytes(KVC_OP_ENCODE or KVC_OP_DECODE,
 *                 desc, preds, n_layers).  It holds the call's layer table and
 *                 its per-tile counters, so calls in flight at the same time
 *                 need workspaces of their own.
 * A device wait that runs out (bounded, about two seconds) ends the launch and
 * is reported by kvc_get_device_error as KVC_ERR_DEVICE_TIMEOUT.
 * With bf16, head_dim 128, scalar residual codes and equal ranks in {0, 64,
 * 128} the call is one persistent tensor-core launch that walks (layer, token
 * tile) items in layer order; the tile of layer i waits (bounded) for the same
 * tile of layer i-1, so the layers' wave tails overlap.  Other shapes run the
 * layers in turn.  The INT4 anchor layer is a separate kvc_encode_layer. */
KVC_API kvc_status kvc_encode_layers(const kvc_layer_desc* desc, const kvc_predictor* preds, int n_layers,
                                     const void* const* K, const void* const* V, const void* K_src,
                                     const void* V_src, const kvc_codes* out, void* const* K_rec,
                                     void* const* V_rec, void* ws, size_t ws_bytes, void* stream);
KVC_API kvc_status kvc_decode_layers(const kvc_layer_desc* desc, const kvc_predictor* preds, int n_layers,
                                     const kvc_codes* codes, const void* K_src, const void* V_src,
                                     void* const* K_rec, void* const* V_rec, void* ws, size_t ws_bytes,
                                     void* stream);
/* Workspace bytes of kvc_encode_layers (op KVC_OP_ENCODE) or kvc_decode_layers
 * (KVC_OP_DECODE); 0 for an invalid description. */
KVC_API size_t kvc_layers_workspace_bytes(int op, const kvc_layer_desc* desc, const kvc_predictor* preds,
                                          int n_layers);

/* Softmax attention of Q [n_q][H][D] (H = desc->q_heads when set) over this layer's compressed history,
 * followed by n_self uncompressed tokens K_self / V_self [n_self][H][D]
 * (non-causal; n_self may be 0 and the pointers NULL):
 *   O = softmax(scale * Q [K_hist; K_self]^T) [V_hist; V_self].
 * NONE / XLAYER: the history is decoded once (the codec's decode, into
 * K_rec_opt / V_rec_opt when given, else into the workspace) and attended with
 * the chunk's own keys (bf16, D = 128: a tensor-core flash attention).  CLUSTER:
 * scores and values are computed on the stored coefficients, q.c_a +
 * (W_dec^T q).coef, without rebuilding full keys ("NanoKV ...", abstract: the
 * Fast variant); n_self must be 0.  TEMPORAL: KVC_ERR_UNSUPPORTED.
 * O [n_q][H][D] is written.
 *  K_rec_opt, V_rec_opt: optional [T][H][D] outputs (NULL = not wanted) that
 *    receive the decoded history, the same values kvc_decode_layer writes,
 *    e.g. as the next layer's K_src / V_src; CLUSTER runs its decode for them.
 *    With n_q = 0 the call does nothing at all (kvc_decode_layer decodes a
 *    history alone). */
KVC_API kvc_status kvc_attend_compressed(const kvc_layer_desc* desc, const kvc_predictor* pred, const void* Q,
                                 int64_t n_q, const kvc_codes* codes, const void* K_src, const void* V_src,
                                 const void* K_self, const void* V_self, int64_t n_self, float scale,
                                 void* O, void* K_rec_opt, void* V_rec_opt, void* ws, size_t ws_bytes,
                                 void* stream);

/* kvc_attend_compressed with the Jensen-bias correction of the quantized
 * history (the abstract on the "Jensen bias" of INT2 key caches, among the
 * related papers listed on the "CORAL-KV ..." page): quantization noise on a
 * cached key inflates E[exp(score)], so history keys steal attention mass from
 * the uncompressed chunk.  Each history key t's score (never a K_self key's) is
 * lowered, for each query and head, by
 *     0.5 * scale^2 * sum_g |q_g|^2 * s_{t,g}^2 / 12,
 * g over the key row's quantization groups, q_g the query's channels of group
 * g and s_{t,g} the stored residual scale: the second-order exponent of a
 * uniform rounding error of step s, which the correction removes in
 * expectation.  It reads only the stored scales (no extra memory).  Same
 * arguments and outputs as kvc_attend_compressed; implemented for the
 * tensor-core attention over a cross-layer history with scalar residual codes
 * (KVC_PRED_XLAYER_DPLR, KVC_RESIDUAL_RTN, bf16, head_dim 128, fp16 params,
 * group 32 or 64, T > 0); other layers return KVC_ERR_UNSUPPORTED. */
KVC_API kvc_status kvc_attend_compressed_debiased(const kvc_layer_desc* desc, const kvc_predictor* pred,
                                                  const void* Q, int64_t n_q, const kvc_codes* codes,
                                                  const void* K_src, const void* V_src, const void* K_self,
                                                  const void* V_self, int64_t n_self, float scale, void* O,
                                                  void* K_rec_opt, void* V_rec_opt, void* ws, size_t ws_bytes,
                                                  void* stream);

/* Video-adapted block-DPLR refit ("CORAL-KV ...", Fig. 4: the low-rank
 * factors stay fixed and the per-head block-diagonal terms are refitted for
 * each filled cache block): for each head h,
 *     block_h^T = (X_h^T X_h + ridge I)^{-1} X_h^T (Y_h - LR_h)
 * over the desc->n_tokens tokens of the block, LR the fixed low-rank term
 * (X_flat W^T) U^T of pred (rank may be 0).
 *  tensor 0 (K): X0 = K^_{l-1} [T][H][D] (X1 ignored), Y = K_l, W/U = k_w/k_u;
 *                block_out [H][D][D] (a k_block).
 *  tensor 1 (V): X0 = K^_l, X1 = V^_{l-1} [T][H][D], Y = V_l, W/U = v_w/v_u;
 *                block_out [H][D][2D] (a v_block).
 * Since V's input is the reconstructed K of the same layer, a video-adapted
 * layer refits K, encodes (for K^_l), refits V, and encodes again.  Computed in
 * fp32 on the CUDA cores (Gram matrices, then a Cholesky solve per head) and
 * written in the layer dtype; ridge >= 0 must make X_h^T X_h + ridge I
 * positive definite.  KVC_PRED_XLAYER_DPLR only; ws of
 * kvc_workspace_bytes(KVC_OP_REFIT_K / KVC_OP_REFIT_V, ...). */
KVC_API kvc_status kvc_refit_block_diag(const kvc_layer_desc* desc, const kvc_predictor* pred, int tensor,
                                        const void* X0, const void* X1, const void* Y, float ridge, void* block_out,
                                        void* ws, size_t ws_bytes, void* stream);

/* Pack n codes (uint8, each < 2^bits) into n*bits/8 bytes, LSB first;
 * n*bits must be a multiple of 128 (whole 16-byte words). */
KVC_API kvc_status kvc_pack_codes(const uint8_t* codes, int64_t n, int bits, void* packed, void* stream);

/* Inverse of kvc_pack_codes. */
KVC_API kvc_status kvc_unpack_codes(const void* packed, int64_t n, int bits, uint8_t* codes, void* stream);

/* Host <-> device copies for callers that keep the cache's inputs and codes in
 * host memory: one stream-ordered cudaMemcpyAsync of `bytes` bytes (pinned
 * host memory makes it asynchronous).  dst / src: device and host pointers as
 * the names say; KVC_ERR_INVALID_ARGUMENT for NULL pointers with bytes > 0. */
KVC_API kvc_status kvc_copy_to_device(void* dst_device, const void* src_host, size_t bytes, void* stream);
KVC_API kvc_status kvc_copy_to_host(void* dst_host, const void* src_device, size_t bytes, void* stream);

/* Synchronizes `stream`, returns the first device-side error recorded since
 * the last call (KVC_OK if none) and clears it. */
KVC_API kvc_status kvc_get_device_error(void* stream);

/* Static description of a status code. */
KVC_API const char* kvc_status_string(kvc_status status);

/* Text of the last CUDA error seen by this thread's calls (or ""). */
KVC_API const char* kvc_last_cuda_error(void);

/* Number of kernels this process has launched through the library so far
 * (all threads, all devices); for counting launches in a timed region. */
KVC_API uint64_t kvc_launch_counter(void);

/* kvc_encode_layer for the clustered predictor, for callers that cannot
 * allocate device memory when they encode (code inside an allocator or memory
 * pool callback, a runtime that hands out pre-carved device memory, a plugin
 * host that forbids cudaMalloc on its threads).  The pages have no counterpart:
 * this is an interface choice of this library.
 *  Same meaning, layouts and results as kvc_encode_layer with
 *  pred->kind == KVC_PRED_CLUSTER (no K_src / V_src, no workspace); K_rec and
 *  V_rec may be NULL.
 *  The centre tables it needs live in a file-scope __device__ array sized for
 *  at most 256 centres of 128 coefficients (about 264 KB, held by every GPU that
 *  loads the library until the process exits); larger n_clusters or another
 *  code_dim return KVC_ERR_UNSUPPORTED before anything runs.
 *  It calls no cudaMalloc / cudaFree.  The first call on a device (and the
 *  first after that device's context was replaced, e.g. by cudaDeviceReset)
 *  looks up the array's device address (cudaGetSymbolAddress), so make that
 *  first call before any stream capture.  Every call writes the whole table before
 *  reading it, so nothing carries over between calls, but all calls share the
 *  one array: calls that can overlap on the GPU (other streams, other threads)
 *  race and must be serialized by the caller. */
KVC_API kvc_status kvc_encode_layer_cluster_static(const kvc_layer_desc* desc, const kvc_predictor* pred,
                                                   const void* K, const void* V, const kvc_codes* out,
                                                   void* K_rec, void* V_rec, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KVC_H */
