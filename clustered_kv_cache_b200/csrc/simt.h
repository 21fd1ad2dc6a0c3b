// Argument blocks and launchers of the CUDA-core kernels (internal).
#pragma once

#include "common.cuh"

namespace kvc {

// Z[t][j] = sum_c X[t][c] W[j][c] (fp32),  X[t] = [in0[t] | in1[t]] (in1 may be NULL)
template <typename TS>
struct LatentArgs {
  int64_t T;
  int C, r;
  const TS* in0;
  const TS* in1;
  const TS* W;  // [r][Cin]
  float* Z;     // [T][r]
};

// per (token, head) row: pred = [in0 | in1]_h block_h^T + Z U_h^T; encode or decode the residual
template <typename TS, typename TP>
struct HeadsArgs {
  int64_t T;
  int H, bits, group, r;
  const TS* in0;    // [T][H][D] (NULL with block == NULL)
  const TS* in1;    // [T][H][D] or NULL
  const TS* block;  // [H][D][Din] or NULL (no block term)
  const float* Z;   // [T][r] latent, fp32 (r > 0)
  const TS* U;      // [C][r]
  const TS* x;      // clean rows (encode)
  uint8_t* codes;   // [T][H][D*bits/8]
  Pair<TP>* params; // [T][H][D/group] (H64 / EDEN-2: [T][H][D/64] scales of type TP)
  TS* rec;          // [T][H][D] or NULL
  const float* codebook;  // H64 / EDEN-2 points [16][2], or NULL for the scalar quantizer
};

template <typename TS, typename TP>
struct TemporalArgs {
  int64_t T, F;
  int H, bits, anchor_bits, group;  // anchor_bits == 0: continue from ksrc / vsrc
  const TS* K;
  const TS* V;
  const TS* ksrc;  // [2][F][H][D] reconstructed K of the two frames before this call
  const TS* vsrc;  // [F][H][D] reconstructed V of the frame before this call
  const TS* ak;  // [H][D][2D]
  const TS* av;
  uint8_t* kcodes;
  Pair<TP>* kparams;
  uint8_t* vcodes;
  Pair<TP>* vparams;
  TS* krec;
  TS* vrec;
};

template <typename TS>
struct ClusterPrepArgs {
  int n_c, C, m;
  const TS* cent;  // [n_c][C]
  const TS* enc;   // [m][C]
  float* cnorm;    // [n_c]
  float* P;        // [n_c][m]
};

template <typename TS, typename TP>
struct ClusterArgs {
  int64_t T;
  int C, m, n_c, bits, group;
  const TS* X;      // [T][C] (encode)
  const TS* cent;   // [n_c][C]
  const TS* enc;    // [m][C]
  const TS* dec;    // [C][m]
  const float* cnorm;
  const float* P;
  uint8_t* codes;   // [T][m*bits/8]
  Pair<TP>* params; // [T][m/group]
  uint8_t* assign;  // [T]
  TS* rec;          // [T][C] or NULL
};

template <typename TS>
struct AttnArgs {
  int64_t n_q, n_hist, n_self;
  int H;
  int Hq;  // query heads, a multiple of H (Q and O are [n_q][Hq][D])
  float scale;
  const TS* Q;
  const TS* Kh;
  const TS* Vh;
  const TS* Ks;
  const TS* Vs;
  TS* O;
};

template <typename TS, typename TP>
struct MixedArgs {
  int64_t n_q, T;
  int H, D, C, n_c, bits, group;
  float scale;
  const TS* Q;
  const TS* cent_k;
  const TS* dec_k;  // [C][128]
  const TS* cent_v;
  const TS* dec_v;
  const uint8_t* codes_k;
  const Pair<TP>* params_k;
  const uint8_t* assign_k;
  const uint8_t* codes_v;
  const Pair<TP>* params_v;
  const uint8_t* assign_v;
  TS* O;
};

template <typename TS>
cudaError_t launch_latent(const LatentArgs<TS>& a, cudaStream_t st);
template <typename TS, typename TP>
cudaError_t launch_heads(const HeadsArgs<TS, TP>& a, int D, bool encode, cudaStream_t st);
template <typename TS, typename TP>
cudaError_t launch_temporal(const TemporalArgs<TS, TP>& a, int D, bool encode, cudaStream_t st);
template <typename TS>
cudaError_t launch_cluster_prep(const ClusterPrepArgs<TS>& a, cudaStream_t st);
template <typename TS>
cudaError_t launch_cluster_norms(const ClusterPrepArgs<TS>& a, cudaStream_t st);  // cnorm only
template <typename TS, typename TP>
cudaError_t launch_cluster(const ClusterArgs<TS, TP>& a, bool encode, cudaStream_t st);
template <typename TS>
cudaError_t launch_attention(const AttnArgs<TS>& a, int D, cudaStream_t st);
template <typename TS, typename TP>
cudaError_t launch_mixed_attention(const MixedArgs<TS, TP>& a, cudaStream_t st);
// video-adapted refit of the per-head blocks (refit.cu); X1 == NULL: the K block
size_t refit_workspace(int64_t T, int H, int D, int r, bool v);
template <typename TS>
cudaError_t launch_refit(int64_t T, int H, int D, int r, const TS* X0, const TS* X1, const TS* Y, const TS* W,
                         const TS* U, float ridge, TS* block, void* ws, cudaStream_t st);
cudaError_t launch_pack(const uint8_t* codes, int64_t n, int bits, void* packed, cudaStream_t st);
cudaError_t launch_unpack(const void* packed, int64_t n, int bits, uint8_t* codes, cudaStream_t st);

}  // namespace kvc
