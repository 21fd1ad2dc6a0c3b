// Video-adapted block-DPLR refit ("CORAL-KV: Compact Cross-Layer Prediction and
// Residual Coding for Autoregressive Video KV Caches", Fig. 4: the
// video-adapted predictor keeps its low-rank factors fixed and refits the
// per-head block-diagonal terms for each filled cache block).  Each head's
// block is the ridge least-squares fit
//     B_h^T = (X_h^T X_h + ridge I)^{-1} X_h^T (Y_h - LR_h)
// of the target left after the fixed low-rank term LR = (X_flat W^T) U^T, over
// the block's tokens; X_h is the head's predictor input (K: K^_{l-1,h};
// V: [K^_{l,h} | V^_{l-1,h}]).
//
// Three CUDA-core kernels (fp32):
//  1. refit_residual_kernel: R = Y - Z U_h^T per (token tile, head), with the
//     latent Z = X_flat W^T from latent_kernel;
//  2. refit_gram_kernel: per (head, 64 x 64 tile, token split), the partial sums
//     over the split's tokens of x x^T (the Gram matrix, columns < din) and of
//     x R^T (the right-hand sides, columns >= din);
//  3. refit_solve_kernel: one CTA per head sums the splits in a fixed order,
//     factors G + ridge I = L L^T in shared memory (packed lower triangle) and
//     solves for the D right-hand sides in chunks of 32 columns.
// The splits are summed in a fixed order, so the result does not depend on
// scheduling.
#include "common.cuh"
#include "simt.h"

namespace kvc {
namespace {

constexpr int kRefitThreads = 256;
constexpr int kSplits = 8;  // token splits of the Gram sums

__host__ __device__ inline int64_t tri(int i, int j) { return (int64_t)i * (i + 1) / 2 + j; }

// R[t][h][o] = Y[t][h][o] - sum_j Z[t][j] U[h D + o][j] (r == 0: R = Y)
template <typename TS>
__global__ void __launch_bounds__(kRefitThreads) refit_residual_kernel(int64_t T, int H, int D, int r,
                                                                       const float* Z, const TS* U, const TS* Y,
                                                                       float* R) {
  extern __shared__ float sm[];
  float* sZ = sm;           // [32][r]
  float* sU = sZ + 32 * r;  // [D][r + 1]
  const int h = blockIdx.y;
  const int64_t t0 = (int64_t)blockIdx.x * 32;
  for (int i = threadIdx.x; i < 32 * r; i += blockDim.x) {
    const int64_t t = t0 + i / r;
    sZ[i] = t < T ? Z[t * r + i % r] : 0.f;
  }
  for (int i = threadIdx.x; i < D * r; i += blockDim.x) sU[(i / r) * (r + 1) + i % r] = to_f(U[((int64_t)h * D + i / r) * r + i % r]);
  __syncthreads();
  for (int i = threadIdx.x; i < 32 * D; i += blockDim.x) {
    const int tt = i / D, o = i % D;
    const int64_t t = t0 + tt;
    if (t >= T) continue;
    float acc = 0.f;
    for (int j = 0; j < r; ++j) acc = fmaf(sZ[tt * r + j], sU[o * (r + 1) + j], acc);
    const int64_t e = (t * H + h) * D + o;
    R[e] = to_f(Y[e]) - acc;
  }
}

// Partial sums over the tokens of split s of P[m][n] = sum_t x_t[m] b_t[n], with
// x_t = [X0[t][h] | X1[t][h]] (din values) and b_t = [x_t | R[t][h]]; one CTA per
// (64 x 64 tile of P, head, split).
template <typename TS>
__global__ void __launch_bounds__(kRefitThreads) refit_gram_kernel(int64_t T, int H, int D, int din, const TS* X0,
                                                                   const TS* X1, const float* R, float* part) {
  __shared__ float sA[32][64 + 1];
  __shared__ float sB[32][64 + 1];
  const int nt_n = (din + D) / 64;
  const int m0 = (blockIdx.x / nt_n) * 64, n0 = (blockIdx.x % nt_n) * 64;
  const int h = blockIdx.y, s = blockIdx.z;
  const int64_t per = (T + kSplits - 1) / kSplits;
  const int64_t ta = (int64_t)s * per, tb = ta + per < T ? ta + per : T;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;  // 16 x 16 threads, 4 x 4 outputs each
  auto xin = [&](int64_t t, int m) -> float {
    const int64_t row = t * H + h;
    return m < D ? to_f(X0[row * D + m]) : to_f(X1[row * D + (m - D)]);
  };
  auto bin = [&](int64_t t, int n) -> float { return n < din ? xin(t, n) : R[(t * H + h) * D + (n - din)]; };
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int64_t tc = ta; tc < tb; tc += 32) {
    for (int i = threadIdx.x; i < 32 * 64; i += blockDim.x) {
      const int k = i / 64, c = i % 64;
      const int64_t t = tc + k;
      const bool ok = t < tb;
      sA[k][c] = ok ? xin(t, m0 + c) : 0.f;
      sB[k][c] = ok ? bin(t, n0 + c) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < 32; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = sA[k][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = sB[k][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* P = part + (((int64_t)s * H + h) * din) * (din + D);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) P[(int64_t)(m0 + ty * 4 + i) * (din + D) + n0 + tx * 4 + j] = acc[i][j];
}

// One CTA per head: G = sum of the splits + ridge I, its Cholesky factor in
// shared memory (packed lower triangle), then the D right-hand sides in chunks
// of 32 columns (8 threads per column), written to block[h][o][:].
template <typename TS>
__global__ void __launch_bounds__(kRefitThreads) refit_solve_kernel(int H, int D, int din, float ridge,
                                                                    const float* part, TS* block) {
  extern __shared__ float sm[];
  float* L = sm;                    // packed lower triangle, din (din + 1) / 2
  float* Bc = L + tri(din, 0);      // [din][32] right-hand sides, then solutions
  const int h = blockIdx.x;
  const int ncol = din + D;
  auto psum = [&](int i, int n) {
    float v = 0.f;
    for (int s = 0; s < kSplits; ++s) v += part[(((int64_t)s * H + h) * din + i) * ncol + n];
    return v;
  };
  for (int64_t e = threadIdx.x; e < tri(din, 0); e += blockDim.x) {
    // row i of the packed index e: the largest i with i (i + 1) / 2 <= e
    int i = (int)((sqrtf(8.f * (float)e + 1.f) - 1.f) * 0.5f);
    while (tri(i + 1, 0) <= e) ++i;
    while (tri(i, 0) > e) --i;
    const int j = (int)(e - tri(i, 0));
    L[e] = psum(i, j) + (i == j ? ridge : 0.f);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // right-looking Cholesky
  for (int j = 0; j < din; ++j) {
    if (threadIdx.x == 0) L[tri(j, j)] = sqrtf(L[tri(j, j)]);
    __syncthreads();
    const float ljj = L[tri(j, j)];
    for (int i = j + 1 + threadIdx.x; i < din; i += blockDim.x) L[tri(i, j)] /= ljj;
    __syncthreads();
    for (int i = j + 1 + warp; i < din; i += kRefitThreads / 32) {
      const float lij = L[tri(i, j)];
      for (int k = j + 1 + lane; k <= i; k += 32) L[tri(i, k)] -= lij * L[tri(k, j)];
    }
    __syncthreads();
  }
  // 32 columns per chunk; column c of the chunk owned by the 8 threads 8c .. 8c + 7
  const int c = threadIdx.x >> 3, sub = threadIdx.x & 7;
  const unsigned gmask = 0xffu << ((threadIdx.x & 31) & ~7);
  for (int o0 = 0; o0 < D; o0 += 32) {
    for (int i = threadIdx.x; i < din * 32; i += blockDim.x) Bc[i] = psum(i / 32, din + o0 + i % 32);
    __syncthreads();
    // forward: L z = b
    for (int i = 0; i < din; ++i) {
      float v = 0.f;
      for (int k = sub; k < i; k += 8) v = fmaf(L[tri(i, k)], Bc[k * 32 + c], v);
#pragma unroll
      for (int o = 4; o; o >>= 1) v += __shfl_xor_sync(gmask, v, o);
      if (sub == 0) Bc[i * 32 + c] = (Bc[i * 32 + c] - v) / L[tri(i, i)];
      __syncwarp();
    }
    // backward: L^T x = z
    for (int i = din - 1; i >= 0; --i) {
      float v = 0.f;
      for (int k = i + 1 + sub; k < din; k += 8) v = fmaf(L[tri(k, i)], Bc[k * 32 + c], v);
#pragma unroll
      for (int o = 4; o; o >>= 1) v += __shfl_xor_sync(gmask, v, o);
      if (sub == 0) Bc[i * 32 + c] = (Bc[i * 32 + c] - v) / L[tri(i, i)];
      __syncwarp();
    }
    __syncthreads();
    for (int i = threadIdx.x; i < din * 32; i += blockDim.x) {
      const int o = o0 + i / din, k = i % din;
      block[((int64_t)h * D + o) * din + k] = from_f<TS>(Bc[k * 32 + (i / din)]);
    }
    __syncthreads();
  }
}

}  // namespace

size_t refit_workspace(int64_t T, int H, int D, int r, bool v) {
  const int din = v ? 2 * D : D;
  auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  return a256((size_t)T * (r > 0 ? r : 1) * 4) + a256((size_t)T * H * D * 4) +
         a256((size_t)kSplits * H * din * (din + D) * 4);
}

template <typename TS>
cudaError_t launch_refit(int64_t T, int H, int D, int r, const TS* X0, const TS* X1, const TS* Y, const TS* W,
                         const TS* U, float ridge, TS* block, void* ws, cudaStream_t st) {
  const bool v = X1 != nullptr;
  const int din = v ? 2 * D : D, C = H * D;
  auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  char* w = static_cast<char*>(ws);
  float* Z = reinterpret_cast<float*>(w);
  float* R = reinterpret_cast<float*>(w + a256((size_t)T * (r > 0 ? r : 1) * 4));
  float* part = reinterpret_cast<float*>(reinterpret_cast<char*>(R) + a256((size_t)T * H * D * 4));
  cudaError_t e;
  if (r > 0) {
    LatentArgs<TS> la{T, C, r, X0, X1, W, Z};
    if ((e = launch_latent(la, st)) != cudaSuccess) return e;
  }
  {
    const size_t smem = (size_t)(32 * r + D * (r + 1)) * sizeof(float);
    auto k = refit_residual_kernel<TS>;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
      return e;
    k<<<dim3((unsigned)((T + 31) / 32), (unsigned)H), kRefitThreads, smem, st>>>(T, H, D, r, Z, U, Y, R);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    const unsigned tiles = (unsigned)((din / 64) * ((din + D) / 64));
    refit_gram_kernel<TS><<<dim3(tiles, (unsigned)H, kSplits), kRefitThreads, 0, st>>>(T, H, D, din, X0, X1, R, part);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    const size_t smem = (size_t)(tri(din, 0) + din * 32) * sizeof(float);
    auto k = refit_solve_kernel<TS>;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
      return e;
    k<<<(unsigned)H, kRefitThreads, smem, st>>>(H, D, din, ridge, part, block);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template cudaError_t launch_refit<float>(int64_t, int, int, int, const float*, const float*, const float*,
                                         const float*, const float*, float, float*, void*, cudaStream_t);
template cudaError_t launch_refit<__nv_bfloat16>(int64_t, int, int, int, const __nv_bfloat16*,
                                                 const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*,
                                                 const __nv_bfloat16*, float, __nv_bfloat16*, void*, cudaStream_t);

}  // namespace kvc
