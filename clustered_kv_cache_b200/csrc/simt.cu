// CUDA-core (FMA) kernels of the codec and of attention over the compressed
// history.  They serve every shape and both state dtypes (fp32 data must not be
// rounded to TF32, so the fp32 path lives here); the bf16 / D = 128 hot path
// has tensor-core kernels of its own.
//
// Every kernel runs 256 threads.  Tiles are 32 tokens; the small GEMMs share
// one FMA tile routine (gemm_tile) that stages 32-wide K slices of both
// operands in shared memory.
#include "common.cuh"
#include "simt.h"

namespace kvc {

constexpr int kThreads = 256;

// acc[i][j] += sum_k A(row = ty*4 + i, k) * W(row = tx + 32*j, k), k < K.
// sA holds [32][33] floats, sW [32*NJ][33].
template <int NJ, class LA, class LW>
__device__ __forceinline__ void gemm_tile(float (&acc)[4][NJ], int K, const LA& la, const LW& lw, float* sA,
                                          float* sW) {
  const int tid = threadIdx.x, tx = tid & 31, ty = tid >> 5;
  for (int k0 = 0; k0 < K; k0 += 32) {
    __syncthreads();
    for (int e = tid; e < 32 * 32; e += kThreads) {
      const int row = e >> 5, col = e & 31;
      sA[row * 33 + col] = (k0 + col < K) ? la(row, k0 + col) : 0.f;
    }
    for (int e = tid; e < 32 * NJ * 32; e += kThreads) {
      const int row = e >> 5, col = e & 31;
      sW[row * 33 + col] = (k0 + col < K) ? lw(row, k0 + col) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      float a[4], w[NJ];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = sA[(ty * 4 + i) * 33 + kk];
#pragma unroll
      for (int j = 0; j < NJ; ++j) w[j] = sW[(tx + 32 * j) * 33 + kk];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < NJ; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
  }
  __syncthreads();
}

template <int NJ>
__device__ __forceinline__ void zero_acc(float (&acc)[4][NJ]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < NJ; ++j) acc[i][j] = 0.f;
}

// ============================================================== latent z = x W^T (fp32, not rounded)

template <typename TS, int NJ>
__global__ void __launch_bounds__(kThreads) latent_kernel(LatentArgs<TS> a) {
  extern __shared__ float smem[];
  float* sA = smem;
  float* sW = sA + 32 * 33;
  const int64_t t0 = (int64_t)blockIdx.x * 32;
  const int C = a.C;
  const int Cin = a.in1 ? 2 * C : C;
  float acc[4][NJ];
  zero_acc(acc);
  auto la = [&](int row, int k) -> float {
    const int64_t t = t0 + row;
    if (t >= a.T) return 0.f;
    return k < C ? to_f(a.in0[t * C + k]) : to_f(a.in1[t * C + (k - C)]);
  };
  auto lw = [&](int row, int k) -> float { return row < a.r ? to_f(a.W[(int64_t)row * Cin + k]) : 0.f; };
  gemm_tile<NJ>(acc, Cin, la, lw, sA, sW);
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t t = t0 + ty * 4 + i;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int jj = tx + 32 * j;
      if (t < a.T && jj < a.r) a.Z[t * a.r + jj] = acc[i][j];
    }
  }
}

// ============================================================== H64 / EDEN-2 rows
//
// "CORAL-KV: Compact Cross-Layer Prediction and Residual Coding for
// Autoregressive Video KV Caches", Fig. 5 (H_n on each non-overlapping group of
// n residual channels; one shared scale per 64 values) and Fig. 9 (16 EDEN-2
// points over pairs of H64-transformed residuals).  A row of D = 32 E values
// is held by a warp, lane l holding elements [l E, (l + 1) E); a 64-channel
// group spans 64 / E lanes.  The orthonormal Walsh-Hadamard transform
// y_i = (1/8) sum_j (-1)^popcount(i & j) r_j runs as six butterfly stages, the
// low log2(E) index bits inside a lane and the others across lanes by xor
// shuffles.  Pairs (y_2p, y_2p+1) sit inside a lane.

template <int E>
__device__ __forceinline__ void walsh64(float (&v)[E]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int b = 1; b < E; b <<= 1)  // index bits inside the lane
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (!(e & b)) {
        const float a = v[e], c = v[e + b];
        v[e] = a + c;
        v[e + b] = a - c;
      }
#pragma unroll
  for (int o = 1; o < 64 / E; o <<= 1) {  // index bits across lanes
    const bool upper = lane & o;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float w = __shfl_xor_sync(0xffffffffu, v[e], o);
      v[e] = upper ? w - v[e] : v[e] + w;
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) v[e] *= 0.125f;
}

// sum over the lanes of this lane's 64-channel group
template <int E>
__device__ __forceinline__ float group_sum64(float x) {
#pragma unroll
  for (int o = 1; o < 64 / E; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Encodes the residual r of this lane's elements; writes the pair indices and
// the group scale, returns the decoded residual in rh.  cb: 16 points in
// shared memory.
template <int E, typename TP>
__device__ __forceinline__ void eden2_encode(const float (&r)[E], const float* cb, uint8_t* row_codes,
                                             TP* row_scales, float (&rh)[E]) {
  static_assert(E % 2 == 0, "pairs inside a lane");
  const int lane = threadIdx.x & 31;
  float y[E];
#pragma unroll
  for (int e = 0; e < E; ++e) y[e] = r[e];
  walsh64<E>(y);
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) ss = fmaf(y[e], y[e], ss);
  const float sumsq = group_sum64<E>(ss);
  int k[E / 2];
  float dot = 0.f;
  const float inv_sigma = sumsq > 0.f ? 1.f / sqrtf(sumsq * (1.f / 64.f)) : 0.f;
#pragma unroll
  for (int i = 0; i < E / 2; ++i) {
    const float u0 = y[2 * i] * inv_sigma, u1 = y[2 * i + 1] * inv_sigma;
    int best = 0;
    float bd = INFINITY;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float d0 = u0 - cb[2 * j], d1 = u1 - cb[2 * j + 1];
      const float d = fmaf(d0, d0, d1 * d1);
      if (d < bd) {  // strict: ties keep the lowest index
        bd = d;
        best = j;
      }
    }
    k[i] = sumsq > 0.f ? best : 0;
    dot = fmaf(y[2 * i], cb[2 * k[i]], fmaf(y[2 * i + 1], cb[2 * k[i] + 1], dot));
  }
  dot = group_sum64<E>(dot);
  const TP S = from_f<TP>(sumsq > 0.f && dot > 0.f ? sumsq / dot : 0.f);
  const float sf = to_f(S);
  if ((lane % (64 / E)) == 0) row_scales[lane / (64 / E)] = S;
  // indices: pair p of the row at bits [4p, 4p + 4); this lane holds pairs lane E/2 + i
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < E / 2; ++i) w |= (uint32_t)k[i] << (4 * i);
  if (E >= 4) {
    if (E == 4) row_codes[lane] = (uint8_t)w;
    else *reinterpret_cast<uint16_t*>(row_codes + lane * (E / 4)) = (uint16_t)w;
  } else {  // one pair per lane: two lanes per byte
    const uint32_t hi = __shfl_xor_sync(0xffffffffu, w, 1);
    if (!(lane & 1)) row_codes[lane / 2] = (uint8_t)(w | (hi << 4));
  }
#pragma unroll
  for (int i = 0; i < E / 2; ++i) {
    rh[2 * i] = sf * cb[2 * k[i]];
    rh[2 * i + 1] = sf * cb[2 * k[i] + 1];
  }
  walsh64<E>(rh);
}

template <int E, typename TP>
__device__ __forceinline__ void eden2_decode(const uint8_t* row_codes, const TP* row_scales, const float* cb,
                                             float (&rh)[E]) {
  const int lane = threadIdx.x & 31;
  uint32_t w;
  if (E == 4) w = row_codes[lane];
  else if (E > 4) w = *reinterpret_cast<const uint16_t*>(row_codes + lane * (E / 4));
  else w = (uint32_t)row_codes[lane / 2] >> ((lane & 1) * 4);
  const float sf = to_f(row_scales[lane / (64 / E)]);
#pragma unroll
  for (int i = 0; i < E / 2; ++i) {
    const int k = (w >> (4 * i)) & 15;
    rh[2 * i] = sf * cb[2 * k];
    rh[2 * i + 1] = sf * cb[2 * k + 1];
  }
  walsh64<E>(rh);
}

// ============================================================== per-head codec rows

template <typename TS, typename TP, int D, bool ENC>
__global__ void __launch_bounds__(kThreads) heads_kernel(HeadsArgs<TS, TP> a) {
  extern __shared__ float smem[];
  float* sA = smem;
  float* sW = sA + 32 * 33;
  float* sP = sW + D * 33;
  constexpr int NJ = D / 32;
  constexpr int E = D / 32;
  const int64_t t0 = (int64_t)blockIdx.x * 32;
  const int h = blockIdx.y;
  const int H = a.H;
  float acc[4][NJ];
  zero_acc(acc);
  if (a.block) {
    const int Din = a.in1 ? 2 * D : D;
    auto la = [&](int row, int k) -> float {
      const int64_t t = t0 + row;
      if (t >= a.T) return 0.f;
      return k < D ? to_f(a.in0[(t * H + h) * D + k]) : to_f(a.in1[(t * H + h) * D + (k - D)]);
    };
    auto lw = [&](int row, int k) -> float { return to_f(a.block[((int64_t)h * D + row) * Din + k]); };
    gemm_tile<NJ>(acc, Din, la, lw, sA, sW);
  }
  if (a.r > 0) {
    auto la = [&](int row, int k) -> float {
      const int64_t t = t0 + row;
      return t < a.T ? a.Z[t * a.r + k] : 0.f;
    };
    auto lw = [&](int row, int k) -> float { return to_f(a.U[((int64_t)h * D + row) * a.r + k]); };
    gemm_tile<NJ>(acc, a.r, la, lw, sA, sW);
  }
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5, lane = tx, warp = ty;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < NJ; ++j) sP[(ty * 4 + i) * D + tx + 32 * j] = acc[i][j];
  __shared__ float sCb[32];  // the H64 / EDEN-2 points
  if (a.codebook && threadIdx.x < 32) sCb[threadIdx.x] = a.codebook[threadIdx.x];
  __syncthreads();
  RowCodec<E> rc{a.bits, a.group};
  const int row_bytes = D * a.bits / 8;
  const int row_groups = D / a.group;
  for (int i = warp; i < 32; i += 8) {
    const int64_t t = t0 + i;
    if (t >= a.T) break;
    const int64_t row = t * H + h;
    float p[E];
#pragma unroll
    for (int e = 0; e < E; ++e) p[e] = sP[i * D + lane * E + e];
    if (a.codebook) {  // H64 / EDEN-2 residuals: D/4 code bytes and D/64 scales per row
      uint8_t* rcodes = a.codes + row * (D / 4);
      TP* rsc = reinterpret_cast<TP*>(a.params) + row * (D / 64);
      float rh[E];
      if (ENC) {
        float x[E], r[E];
        load_vec<TS, E>(a.x + row * D + lane * E, x);
#pragma unroll
        for (int e = 0; e < E; ++e) r[e] = x[e] - p[e];
        eden2_encode<E, TP>(r, sCb, rcodes, rsc, rh);
      } else {
        eden2_decode<E, TP>(rcodes, rsc, sCb, rh);
      }
      if (a.rec) {
        float o[E];
#pragma unroll
        for (int e = 0; e < E; ++e) o[e] = p[e] + rh[e];
        store_vec<TS, E>(a.rec + row * D + lane * E, o);
      }
      continue;
    }
    int q[E];
    float s, z;
    uint8_t* rcodes = a.codes + row * row_bytes;
    Pair<TP>* rpar = a.params + row * row_groups;
    if (ENC) {
      float x[E], r[E];
      load_vec<TS, E>(a.x + row * D + lane * E, x);
#pragma unroll
      for (int e = 0; e < E; ++e) r[e] = x[e] - p[e];
      rc.quantize(r, q, s, z, rcodes, rpar);
    } else {
      rc.load_codes(rcodes, q);
      rc.load_params(rpar, s, z);
    }
    if (a.rec) {
      float o[E];
#pragma unroll
      for (int e = 0; e < E; ++e) o[e] = p[e] + fmaf(s, (float)q[e], z);
      store_vec<TS, E>(a.rec + row * D + lane * E, o);
    }
  }
}

// ============================================================== temporal codec (frame walk)

template <typename TS, typename TP, int D, bool ENC>
__global__ void __launch_bounds__(kThreads) temporal_kernel(TemporalArgs<TS, TP> a) {
  extern __shared__ float smem[];
  float* sA = smem;
  float* sW = sA + 32 * 33;
  float* sP = sW + D * 33;
  float* buf[5];
  for (int b = 0; b < 5; ++b) buf[b] = sP + 32 * D * (b + 1);
  float* Kp1 = buf[0];
  float* Kp2 = buf[1];
  float* Kc = buf[2];
  float* Vp1 = buf[3];
  float* Vc = buf[4];
  constexpr int NJ = D / 32;
  constexpr int E = D / 32;
  const int s0 = blockIdx.x * 32;
  const int h = blockIdx.y;
  const int H = a.H;
  const int64_t F = a.F;
  const int64_t n_frames = (a.T + F - 1) / F;
  const bool cont = a.anchor_bits == 0;  // continues a sequence from K_src / V_src
  const int64_t F0 = cont ? 0 : (F < a.T ? F : a.T);
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5, lane = tx, warp = ty;
  const int row_groups = D / a.group;
  for (int e = threadIdx.x; e < 5 * 32 * D; e += kThreads) buf[0][e] = 0.f;
  __syncthreads();
  if (cont) {
    // history: K_src = [K^ of frame f0-2 ; K^ of frame f0-1], V_src = V^ of frame f0-1
    for (int e = threadIdx.x; e < 32 * D; e += kThreads) {
      const int i = e / D, d = e % D;
      const int64_t s = s0 + i;
      if (s >= F) continue;
      Kp2[e] = to_f(a.ksrc[(s * H + h) * D + d]);
      Kp1[e] = to_f(a.ksrc[((F + s) * H + h) * D + d]);
      Vp1[e] = to_f(a.vsrc[(s * H + h) * D + d]);
    }
    __syncthreads();
  }

  for (int64_t f = 0; f < n_frames; ++f) {
    const int64_t n_f = (a.T - f * F) < F ? (a.T - f * F) : F;
    const bool anchor = f == 0 && !cont;
    const int bits = anchor ? a.anchor_bits : a.bits;
    const int row_bytes = D * bits / 8;
    const int anchor_row_bytes = D * a.anchor_bits / 8;
    RowCodec<E> rc{bits, a.group};
    for (int pass = 0; pass < 2; ++pass) {  // 0: K, 1: V
      float acc[4][NJ];
      zero_acc(acc);
      if (!anchor) {
        const float* in0 = pass == 0 ? Kp1 : Kc;
        const float* in1 = pass == 0 ? Kp2 : Vp1;
        const TS* W = (pass == 0 ? a.ak : a.av) + (int64_t)h * D * 2 * D;
        auto la = [&](int row, int k) -> float { return k < D ? in0[row * D + k] : in1[row * D + k - D]; };
        auto lw = [&](int row, int k) -> float { return to_f(W[(int64_t)row * 2 * D + k]); };
        gemm_tile<NJ>(acc, 2 * D, la, lw, sA, sW);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < NJ; ++j) sP[(ty * 4 + i) * D + tx + 32 * j] = acc[i][j];
      __syncthreads();
      float* out = pass == 0 ? Kc : Vc;
      const TS* X = pass == 0 ? a.K : a.V;
      uint8_t* codes = pass == 0 ? a.kcodes : a.vcodes;
      Pair<TP>* params = pass == 0 ? a.kparams : a.vparams;
      TS* rec = pass == 0 ? a.krec : a.vrec;
      for (int i = warp; i < 32; i += 8) {
        const int64_t s = s0 + i;
        if (s >= n_f) break;
        const int64_t t = f * F + s;
        const int64_t row = t * H + h;
        const int64_t cofs = row < F0 * H ? row * anchor_row_bytes
                                          : F0 * H * anchor_row_bytes + (row - F0 * H) * row_bytes;
        float p[E];
#pragma unroll
        for (int e = 0; e < E; ++e) p[e] = sP[i * D + lane * E + e];
        int q[E];
        float sc, zc;
        if (ENC) {
          float x[E], r[E];
          load_vec<TS, E>(X + row * D + lane * E, x);
#pragma unroll
          for (int e = 0; e < E; ++e) r[e] = x[e] - p[e];
          rc.quantize(r, q, sc, zc, codes + cofs, params + row * row_groups);
        } else {
          rc.load_codes(codes + cofs, q);
          rc.load_params(params + row * row_groups, sc, zc);
        }
        float o[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
          o[e] = round_as<TS>(p[e] + fmaf(sc, (float)q[e], zc));
          out[i * D + lane * E + e] = o[e];
        }
        if (rec) store_vec<TS, E>(rec + row * D + lane * E, o);
      }
      __syncthreads();
    }
    // rotate the frame history: K_{f-2} <- K_{f-1} <- K_f, V_{f-1} <- V_f
    float* old = Kp2;
    Kp2 = Kp1;
    Kp1 = Kc;
    Kc = old;
    float* tv = Vp1;
    Vp1 = Vc;
    Vc = tv;
  }
}

// ============================================================== clustered codec

// cnorm[j] = |c_j|^2 (fp32), one warp per centre: the norms alone, for the
// tensor-core encode, which forms P on the tensor cores
template <typename TS>
__global__ void __launch_bounds__(kThreads) cluster_norms_kernel(ClusterPrepArgs<TS> a) {
  const int tx = threadIdx.x & 31;
  const int jc = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
  if (jc >= a.n_c) return;
  float s = 0.f;
  for (int k = tx; k < a.C; k += 32) {
    const float v = to_f(a.cent[(int64_t)jc * a.C + k]);
    s = fmaf(v, v, s);
  }
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (tx == 0) a.cnorm[jc] = s;
}

// cnorm[j] = |c_j|^2, P[j][i] = enc_i . c_j (fp32)
template <typename TS>
__global__ void __launch_bounds__(kThreads) cluster_prep_kernel(ClusterPrepArgs<TS> a) {
  extern __shared__ float smem[];
  float* sA = smem;
  float* sW = sA + 32 * 33;
  const int j0 = blockIdx.x * 32;
  const int C = a.C;
  float acc[4][4];
  zero_acc(acc);
  auto la = [&](int row, int k) -> float { return j0 + row < a.n_c ? to_f(a.cent[(int64_t)(j0 + row) * C + k]) : 0.f; };
  auto lw = [&](int row, int k) -> float { return row < a.m ? to_f(a.enc[(int64_t)row * C + k]) : 0.f; };
  gemm_tile<4>(acc, C, la, lw, sA, sW);
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int jc = j0 + ty * 4 + i, mi = tx + 32 * j;
      if (jc < a.n_c && mi < a.m) a.P[jc * a.m + mi] = acc[i][j];
    }
  // norms: one warp per centre
  for (int i = ty; i < 32; i += 8) {
    const int jc = j0 + i;
    if (jc >= a.n_c) break;
    float s = 0.f;
    for (int k = tx; k < C; k += 32) {
      const float v = to_f(a.cent[(int64_t)jc * C + k]);
      s = fmaf(v, v, s);
    }
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (tx == 0) a.cnorm[jc] = s;
  }
}

// reconstruct 32 tokens: rec[t][c] = cent[a_t][c] + sum_i coef[t][i] dec[c][i]
template <typename TS, int NJ_M>
__device__ __forceinline__ void cluster_reconstruct(int64_t t0, int64_t T, int C, int m, const float* sCoef,
                                                    const int* sAssign, const TS* cent, const TS* dec, TS* rec,
                                                    float* sA, float* sW) {
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int n0 = 0; n0 < C; n0 += 128) {
    float acc[4][4];
    zero_acc(acc);
    auto la = [&](int row, int k) -> float { return sCoef[row * 128 + k]; };
    auto lw = [&](int row, int k) -> float { return n0 + row < C ? to_f(dec[(int64_t)(n0 + row) * m + k]) : 0.f; };
    gemm_tile<4>(acc, m, la, lw, sA, sW);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rr = ty * 4 + i;
      const int64_t t = t0 + rr;
      if (t >= T) continue;
      const int at = sAssign[rr];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = n0 + tx + 32 * j;
        if (c < C) rec[t * C + c] = from_f<TS>(to_f(cent[(int64_t)at * C + c]) + acc[i][j]);
      }
    }
  }
}

template <typename TS, typename TP, bool ENC>
__global__ void __launch_bounds__(kThreads) cluster_kernel(ClusterArgs<TS, TP> a) {
  extern __shared__ float smem[];
  float* sA = smem;
  float* sW = sA + 32 * 33;              // [256][33]
  float* sCoef = sW + 256 * 33;          // [32][128]
  int* sAssign = reinterpret_cast<int*>(sCoef + 32 * 128);
  const int64_t t0 = (int64_t)blockIdx.x * 32;
  const int C = a.C, m = a.m;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5, lane = tx, warp = ty;
  constexpr int E = 4;  // m == 128
  RowCodec<E> rc{a.bits, a.group};
  const int row_bytes = m * a.bits / 8;
  const int row_groups = m / a.group;
  if (ENC) {
    // 1. nearest centre: argmin_j |c_j|^2 - 2 x.c_j, ties to the lowest j
    {
      float acc[4][8];
      zero_acc(acc);
      auto la = [&](int row, int k) -> float {
        const int64_t t = t0 + row;
        return t < a.T ? to_f(a.X[t * C + k]) : 0.f;
      };
      auto lw = [&](int row, int k) -> float { return row < a.n_c ? to_f(a.cent[(int64_t)row * C + k]) : 0.f; };
      gemm_tile<8>(acc, C, la, lw, sA, sW);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float best = INFINITY;
        int bj = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int jc = tx + 32 * j;
          if (jc < a.n_c) {
            const float sc = a.cnorm[jc] - 2.f * acc[i][j];
            if (sc < best) {
              best = sc;
              bj = jc;
            }
          }
        }
        for (int o = 16; o; o >>= 1) {
          const float ob = __shfl_xor_sync(0xffffffffu, best, o);
          const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
          if (ob < best || (ob == best && oj < bj)) {
            best = ob;
            bj = oj;
          }
        }
        if (tx == 0) sAssign[ty * 4 + i] = bj;
      }
    }
    __syncthreads();
    // 2. coefficients enc (x - c_a) = enc x - P[a]
    {
      float acc[4][4];
      zero_acc(acc);
      auto la = [&](int row, int k) -> float {
        const int64_t t = t0 + row;
        return t < a.T ? to_f(a.X[t * C + k]) : 0.f;
      };
      auto lw = [&](int row, int k) -> float { return row < m ? to_f(a.enc[(int64_t)row * C + k]) : 0.f; };
      gemm_tile<4>(acc, C, la, lw, sA, sW);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int rr = ty * 4 + i, mi = tx + 32 * j;
          sCoef[rr * 128 + mi] = acc[i][j] - a.P[sAssign[rr] * m + mi];
        }
    }
    __syncthreads();
  }
  // 3. rows of coefficients: quantize (encode) or unpack (decode), keep the dequantized values
  for (int i = warp; i < 32; i += 8) {
    const int64_t t = t0 + i;
    if (t >= a.T) {
      for (int e = 0; e < E; ++e) sCoef[i * 128 + lane * E + e] = 0.f;
      if (lane == 0) sAssign[i] = 0;
      continue;
    }
    int q[E];
    float s, z;
    if (ENC) {
      float r[E];
#pragma unroll
      for (int e = 0; e < E; ++e) r[e] = sCoef[i * 128 + lane * E + e];
      rc.quantize(r, q, s, z, a.codes + t * row_bytes, a.params + t * row_groups);
      if (lane == 0) a.assign[t] = (uint8_t)sAssign[i];
    } else {
      rc.load_codes(a.codes + t * row_bytes, q);
      rc.load_params(a.params + t * row_groups, s, z);
      if (lane == 0) sAssign[i] = a.assign[t];
    }
#pragma unroll
    for (int e = 0; e < E; ++e) sCoef[i * 128 + lane * E + e] = fmaf(s, (float)q[e], z);
  }
  __syncthreads();
  if (a.rec) cluster_reconstruct<TS, 4>(t0, a.T, C, m, sCoef, sAssign, a.cent, a.dec, a.rec, sA, sW);
}

// ============================================================== attention (flash, FMA)

template <typename TS, int D>
__global__ void __launch_bounds__(kThreads) attention_kernel(AttnArgs<TS> a) {
  extern __shared__ float smem[];
  float* sQ = smem;                 // [32][D]
  float* sK = sQ + 32 * D;          // [32][D+1]
  float* sV = sK + 32 * (D + 1);    // [32][D]
  float* sS = sV + 32 * D;          // [32][33]
  constexpr int DJ = D / 8;
  const int64_t q0 = (int64_t)blockIdx.x * 32;
  const int hq = blockIdx.y;        // query head
  const int h = hq / (a.Hq / a.H);  // its KV head (grouped-query attention when Hq > H)
  const int H = a.H;
  const int tid = threadIdx.x;
  const int qr = tid >> 3, sub = tid & 7;
  for (int e = tid; e < 32 * D; e += kThreads) {
    const int r = e / D, d = e % D;
    const int64_t q = q0 + r;
    sQ[e] = q < a.n_q ? to_f(a.Q[(q * a.Hq + hq) * D + d]) : 0.f;
  }
  float o[DJ];
#pragma unroll
  for (int j = 0; j < DJ; ++j) o[j] = 0.f;
  float mrow = -INFINITY, lrow = 0.f;
  const int64_t n_keys = a.n_hist + a.n_self;
  for (int64_t k0 = 0; k0 < n_keys; k0 += 32) {
    __syncthreads();
    for (int e = tid; e < 32 * D; e += kThreads) {
      const int r = e / D, d = e % D;
      const int64_t k = k0 + r;
      float kv = 0.f, vv = 0.f;
      if (k < a.n_hist) {
        kv = to_f(a.Kh[(k * H + h) * D + d]);
        vv = to_f(a.Vh[(k * H + h) * D + d]);
      } else if (k < n_keys) {
        kv = to_f(a.Ks[((k - a.n_hist) * H + h) * D + d]);
        vv = to_f(a.Vs[((k - a.n_hist) * H + h) * D + d]);
      }
      sK[r * (D + 1) + d] = kv;
      sV[r * D + d] = vv;
    }
    __syncthreads();
    float s[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int kc = sub * 4 + i;
      float acc = 0.f;
#pragma unroll 8
      for (int d = 0; d < D; ++d) acc = fmaf(sQ[qr * D + d], sK[kc * (D + 1) + d], acc);
      s[i] = (k0 + kc < n_keys) ? acc * a.scale : -INFINITY;
    }
    float mx = fmaxf(fmaxf(s[0], s[1]), fmaxf(s[2], s[3]));
    for (int off = 1; off < 8; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float mnew = fmaxf(mrow, mx);
    const float alpha = (mrow == -INFINITY) ? 0.f : expf(mrow - mnew);
    float psum = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float p = (s[i] == -INFINITY) ? 0.f : expf(s[i] - mnew);
      sS[qr * 33 + sub * 4 + i] = p;
      psum += p;
    }
    for (int off = 1; off < 8; off <<= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
    lrow = lrow * alpha + psum;
    mrow = mnew;
    __syncwarp();
#pragma unroll
    for (int j = 0; j < DJ; ++j) {
      const int d = sub + 8 * j;
      float acc = o[j] * alpha;
#pragma unroll 8
      for (int kc = 0; kc < 32; ++kc) acc = fmaf(sS[qr * 33 + kc], sV[kc * D + d], acc);
      o[j] = acc;
    }
  }
  const int64_t q = q0 + qr;
  if (q < a.n_q) {
    const float inv = 1.f / lrow;
#pragma unroll
    for (int j = 0; j < DJ; ++j) a.O[(q * a.Hq + hq) * D + sub + 8 * j] = from_f<TS>(o[j] * inv);
  }
}

// ============================================================== mixed-dimensional attention (clustered)

template <typename TS, typename TP>
__global__ void __launch_bounds__(kThreads) mixed_attention_kernel(MixedArgs<TS, TP> a) {
  extern __shared__ float smem[];
  constexpr int QT = 16, KT = 32, M = 128;
  const int n_c = a.n_c, D = a.D, C = a.C;
  float* sQ = smem;                   // [QT][D]
  float* sTab = sQ + QT * D;          // [QT][n_c]
  float* sQt = sTab + QT * 256;       // [QT][M]
  float* sMass = sQt + QT * M;        // [QT][n_c]
  float* sCbar = sMass + QT * 256;    // [QT][M]
  float* sCk = sCbar + QT * M;        // [KT][M+1]
  float* sCv = sCk + KT * (M + 1);    // [KT][M]
  float* sS = sCv + KT * M;           // [QT][KT]
  float* sAlpha = sS + QT * KT;       // [QT]
  int* sAk = reinterpret_cast<int*>(sAlpha + QT);
  int* sAv = sAk + KT;
  const int64_t q0 = (int64_t)blockIdx.x * QT;
  const int h = blockIdx.y;
  const int H = a.H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < QT * D; e += kThreads) {
    const int r = e / D, d = e % D;
    const int64_t q = q0 + r;
    sQ[e] = q < a.n_q ? to_f(a.Q[(q * H + h) * D + d]) : 0.f;
  }
  __syncthreads();
  for (int e = tid; e < QT * n_c; e += kThreads) {
    const int r = e / n_c, j = e % n_c;
    float acc = 0.f;
    for (int d = 0; d < D; ++d) acc = fmaf(sQ[r * D + d], to_f(a.cent_k[(int64_t)j * C + h * D + d]), acc);
    sTab[r * 256 + j] = acc;
    sMass[r * 256 + j] = 0.f;
  }
  for (int e = tid; e < QT * M; e += kThreads) {
    const int r = e / M, i = e % M;
    float acc = 0.f;
    for (int d = 0; d < D; ++d) acc = fmaf(sQ[r * D + d], to_f(a.dec_k[(int64_t)(h * D + d) * M + i]), acc);
    sQt[e] = acc;
    sCbar[e] = 0.f;
  }
  float mrow = -INFINITY, lrow = 0.f;  // warp w owns rows w and w + 8
  float mrow2 = -INFINITY, lrow2 = 0.f;
  RowCodec<4> rc{a.bits, a.group};
  const int row_bytes = M * a.bits / 8;
  const int row_groups = M / a.group;
  for (int64_t k0 = 0; k0 < a.T; k0 += KT) {
    __syncthreads();
    for (int i = warp; i < KT; i += 8) {
      const int64_t t = k0 + i;
      int q[4];
      float s, z;
      if (t < a.T) {
        rc.load_codes(a.codes_k + t * row_bytes, q);
        rc.load_params(a.params_k + t * row_groups, s, z);
        for (int e = 0; e < 4; ++e) sCk[i * (M + 1) + lane * 4 + e] = fmaf(s, (float)q[e], z);
        rc.load_codes(a.codes_v + t * row_bytes, q);
        rc.load_params(a.params_v + t * row_groups, s, z);
        for (int e = 0; e < 4; ++e) sCv[i * M + lane * 4 + e] = fmaf(s, (float)q[e], z);
        if (lane == 0) {
          sAk[i] = a.assign_k[t];
          sAv[i] = a.assign_v[t];
        }
      } else {
        for (int e = 0; e < 4; ++e) {
          sCk[i * (M + 1) + lane * 4 + e] = 0.f;
          sCv[i * M + lane * 4 + e] = 0.f;
        }
        if (lane == 0) {
          sAk[i] = 0;
          sAv[i] = 0;
        }
      }
    }
    __syncthreads();
    for (int e = tid; e < QT * KT; e += kThreads) {
      const int r = e / KT, kc = e % KT;
      float acc = sTab[r * 256 + sAk[kc]];
      for (int i = 0; i < M; ++i) acc = fmaf(sQt[r * M + i], sCk[kc * (M + 1) + i], acc);
      sS[e] = (k0 + kc < a.T) ? acc * a.scale : -INFINITY;
    }
    __syncthreads();
    for (int rr = 0; rr < 2; ++rr) {
      const int r = warp + 8 * rr;
      float& mr = rr ? mrow2 : mrow;
      float& lr = rr ? lrow2 : lrow;
      const float s = sS[r * KT + lane];
      float mx = s;
      for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float mnew = fmaxf(mr, mx);
      const float alpha = (mr == -INFINITY) ? 0.f : expf(mr - mnew);
      const float p = (s == -INFINITY) ? 0.f : expf(s - mnew);
      float ps = p;
      for (int off = 16; off; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      lr = lr * alpha + ps;
      mr = mnew;
      sS[r * KT + lane] = p;
      if (lane == 0) sAlpha[r] = alpha;
    }
    __syncthreads();
    for (int e = tid; e < QT * 256; e += kThreads) sMass[e] *= sAlpha[e / 256];
    for (int e = tid; e < QT * M; e += kThreads) {
      const int r = e / M, i = e % M;
      float acc = sCbar[e] * sAlpha[r];
      for (int kc = 0; kc < KT; ++kc) acc = fmaf(sS[r * KT + kc], sCv[kc * M + i], acc);
      sCbar[e] = acc;
    }
    __syncthreads();
    for (int e = tid; e < QT * KT; e += kThreads) {
      const int r = e / KT, kc = e % KT;
      atomicAdd(&sMass[r * 256 + sAv[kc]], sS[e]);
    }
  }
  __syncthreads();
  // normalisers to shared memory (reuse sAlpha)
  if (lane == 0) {
    sAlpha[warp] = lrow;
    sAlpha[warp + 8] = lrow2;
  }
  __syncthreads();
  for (int e = tid; e < QT * D; e += kThreads) {
    const int r = e / D, d = e % D;
    const int64_t q = q0 + r;
    if (q >= a.n_q) continue;
    float acc = 0.f;
    for (int j = 0; j < n_c; ++j) acc = fmaf(sMass[r * 256 + j], to_f(a.cent_v[(int64_t)j * C + h * D + d]), acc);
    for (int i = 0; i < M; ++i) acc = fmaf(sCbar[r * M + i], to_f(a.dec_v[(int64_t)(h * D + d) * M + i]), acc);
    a.O[(q * H + h) * D + d] = from_f<TS>(acc / sAlpha[r]);
  }
}

// ============================================================== pack / unpack (16-byte words)

__global__ void pack_kernel(const uint8_t* codes, int64_t n_words, int bits, uint4* packed) {
  const int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (w >= n_words) return;
  const int per_word = 128 / bits;
  const uint8_t* c = codes + w * per_word;
  uint32_t out[4] = {0, 0, 0, 0};
  for (int j = 0; j < per_word; ++j) {
    const int bit = j * bits;
    out[bit >> 5] |= (uint32_t)c[j] << (bit & 31);
  }
  packed[w] = make_uint4(out[0], out[1], out[2], out[3]);
}

__global__ void unpack_kernel(const uint4* packed, int64_t n_words, int bits, uint8_t* codes) {
  const int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (w >= n_words) return;
  const int per_word = 128 / bits;
  const uint4 v = packed[w];
  const uint32_t in[4] = {v.x, v.y, v.z, v.w};
  const uint32_t mask = (1u << bits) - 1u;
  uint8_t* c = codes + w * per_word;
  for (int j = 0; j < per_word; ++j) {
    const int bit = j * bits;
    c[j] = (uint8_t)((in[bit >> 5] >> (bit & 31)) & mask);
  }
}

// ============================================================== launchers

static inline int div_up(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }

template <typename K>
static cudaError_t set_smem(K kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <typename TS>
cudaError_t launch_latent(const LatentArgs<TS>& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const int nj = (a.r + 31) / 32;
  const size_t smem = (32 * 33 + 32 * 4 * 33) * sizeof(float);
  dim3 grid(div_up(a.T, 32));
#define KVC_LAT(NJ)                                                  \
  {                                                                  \
    auto k = latent_kernel<TS, NJ>;                                  \
    cudaError_t e = set_smem(k, smem);                               \
    if (e != cudaSuccess) return e;                                  \
    k<<<grid, kThreads, smem, st>>>(a);                              \
    count_launches(1);                                               \
    return cudaGetLastError();                                       \
  }
  if (nj == 1) KVC_LAT(1) else if (nj == 2) KVC_LAT(2) else if (nj == 3) KVC_LAT(3) else KVC_LAT(4)
#undef KVC_LAT
}

template <typename TS, typename TP>
cudaError_t launch_heads(const HeadsArgs<TS, TP>& a, int D, bool encode, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  dim3 grid(div_up(a.T, 32), a.H);
  const size_t smem = (32 * 33 + D * 33 + 32 * D) * sizeof(float);
#define KVC_HEADS(DD, ENC)                                           \
  {                                                                  \
    auto k = heads_kernel<TS, TP, DD, ENC>;                          \
    cudaError_t e = set_smem(k, smem);                               \
    if (e != cudaSuccess) return e;                                  \
    k<<<grid, kThreads, smem, st>>>(a);                              \
    count_launches(1);                                               \
    return cudaGetLastError();                                       \
  }
  if (D == 128) {
    if (encode) KVC_HEADS(128, true) else KVC_HEADS(128, false)
  } else {
    if (encode) KVC_HEADS(64, true) else KVC_HEADS(64, false)
  }
#undef KVC_HEADS
}

template <typename TS, typename TP>
cudaError_t launch_temporal(const TemporalArgs<TS, TP>& a, int D, bool encode, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const int64_t F = a.F < a.T ? a.F : a.T;
  dim3 grid(div_up(F, 32), a.H);
  const size_t smem = (32 * 33 + D * 33 + 6 * 32 * D) * sizeof(float);
#define KVC_TEMP(DD, ENC)                                            \
  {                                                                  \
    auto k = temporal_kernel<TS, TP, DD, ENC>;                       \
    cudaError_t e = set_smem(k, smem);                               \
    if (e != cudaSuccess) return e;                                  \
    k<<<grid, kThreads, smem, st>>>(a);                              \
    count_launches(1);                                               \
    return cudaGetLastError();                                       \
  }
  if (D == 128) {
    if (encode) KVC_TEMP(128, true) else KVC_TEMP(128, false)
  } else {
    if (encode) KVC_TEMP(64, true) else KVC_TEMP(64, false)
  }
#undef KVC_TEMP
}

template <typename TS>
cudaError_t launch_cluster_norms(const ClusterPrepArgs<TS>& a, cudaStream_t st) {
  cluster_norms_kernel<TS><<<div_up(a.n_c, kThreads / 32), kThreads, 0, st>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

template <typename TS>
cudaError_t launch_cluster_prep(const ClusterPrepArgs<TS>& a, cudaStream_t st) {
  const size_t smem = (32 * 33 + 128 * 33) * sizeof(float);
  auto k = cluster_prep_kernel<TS>;
  cudaError_t e = set_smem(k, smem);
  if (e != cudaSuccess) return e;
  k<<<div_up(a.n_c, 32), kThreads, smem, st>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

template <typename TS, typename TP>
cudaError_t launch_cluster(const ClusterArgs<TS, TP>& a, bool encode, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const size_t smem = (32 * 33 + 256 * 33 + 32 * 128) * sizeof(float) + 32 * sizeof(int);
  cudaError_t e;
  if (encode) {
    auto k = cluster_kernel<TS, TP, true>;
    if ((e = set_smem(k, smem)) != cudaSuccess) return e;
    k<<<div_up(a.T, 32), kThreads, smem, st>>>(a);
    count_launches(1);
  } else {
    auto k = cluster_kernel<TS, TP, false>;
    if ((e = set_smem(k, smem)) != cudaSuccess) return e;
    k<<<div_up(a.T, 32), kThreads, smem, st>>>(a);
    count_launches(1);
  }
  return cudaGetLastError();
}

template <typename TS>
cudaError_t launch_attention(const AttnArgs<TS>& a, int D, cudaStream_t st) {
  if (a.n_q == 0) return cudaSuccess;
  dim3 grid(div_up(a.n_q, 32), a.Hq);
  const size_t smem = (32 * D + 32 * (D + 1) + 32 * D + 32 * 33) * sizeof(float);
  cudaError_t e;
  if (D == 128) {
    auto k = attention_kernel<TS, 128>;
    if ((e = set_smem(k, smem)) != cudaSuccess) return e;
    k<<<grid, kThreads, smem, st>>>(a);
    count_launches(1);
  } else {
    auto k = attention_kernel<TS, 64>;
    if ((e = set_smem(k, smem)) != cudaSuccess) return e;
    k<<<grid, kThreads, smem, st>>>(a);
    count_launches(1);
  }
  return cudaGetLastError();
}

template <typename TS, typename TP>
cudaError_t launch_mixed_attention(const MixedArgs<TS, TP>& a, cudaStream_t st) {
  if (a.n_q == 0) return cudaSuccess;
  dim3 grid(div_up(a.n_q, 16), a.H);
  const size_t smem = (16 * a.D + 16 * 256 + 16 * 128 + 16 * 256 + 16 * 128 + 32 * 129 + 32 * 128 + 16 * 32 + 16) *
                          sizeof(float) + 64 * sizeof(int);
  auto k = mixed_attention_kernel<TS, TP>;
  cudaError_t e = set_smem(k, smem);
  if (e != cudaSuccess) return e;
  k<<<grid, kThreads, smem, st>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_pack(const uint8_t* codes, int64_t n, int bits, void* packed, cudaStream_t st) {
  const int64_t words = n * bits / 128;
  if (words == 0) return cudaSuccess;
  pack_kernel<<<div_up(words, 256), 256, 0, st>>>(codes, words, bits, reinterpret_cast<uint4*>(packed));
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_unpack(const void* packed, int64_t n, int bits, uint8_t* codes, cudaStream_t st) {
  const int64_t words = n * bits / 128;
  if (words == 0) return cudaSuccess;
  unpack_kernel<<<div_up(words, 256), 256, 0, st>>>(reinterpret_cast<const uint4*>(packed), words, bits, codes);
  count_launches(1);
  return cudaGetLastError();
}

// explicit instantiations
#define KVC_INST(TS, TP)                                                                          \
  template cudaError_t launch_heads<TS, TP>(const HeadsArgs<TS, TP>&, int, bool, cudaStream_t);    \
  template cudaError_t launch_temporal<TS, TP>(const TemporalArgs<TS, TP>&, int, bool, cudaStream_t); \
  template cudaError_t launch_cluster<TS, TP>(const ClusterArgs<TS, TP>&, bool, cudaStream_t);     \
  template cudaError_t launch_mixed_attention<TS, TP>(const MixedArgs<TS, TP>&, cudaStream_t);
KVC_INST(float, float)
KVC_INST(float, __half)
KVC_INST(__nv_bfloat16, float)
KVC_INST(__nv_bfloat16, __half)
#undef KVC_INST
template cudaError_t launch_latent<float>(const LatentArgs<float>&, cudaStream_t);
template cudaError_t launch_latent<__nv_bfloat16>(const LatentArgs<__nv_bfloat16>&, cudaStream_t);
template cudaError_t launch_cluster_prep<float>(const ClusterPrepArgs<float>&, cudaStream_t);
template cudaError_t launch_cluster_norms<__nv_bfloat16>(const ClusterPrepArgs<__nv_bfloat16>&, cudaStream_t);
template cudaError_t launch_cluster_prep<__nv_bfloat16>(const ClusterPrepArgs<__nv_bfloat16>&, cudaStream_t);
template cudaError_t launch_attention<float>(const AttnArgs<float>&, int, cudaStream_t);
template cudaError_t launch_attention<__nv_bfloat16>(const AttnArgs<__nv_bfloat16>&, int, cudaStream_t);

}  // namespace kvc
