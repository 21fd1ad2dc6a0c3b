// Internal helpers shared by the kernels of libkvc.so (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kvc.h"

namespace kvc {

// ---------------------------------------------------------------- value types

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f(__half x) { return __half2float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }
template <>
__device__ __forceinline__ __half from_f<__half>(float x) { return __float2half_rn(x); }

// value of x after rounding to T, as float
template <typename T>
__device__ __forceinline__ float round_as(float x) { return to_f(from_f<T>(x)); }

// (scale, zero) pair of one group
template <typename TP>
struct Pair {
  TP s, z;
};

// Loads E consecutive elements of type T (E*sizeof(T) is 4, 8 or 16 bytes) as floats.
template <typename T, int E>
__device__ __forceinline__ void load_vec(const T* p, float (&v)[E]) {
  if constexpr (sizeof(T) * E == 16) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
    for (int i = 0; i < E; ++i) v[i] = to_f(e[i]);
  } else if constexpr (sizeof(T) * E == 8) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
    for (int i = 0; i < E; ++i) v[i] = to_f(e[i]);
  } else {
#pragma unroll
    for (int i = 0; i < E; ++i) v[i] = to_f(p[i]);
  }
}

template <typename T, int E>
__device__ __forceinline__ void store_vec(T* p, const float (&v)[E]) {
  if constexpr (sizeof(T) * E == 16) {
    uint4 u;
    T* e = reinterpret_cast<T*>(&u);
#pragma unroll
    for (int i = 0; i < E; ++i) e[i] = from_f<T>(v[i]);
    *reinterpret_cast<uint4*>(p) = u;
  } else if constexpr (sizeof(T) * E == 8) {
    uint2 u;
    T* e = reinterpret_cast<T*>(&u);
#pragma unroll
    for (int i = 0; i < E; ++i) e[i] = from_f<T>(v[i]);
    *reinterpret_cast<uint2*>(p) = u;
  } else {
#pragma unroll
    for (int i = 0; i < E; ++i) p[i] = from_f<T>(v[i]);
  }
}

// ---------------------------------------------------------------- one coded row held by a warp
//
// A row of N = 32*E values is spread over the 32 lanes of a warp, lane l
// holding the E consecutive elements [l*E, (l+1)*E).  A quantization group of
// G elements then spans G/E consecutive lanes, so its min / max is a
// butterfly of xor-shuffles inside that aligned lane segment.

template <int E>
struct RowCodec {
  int bits;
  int group;  // elements per group, a multiple of E, G/E a power of two <= 32

  __device__ __forceinline__ int lanes_per_group() const { return group / E; }

  // Quantizes the residual r; returns the codes, the group's stored (s, z)
  // as floats, and writes params (first lane of each group) and the packed
  // codes of this row.
  template <typename TP>
  __device__ __forceinline__ void quantize(const float (&r)[E], int (&q)[E], float& sf, float& zf,
                                           uint8_t* row_codes, Pair<TP>* row_params) const {
    const int lane = threadIdx.x & 31;
    const int lpg = lanes_per_group();
    const int levels = (1 << bits) - 1;
    float mn = r[0], mx = r[0];
#pragma unroll
    for (int e = 1; e < E; ++e) {
      mn = fminf(mn, r[e]);
      mx = fmaxf(mx, r[e]);
    }
    for (int o = 1; o < lpg; o <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    TP s = from_f<TP>((mx - mn) / (float)levels);
    TP z = from_f<TP>(mn);
    sf = to_f(s);
    zf = to_f(z);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      int v = 0;
      if (sf > 0.f) {
        float t = rintf((r[e] - zf) / sf);
        t = fminf(fmaxf(t, 0.f), (float)levels);
        v = (int)t;
      }
      q[e] = v;
    }
    if ((lane % lpg) == 0) row_params[lane / lpg] = Pair<TP>{s, z};
    store_codes(q, row_codes);
  }

  __device__ __forceinline__ void store_codes(const int (&q)[E], uint8_t* row_codes) const {
    const int lane = threadIdx.x & 31;
    const int pbits = E * bits;  // bits held by this lane
    uint32_t w = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) w |= (uint32_t)q[e] << (e * bits);
    if (pbits >= 8) {
      uint8_t* dst = row_codes + lane * (pbits / 8);
      if (pbits == 8) {
        dst[0] = (uint8_t)w;
      } else if (pbits == 16) {
        *reinterpret_cast<uint16_t*>(dst) = (uint16_t)w;
      } else {
        *reinterpret_cast<uint32_t*>(dst) = w;
      }
    } else {
      // pbits in {2, 4}: 8/pbits lanes share one byte
      const int lpb = 8 / pbits;
      uint32_t acc = w << ((lane % lpb) * pbits);
      for (int o = 1; o < lpb; o <<= 1) acc |= __shfl_xor_sync(0xffffffffu, acc, o);
      if ((lane % lpb) == 0) row_codes[lane / lpb] = (uint8_t)acc;
    }
  }

  __device__ __forceinline__ void load_codes(const uint8_t* row_codes, int (&q)[E]) const {
    const int lane = threadIdx.x & 31;
    const int pbits = E * bits;
    const uint32_t mask = (1u << bits) - 1u;
    uint32_t w;
    if (pbits >= 8) {
      const uint8_t* src = row_codes + lane * (pbits / 8);
      if (pbits == 8) {
        w = src[0];
      } else if (pbits == 16) {
        w = *reinterpret_cast<const uint16_t*>(src);
      } else {
        w = *reinterpret_cast<const uint32_t*>(src);
      }
    } else {
      const int lpb = 8 / pbits;
      w = (uint32_t)row_codes[lane / lpb] >> ((lane % lpb) * pbits);
    }
#pragma unroll
    for (int e = 0; e < E; ++e) q[e] = (int)((w >> (e * bits)) & mask);
  }

  template <typename TP>
  __device__ __forceinline__ void load_params(const Pair<TP>* row_params, float& sf, float& zf) const {
    const int lane = threadIdx.x & 31;
    Pair<TP> p = row_params[lane / lanes_per_group()];
    sf = to_f(p.s);
    zf = to_f(p.z);
  }
};

// ---------------------------------------------------------------- launch accounting

// adds n to the process-wide launch counter (kvc_launch_counter)
void count_launches(unsigned long long n);
// Records the text of a failed CUDA call for kvc_last_cuda_error() and returns KVC_ERR_CUDA.
kvc_status record_cuda_error(cudaError_t e);

}  // namespace kvc
