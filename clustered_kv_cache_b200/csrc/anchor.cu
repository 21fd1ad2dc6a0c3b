// The anchor layer (no predictor): plain asymmetric min/max quantization of
// each G-value group of K and V, their reconstruction, and the decode.
//
// ("CORAL-KV: Compact Cross-Layer Prediction and Residual Coding ...", Fig. 3:
// the first layer of the chain is coded on its own, without a prediction; the
// group quantizer is that of every residual, CORAL Fig. 5 and Table 9.)
//
// With no prediction a tensor [T][H][D] is one contiguous run of groups, and
// its codes, (scale, zero) pairs and reconstruction are contiguous runs too.
// So the kernel streams it: a thread codes one 16-byte chunk of 8 values, the
// G / 8 threads of a group (adjacent lanes) reduce its min and max with
// shuffles, and every load and store of a warp is contiguous.  The
// quantization is the tensor-core epilogues' (quant8 / dequant8), so a decode
// replays its encode bit for bit.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "tc.h"
#include "tc_ptx.cuh"

namespace kvc {
namespace anchor {

using tc::dequant8;
using tc::pack_bf16x2;
using tc::quant8;
using tc::unpack_bf16x8;

constexpr int kThreads = 256;

struct Tensor {
  const __nv_bfloat16* x;  // encode input [n]
  uint8_t* codes;          // [n * BITS / 8]
  __half2* params;         // [n / G] (scale, zero)
  __nv_bfloat16* rec;      // reconstruction [n], or null (encode only)
};
struct Args {
  Tensor t[2];  // K, V
  int64_t chunks;  // 8-value chunks of one tensor
};

template <bool ENC, int BITS, int G>
__global__ void __launch_bounds__(kThreads) anchor_kernel(const Args a) {
  constexpr int LANES = G / 8;  // threads of a group
  constexpr float levels = (float)((1 << BITS) - 1);
  const Tensor T = blockIdx.y ? a.t[1] : a.t[0];  // (a select: no indexed copy of the parameters)
  const float zero8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  const int lane = threadIdx.x & 31;
  // The loop is uniform over a warp (its shuffles take every lane); a lane past
  // the end works on zeros and stores nothing.  A chunk count is a multiple of
  // LANES, so a group's lanes are all in range or all past it.
  for (int64_t c0 = (int64_t)blockIdx.x * kThreads + (threadIdx.x & ~31); c0 < a.chunks; c0 += stride) {
    const int64_t c = c0 + lane;
    const bool valid = c < a.chunks;
    const int64_t g = c / LANES;
    float r[8];
    if constexpr (ENC) {
      float x[8];
      unpack_bf16x8(valid ? __ldcs(reinterpret_cast<const uint4*>(T.x) + c) : make_uint4(0, 0, 0, 0), x, 0);
      float mn = x[0], mx = x[0];
#pragma unroll
      for (int i = 1; i < 8; ++i) {
        mn = fminf(mn, x[i]);
        mx = fmaxf(mx, x[i]);
      }
#pragma unroll
      for (int o = 1; o < LANES; o <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      const __half sh = __float2half_rn((mx - mn) / levels);
      const __half zh = __float2half_rn(mn);
      const float sf = __half2float(sh), zf = __half2float(zh);
      const float inv = sf > 0.f ? 1.f / sf : 0.f;
      const uint32_t q = quant8<BITS>(x, zero8, sf, zf, inv, r);
      if (!valid) continue;
      if constexpr (BITS == 4)
        __stcs(reinterpret_cast<uint32_t*>(T.codes) + c, q);
      else
        __stcs(reinterpret_cast<unsigned short*>(T.codes) + c, (unsigned short)q);
      if ((c & (LANES - 1)) == 0) __stcs(T.params + g, __halves2half2(sh, zh));
      if (!T.rec) continue;
    } else {
      if (!valid) continue;
      const uint32_t q = BITS == 4 ? __ldcs(reinterpret_cast<const uint32_t*>(T.codes) + c)
                                   : (uint32_t)__ldcs(reinterpret_cast<const unsigned short*>(T.codes) + c);
      const float2 sz = __half22float2(__ldg(T.params + g));
      dequant8<BITS>(q, 0, sz.x, sz.y, zero8, r);
    }
    __stcs(reinterpret_cast<uint4*>(T.rec) + c, make_uint4(pack_bf16x2(r[0], r[1]), pack_bf16x2(r[2], r[3]),
                                                           pack_bf16x2(r[4], r[5]), pack_bf16x2(r[6], r[7])));
  }
}

template <bool ENC, int BITS, int G>
static cudaError_t launch(const Args& a, cudaStream_t st) {
  int sms = 0, dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int64_t want = (a.chunks + kThreads - 1) / kThreads;
  const int64_t cap = (int64_t)sms * 8;  // 8 CTAs of 256 threads per SM, grid-striding
  const dim3 grid((unsigned)(want < cap ? want : cap), 2u);
  anchor_kernel<ENC, BITS, G><<<grid, kThreads, 0, st>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace anchor

bool anchor_supported(const kvc_layer_desc* d, const kvc_predictor* p) {
  return p->kind == KVC_PRED_NONE && d->dtype == KVC_BF16 && d->param_dtype == KVC_F16 &&
         d->residual_codec == KVC_RESIDUAL_RTN && (d->bits == 2 || d->bits == 4) &&
         (d->group == 32 || d->group == 64) && d->head_dim % d->group == 0;
}

cudaError_t anchor_layer(const kvc_layer_desc* d, bool enc, const void* K, const void* V, const kvc_codes* c,
                         void* Kr, void* Vr, cudaStream_t st) {
  if (d->n_tokens == 0) return cudaSuccess;
  anchor::Args a;
  a.chunks = d->n_tokens * d->n_heads * d->head_dim / 8;
  a.t[0] = anchor::Tensor{(const __nv_bfloat16*)K, (uint8_t*)c->k_codes, (__half2*)c->k_params, (__nv_bfloat16*)Kr};
  a.t[1] = anchor::Tensor{(const __nv_bfloat16*)V, (uint8_t*)c->v_codes, (__half2*)c->v_params, (__nv_bfloat16*)Vr};
  const bool g64 = d->group == 64;
  if (enc) {
    if (d->bits == 2) return g64 ? anchor::launch<true, 2, 64>(a, st) : anchor::launch<true, 2, 32>(a, st);
    return g64 ? anchor::launch<true, 4, 64>(a, st) : anchor::launch<true, 4, 32>(a, st);
  }
  if (d->bits == 2) return g64 ? anchor::launch<false, 2, 64>(a, st) : anchor::launch<false, 2, 32>(a, st);
  return g64 ? anchor::launch<false, 4, 64>(a, st) : anchor::launch<false, 4, 32>(a, st);
}

}  // namespace kvc
