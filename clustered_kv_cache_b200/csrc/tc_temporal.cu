// Temporal predictive codec on tcgen05 ("TempoKV: Predictive KV Cache
// Quantization for Autoregressive Video Generation", Fig. 2(b): K of frame f is
// predicted from the reconstructed K of frames f-1 and f-2 at the same spatial
// position, V of frame f from the aligned reconstructed K of frame f and V of
// frame f-1; only the low-bit residual is stored).
//
// One CTA per (128-position tile, head) walks every frame of the call in order.
// The head's two 128x256 maps stay in shared memory; the reconstructed state
// lives in three bf16 tiles (K of frames f and f-1, V of frame f-1) that serve
// directly as MMA operands: each new reconstruction overwrites the tile that
// its own prediction was the last to read.  Per frame the MMA of V(f) and of
// K(f+1) are issued together once K^_f exists, and two epilogue groups
// quantize V(f) and K(f+1) side by side.
//
// Warp roles: 0 TMA (maps, history), 1 MMA + TMEM, 2-5 K epilogue, 6-9 V epilogue.
#include <cuda.h>
#include <string.h>

#include "tc.h"
#include "tc_ptx.cuh"

namespace kvc {
namespace tc {

bool map2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);

namespace temporal {

constexpr int kThreads = 320;
constexpr int kKb = 0;                   // K^ tiles [2] (frame f in buffer f & 1)
constexpr int kVb = kKb + 2 * 32768;     // V^ tile
constexpr int kAK = kVb + 32768;         // AK_h as 4 sub-tiles [128 out][64 in]
constexpr int kAV = kAK + 65536;         // AV_h
constexpr int kBar = kAV + 65536;
constexpr int kSmem = kBar + 1024 + 1024;

struct Maps {
  CUtensorMap ak, av;      // [H*128][256]
  CUtensorMap ksrc, vsrc;  // history: [2F][C], [F][C] (continuation only)
};

struct Args {
  unsigned* err;
  int64_t T, F;
  int H, bits, anchor_bits;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  uint8_t* kcodes;
  __half2* kparams;
  uint8_t* vcodes;
  __half2* vparams;
  __nv_bfloat16* krec;  // optional
  __nv_bfloat16* vrec;  // optional
};

template <bool ENC, int G>
__global__ void __launch_bounds__(kThreads, 1) temporal_kernel(const __grid_constant__ Maps maps, const Args a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBar);
  uint64_t* w_full = bars;           // maps (+ history) landed
  uint64_t* kacc_full = bars + 1;    // K prediction of a frame in TMEM
  uint64_t* vacc_full = bars + 2;    // V prediction of a frame in TMEM
  uint64_t* kready = bars + 3;       // K^ of a frame in its tile (K epilogue, 128 arrivals)
  uint64_t* vready = bars + 4;       // V^ of a frame in its tile (V epilogue)
  uint64_t* mma_done = bars + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 6);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int s0 = blockIdx.x * 128;
  const int H = a.H;
  const int64_t C = (int64_t)H * 128;
  const int64_t F = a.F;
  const int nf = (int)((a.T + F - 1) / F);
  const bool cont = a.anchor_bits == 0;
  auto Kb = [&](int f) { return smem + kKb + (f & 1) * 32768; };
  uint8_t* Vb = smem + kVb;

  if (threadIdx.x == 0) {
    mbar_init(w_full, 1);
    mbar_init(kacc_full, 1);
    mbar_init(vacc_full, 1);
    mbar_init(kready, 128);
    mbar_init(vready, 128);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_async_smem();
  }
  // without a history the lag-2 input of frame 1 is zero: clear the tile of frame -1
  if (!cont)
    for (int e = threadIdx.x; e < 32768 / 16; e += kThreads) reinterpret_cast<uint4*>(Kb(1))[e] = make_uint4(0, 0, 0, 0);
  fence_async_smem();
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;  // K accumulator cols [0,128), V accumulator [128,256)

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      mbar_arrive_expect_tx(w_full, 131072u + (cont ? 98304u : 0u));
      for (int c = 0; c < 4; ++c) {
        tma_load(smem + kAK + c * 16384, &maps.ak, c * 64, h * 128, w_full, pol);
        tma_load(smem + kAV + c * 16384, &maps.av, c * 64, h * 128, w_full, pol);
      }
      if (cont) {  // K^ of frames -1 (tile 1) and -2 (tile 0), V^ of frame -1
        for (int c = 0; c < 2; ++c) {
          tma_load(Kb(1) + c * 16384, &maps.ksrc, h * 128 + c * 64, (int)(F + s0), w_full, pol);
          tma_load(Kb(0) + c * 16384, &maps.ksrc, h * 128 + c * 64, s0, w_full, pol);
          tma_load(Vb + c * 16384, &maps.vsrc, h * 128 + c * 64, s0, w_full, pol);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = wait(w_full, 0, abort_flag, a.err, 0x2100u);
      tc_fence_after();
      const uint32_t id = idesc_bf16(128, 128);
      // D = [A0 | A1] W^T over 256 inputs: W as 4 sub-tiles of 64 inputs
      auto mma256 = [&](uint32_t d, const uint8_t* A0, const uint8_t* A1, const uint8_t* W) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint64_t ad = desc_sw128(smem_u32((c < 2 ? A0 : A1) + (c & 1) * 16384));
          const uint64_t bd = desc_sw128(smem_u32(W + c * 16384));
#pragma unroll
          for (int k = 0; k < 4; ++k) umma(d, ad + 2 * k, bd + 2 * k, id, (c == 0 && k == 0) ? 0u : 1u);
        }
      };
      int kr = 0, vr = 0;  // completions of kready / vready seen
      // frame f's K prediction: [K^_{f-1} | K^_{f-2}] AK^T; K^_{f-2} sits in the tile of frame f
      auto issue_k = [&](int f) {
        mma256(tmem, Kb(f - 1), Kb(f), smem + kAK);
        umma_commit(kacc_full);
      };
      if (cont && ok) issue_k(0);
      for (int f = 0; f < nf && ok; ++f) {
        // K^_f is needed by K(f+1) and V(f); K(f+1) goes first, it is the next link
        // of the K chain, while V(f) may still wait for V^_{f-1}
        if (!wait(kready, kr++ & 1, abort_flag, a.err, 0x2110u)) ok = false;
        tc_fence_after();
        if (ok && f + 1 < nf) issue_k(f + 1);
        if (ok && (f > 0 || cont)) {  // the anchor frame has no prediction
          // V(f) reads V^_{f-1}: wait for its epilogue unless it is the supplied history
          if (f > 0 && !wait(vready, vr++ & 1, abort_flag, a.err, 0x2111u)) ok = false;
          tc_fence_after();
          if (ok) {
            mma256(tmem + 128, Kb(f), Vb, smem + kAV);
            umma_commit(vacc_full);
          }
        }
      }
      umma_commit(mma_done);
      const long long w0 = clock64();
      while (!mbar_test(mma_done, 0) && clock64() - w0 < kWaitBudget) {
      }
    }
  } else {
    // ================================================================ epilogues: warps 2-5 K, 6-9 V
    const bool isv = warp >= 6;
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int64_t s = s0 + row;
    const uint32_t acc_addr = tmem + ((uint32_t)(q * 32) << 16) + (isv ? 128 : 0);
    uint64_t* acc_full = isv ? vacc_full : kacc_full;
    int acc_use = 0;
    const int64_t F0 = cont ? 0 : (F < a.T ? F : a.T);
    const int arb = 128 * a.anchor_bits / 8;
    wait(w_full, 0, abort_flag, a.err, 0x2200u);
    for (int f = 0; f < nf; ++f) {
      const int64_t n_f = (a.T - f * F) < F ? (a.T - f * F) : F;
      const bool valid = s < n_f;
      const bool anchor = f == 0 && !cont;
      const int bits = anchor ? a.anchor_bits : a.bits;
      const int levels = (1 << bits) - 1;
      const int64_t t = f * F + s;
      const int64_t rowi = t * H + h;
      const int row_bytes = 128 * bits / 8;
      const int64_t cofs = rowi < F0 * H ? rowi * arb : F0 * H * arb + (rowi - F0 * H) * row_bytes;
      uint8_t* codes = (isv ? a.vcodes : a.kcodes) + cofs;
      __half2* params = (isv ? a.vparams : a.kparams) + rowi * (128 / G);
      constexpr int NG = 128 / G, NP = G / 32;
      uint4 xin[16];
      uint4 cin[4];
      __half2 pin[NG];
      if (ENC) {
        const __nv_bfloat16* X = (isv ? a.V : a.K) + t * C + h * 128;
#pragma unroll
        for (int i = 0; i < 16; ++i)
          xin[i] = valid ? __ldcs(reinterpret_cast<const uint4*>(X) + i) : make_uint4(0, 0, 0, 0);
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          cin[i] = (valid && i * 16 < row_bytes) ? __ldcs(reinterpret_cast<const uint4*>(codes) + i)
                                                 : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int g = 0; g < NG; ++g) pin[g] = valid ? params[g] : __floats2half2_rn(0.f, 0.f);
      }
      // V(f) reads K^_f: the V epilogue of frame f starts after the K epilogue of f
      if (!anchor) {
        wait(acc_full, acc_use & 1, abort_flag, a.err, 0x2210u + isv);
        acc_use++;
        tc_fence_after();
      }
      uint8_t* tile = isv ? Vb : Kb(f);
      uint32_t cw[16] = {0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0};
      const uint32_t* cwin = reinterpret_cast<const uint32_t*>(cin);
      __nv_bfloat16* rec = isv ? a.vrec : a.krec;
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        float sf, zf;
        if (ENC) {
          float mn = INFINITY, mx = -INFINITY;
#pragma unroll
          for (int pc = 0; pc < NP; ++pc) {
            float p[32];
            if (anchor) {
#pragma unroll
              for (int i = 0; i < 32; ++i) p[i] = 0.f;
            } else {
              tmem_ld32(acc_addr + g * G + pc * 32, p);
            }
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
              float x[8];
              unpack_bf16x8(xin[(g * G + pc * 32) / 8 + ch], x, 0);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float r = x[i] - p[ch * 8 + i];
                mn = fminf(mn, r);
                mx = fmaxf(mx, r);
              }
            }
          }
          const __half sh = __float2half_rn((mx - mn) / (float)levels);
          const __half zh = __float2half_rn(mn);
          sf = __half2float(sh);
          zf = __half2float(zh);
          if (valid) params[g] = __halves2half2(sh, zh);
        } else {
          const float2 fz = __half22float2(pin[g]);
          sf = fz.x;
          zf = fz.y;
        }
        const float inv = sf > 0.f ? 1.f / sf : 0.f;
#pragma unroll
        for (int pc = 0; pc < NP; ++pc) {
          const int e0 = g * G + pc * 32;
          float p[32];
          if (anchor) {
#pragma unroll
            for (int i = 0; i < 32; ++i) p[i] = 0.f;
          } else {
            tmem_ld32(acc_addr + e0, p);
          }
          uint4 recw[4];
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            const int e = e0 + ch * 8;
            float r[8];  // reconstruction
            if (ENC) {
              float x[8];
              unpack_bf16x8(xin[e / 8], x, 0);
              if (bits == 2)
                cw[e / 16] |= quant8<2>(x, &p[ch * 8], sf, zf, inv, r) << ((e % 16) * 2);
              else
                cw[e / 8] = quant8<4>(x, &p[ch * 8], sf, zf, inv, r);
            } else {
              if (bits == 2)
                dequant8<2>(cwin[e / 16], e, sf, zf, &p[ch * 8], r);
              else
                dequant8<4>(cwin[e / 8], e, sf, zf, &p[ch * 8], r);
            }
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) w[i] = pack_bf16x2(r[2 * i], r[2 * i + 1]);
            recw[ch] = make_uint4(w[0], w[1], w[2], w[3]);
          }
          // the tile of K^_f is being read by K(f)'s MMA (lag 2) until acc_full: safe now
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            const int e = e0 + ch * 8;
            *reinterpret_cast<uint4*>(tile + (e / 64) * 16384 + sw128_off(row, (e % 64) / 8)) = recw[ch];
            if (rec && valid) reinterpret_cast<uint4*>(rec + t * C + h * 128 + e)[0] = recw[ch];
          }
        }
      }
      if (ENC && valid) {
        uint4* dst = reinterpret_cast<uint4*>(codes);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (i * 16 < row_bytes) dst[i] = make_uint4(cw[4 * i], cw[4 * i + 1], cw[4 * i + 2], cw[4 * i + 3]);
      }
      tc_fence_before();
      fence_async_smem();
      mbar_arrive(isv ? vready : kready);
      // the V epilogue of frame f needs K^_f in the tile before the MMA of V(f) reads both;
      // the MMA waits kready(f) and vready(f-1), so no extra ordering is needed here
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <bool ENC, int G>
static cudaError_t launch(const Maps& m, const Args& a, cudaStream_t st) {
  auto k = temporal_kernel<ENC, G>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  const int64_t Fp = a.F < a.T ? a.F : a.T;
  dim3 grid((unsigned)((Fp + 127) / 128), (unsigned)a.H);
  k<<<grid, kThreads, kSmem, st>>>(m, a);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace temporal
}  // namespace tc

bool tc_temporal_supported(const kvc_layer_desc* d, const kvc_predictor* p) {
  if (p->kind != KVC_PRED_TEMPORAL) return false;
  if (d->dtype != KVC_BF16 || d->head_dim != 128 || d->param_dtype != KVC_F16) return false;
  if (d->bits != 2 && d->bits != 4) return false;
  if (d->anchor_bits != 0 && d->anchor_bits != 2 && d->anchor_bits != 4) return false;
  if (d->group != 32 && d->group != 64) return false;
  return d->n_tokens >= 1;
}

cudaError_t tc_temporal_layer(const kvc_layer_desc* d, const kvc_predictor* p, bool enc, const void* K, const void* V,
                              const void* Ks, const void* Vs, const kvc_codes* c, void* Kr, void* Vr,
                              cudaStream_t st) {
  const uint64_t H = d->n_heads, C = H * 128, F = d->frame_tokens;
  tc::temporal::Maps m;
  memset(&m, 0, sizeof(m));
  bool ok = tc::map2d(&m.ak, p->k_block, H * 128, 256, 128) && tc::map2d(&m.av, p->v_block, H * 128, 256, 128);
  if (ok && d->anchor_bits == 0) ok = tc::map2d(&m.ksrc, Ks, 2 * F, C, 128) && tc::map2d(&m.vsrc, Vs, F, C, 128);
  if (!ok) return cudaErrorInvalidValue;
  unsigned* err = tc_error_word();
  if (!err) return cudaErrorInvalidDevice;
  tc::temporal::Args a{err, d->n_tokens, (int64_t)F, (int)H, d->bits, d->anchor_bits,
                       (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, (uint8_t*)c->k_codes,
                       (__half2*)c->k_params, (uint8_t*)c->v_codes, (__half2*)c->v_params,
                       (__nv_bfloat16*)Kr, (__nv_bfloat16*)Vr};
  if (d->group == 32)
    return enc ? tc::temporal::launch<true, 32>(m, a, st) : tc::temporal::launch<false, 32>(m, a, st);
  return enc ? tc::temporal::launch<true, 64>(m, a, st) : tc::temporal::launch<false, 64>(m, a, st);
}

}  // namespace kvc
