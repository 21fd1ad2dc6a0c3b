// Clustered codec on the tensor cores (tcgen05 + TMEM + TMA), one tensor (K or V)
// of one layer per call.
//
// ("NanoKV: High-Ratio KV Cache Compression for Autoregressive Video
// Generation", abstract: each row is predicted by its nearest cluster centre
// over the head-concatenated dimension and the residual is coded as a few
// coefficients.)  Per 128-token tile:
//
//   encode: S = X C^T (N = 256 centres) and Y = X E^T (N = 128 coefficients)
//           accumulate together over 64-channel chunks of X; then per token
//           a = argmin_j |c_j|^2 - 2 S_j (ties to the lowest j), coef = Y - P[a]
//           with P = C E^T, group quantization of coef, codes / params / a.
//   decode: x^ = c_a + coef^ W_dec^T, coef^ carried into the MMA as a bf16
//           hi + lo pair (error <= 2^-16 relative), N = 256 output chunks
//           double-buffered in TMEM; the centre row is added in the epilogue.
//
// Warp roles: 0 TMA producer, 1 MMA issuer (TMEM owner), then the epilogue
// warps (4 for the encode, 8 for the decode: two groups, one per half of an
// output chunk).  Every wait is bounded.
#include <cuda.h>
#include <string.h>

#include "tc.h"
#include "tc_ptx.cuh"

namespace kvc {
namespace tc {

bool map2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);
bool map2d_bytes(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                 uint32_t box_rows);
bool map2d_bytes_sw64(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);

namespace cluster {

// ---------------------------------------------------------------- encode

constexpr int kEncThreads = 192;
constexpr int kEncStages = 3;
constexpr int kEncStage = 65536;  // X 16 KB + centres 32 KB + encoder 16 KB
constexpr int kEncBar = kEncStages * kEncStage;
constexpr int kEncCn = kEncBar + 512;  // |c_j|^2, 256 floats
constexpr int kEncSmem = kEncCn + 1024 + 1024;

struct EncMaps {
  CUtensorMap x, cent, enc;  // [T][C], [n_c][C] (box 256 rows), [128][C]
};
struct EncArgs {
  unsigned* err;
  int64_t T;
  int C, n_c;
  const float* cnorm;  // [n_c]
  float* P;            // [n_c][128]: read by the encode, written in PMODE
  uint8_t* codes;      // [T][128 * bits / 8]
  __half2* params;     // [T][128 / G]
  uint8_t* assign;     // [T]
};

// PMODE: the rows are the centres themselves and the kernel writes Y = C E^T to
// P (fp32), so that a token equal to its centre gets Y - P[a] = 0 exactly (the
// same products summed in the same order); it loads no centre box and issues
// no S products, which P does not need.  blockIdx.y selects the tensor
// (maps0 / a0 or maps1 / a1), so the short P passes of K and V share a launch.
template <int BITS, int G, bool PMODE>
__global__ void __launch_bounds__(kEncThreads, 1)
    enc_kernel(const __grid_constant__ EncMaps maps0, const EncArgs a0, const __grid_constant__ EncMaps maps1,
               const EncArgs a1) {
  const EncMaps& maps = blockIdx.y ? maps1 : maps0;
  const EncArgs a = blockIdx.y ? a1 : a0;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kEncBar);
  uint64_t* full = bars;                  // [kEncStages]
  uint64_t* empty = full + kEncStages;    // [kEncStages]
  uint64_t* acc_full = empty + kEncStages;
  uint64_t* mma_done = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* cn = reinterpret_cast<float*>(smem + kEncCn);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * 128;
  const int NCH = a.C / 64;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kEncStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_async_smem();
  }
  for (int j = threadIdx.x; j < 256; j += blockDim.x) cn[j] = j < a.n_c ? a.cnorm[j] : INFINITY;
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t SC = tmem, YC = tmem + 256;  // scores (256 columns), coefficients (128)
  auto stX = [&](int s) { return smem + s * kEncStage; };
  auto stC = [&](int s) { return smem + s * kEncStage + 16384; };
  auto stE = [&](int s) { return smem + s * kEncStage + 49152; };

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      int s = 0;
      uint32_t ph = 0;
      int issued[kEncStages] = {};
      uint32_t issued_ph[kEncStages] = {};
      for (int c = 0; c < NCH; ++c) {
        if (!wait(&empty[s], ph ^ 1, abort_flag, a.err, 0x3100u + s)) break;
        // the P pass needs Y only: no centre box, and no S products below
        mbar_arrive_expect_tx(&full[s], PMODE ? 32768u : (uint32_t)kEncStage);
        tma_load(stX(s), &maps.x, c * 64, t0, &full[s], pol_stream);
        if (!PMODE) tma_load(stC(s), &maps.cent, c * 64, 0, &full[s], pol_keep);
        tma_load(stE(s), &maps.enc, c * 64, 0, &full[s], pol_keep);
        issued[s] = 1;
        issued_ph[s] = ph;
        if (++s == kEncStages) {
          s = 0;
          ph ^= 1;
        }
      }
      if (*abort_flag) {
        for (int i = 0; i < kEncStages; ++i) {
          if (!issued[i]) continue;
          const long long w0 = clock64();
          while (!mbar_test(&full[i], issued_ph[i]) && clock64() - w0 < kWaitBudget) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint32_t id256 = idesc_bf16(128, 256), id128 = idesc_bf16(128, 128);
      int s = 0;
      uint32_t ph = 0;
      for (int c = 0; c < NCH; ++c) {
        if (!wait(&full[s], ph, abort_flag, a.err, 0x3200u + s)) break;
        tc_fence_after();
        const uint64_t ad = desc_sw128(smem_u32(stX(s)));
        const uint64_t cd = desc_sw128(smem_u32(stC(s)));
        const uint64_t ed = desc_sw128(smem_u32(stE(s)));
        if (!PMODE) {
#pragma unroll
          for (int k = 0; k < 4; ++k) umma(SC, ad + 2 * k, cd + 2 * k, id256, (c == 0 && k == 0) ? 0u : 1u);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) umma(YC, ad + 2 * k, ed + 2 * k, id128, (c == 0 && k == 0) ? 0u : 1u);
        umma_commit(&empty[s]);
        if (++s == kEncStages) {
          s = 0;
          ph ^= 1;
        }
      }
      umma_commit(acc_full);
      umma_commit(mma_done);
      const long long w0 = clock64();
      while (!mbar_test(mma_done, 0) && clock64() - w0 < kWaitBudget) {
      }
    }
  } else {
    // ================================================================ epilogue (warps 2-5), one token per thread
    const int qd = warp & 3;
    const int row = qd * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(qd * 32) << 16);
    const int64_t t = (int64_t)t0 + row;
    const bool valid = t < a.T;
    constexpr int LEVELS = (1 << BITS) - 1;
    constexpr int NG = 128 / G, NP = G / 32;
    constexpr int GW = G * BITS / 32;  // code words of a group
    wait(acc_full, 0, abort_flag, a.err, 0x3300u);
    tc_fence_after();
    if (PMODE) {
      float* dst = a.P + t * 128;
      for (int pc = 0; pc < 4; ++pc) {
        float v[32];
        tmem_ld32(lane_addr + (YC - tmem) + pc * 32, v);
        if (valid) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            reinterpret_cast<float4*>(dst + pc * 32)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
      }
    } else {
      // nearest centre: |c_j|^2 - 2 x.c_j, ascending j, strict <, so ties go to the lowest j
      float best = INFINITY;
      int bj = 0;
      for (int jb = 0; jb < 8; ++jb) {
        float v[32];
        tmem_ld32(lane_addr + (SC - tmem) + jb * 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float sc = cn[jb * 32 + i] - 2.f * v[i];
          if (sc < best) {
            best = sc;
            bj = jb * 32 + i;
          }
        }
      }
      const float* Pa = a.P + (int64_t)bj * 128;
      uint32_t* codes = reinterpret_cast<uint32_t*>(a.codes + t * (128 * BITS / 8));
      for (int g = 0; g < NG; ++g) {
        // coef = X E^T - P[a] over the group's NP passes of 32
        float r[NP][32];
        float mn = INFINITY, mx = -INFINITY;
#pragma unroll
        for (int pc = 0; pc < NP; ++pc) {
          tmem_ld32(lane_addr + (YC - tmem) + g * G + pc * 32, r[pc]);
          const float4* pp = reinterpret_cast<const float4*>(Pa + g * G + pc * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 p4 = __ldg(pp + i);
            r[pc][4 * i] -= p4.x;
            r[pc][4 * i + 1] -= p4.y;
            r[pc][4 * i + 2] -= p4.z;
            r[pc][4 * i + 3] -= p4.w;
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            mn = fminf(mn, r[pc][i]);
            mx = fmaxf(mx, r[pc][i]);
          }
        }
        const __half sh = __float2half_rn((mx - mn) / (float)LEVELS);
        const __half zh = __float2half_rn(mn);
        const float sf = __half2float(sh), zf = __half2float(zh);
        const float inv = sf > 0.f ? 1.f / sf : 0.f;
        const float top = kGridMagic + (float)LEVELS;
        uint32_t gw[GW];
#pragma unroll
        for (int i = 0; i < GW; ++i) gw[i] = 0;
#pragma unroll
        for (int pc = 0; pc < NP; ++pc)
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t v = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i)
              v += __float_as_uint(grid_point(r[pc][ch * 8 + i] - zf, inv, top)) << (i * BITS);
            v -= grid_pack_bias(BITS, 8);
            const int eg = pc * 32 + ch * 8;  // element within the group
            if (BITS == 2)
              gw[eg / 16] |= v << ((eg % 16) * 2);
            else
              gw[eg / 8] = v;
          }
        if (valid) {
#pragma unroll
          for (int i = 0; i < GW; i += 2) *reinterpret_cast<uint2*>(codes + g * GW + i) = make_uint2(gw[i], gw[i + 1]);
          a.params[t * NG + g] = __halves2half2(sh, zh);
        }
      }
      if (valid) a.assign[t] = (uint8_t)bj;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- decode

constexpr int kDecThreads = 320;
constexpr int kDecStages = 2;
constexpr int kDecStage = 65536;  // W_dec rows of one 256-wide output chunk, two [256][64] sub-tiles
constexpr int kDecA = kDecStages * kDecStage;  // [coef^ hi | coef^ lo], four [128][64] sub-tiles
constexpr int kDecOut = kDecA + 65536;          // output boxes [32 rows][64 bytes], two per epilogue warp
constexpr int kDecBar = kDecOut + 8 * 2 * 2048;
constexpr int kDecSmem = kDecBar + 1024 + 1024;

struct DecMaps {
  CUtensorMap dec;  // [C][128], box 256 rows
  CUtensorMap out;  // x^ [T][C] as bytes, box 32 rows x 64 bytes, 64-byte swizzle
};
struct DecArgs {
  unsigned* err;
  int64_t T;
  int C, n_c;
  const uint8_t* codes;
  const __half2* params;
  const uint8_t* assign;
  const __nv_bfloat16* cent;  // [n_c][C]
  __nv_bfloat16* out;         // [T][C]
};

// blockIdx.y selects the tensor (maps0 / a0 or maps1 / a1): the K and V decodes
// of a layer share one launch, so that their 2 x 256 tiles fill the SMs' waves
// together.
template <int BITS, int G>
__global__ void __launch_bounds__(kDecThreads, 1)
    dec_kernel(const __grid_constant__ DecMaps maps0, const DecArgs a0, const __grid_constant__ DecMaps maps1,
               const DecArgs a1) {
  const DecMaps& maps = blockIdx.y ? maps1 : maps0;
  const DecArgs a = blockIdx.y ? a1 : a0;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kDecBar);
  uint64_t* full = bars;                 // [kDecStages]
  uint64_t* empty = full + kDecStages;   // [kDecStages]
  uint64_t* a_ready = empty + kDecStages;
  uint64_t* acc_full = a_ready + 1;      // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * 128;
  const int NN = a.C / 256;  // output chunks

  if (threadIdx.x == 0) {
    for (int i = 0; i < kDecStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(a_ready, 256);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 256);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto stB = [&](int s) { return smem + s * kDecStage; };
  uint8_t* At = smem + kDecA;

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      const uint64_t pol_keep = policy_evict_last();
      int s = 0;
      uint32_t ph = 0;
      int issued[kDecStages] = {};
      uint32_t issued_ph[kDecStages] = {};
      for (int n = 0; n < NN; ++n) {
        if (!wait(&empty[s], ph ^ 1, abort_flag, a.err, 0x3400u + s)) break;
        mbar_arrive_expect_tx(&full[s], (uint32_t)kDecStage);
        tma_load(stB(s), &maps.dec, 0, n * 256, &full[s], pol_keep);
        tma_load(stB(s) + 32768, &maps.dec, 64, n * 256, &full[s], pol_keep);
        issued[s] = 1;
        issued_ph[s] = ph;
        if (++s == kDecStages) {
          s = 0;
          ph ^= 1;
        }
      }
      if (*abort_flag) {
        for (int i = 0; i < kDecStages; ++i) {
          if (!issued[i]) continue;
          const long long w0 = clock64();
          while (!mbar_test(&full[i], issued_ph[i]) && clock64() - w0 < kWaitBudget) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint32_t id256 = idesc_bf16(128, 256);
      const uint64_t ad = desc_sw128(smem_u32(At));
      int s = 0;
      uint32_t ph = 0;
      bool ok = wait(a_ready, 0, abort_flag, a.err, 0x3500u);
      for (int n = 0; n < NN && ok; ++n) {
        const int b = n & 1;
        if (n >= 2 && !wait(&acc_empty[b], ((n - 2) >> 1) & 1, abort_flag, a.err, 0x3510u + b)) break;
        if (!wait(&full[s], ph, abort_flag, a.err, 0x3520u + s)) break;
        tc_fence_after();
        const uint64_t bd = desc_sw128(smem_u32(stB(s)));
        // K = 256: coef^ hi (A sub-tiles 0, 1) then coef^ lo (A sub-tiles 2, 3), both against the
        // same two W_dec sub-tiles
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const uint32_t aoff = (k >> 2) * (16384 >> 4) + (k & 3) * 2;
          const uint32_t boff = ((k >> 2) & 1) * (32768 >> 4) + (k & 3) * 2;
          umma(tmem + b * 256, ad + aoff, bd + boff, id256, k == 0 ? 0u : 1u);
        }
        umma_commit(&empty[s]);
        umma_commit(&acc_full[b]);
        if (++s == kDecStages) {
          s = 0;
          ph ^= 1;
        }
      }
      umma_commit(mma_done);
      const long long w0 = clock64();
      while (!mbar_test(mma_done, 0) && clock64() - w0 < kWaitBudget) {
      }
    }
  } else {
    // ================================================================ epilogue (warps 2-9): two groups of 4
    const int grp = (warp - 2) >> 2;  // 0: columns [0, 128) of a chunk, 1: [128, 256)
    const int qd = warp & 3;
    const int row = qd * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(qd * 32) << 16);
    const int64_t t = (int64_t)t0 + row;
    const bool valid = t < a.T;
    constexpr int NGH = 64 / G > 0 ? 64 / G : 1;  // groups touched by one half of the coefficients
    // coef^ of this token's half of the coefficients -> hi / lo bf16 A sub-tiles
    {
      constexpr int RB = 128 * BITS / 8;
      uint32_t cw[RB / 8];  // the half's code words
      const uint4* src = reinterpret_cast<const uint4*>(a.codes + t * RB + grp * (RB / 2));
#pragma unroll
      for (int i = 0; i < RB / 32; ++i) {
        const uint4 w = valid ? __ldcs(src + i) : make_uint4(0, 0, 0, 0);
        cw[4 * i] = w.x;
        cw[4 * i + 1] = w.y;
        cw[4 * i + 2] = w.z;
        cw[4 * i + 3] = w.w;
      }
      const float zero[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int e = 0; e < 64; e += 8) {
        const int ge = grp * 64 + e;  // coefficient index
        const __half2 pz = valid ? a.params[t * (128 / G) + ge / G] : __floats2half2_rn(0.f, 0.f);
        const float2 f = __half22float2(pz);
        float r[8];
        dequant8<BITS>(cw[BITS == 2 ? e / 16 : e / 8], e, f.x, f.y, zero, r);
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(r[2 * i], r[2 * i + 1]);
          const float2 hf = __bfloat1622float2(h2);
          hi[i] = *reinterpret_cast<const uint32_t*>(&h2);
          lo[i] = pack_bf16x2(r[2 * i] - hf.x, r[2 * i + 1] - hf.y);
        }
        *reinterpret_cast<uint4*>(At + grp * 16384 + sw128_off(row, e / 8)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(At + (2 + grp) * 16384 + sw128_off(row, e / 8)) =
            make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      (void)NGH;
      fence_async_smem();
      mbar_arrive(a_ready);
    }
    // The centre rows are gathered coalesced: lane l fetches the 16-byte piece
    // l & 3 of the 64 bytes a box holds for rows (l >> 2) + 8 j, j = 0..3, of
    // this warp's 32 tokens (a load instruction covers 8 rows x 64 contiguous
    // bytes; a row per lane would touch 32 lines per instruction).
    int c = t < a.T ? (int)a.assign[t] : 0;
    c = c < a.n_c ? c : a.n_c - 1;
    const __nv_bfloat16* cbase[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int cj = __shfl_sync(0xffffffffu, c, (lane >> 2) + 8 * j);
      cbase[j] = a.cent + (int64_t)cj * a.C + (lane & 3) * 8;
    }
    // x^ leaves through shared memory and TMA stores (row-per-thread global
    // stores cost a request per 16 bytes): per 32 columns the warp fills one of
    // its two [32 rows][64 bytes] boxes, laid out with the 64-byte swizzle (the
    // store's tensor map undoes it): piece q of row r at chunk q ^ ((r >> 1) & 3).
    // The gathered centre pieces are first written to the box (8 whole rows per
    // instruction); each lane then reads its own row's four pieces, adds the
    // product and writes the result in place.  The swizzle spreads a row-per-lane
    // access of one piece over eight bank groups.
    auto sw = [](int r, int q) { return r * 64 + ((q ^ ((r >> 1) & 3)) << 4); };
    uint8_t* obox = smem + kDecOut + (warp - 2) * 4096;
    int ob = 0;
    for (int n = 0; n < NN; ++n) {
      const int b = n & 1;
      // this half chunk's centre pieces, fetched while the MMAs run
      uint4 cv[16];
#pragma unroll
      for (int cb = 0; cb < 4; ++cb)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          cv[cb * 4 + j] = __ldg(reinterpret_cast<const uint4*>(cbase[j] + n * 256 + grp * 128 + cb * 32));
      wait(&acc_full[b], (n >> 1) & 1, abort_flag, a.err, 0x3600u + b);
      tc_fence_after();
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) {
        const int col = n * 256 + grp * 128 + cb * 32;  // output channel
        float v[32];
        tmem_ld32(lane_addr + b * 256 + grp * 128 + cb * 32, v);
        uint8_t* box = obox + ob * 2048;
        if (lane == 0) bulk_wait_read1();  // the store that last read this box is done with it
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<uint4*>(box + sw((lane >> 2) + 8 * j, lane & 3)) = cv[cb * 4 + j];
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint4* piece = reinterpret_cast<uint4*>(box + sw(lane, i));
          float cc[8];
          unpack_bf16x8(*piece, cc, 0);
          const float* vi = v + 8 * i;
          *piece = make_uint4(pack_bf16x2(cc[0] + vi[0], cc[1] + vi[1]), pack_bf16x2(cc[2] + vi[2], cc[3] + vi[3]),
                              pack_bf16x2(cc[4] + vi[4], cc[5] + vi[5]), pack_bf16x2(cc[6] + vi[6], cc[7] + vi[7]));
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0 && t0 + qd * 32 < a.T) {  // the tensor map clips rows past T
          tma_store(&maps.out, col * 2, t0 + qd * 32, box);
          bulk_commit();
        }
        ob ^= 1;
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[b]);
    }
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// one tensor (n = 1) or two of the same row count (n = 2: m1 / a1 as the second)
template <int BITS, int G, bool PMODE = false>
static cudaError_t launch_enc(const EncMaps& m, const EncArgs& a, cudaStream_t st, int n = 1,
                              const EncMaps* m1 = nullptr, const EncArgs* a1 = nullptr) {
  auto k = enc_kernel<BITS, G, PMODE>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kEncSmem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((a.T + 127) / 128), (unsigned)n);
  k<<<grid, kEncThreads, kEncSmem, st>>>(m, a, n == 2 ? *m1 : m, n == 2 ? *a1 : a);
  count_launches(1);
  return cudaGetLastError();
}
// one tensor (n = 1) or two of the same row count (n = 2: m[1] / a[1] as the second)
template <int BITS, int G>
static cudaError_t launch_dec(const DecMaps* m, const DecArgs* a, int n, cudaStream_t st) {
  auto k = dec_kernel<BITS, G>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((a[0].T + 127) / 128), (unsigned)n);
  k<<<grid, kDecThreads, kDecSmem, st>>>(m[0], a[0], m[n - 1], a[n - 1]);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace cluster
}  // namespace tc

bool tc_cluster_supported(const kvc_layer_desc* d, const kvc_predictor* p) {
  if (p->kind != KVC_PRED_CLUSTER) return false;
  if (d->dtype != KVC_BF16 || d->param_dtype != KVC_F16) return false;
  if (d->bits != 2 && d->bits != 4) return false;
  if (d->group != 32 && d->group != 64) return false;
  const int64_t C = (int64_t)d->n_heads * d->head_dim;
  if (p->code_dim != 128 || p->n_clusters < 1 || p->n_clusters > 256) return false;
  if (C % 256 != 0 || C * 2 > (1 << 20) || d->n_tokens < 1) return false;
  return true;
}

cudaError_t tc_cluster_encode(const kvc_layer_desc* d, const kvc_predictor* p, const void* const X[2],
                              const float* const cnorm[2], float* const P[2], void* const codes[2],
                              void* const params[2], void* const assign[2], cudaStream_t st) {
  const uint64_t T = (uint64_t)d->n_tokens, C = (uint64_t)d->n_heads * d->head_dim;
  const void* cent[2] = {p->k_centroids, p->v_centroids};
  const void* enc[2] = {p->k_enc, p->v_enc};
  unsigned* err = tc_error_word();
  if (!err) return cudaErrorInvalidDevice;
  tc::cluster::EncMaps m[2];
  tc::cluster::EncArgs a[2];
  for (int w = 0; w < 2; ++w) {
    memset(&m[w], 0, sizeof(m[w]));
    if (!(tc::map2d(&m[w].x, X[w], T, C, 128) && tc::map2d(&m[w].cent, cent[w], (uint64_t)p->n_clusters, C, 256) &&
          tc::map2d(&m[w].enc, enc[w], 128, C, 128)))
      return cudaErrorInvalidValue;
    a[w] = tc::cluster::EncArgs{err, (int64_t)T, (int)C, p->n_clusters, cnorm[w], P[w], (uint8_t*)codes[w],
                                (__half2*)params[w], (uint8_t*)assign[w]};
  }
  using namespace tc::cluster;
  if (d->bits == 2)
    return d->group == 32 ? launch_enc<2, 32>(m[0], a[0], st, 2, &m[1], &a[1])
                          : launch_enc<2, 64>(m[0], a[0], st, 2, &m[1], &a[1]);
  return d->group == 32 ? launch_enc<4, 32>(m[0], a[0], st, 2, &m[1], &a[1])
                        : launch_enc<4, 64>(m[0], a[0], st, 2, &m[1], &a[1]);
}

cudaError_t tc_cluster_prepare(const kvc_layer_desc* d, const kvc_predictor* p, const float* const cnorm[2],
                               float* const P[2], cudaStream_t st) {
  const uint64_t C = (uint64_t)d->n_heads * d->head_dim;
  const void* cent[2] = {p->k_centroids, p->v_centroids};
  const void* enc[2] = {p->k_enc, p->v_enc};
  unsigned* err = tc_error_word();
  if (!err) return cudaErrorInvalidDevice;
  tc::cluster::EncMaps m[2];
  tc::cluster::EncArgs a[2];
  for (int w = 0; w < 2; ++w) {
    memset(&m[w], 0, sizeof(m[w]));
    if (!(tc::map2d(&m[w].x, cent[w], (uint64_t)p->n_clusters, C, 128) &&
          tc::map2d(&m[w].cent, cent[w], (uint64_t)p->n_clusters, C, 256) && tc::map2d(&m[w].enc, enc[w], 128, C, 128)))
      return cudaErrorInvalidValue;
    a[w] = tc::cluster::EncArgs{err, (int64_t)p->n_clusters, (int)C, p->n_clusters, cnorm[w], P[w],
                                nullptr, nullptr, nullptr};
  }
  return tc::cluster::launch_enc<4, 32, true>(m[0], a[0], st, 2, &m[1], &a[1]);
}

cudaError_t tc_cluster_decode(const kvc_layer_desc* d, const kvc_predictor* p, const void* const codes[2],
                              const void* const params[2], const void* const assign[2], void* const out[2],
                              cudaStream_t st) {
  const uint64_t T = (uint64_t)d->n_tokens, C = (uint64_t)d->n_heads * d->head_dim;
  const void* cent[2] = {p->k_centroids, p->v_centroids};
  const void* dec[2] = {p->k_dec, p->v_dec};
  unsigned* err = tc_error_word();
  if (!err) return cudaErrorInvalidDevice;
  tc::cluster::DecMaps m[2];
  tc::cluster::DecArgs a[2];
  int n = 0;
  for (int w = 0; w < 2; ++w) {
    if (!out[w]) continue;
    memset(&m[n], 0, sizeof(m[n]));
    if (!tc::map2d(&m[n].dec, dec[w], C, 128, 256) || !tc::map2d_bytes_sw64(&m[n].out, out[w], T, C * 2, 32))
      return cudaErrorInvalidValue;
    a[n] = tc::cluster::DecArgs{err, (int64_t)T, (int)C, p->n_clusters, (const uint8_t*)codes[w],
                                (const __half2*)params[w], (const uint8_t*)assign[w], (const __nv_bfloat16*)cent[w],
                                (__nv_bfloat16*)out[w]};
    ++n;
  }
  if (n == 0) return cudaSuccess;
  using namespace tc::cluster;
  if (d->bits == 2)
    return d->group == 32 ? launch_dec<2, 32>(m, a, n, st) : launch_dec<2, 64>(m, a, n, st);
  return d->group == 32 ? launch_dec<4, 32>(m, a, n, st) : launch_dec<4, 64>(m, a, n, st);
}

}  // namespace kvc
