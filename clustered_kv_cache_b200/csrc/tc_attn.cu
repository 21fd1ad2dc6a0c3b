// Attention over a compressed cross-layer history (tcgen05 + TMEM + TMA).
//
//   O = softmax(scale Q [K^_hist ; K_self]^T) [V^_hist ; V_self]
//
// ("NanoKV: High-Ratio KV Cache Compression for Autoregressive Video
// Generation", abstract: attention over the compressed history is the
// bottleneck; "CORAL-KV ...", Fig. 3: the history of layer l is decoded from
// its codes and the reconstruction of layer l-1.)  One CTA per (head, 128-query
// tile).  The history is decoded tile by tile on chip and never written to
// device memory: for each 128-key tile the CTA runs the block-DPLR prediction on
// the tensor cores (the layer's low-rank latents come precomputed, as bf16
// hi / lo pairs, from the latent-only codec kernel), adds the dequantized codes
// and keeps the bf16 K^ / V^ tile in shared memory.  Then S = Q K^T and
// O += P V^ run on tcgen05 with the softmax on four warps.
//
// Warp roles: 0 TMA producer, 1 MMA issuer (and TMEM owner), 2-5 decode
// epilogue (TMEM -> K^ / V^ tiles), 6-9 softmax (S -> P, running max / sum,
// lazy rescaling of O, final normalisation).  TMEM: decode-K accumulator, decode-V
// accumulator, S, O (128 columns each).
#include <cuda.h>
#include <string.h>

#include "tc.h"
#include "tc_ptx.cuh"

namespace kvc {
namespace tc {

bool map2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);
bool map2d_bytes(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                 uint32_t box_rows);

namespace attn {

constexpr int kThreads = 320;
constexpr int kStages = 2;
constexpr int kStage = 32768;
// shared memory (offsets from a 1024-aligned base)
constexpr int kQ = 0;                        // Q tile, 2 sub-tiles
constexpr int kK = kQ + 32768;               // K^ tiles [2]
constexpr int kV = kK + 2 * 32768;           // V^ tile
constexpr int kP = kV + 32768;               // P tile
constexpr int kSt = kP + 32768;              // operand stages
constexpr int kBar = kSt + kStages * kStage;
constexpr int kSmem = kBar + 1024 + 1024;    // + barriers + alignment slack

struct Maps {
  CUtensorMap q;             // [n_q][C]
  CUtensorMap ks, vs;        // reconstructions of layer l-1 [T][C]
  CUtensorMap kself, vself;  // [n_self][C]
  CUtensorMap bk, bv;        // [H*128][128], [H*128][256]
  CUtensorMap uk, uv;        // [C][r]
  CUtensorMap zkh, zkl, zvh, zvl;  // latents [T][r]
  CUtensorMap ck, cv, pk, pv;      // codes / params as bytes, for L2 prefetches
};

struct Args {
  unsigned* err;
  int64_t n_q, T, n_self;
  int H, bits, group;
  float scale_log2;  // softmax scale * log2(e)
  const uint8_t* kcodes;
  const __half2* kparams;
  const uint8_t* vcodes;
  const __half2* vparams;
  __nv_bfloat16* O;  // [n_q][H][128]
};

// MN-major operand (N contiguous), 128-byte swizzle: sub-tiles of 64 N values
// lbo bytes apart, 8 K-rows per 1024-byte core group.
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t saddr, uint32_t lbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
__host__ __device__ constexpr uint32_t idesc_bf16_bmn(int M, int N) { return idesc_bf16(M, N) | (1u << 16); }

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]),
      "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]),
      "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]),
      "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

template <int RC>
__global__ void __launch_bounds__(kThreads, 1) attend_xlayer_kernel(const __grid_constant__ Maps maps, const Args a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBar);
  uint64_t* full = bars;                  // [kStages]
  uint64_t* empty = bars + kStages;       // [kStages]
  uint64_t* q_full = bars + 2 * kStages;
  uint64_t* d0_full = q_full + 1;         // decode-K accumulator ready
  uint64_t* d1_full = d0_full + 1;        // decode-V accumulator ready
  uint64_t* kt_ready = d1_full + 1;       // [2] K tile in smem (decode warps)
  uint64_t* vt_ready = kt_ready + 2;      // V tile in smem (decode warps)
  uint64_t* s_full = vt_ready + 1;
  uint64_t* p_full = s_full + 1;          // P written (softmax warps)
  uint64_t* pv_done = p_full + 1;         // a PV product finished (O stable, P / V tiles free)
  uint64_t* kt_free = pv_done + 1;        // [2] S and DEC_V of a K tile finished
  uint64_t* self_kfull = kt_free + 2;     // [2] a K_self tile landed
  uint64_t* self_vfull = self_kfull + 2;  // a V_self tile landed
  uint64_t* o_done = self_vfull + 1;
  uint64_t* mma_done = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  constexpr int R = RC * 64;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int q0 = blockIdx.x * 128;
  const int NH = (int)((a.T + 127) / 128);       // history key tiles
  const int NS = (int)((a.n_self + 127) / 128);  // chunk key tiles
  const int NT = NH + NS;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(d0_full, 1);
    mbar_init(d1_full, 1);
    mbar_init(&kt_ready[0], 128);
    mbar_init(&kt_ready[1], 128);
    mbar_init(vt_ready, 128);
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(&kt_free[0], 1);
    mbar_init(&kt_free[1], 1);
    mbar_init(&self_kfull[0], 1);
    mbar_init(&self_kfull[1], 1);
    mbar_init(self_vfull, 1);
    mbar_init(o_done, 1);
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
  const uint32_t D0 = tmem, D1 = tmem + 128, SC = tmem + 256, OC = tmem + 384;

  auto stA = [&](int s) { return smem + kSt + s * kStage; };
  auto stB = [&](int s) { return smem + kSt + s * kStage + 16384; };
  uint8_t* Qs = smem + kQ;
  auto Kt = [&](int b) { return smem + kK + b * 32768; };
  uint8_t* Vt = smem + kV;
  uint8_t* Ps = smem + kP;

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* ma, int ax, int ay, const CUtensorMap* mb, int bx, int by) {
        if (!ok) return;
        if (!wait(&empty[s], ph ^ 1, abort_flag, a.err, 0x1100u + s)) {
          ok = false;
          return;
        }
        mbar_arrive_expect_tx(&full[s], (ma ? 16384u : 0u) + 16384u);
        if (ma) tma_load(stA(s), ma, ax, ay, &full[s], pol_stream);
        tma_load(stB(s), mb, bx, by, &full[s], pol_keep);
        if (++s == kStages) {
          s = 0;
          ph ^= 1;
        }
      };
      mbar_arrive_expect_tx(q_full, 32768u);
      tma_load(Qs, &maps.q, h * 128, q0, q_full, pol_stream);
      tma_load(Qs + 16384, &maps.q, h * 128 + 64, q0, q_full, pol_stream);
      for (int j = 0; j < NT && ok; ++j) {
        const int b = j & 1;
        if (j < NH) {
          const int t0 = j * 128;
          const int rbytes = 128 * a.bits / 8;
          tma_prefetch(&maps.ck, h * rbytes, t0);
          tma_prefetch(&maps.cv, h * rbytes, t0);
          if (a.group == 32) {
            tma_prefetch(&maps.pk, h * 16, t0);
            tma_prefetch(&maps.pv, h * 16, t0);
          }
          // decode K: K^_{l-1,h} B_h^T + [Z_K hi | lo] U_h^T
          for (int c = 0; c < 2; ++c) load(&maps.ks, h * 128 + c * 64, t0, &maps.bk, c * 64, h * 128);
          for (int c = 0; c < RC; ++c) {
            load(&maps.zkh, c * 64, t0, &maps.uk, c * 64, h * 128);
            load(&maps.zkl, c * 64, t0, &maps.uk, c * 64, h * 128);
          }
          // decode V: [K^_{l,h} (resident) | V^_{l-1,h}] BV_h^T + [Z_V hi | lo] UV_h^T
          for (int c = 0; c < 2; ++c) load(nullptr, 0, 0, &maps.bv, c * 64, h * 128);
          for (int c = 0; c < 2; ++c) load(&maps.vs, h * 128 + c * 64, t0, &maps.bv, 128 + c * 64, h * 128);
          for (int c = 0; c < RC; ++c) {
            load(&maps.zvh, c * 64, t0, &maps.uv, c * 64, h * 128);
            load(&maps.zvl, c * 64, t0, &maps.uv, c * 64, h * 128);
          }
        } else {
          // chunk tile: K_self into the K tile once S and DEC_V of tile j-2 are done,
          // V_self into the V tile once PV(j-1) is done (PV(j-1) follows S(j))
          const int s0 = (j - NH) * 128;
          if (j >= 2 && !wait(&kt_free[b], ((j - 2) >> 1) & 1, abort_flag, a.err, 0x1200u + b)) ok = false;
          if (!ok) break;
          mbar_arrive_expect_tx(&self_kfull[b], 32768u);
          tma_load(Kt(b), &maps.kself, h * 128, s0, &self_kfull[b], pol_stream);
          tma_load(Kt(b) + 16384, &maps.kself, h * 128 + 64, s0, &self_kfull[b], pol_stream);
          if (j >= 1 && !wait(pv_done, (j - 1) & 1, abort_flag, a.err, 0x1210u)) ok = false;
          if (!ok) break;
          mbar_arrive_expect_tx(self_vfull, 32768u);
          tma_load(Vt, &maps.vself, h * 128, s0, self_vfull, pol_stream);
          tma_load(Vt + 16384, &maps.vself, h * 128 + 64, s0, self_vfull, pol_stream);
        }
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      const uint32_t id128 = idesc_bf16(128, 128);
      auto chunk = [&](uint32_t d, bool first, const uint8_t* resA) {
        if (!ok) return;
        if (!wait(&full[s], ph, abort_flag, a.err, 0x1300u + s)) {
          ok = false;
          return;
        }
        tc_fence_after();
        const uint64_t ad = desc_sw128(smem_u32(resA ? resA : stA(s)));
        const uint64_t bd = desc_sw128(smem_u32(stB(s)));
#pragma unroll
        for (int k = 0; k < 4; ++k) umma(d, ad + 2 * k, bd + 2 * k, id128, (first && k == 0) ? 0u : 1u);
        umma_commit(&empty[s]);
        if (++s == kStages) {
          s = 0;
          ph ^= 1;
        }
      };
      auto dec_k = [&]() {
        for (int c = 0; c < 2; ++c) chunk(D0, c == 0, nullptr);
        for (int c = 0; c < 2 * RC; ++c) chunk(D0, false, nullptr);
        if (ok) umma_commit(d0_full);
      };
      int kt_use[2] = {0, 0};
      if (!wait(q_full, 0, abort_flag, a.err, 0x1310u)) ok = false;
      tc_fence_after();
      if (NH > 0) dec_k();
      for (int j = 0; j < NT && ok; ++j) {
        const int b = j & 1;
        if (!wait(&kt_ready[b], kt_use[b] & 1, abort_flag, a.err, 0x1320u + b)) ok = false;
        kt_use[b]++;
        // S(j) = Q K^(j)^T; the S columns are free once the softmax of tile j-1 wrote P
        if (ok && j >= 1 && !wait(p_full, (j - 1) & 1, abort_flag, a.err, 0x1330u)) ok = false;
        if (!ok) break;
        tc_fence_after();
        {
          const uint64_t qd = desc_sw128(smem_u32(Qs));
          const uint64_t kd = desc_sw128(smem_u32(Kt(b)));
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t off = (k >> 2) * (16384 >> 4) + (k & 3) * 2;
            umma(SC, qd + off, kd + off, id128, k == 0 ? 0u : 1u);
          }
          umma_commit(s_full);
        }
        // PV(j-1): O += P V^(j-1)
        if (j >= 1) {
          if (!wait(vt_ready, (j - 1) & 1, abort_flag, a.err, 0x1340u)) ok = false;
          tc_fence_after();
          if (ok) {
            const uint64_t pd = desc_sw128(smem_u32(Ps));
            const uint64_t vd = desc_mn_sw128(smem_u32(Vt), 16384);
            const uint32_t idv = idesc_bf16_bmn(128, 128);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint64_t poff = (k >> 2) * (16384 >> 4) + (k & 3) * 2;
              const uint64_t voff = (uint64_t)k * (2048 >> 4);
              umma(OC, pd + poff, vd + voff, idv, j == 1 && k == 0 ? 0u : 1u);
            }
            umma_commit(pv_done);
          }
        }
        // decode V(j) (needs K^(j) as an operand) and K(j+1)
        if (j < NH) {
          for (int c = 0; c < 2; ++c) chunk(D1, c == 0, Kt(b) + c * 16384);
          for (int c = 0; c < 2; ++c) chunk(D1, false, nullptr);
          for (int c = 0; c < 2 * RC; ++c) chunk(D1, false, nullptr);
          if (ok) umma_commit(d1_full);
        }
        if (ok) umma_commit(&kt_free[b]);
        if (j + 1 < NH) dec_k();
      }
      // last PV
      if (ok && NT >= 1) {
        const int j = NT;
        if (!wait(p_full, (j - 1) & 1, abort_flag, a.err, 0x1350u)) ok = false;
        if (ok && !wait(vt_ready, (j - 1) & 1, abort_flag, a.err, 0x1351u)) ok = false;
        tc_fence_after();
        if (ok) {
          const uint64_t pd = desc_sw128(smem_u32(Ps));
          const uint64_t vd = desc_mn_sw128(smem_u32(Vt), 16384);
          const uint32_t idv = idesc_bf16_bmn(128, 128);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint64_t poff = (k >> 2) * (16384 >> 4) + (k & 3) * 2;
            const uint64_t voff = (uint64_t)k * (2048 >> 4);
            umma(OC, pd + poff, vd + voff, idv, j == 1 && k == 0 ? 0u : 1u);
          }
          umma_commit(pv_done);
        }
      }
      umma_commit(o_done);
      umma_commit(mma_done);
      const long long w0 = clock64();
      while (!mbar_test(mma_done, 0) && clock64() - w0 < kWaitBudget) {
      }
    }
  } else if (warp < 6) {
    // ================================================================ decode epilogue (warps 2-5)
    const int qd = warp & 3;
    const int row = qd * 32 + lane;  // key row of the tile (TMEM lane)
    const uint32_t lane_addr = tmem + ((uint32_t)(qd * 32) << 16);
    const int bits = a.bits, levels = (1 << bits) - 1, G = a.group;
    const int row_bytes = 128 * bits / 8;
    int d0_use = 0, d1_use = 0, kself_use[2] = {0, 0}, vself_use = 0;
    // TMEM accumulator + dequantized codes -> bf16 row of a K^ / V^ tile
    auto emit = [&](uint32_t acc, const uint8_t* codes, const __half2* params, bool valid, uint8_t* tile) {
      uint32_t cw[16];
      __half2 pr[4];
#pragma unroll
      for (int i = 0; i < 16; ++i) cw[i] = 0;
      if (valid) {
        const uint4* cp = reinterpret_cast<const uint4*>(codes);
        const int nw = row_bytes / 16;
        for (int i = 0; i < nw; ++i) reinterpret_cast<uint4*>(cw)[i] = __ldcs(cp + i);
        for (int g = 0; g < 128 / G; ++g) pr[g] = params[g];
      }
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        float p[32];
        tmem_ld32(lane_addr + acc + pc * 32, p);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const int e = pc * 32 + ch * 8;  // element of the row
          float sf = 0.f, zf = 0.f;
          if (valid) {
            const float2 f = __half22float2(pr[e / G]);
            sf = f.x;
            zf = f.y;
          }
          const uint32_t v = bits == 2 ? (cw[e / 16] >> ((e % 16) * 2)) : cw[e / 8];
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float c0 = grid_code(grid_from_code((v >> ((2 * i) * bits)) & levels));
            const float c1 = grid_code(grid_from_code((v >> ((2 * i + 1) * bits)) & levels));
            w[i] = pack_bf16x2(p[ch * 8 + 2 * i] + fmaf(sf, c0, zf), p[ch * 8 + 2 * i + 1] + fmaf(sf, c1, zf));
          }
          *reinterpret_cast<uint4*>(tile + (e / 64) * 16384 + sw128_off(row, (e % 64) / 8)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      tc_fence_before();
      fence_async_smem();
    };
    for (int j = 0; j < NT; ++j) {
      const int b = j & 1;
      if (j < NH) {
        const int64_t t = (int64_t)j * 128 + row;
        const bool valid = t < a.T;
        const int64_t rowi = t * a.H + h;
        wait(d0_full, d0_use++ & 1, abort_flag, a.err, 0x1400u);
        tc_fence_after();
        emit(0, a.kcodes + rowi * row_bytes, a.kparams + rowi * (128 / G), valid, Kt(b));
        mbar_arrive(&kt_ready[b]);
        wait(d1_full, d1_use++ & 1, abort_flag, a.err, 0x1401u);
        tc_fence_after();
        emit(128, a.vcodes + rowi * row_bytes, a.vparams + rowi * (128 / G), valid, Vt);
        mbar_arrive(vt_ready);
      } else {
        wait(&self_kfull[b], kself_use[b]++ & 1, abort_flag, a.err, 0x1402u + b);
        mbar_arrive(&kt_ready[b]);
        wait(self_vfull, vself_use++ & 1, abort_flag, a.err, 0x1404u);
        mbar_arrive(vt_ready);
      }
    }
  } else {
    // ================================================================ softmax (warps 6-9)
    const int qd = warp & 3;
    const int row = qd * 32 + lane;  // query row
    const uint32_t lane_addr = tmem + ((uint32_t)(qd * 32) << 16);
    const float c = a.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    for (int j = 0; j < NT; ++j) {
      wait(s_full, j & 1, abort_flag, a.err, 0x1500u);
      tc_fence_after();
      const int64_t kbase = j < NH ? (int64_t)j * 128 : (int64_t)(j - NH) * 128;
      const int64_t klim = j < NH ? a.T : a.n_self;
      const int nvalid = klim - kbase < 128 ? (int)(klim - kbase) : 128;
      float mt = -INFINITY;
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        float sv[32];
        tmem_ld32(lane_addr + (SC - tmem) + pc * 32, sv);
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (pc * 32 + i < nvalid) mt = fmaxf(mt, sv[i] * c);
      }
      // lazy rescale: only when the tile's max exceeds the one in use by 2^8
      const bool need = mt > m_used + 8.f;
      if (__any_sync(0xffffffffu, need && j > 0)) {
        wait(pv_done, (j - 1) & 1, abort_flag, a.err, 0x1501u);  // O holds PV(j-1)
        tc_fence_after();
        const float alpha = need ? exp2f(m_used - mt) : 1.f;
#pragma unroll
        for (int pc = 0; pc < 4; ++pc) {
          float ov[32];
          tmem_ld32(lane_addr + (OC - tmem) + pc * 32, ov);
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] *= alpha;
          tmem_st32(lane_addr + (OC - tmem) + pc * 32, ov);
        }
      }
      if (need) {
        l = (m_used == -INFINITY) ? 0.f : l * exp2f(m_used - mt);
        m_used = mt;
      }
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        float sv[32];
        tmem_ld32(lane_addr + (SC - tmem) + pc * 32, sv);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int k0 = pc * 32 + ch * 8 + 2 * i;
            const float p0 = k0 < nvalid ? exp2f(sv[ch * 8 + 2 * i] * c - m_used) : 0.f;
            const float p1 = k0 + 1 < nvalid ? exp2f(sv[ch * 8 + 2 * i + 1] * c - m_used) : 0.f;
            l += p0 + p1;
            w[i] = pack_bf16x2(p0, p1);
          }
          const int e = pc * 32 + ch * 8;
          *reinterpret_cast<uint4*>(Ps + (e / 64) * 16384 + sw128_off(row, (e % 64) / 8)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      tc_fence_before();
      fence_async_smem();
      mbar_arrive(p_full);
    }
    wait(o_done, 0, abort_flag, a.err, 0x1502u);
    tc_fence_after();
    const int64_t qrow = (int64_t)q0 + row;
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int pc = 0; pc < 4; ++pc) {
      float ov[32];
      tmem_ld32(lane_addr + (OC - tmem) + pc * 32, ov);
      if (qrow < a.n_q) {
        uint4* dst = reinterpret_cast<uint4*>(a.O + (qrow * a.H + h) * 128 + pc * 32);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) w[i] = pack_bf16x2(ov[ch * 8 + 2 * i] * inv, ov[ch * 8 + 2 * i + 1] * inv);
          dst[ch] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int RC>
static cudaError_t launch(const Maps& m, const Args& a, cudaStream_t st) {
  auto k = attend_xlayer_kernel<RC>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((a.n_q + 127) / 128), (unsigned)a.H);
  k<<<grid, kThreads, kSmem, st>>>(m, a);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace attn

cudaError_t latent_layer(const kvc_layer_desc* d, const kvc_predictor* p, const kvc_codes* c, const void* Ks,
                         const void* Vs, void* zk_hi, void* zk_lo, void* zv_hi, void* zv_lo, cudaStream_t st);

}  // namespace tc

bool tc_attend_supported(const kvc_layer_desc* d, const kvc_predictor* p, int64_t n_self) {
  (void)n_self;
  if (p->kind != KVC_PRED_XLAYER_DPLR) return false;
  if (d->dtype != KVC_BF16 || d->head_dim != 128 || d->param_dtype != KVC_F16) return false;
  if (d->bits != 2 && d->bits != 4) return false;
  if (d->group != 32 && d->group != 64) return false;
  if (p->rank != 0 && p->rank != 64 && p->rank != 128) return false;
  return tc_codec_supported(d, p) || d->n_tokens == 0;
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

size_t tc_attend_workspace(const kvc_layer_desc* d, const kvc_predictor* p) {
  return 4 * align256((size_t)d->n_tokens * (size_t)p->rank * 2);
}

cudaError_t tc_attend(const kvc_layer_desc* d, const kvc_predictor* p, const void* Q, int64_t n_q, const kvc_codes* c,
                      const void* Ks, const void* Vs, const void* K_self, const void* V_self, int64_t n_self,
                      float scale, void* O, void* ws, size_t ws_bytes, cudaStream_t st) {
  const uint64_t T = (uint64_t)d->n_tokens, H = d->n_heads, C = H * 128, r = (uint64_t)p->rank;
  if (ws_bytes < tc_attend_workspace(d, p)) return cudaErrorInvalidValue;
  char* w = static_cast<char*>(ws);
  const size_t zb = align256(T * r * 2);
  void* zkh = w;
  void* zkl = w + zb;
  void* zvh = w + 2 * zb;
  void* zvl = w + 3 * zb;
  cudaError_t e;
  if (r > 0 && T > 0) {
    if ((e = tc::latent_layer(d, p, c, Ks, Vs, zkh, zkl, zvh, zvl, st)) != cudaSuccess) return e;
  }
  tc::attn::Maps m;
  memset(&m, 0, sizeof(m));
  const uint64_t Th = T > 0 ? T : 1;  // maps need a non-empty extent; no history tile is read when T = 0
  bool ok = tc::map2d(&m.q, Q, (uint64_t)n_q, C, 128) && tc::map2d(&m.ks, T ? Ks : Q, Th, C, 128) &&
            tc::map2d(&m.vs, T ? Vs : Q, Th, C, 128) && tc::map2d(&m.bk, p->k_block, H * 128, 128, 128) &&
            tc::map2d(&m.bv, p->v_block, H * 128, 256, 128);
  if (ok && n_self > 0)
    ok = tc::map2d(&m.kself, K_self, (uint64_t)n_self, C, 128) && tc::map2d(&m.vself, V_self, (uint64_t)n_self, C, 128);
  if (ok && r > 0 && T > 0)
    ok = tc::map2d(&m.uk, p->k_u, C, r, 128) && tc::map2d(&m.uv, p->v_u, C, r, 128) &&
         tc::map2d(&m.zkh, zkh, T, r, 128) && tc::map2d(&m.zkl, zkl, T, r, 128) &&
         tc::map2d(&m.zvh, zvh, T, r, 128) && tc::map2d(&m.zvl, zvl, T, r, 128);
  const uint64_t rb = 128 * (uint64_t)d->bits / 8;
  if (ok && T > 0)
    ok = tc::map2d_bytes(&m.ck, c->k_codes, T, H * rb, (uint32_t)rb, 128) &&
         tc::map2d_bytes(&m.cv, c->v_codes, T, H * rb, (uint32_t)rb, 128) &&
         (d->group != 32 || (tc::map2d_bytes(&m.pk, c->k_params, T, H * 16, 16, 128) &&
                             tc::map2d_bytes(&m.pv, c->v_params, T, H * 16, 16, 128)));
  if (!ok) return cudaErrorInvalidValue;
  unsigned* err = tc_error_word();
  if (!err) return cudaErrorInvalidDevice;
  tc::attn::Args a{err, n_q, (int64_t)T, n_self, (int)H, d->bits, d->group, scale * 1.4426950408889634f,
                   (const uint8_t*)c->k_codes, (const __half2*)c->k_params, (const uint8_t*)c->v_codes,
                   (const __half2*)c->v_params, (__nv_bfloat16*)O};
  if (r == 0) return tc::attn::launch<0>(m, a, st);
  if (r == 64) return tc::attn::launch<1>(m, a, st);
  return tc::attn::launch<2>(m, a, st);
}

}  // namespace kvc
