// Mixed-dimensional attention over the clustered codec (tcgen05 + TMEM + TMA).
//
// ("NanoKV: High-Ratio KV Cache Compression for Autoregressive Video
// Generation", abstract and the Fast variant: the score of a key is computed
// from its cluster centre and its stored coefficients, without reconstructing
// the full-dimension key.)  With a(t) the key's cluster, coef^ its dequantized
// coefficients and W_dec,h the head's rows of the decoder:
//
//   s(q, t) = scale * (q_h . c_{a(t),h} + (q_h W_dec,h) . coef^_t)
//           = scale * [q_h | q_h W_dec,h] . [c_{a(t),h} | coef^_t]
//   o_h     = sum_t p_t c^V_{a_v(t),h} + W^V_dec,h (sum_t p_t coef^V_t)
//
// so per (128-query tile, head) the kernel is a flash attention with 256-wide
// rows on both sides: A = [q_h | q_h W_dec,h] (its second half computed on the
// tensor cores at the start; the score MMAs read A from tensor memory, so only
// the key tile comes from shared memory), 64-key tiles [centre rows | coefficients] for the
// keys and for the values, double-buffered so that a tile's gather and load
// overlap the MMAs of the one before; the value product accumulates
// [O_c | cbar] (256 TMEM columns) and the end adds cbar W^V_dec,h^T.  The sum
// over p_t c_{a(t)} equals the oracle's sum over clusters of the per-cluster
// mass times the centre (the same terms, grouped differently).
//
// The coefficients of all tokens are dequantized once per call into the
// workspace as bf16 [T][128] (the compressed-domain representation, 1/16 of
// the history's size), because every head and every query tile reads them.
//
// Warp roles: 0 TMA producer, 1 MMA issuer (TMEM owner), 2-5 prep (centre rows
// gathered into the key / value tiles; q W_dec and cbar converted to bf16),
// 6-9 softmax (P written over S in TMEM, lazy rescaling, final output).
#include <cuda.h>
#include <string.h>

#include "tc.h"
#include "tc_ptx.cuh"

namespace kvc {
namespace tc {

bool map2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);

namespace mixed {

// 16 consecutive 32-bit TMEM columns of this thread's lane (no wait)
__device__ __forceinline__ void tmem_st16w(uint32_t taddr, const uint32_t (&w)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]), "r"(w[8]), "r"(w[9]),
      "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15])
      : "memory");
}

constexpr int kThreads = 320;
constexpr int kKeys = 64;  // keys per tile
// shared memory (offsets from a 1024-aligned base)
constexpr int kA = 0;              // [q_h | q_h W_dec,h], four [128][64] bf16 sub-tiles
constexpr int kKt = kA + 65536;    // key tiles [2], each [centre rows | coef] as four [64][64] sub-tiles;
                                   // at the start W_dec,h, at the end cbar (both [128][64] x 2)
constexpr int kVt = kKt + 65536;   // value tiles [2] (MN-major B: four 64-wide N sub-tiles of 64 keys);
                                   // at the end W^V_dec,h
constexpr int kTile = 32768;
constexpr int kSub = 8192;         // [64 rows][64] sub-tile of a key / value tile
constexpr int kBar = kVt + 65536;
constexpr int kSmem = kBar + 1024 + 1024;

struct Maps {
  CUtensorMap q;           // [n_q][C]
  CUtensorMap deck, decv;  // [C][128]
  CUtensorMap ckh, cvh;    // dequantized coefficients [T][128]
};

struct Args {
  unsigned* err;
  int64_t n_q, T;
  int H, n_c;
  float scale_log2;  // softmax scale * log2(e)
  const __nv_bfloat16* cent_k;  // [n_c][C]
  const __nv_bfloat16* cent_v;
  const uint8_t* assign_k;  // [T]
  const uint8_t* assign_v;
  __nv_bfloat16* O;  // [n_q][H][128]
  // key splits: with ks > 1 this launch's keys are one split of the history
  // and the kernel writes its unnormalised output, running max and sum to
  // opart [n_q][H][128] and ml [n_q][H][2] (this split's part of the workspace)
  int ks;
  float* opart;
  float* ml;
};

__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t saddr, uint32_t lbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
__host__ __device__ constexpr uint32_t idesc_bf16_bmn(int M, int N) { return idesc_bf16(M, N) | (1u << 16); }

__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, float (&v)[32]) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// keeps the compiler from touching v before this point
__device__ __forceinline__ void tie32(float (&v)[32]) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
                 "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]),
                 "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}
__device__ __forceinline__ void tmem_ld_wait2(float (&a)[32], float (&b)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  tie32(a);
  tie32(b);
}
__device__ __forceinline__ void tmem_ld_wait4(float (&a)[32], float (&b)[32], float (&c)[32], float (&d)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  tie32(a);
  tie32(b);
  tie32(c);
  tie32(d);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&w)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]), "r"(w[8]), "r"(w[9]),
      "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15])
      : "memory");
}
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
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------- coefficient dequantization

// coef^ = s q + z of every token (128 coefficients, groups of G), as bf16 rows.
template <int BITS, int G>
__global__ void coef_dequant_kernel(const uint8_t* codes, const __half2* params, int64_t T, __nv_bfloat16* out) {
  constexpr int RB = 128 * BITS / 8;
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  uint32_t cw[RB / 4];
#pragma unroll
  for (int i = 0; i < RB / 16; ++i) {
    const uint4 w = __ldcs(reinterpret_cast<const uint4*>(codes + t * RB) + i);
    cw[4 * i] = w.x;
    cw[4 * i + 1] = w.y;
    cw[4 * i + 2] = w.z;
    cw[4 * i + 3] = w.w;
  }
  const float zero[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  uint4* dst = reinterpret_cast<uint4*>(out + t * 128);
#pragma unroll
  for (int e = 0; e < 128; e += 8) {
    const float2 f = __half22float2(params[t * (128 / G) + e / G]);
    float r[8];
    dequant8<BITS>(cw[BITS == 2 ? e / 16 : e / 8], e, f.x, f.y, zero, r);
    dst[e / 8] = make_uint4(pack_bf16x2(r[0], r[1]), pack_bf16x2(r[2], r[3]), pack_bf16x2(r[4], r[5]),
                            pack_bf16x2(r[6], r[7]));
  }
}

// ---------------------------------------------------------------- the attention kernel

// blockIdx.z picks the key split (maps0 / a0 or maps1 / a1: the split's keys,
// assignments and coefficients, offsets applied by the host)
__global__ void __launch_bounds__(kThreads, 1)
    mixed_kernel(const __grid_constant__ Maps maps0, const Args a0, const __grid_constant__ Maps maps1, const Args a1) {
  const Maps& maps = blockIdx.z ? maps1 : maps0;
  const Args a = blockIdx.z ? a1 : a0;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBar);
  uint64_t* setup_full = bars;         // q_h and W_dec,h landed
  uint64_t* qw_acc = setup_full + 1;   // q_h W_dec,h in TMEM
  uint64_t* qw_ready = qw_acc + 1;     // ... and [q | q W_dec] as bf16 pairs in TMEM (prep)
  uint64_t* kfull = qw_ready + 1;      // [2] key tile complete (producer tx + 64 prep arrivals)
  uint64_t* vfull = kfull + 2;         // [2] value tile complete
  uint64_t* kfree = vfull + 2;         // [2] S(j) done: the key tile may be refilled
  uint64_t* vfree = kfree + 2;         // [2] PV(j) done: the value tile may be refilled
  uint64_t* s_full = vfree + 2;        // [2]
  uint64_t* p_full = s_full + 2;       // [2]
  uint64_t* pv_done = p_full + 2;
  uint64_t* acc_done = pv_done + 1;    // the last PV finished: O_c and cbar final
  uint64_t* cbar_ready = acc_done + 1; // cbar as bf16 in the key-tile area (prep)
  uint64_t* dv_full = cbar_ready + 1;  // W^V_dec,h landed in the value-tile area
  uint64_t* o_done = dv_full + 1;
  uint64_t* mma_done = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int q0 = blockIdx.x * 128;
  const int C = a.H * 128;
  const int NT = (int)((a.T + kKeys - 1) / kKeys);

  if (threadIdx.x == 0) {
    mbar_init(setup_full, 1);
    mbar_init(qw_acc, 1);
    mbar_init(qw_ready, 128);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kfull[i], kKeys + 1);
      mbar_init(&vfull[i], kKeys + 1);
      mbar_init(&kfree[i], 1);
      mbar_init(&vfree[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
    }
    mbar_init(pv_done, 1);
    mbar_init(acc_done, 1);
    mbar_init(cbar_ready, 128);
    mbar_init(dv_full, 1);
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
  auto SC = [&](int b) { return tmem + 64 * b; };  // S / P slots, 64 columns each
  const uint32_t OC = tmem + 128;                  // [O_c | cbar], 256 columns
  const uint32_t QW = tmem + 384;                  // q W_dec (setup)
  uint8_t* At = smem + kA;
  uint8_t* Kt = smem + kKt;
  uint8_t* Vt = smem + kVt;
  auto KT = [&](int b) { return Kt + b * kTile; };
  auto VT = [&](int b) { return Vt + b * kTile; };

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      bool ok = true;
      mbar_arrive_expect_tx(setup_full, 65536u);
      tma_load(At, &maps.q, h * 128, q0, setup_full, pol_stream);
      tma_load(At + 16384, &maps.q, h * 128 + 64, q0, setup_full, pol_stream);
      tma_load(Kt, &maps.deck, 0, h * 128, setup_full, pol_keep);  // [K = d][N = i], MN-major B
      tma_load(Kt + 16384, &maps.deck, 64, h * 128, setup_full, pol_keep);
      int k_last = -1, v_last = -1;  // last tile loaded (the loads of it and of the tile before are drained after an abort)
      bool dv_armed = false;
      for (int j = 0; j < NT && ok; ++j) {
        const int b = j & 1;
        // coefficients of the key tile, once S(j-2) is done with the buffer (tile 0: once the
        // q W_dec product is done with W_dec,h, which it overlaps)
        if (j == 0) {
          if (!wait(qw_acc, 0, abort_flag, a.err, 0x2100u)) ok = false;
        } else if (j >= 2 && !wait(&kfree[b], ((j - 2) >> 1) & 1, abort_flag, a.err, 0x2101u)) {
          ok = false;
        }
        if (!ok) break;
        mbar_arrive_expect_tx(&kfull[b], 16384u);
        tma_load(KT(b) + 2 * kSub, &maps.ckh, 0, j * kKeys, &kfull[b], pol_keep);
        tma_load(KT(b) + 3 * kSub, &maps.ckh, 64, j * kKeys, &kfull[b], pol_keep);
        k_last = j;
        if (j >= 2 && !wait(&vfree[b], ((j - 2) >> 1) & 1, abort_flag, a.err, 0x2102u)) ok = false;
        if (!ok) break;
        mbar_arrive_expect_tx(&vfull[b], 16384u);
        tma_load(VT(b) + 2 * kSub, &maps.cvh, 0, j * kKeys, &vfull[b], pol_keep);
        tma_load(VT(b) + 3 * kSub, &maps.cvh, 64, j * kKeys, &vfull[b], pol_keep);
        v_last = j;
      }
      // W^V_dec,h for the final product, once every MMA is done with the value tiles
      if (ok && wait(acc_done, 0, abort_flag, a.err, 0x2103u)) {
        mbar_arrive_expect_tx(dv_full, 32768u);
        tma_load(Vt, &maps.decv, 0, h * 128, dv_full, pol_keep);  // [N = d][K = i], K-major B
        tma_load(Vt + 16384, &maps.decv, 64, h * 128, dv_full, pol_keep);
        dv_armed = true;
      }
      if (*abort_flag) {
        // the loads this thread issued land before the CTA can leave (the prep
        // arrivals of an aborted tile may be missing, so only the bytes are awaited)
        auto drain = [&](uint64_t* bar, uint32_t parity) {
          const long long w0 = clock64();
          while (!mbar_test(bar, parity) && clock64() - w0 < kWaitBudget) {
          }
        };
        drain(setup_full, 0);
        for (int j = k_last - 1; j <= k_last; ++j)
          if (j >= 0) drain(&kfull[j & 1], (j >> 1) & 1);
        for (int j = v_last - 1; j <= v_last; ++j)
          if (j >= 0) drain(&vfull[j & 1], (j >> 1) & 1);
        if (dv_armed) drain(dv_full, 0);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint32_t id128 = idesc_bf16(128, 128);
      const uint64_t ad = desc_sw128(smem_u32(At));
      // q W_dec,h: A = q_h (K = d), B = W_dec,h (MN-major)
      wait(setup_full, 0, abort_flag, a.err, 0x2200u);
      tc_fence_after();
      {
        const uint64_t bd = desc_mn_sw128(smem_u32(Kt), 16384);
        const uint32_t idm = idesc_bf16_bmn(128, 128);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (k >> 2) * (16384 >> 4) + (k & 3) * 2;
          umma(QW, ad + off, bd + (uint64_t)k * (2048 >> 4), idm, k == 0 ? 0u : 1u);
        }
        umma_commit(qw_acc);
      }
      wait(qw_ready, 0, abort_flag, a.err, 0x2201u);
      tc_fence_after();
      const uint32_t id64 = idesc_bf16(128, kKeys);
      const uint32_t idv = idesc_bf16_bmn(128, 256);
      for (int j = 0; j <= NT; ++j) {
        if (j < NT) {
          const int b = j & 1;
          // S(j) = [q | q W_dec] [centres | coef]^T, K = 256, N = 64 keys; A from
          // tensor memory (bf16 pairs, 8 columns a K step), so the MMAs read only
          // the key tile from shared memory
          wait(&kfull[b], (j >> 1) & 1, abort_flag, a.err, 0x2210u + b);
          tc_fence_after();
          const uint64_t kd = desc_sw128(smem_u32(KT(b)));
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const uint32_t boff = (k >> 2) * (kSub >> 4) + (k & 3) * 2;
            umma_ts(SC(b), QW + k * 8, kd + boff, id64, k == 0 ? 0u : 1u);
          }
          umma_commit(&s_full[b]);
          umma_commit(&kfree[b]);
        }
        if (j >= 1) {
          const int t = j - 1, b = t & 1;
          // [O_c | cbar] += P(t) [centres | coef], K = 64 keys, N = 256, P from TMEM
          wait(&p_full[b], (t >> 1) & 1, abort_flag, a.err, 0x2220u + b);
          wait(&vfull[b], (t >> 1) & 1, abort_flag, a.err, 0x2230u + b);
          tc_fence_after();
          const uint64_t vd = desc_mn_sw128(smem_u32(VT(b)), kSub);
#pragma unroll
          for (int k = 0; k < kKeys / 16; ++k)
            umma_ts(OC, SC(b) + k * 8, vd + (uint64_t)k * (2048 >> 4), idv, (t == 0 && k == 0) ? 0u : 1u);
          umma_commit(pv_done);
          umma_commit(&vfree[b]);
        }
      }
      umma_commit(acc_done);
      // O_c += cbar W^V_dec,h^T
      wait(cbar_ready, 0, abort_flag, a.err, 0x2240u);
      wait(dv_full, 0, abort_flag, a.err, 0x2241u);
      tc_fence_after();
      {
        const uint64_t cd = desc_sw128(smem_u32(Kt));
        const uint64_t dd = desc_sw128(smem_u32(Vt));
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (k >> 2) * (16384 >> 4) + (k & 3) * 2;
          umma(OC, cd + off, dd + off, id128, 1u);
        }
      }
      umma_commit(o_done);
      umma_commit(mma_done);
      const long long w0 = clock64();
      while (!mbar_test(mma_done, 0) && clock64() - w0 < kWaitBudget) {
      }
    }
  } else if (warp < 6) {
    // ================================================================ prep (warps 2-5)
    const int qd = warp & 3;
    const int row = qd * 32 + lane;  // key row of a tile, or query row (TMEM lane) for conversions
    const uint32_t lane_addr = tmem + ((uint32_t)(qd * 32) << 16);
    // 128 fp32 TMEM columns of this lane -> bf16 row of a K-major pair of sub-tiles
    auto to_bf16 = [&](uint32_t col, uint8_t* tile) {
      float v[4][32];
      tmem_ld32_async(lane_addr + (col - tmem), v[0]);
      tmem_ld32_async(lane_addr + (col - tmem) + 32, v[1]);
      tmem_ld32_async(lane_addr + (col - tmem) + 64, v[2]);
      tmem_ld32_async(lane_addr + (col - tmem) + 96, v[3]);
      tmem_ld_wait4(v[0], v[1], v[2], v[3]);
#pragma unroll
      for (int c16 = 0; c16 < 16; ++c16) {
        const float* x = &v[c16 / 4][(c16 % 4) * 8];
        *reinterpret_cast<uint4*>(tile + (c16 / 8) * 16384 + sw128_off(row, c16 % 8)) =
            make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                       pack_bf16x2(x[6], x[7]));
      }
      tc_fence_before();
      fence_async_smem();
    };
    // The head's 128 channels (256 bytes) of the centre of each key: the warps
    // of lane quarters 0, 1 gather the 64 rows of a key tile, those of quarters
    // 2, 3 the rows of a value tile, 32 rows per warp.  A half warp reads one
    // row (16 bytes a lane), two rows per instruction, so a load touches two
    // rows' lines rather than 32.  Rows are fetched ahead of the wait for their
    // buffer, then stored into sub-tiles 0, 1 of it.
    const bool is_v = qd >= 2;
    const int r0 = (qd & 1) * 32;  // this warp's first row of a tile
    const int ch = lane & 15;      // 16-byte chunk of a row
    const __nv_bfloat16* cent = is_v ? a.cent_v : a.cent_k;
    const uint8_t* assign = is_v ? a.assign_v : a.assign_k;
    uint64_t* tfull = is_v ? vfull : kfull;
    uint64_t* tfree = is_v ? vfree : kfree;
    auto fetch_row = [&](int j, uint4 (&w)[16]) {
      const int64_t t = (int64_t)j * kKeys + r0 + lane;  // a lane holds the centre of one row
      int c = t < a.T ? (int)assign[t] : 0;
      c = c < a.n_c ? c : a.n_c - 1;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int cr = __shfl_sync(0xffffffffu, c, 2 * i + (lane >> 4));
        w[i] = __ldg(reinterpret_cast<const uint4*>(cent + (int64_t)cr * C + h * 128) + ch);
      }
    };
    wait(setup_full, 0, abort_flag, a.err, 0x2305u);  // q in At (read below through the generic proxy)
    wait(qw_acc, 0, abort_flag, a.err, 0x2300u);      // also: W_dec,h in key buffer 0 is no longer read
    tc_fence_after();
    // A of the score MMAs into tensor memory, over the q W_dec accumulator (this
    // thread's lane): columns [0, 64) q and [64, 128) q W_dec as bf16 pairs.  Block
    // k of 32 fp32 columns of q W_dec becomes 16 columns of pairs at 64 + 16 k,
    // highest block first, so that no block is overwritten before it is read.
    {
#pragma unroll 1
      for (int k = 3; k >= 0; --k) {
        float v[32];
        tmem_ld32(lane_addr + (QW - tmem) + 32 * k, v);
        uint32_t p16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) p16[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
        tmem_st16w(lane_addr + (QW - tmem) + 64 + 16 * k, p16);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      }
#pragma unroll 1
      for (int k = 0; k < 4; ++k) {  // q elements 32 k .. 32 k + 31: chunks 4 k .. 4 k + 3 of the row
        uint32_t p16[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int cc = 4 * k + c;  // 16-byte chunk of the 256-byte row (sub-tile cc / 8)
          const uint4 u = *reinterpret_cast<const uint4*>(At + (cc >> 3) * 16384 + sw128_off(row, cc & 7));
          p16[4 * c] = u.x;
          p16[4 * c + 1] = u.y;
          p16[4 * c + 2] = u.z;
          p16[4 * c + 3] = u.w;
        }
        tmem_st16w(lane_addr + (QW - tmem) + 16 * k, p16);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
    }
    mbar_arrive(qw_ready);
    uint4 w[16];
    fetch_row(0, w);
    for (int j = 0; j < NT; ++j) {
      const int b = j & 1;
      if (j >= 2) wait(&tfree[b], ((j - 2) >> 1) & 1, abort_flag, a.err, 0x2301u + (is_v ? 2 : 0) + b);
      uint8_t* tile = is_v ? VT(b) : KT(b);
#pragma unroll
      for (int i = 0; i < 16; ++i)
        *reinterpret_cast<uint4*>(tile + (ch / 8) * kSub + sw128_off(r0 + 2 * i + (lane >> 4), ch % 8)) = w[i];
      fence_async_smem();
      mbar_arrive(&tfull[b]);
      if (j + 1 < NT) fetch_row(j + 1, w);
    }
    // cbar (TMEM) -> bf16 A operand in the key-tile area, once every S and PV is done
    wait(acc_done, 0, abort_flag, a.err, 0x2303u);
    tc_fence_after();
    to_bf16(OC + 128, Kt);
    mbar_arrive(cbar_ready);
  } else {
    // ================================================================ softmax (warps 6-9)
    const int qd = warp & 3;
    const int row = qd * 32 + lane;  // query row
    const uint32_t lane_addr = tmem + ((uint32_t)(qd * 32) << 16);
    const float c = a.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    for (int j = 0; j < NT; ++j) {
      const int b = j & 1;
      const uint32_t sc = lane_addr + (SC(b) - tmem);
      wait(&s_full[b], (j >> 1) & 1, abort_flag, a.err, 0x2400u + b);
      tc_fence_after();
      const int64_t kbase = (int64_t)j * kKeys;
      const int nvalid = a.T - kbase < kKeys ? (int)(a.T - kbase) : kKeys;
      float sv[2][32];
      tmem_ld32_async(sc, sv[0]);
      tmem_ld32_async(sc + 32, sv[1]);
      tmem_ld_wait2(sv[0], sv[1]);
      if (nvalid < kKeys) {
#pragma unroll
        for (int pc = 0; pc < 2; ++pc)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (pc * 32 + i >= nvalid) sv[pc][i] = -INFINITY;
      }
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int pc = 0; pc < 2; ++pc)
#pragma unroll
        for (int i = 0; i < 32; ++i) mx[i & 3] = fmaxf(mx[i & 3], sv[pc][i]);
      const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * c;
      // lazy rescale: only when the tile's max exceeds the one in use by 2^8
      const bool need = mt > m_used + 8.f;
      float alpha = 1.f;
      if (need) {
        alpha = m_used == -INFINITY ? 0.f : ex2_approx(m_used - mt);
        l *= alpha;
        m_used = mt;
      }
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int pc = 0; pc < 2; ++pc) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = ex2_approx(fmaf(sv[pc][2 * i], c, -m_used));
          const float p1 = ex2_approx(fmaf(sv[pc][2 * i + 1], c, -m_used));
          ls[i & 3] += p0 + p1;
          w[i] = pack_bf16x2(p0, p1);
        }
        tmem_st16(sc + pc * 16, w);
      }
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      // O (both halves) is rescaled before P(j) is handed over
      if (__any_sync(0xffffffffu, need && j > 0)) {
        wait(pv_done, (j - 1) & 1, abort_flag, a.err, 0x2401u);
        tc_fence_after();
#pragma unroll
        for (int pc = 0; pc < 8; ++pc) {
          float ov[32];
          tmem_ld32(lane_addr + (OC - tmem) + pc * 32, ov);
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] *= alpha;
          tmem_st32(lane_addr + (OC - tmem) + pc * 32, ov);
        }
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      mbar_arrive(&p_full[b]);
    }
    wait(o_done, 0, abort_flag, a.err, 0x2402u);
    tc_fence_after();
    const int64_t qrow = (int64_t)q0 + row;
    // one split: O / l as bf16; several: this split's O (relative to 2^m_used)
    // and (m_used, l), merged by the combine kernel
    const bool part = a.ks > 1;
    if (part && qrow < a.n_q) *reinterpret_cast<float2*>(a.ml + (qrow * a.H + h) * 2) = make_float2(m_used, l);
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
    for (int pc = 0; pc < 4; ++pc) {
      float ov[32];
      tmem_ld32(lane_addr + (OC - tmem) + pc * 32, ov);
      if (qrow >= a.n_q) continue;
      if (part) {
        float4* dst = reinterpret_cast<float4*>(a.opart + (qrow * a.H + h) * 128 + pc * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[i] = make_float4(ov[4 * i], ov[4 * i + 1], ov[4 * i + 2], ov[4 * i + 3]);
      } else {
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

// Merge of the key splits of every (query, head) row: with m the largest of the
// splits' running maxima, O = sum_s 2^(m_s - m) O_s / sum_s 2^(m_s - m) l_s.
// One warp per row, four channels a lane.
__global__ void combine_kernel(const float* opart, const float* ml, int ks, int64_t rows, __nv_bfloat16* O) {
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (r >= rows) return;
  const int lane = threadIdx.x & 31;
  float m = -INFINITY;
  for (int s = 0; s < ks; ++s) m = fmaxf(m, ml[(s * rows + r) * 2]);
  float l = 0.f;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < ks; ++s) {
    const float2 sl = *reinterpret_cast<const float2*>(ml + (s * rows + r) * 2);
    const float w = sl.x == -INFINITY ? 0.f : exp2f(sl.x - m);
    l += w * sl.y;
    const float4 v = reinterpret_cast<const float4*>(opart + (s * rows + r) * 128)[lane];
    o.x += w * v.x;
    o.y += w * v.y;
    o.z += w * v.z;
    o.w += w * v.w;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  reinterpret_cast<uint2*>(O + r * 128)[lane] = make_uint2(pack_bf16x2(o.x * inv, o.y * inv), pack_bf16x2(o.z * inv, o.w * inv));
}

}  // namespace mixed
}  // namespace tc

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
namespace {
constexpr int kMaxSplits = 2;
size_t mixed_parts_bytes(const kvc_layer_desc* d, int64_t n_q) {
  const size_t rows = (size_t)(n_q > 0 ? n_q : 0) * d->n_heads;
  return align256(kMaxSplits * rows * 128 * sizeof(float)) + align256(kMaxSplits * rows * 2 * sizeof(float));
}
int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return n;
}
}  // namespace


bool tc_mixed_supported(const kvc_layer_desc* d, const kvc_predictor* p) {
  if (p->kind != KVC_PRED_CLUSTER) return false;
  if (d->dtype != KVC_BF16 || d->head_dim != 128 || d->param_dtype != KVC_F16) return false;
  if (d->bits != 2 && d->bits != 4) return false;
  if (d->group != 32 && d->group != 64) return false;
  if (p->code_dim != 128 || p->n_clusters < 1 || p->n_clusters > 256) return false;
  if (d->n_tokens < 1 || (int64_t)d->n_heads * 128 * 2 > (1 << 20)) return false;
  return true;
}

// dequantized coefficients of K and V, then room for the key splits' partial results
size_t tc_mixed_workspace(const kvc_layer_desc* d, int64_t n_q) {
  return 2 * align256((size_t)d->n_tokens * 128 * 2) + mixed_parts_bytes(d, n_q);
}

cudaError_t tc_mixed_attend(const kvc_layer_desc* d, const kvc_predictor* p, const void* Q, int64_t n_q,
                            const kvc_codes* c, float scale, void* O, void* ws, size_t ws_bytes, cudaStream_t st) {
  const uint64_t T = (uint64_t)d->n_tokens, H = d->n_heads, C = H * 128;
  const size_t coef_bytes = 2 * align256((size_t)T * 128 * 2);
  if (ws_bytes < coef_bytes) return cudaErrorInvalidValue;
  __nv_bfloat16* ckh = static_cast<__nv_bfloat16*>(ws);
  __nv_bfloat16* cvh = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(ws) + align256(T * 128 * 2));
  // dequantized coefficients of every token
  {
    const unsigned blocks = (unsigned)((T + 127) / 128);
    auto k = d->bits == 2 ? (d->group == 32 ? tc::mixed::coef_dequant_kernel<2, 32> : tc::mixed::coef_dequant_kernel<2, 64>)
                          : (d->group == 32 ? tc::mixed::coef_dequant_kernel<4, 32> : tc::mixed::coef_dequant_kernel<4, 64>);
    k<<<blocks, 128, 0, st>>>((const uint8_t*)c->k_codes, (const __half2*)c->k_params, (int64_t)T, ckh);
    k<<<blocks, 128, 0, st>>>((const uint8_t*)c->v_codes, (const __half2*)c->v_params, (int64_t)T, cvh);
    count_launches(2);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  tc::mixed::Maps m;
  memset(&m, 0, sizeof(m));
  bool ok = tc::map2d(&m.q, Q, (uint64_t)n_q, C, 128) && tc::map2d(&m.deck, p->k_dec, C, 128, 128) &&
            tc::map2d(&m.decv, p->v_dec, C, 128, 128) && tc::map2d(&m.ckh, ckh, T, 128, tc::mixed::kKeys) &&
            tc::map2d(&m.cvh, cvh, T, 128, tc::mixed::kKeys);
  if (!ok) return cudaErrorInvalidValue;
  unsigned* err = tc_error_word();
  if (!err) return cudaErrorInvalidDevice;
  // Two key splits when they shorten the run: (query tile, head) CTAs in waves
  // of one per SM, each split half as long; the splits' partials are merged after.
  const int64_t tiles = (n_q + 127) / 128 * (int64_t)H;
  const int64_t nkt = ((int64_t)T + tc::mixed::kKeys - 1) / tc::mixed::kKeys;
  const int sms = device_sms();
  int ks = 1;
  if (sms > 0 && nkt >= 2 && ws_bytes >= coef_bytes + mixed_parts_bytes(d, n_q)) {
    const int64_t w1 = (tiles + sms - 1) / sms, w2 = (2 * tiles + sms - 1) / sms;
    if (w2 < 2 * w1) ks = 2;  // 2 splits of half the work: w2 / 2 < w1
  }
  float* opart = reinterpret_cast<float*>(static_cast<char*>(ws) + coef_bytes);
  float* ml = reinterpret_cast<float*>(static_cast<char*>(ws) + coef_bytes +
                                       align256(kMaxSplits * (size_t)n_q * H * 128 * sizeof(float)));
  const int64_t rows = n_q * (int64_t)H;
  tc::mixed::Args a0{err, n_q, (int64_t)T, (int)H, p->n_clusters, scale * 1.4426950408889634f,
                     (const __nv_bfloat16*)p->k_centroids, (const __nv_bfloat16*)p->v_centroids,
                     (const uint8_t*)c->k_assign, (const uint8_t*)c->v_assign, (__nv_bfloat16*)O, ks, opart, ml};
  tc::mixed::Maps m1 = m;
  tc::mixed::Args a1 = a0;
  if (ks > 1) {  // split 0: the first ceil(tiles / 2) key tiles; split 1: the rest
    const uint64_t T0 = (uint64_t)((nkt + 1) / 2) * tc::mixed::kKeys, T1 = T - T0;
    a0.T = (int64_t)T0;
    a1.T = (int64_t)T1;
    a1.assign_k += T0;
    a1.assign_v += T0;
    a1.opart = opart + rows * 128;
    a1.ml = ml + rows * 2;
    if (!(tc::map2d(&m1.ckh, ckh + T0 * 128, T1, 128, tc::mixed::kKeys) &&
          tc::map2d(&m1.cvh, cvh + T0 * 128, T1, 128, tc::mixed::kKeys)))
      return cudaErrorInvalidValue;
  }
  auto k = tc::mixed::mixed_kernel;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::mixed::kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((n_q + 127) / 128), (unsigned)H, (unsigned)ks);
  k<<<grid, tc::mixed::kThreads, tc::mixed::kSmem, st>>>(m, a0, m1, a1);
  count_launches(1);
  if (ks > 1) {
    tc::mixed::combine_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(opart, ml, ks, rows, (__nv_bfloat16*)O);
    count_launches(1);
  }
  return cudaGetLastError();
}

}  // namespace kvc
