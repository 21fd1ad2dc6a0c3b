// Attention over a decoded history and the chunk's own keys (tcgen05 + TMEM + TMA).
//
//   O = softmax(scale Q [K^_hist ; K_self]^T - J) [V^_hist ; V_self]
//
// ("NanoKV: High-Ratio KV Cache Compression for Autoregressive Video
// Generation", abstract: the later frames attend over the whole compressed
// history; "CORAL-KV ...", Fig. 3: the history of layer l is decoded from its
// codes and the reconstruction of layer l-1.)  The caller decodes the history
// once (the codec kernel, all heads of a token tile per CTA) into bf16 K^ / V^;
// this kernel is a flash attention over it, one CTA per (128-query tile, query
// head), CTAs of one head adjacent in launch order so that the head's K^ / V^
// tiles are served from L2 to every query tile.
//
// J is zero, or, for the debiased attention, the Jensen term of each history
// key (the related-papers abstract on the "Jensen bias" of INT2 key caches,
// listed on the CORAL-KV page): 0.5 scale^2 sum_g |q_g|^2 s_g^2 / 12 over the
// key's quantization groups g (s_g its stored scale).  It is a rank-NG product,
// so it runs on the tensor cores as one more K = 16 MMA into S: A holds
// -|q_g|^2 J' per query row, B holds s_g^2 per key.
//
// Warp roles: 0 TMA producer (Q, then K / V tiles through a ring of stages),
// 1 MMA issuer and TMEM owner, 2-5 softmax (one query row per thread: S -> P in
// TMEM, running max / sum, lazy rescaling of O, final normalisation), 6 (the
// debiased variant only) writes the Jensen operands.  TMEM: S / P slots [2], O.
#include <cuda.h>
#include <string.h>

#include <type_traits>

#include "tc.h"
#include "tc_ptx.cuh"

namespace kvc {
namespace tc {

bool map2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);

namespace flash {

template <bool JC>
struct Cfg {
  static constexpr int kWarps = JC ? 7 : 6;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int S = 3;  // K / V tile pairs in flight
  // shared memory (offsets from a 1024-aligned base)
  // Q tile, two [128][64] sub-tiles.  Once Q is in tensor memory, JC keeps the
  // Jensen operands in its first sub-tile, four K = 16 slices of 16 columns:
  // slice 0 the A operand, slice 1 + s the B operand of stage s.
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + 32768;           // K tiles [S]
  static constexpr int kV = kK + S * 32768;       // V tiles [S]
  static constexpr int kBar = kV + S * 32768;
  static_assert(!JC || S <= 3, "the Jensen tile holds the A slice and one B slice per stage");
  static constexpr int kSmem = kBar + 1024 + 1024;  // + barriers + alignment slack
};

struct Maps {
  CUtensorMap q;             // [n_q][Hq*128]
  CUtensorMap kh, vh;        // decoded history [T][H*128]
  CUtensorMap kself, vself;  // [n_self][H*128]
};

struct Args {
  unsigned* err;
  int64_t n_q, T, n_self;
  int H, Hq, group;
  float scale_log2;          // softmax scale * log2(e)
  const __half2* kparams;    // JC: the history's K (scale, zero) pairs, [T][H][128 / group]
  float jensen_a;            // JC: -0.5 scale / 12 (times |q_g|^2: the A operand, in units of S)
  __nv_bfloat16* O;          // [n_q][Hq][128]
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
// D[tmem] (+)= A[tmem] * B[smem]: A (bf16 pairs per 32-bit column) from tensor memory
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// 32 columns of this thread's TMEM lane, without waiting: the values are valid
// only after tmem_ld_wait on the same arrays
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
__device__ __forceinline__ void tmem_ld_wait(float (&a)[32], float (&b)[32], float (&c)[32], float (&d)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  tie32(a);
  tie32(b);
  tie32(c);
  tie32(d);
}
// 2^x by the hardware approximation (flush-to-zero; softmax weights only)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 2^x on the FMA pipe, for the share of the softmax weights that would
// otherwise queue on the (16 per cycle per SM) exponential unit: x = n + f with
// n = rint(x) (the 1.5 * 2^23 addition leaves n in the low mantissa bits) and
// f in [-0.5, 0.5]; 2^f by a cubic fitted here to the relative error of 2^f on
// that interval (Lawson-weighted least squares on Chebyshev nodes, max relative
// error 7.5e-5, below the 2^-9 of the bf16 the weights are rounded to); 2^n
// added to the exponent field.  x is clamped at -126 (weights below 2^-126 are
// kept at about 2^-126: nothing at that scale survives the fp32 sums).
__device__ __forceinline__ float ex2_cubic(float x) {
  x = fmaxf(x, -126.f);
  const float t = x + 12582912.f;
  const float f = x - (t - 12582912.f);
  const float p = fmaf(fmaf(fmaf(0.0551716648f, f, 0.2426111251f), f, 0.6932609677f), f, 0.9999280572f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&w)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]), "r"(w[8]), "r"(w[9]),
      "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15])
      : "memory");
}

// ---------------------------------------------------------------- the kernel
//
// Key tiles j = 0 .. NH-1 are the history, NH .. NT-1 the chunk's own keys;
// tile j uses stage j mod S.  Per tile: S(j) = Q K(j)^T into TMEM slot j mod 2
// (plus the Jensen MMA for a history tile), the softmax writes P(j) over it as
// bf16 pairs, and O += P(j) V(j) takes P from tensor memory.  The MMA warp
// issues S(j + 1) before it waits for P(j), so the softmax of one tile runs
// under the MMAs of the next.

template <bool JC, int NG>
__global__ void __launch_bounds__(Cfg<JC>::kThreads, 1)
    attend_kernel(const __grid_constant__ Maps maps, const Args a) {
  using L = Cfg<JC>;
  constexpr int S = L::S;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* k_full = bars;           // [S] K tile landed
  uint64_t* v_full = k_full + S;     // [S] V tile landed
  uint64_t* kv_empty = v_full + S;   // [S] stage free (PV of its tile done)
  uint64_t* x_full = kv_empty + S;   // [S] JC: the stage's Jensen B operand written
  uint64_t* q_full = x_full + S;
  uint64_t* qx_full = q_full + 1;    // JC: the Jensen A operand written
  uint64_t* q_tmem = qx_full + 1;    // Q copied into tensor memory (the softmax warps)
  uint64_t* s_full = q_tmem + 1;     // [2]
  uint64_t* p_full = s_full + 2;     // [2]
  uint64_t* pv_done = p_full + 2;
  uint64_t* o_done = pv_done + 1;
  uint64_t* mma_done = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hq = blockIdx.y;        // query head
  const int h = hq / (a.Hq / a.H);  // its KV head (grouped-query attention when Hq > H)
  const int q0 = blockIdx.x * 128;
  const int NH = (int)((a.T + 127) / 128);       // history key tiles
  const int NS = (int)((a.n_self + 127) / 128);  // chunk key tiles
  const int NT = NH + NS;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&x_full[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(qx_full, 1);
    mbar_init(q_tmem, 128);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
    }
    mbar_init(pv_done, 1);
    mbar_init(o_done, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
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
  const uint32_t OC = tmem + 256;
  // Q as bf16 pairs: the A operand of S = Q K^T comes from tensor memory, so the
  // S MMAs read only K from shared memory
  const uint32_t QC = tmem + 384;
  auto SC = [&](int b) { return tmem + 128 * b; };
  uint8_t* Qs = smem + L::kQ;
  auto Kt = [&](int s) { return smem + L::kK + s * 32768; };
  auto Vt = [&](int s) { return smem + L::kV + s * 32768; };
  uint8_t* X = smem + L::kQ;  // JC: the Jensen operands, after Q has moved to tensor memory

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      const uint64_t pol_q = policy_evict_first();
      const uint64_t pol_kv = policy_evict_last();  // read by every query tile of the head
      bool ok = true;
      int issued[S];
      uint32_t issued_ph[S];
      for (int i = 0; i < S; ++i) issued[i] = 0, issued_ph[i] = 0;
      mbar_arrive_expect_tx(q_full, 32768u);
      tma_load(Qs, &maps.q, hq * 128, q0, q_full, pol_q);
      tma_load(Qs + 16384, &maps.q, hq * 128 + 64, q0, q_full, pol_q);
      for (int j = 0; j < NT && ok; ++j) {
        const int s = j % S;
        const uint32_t ph = (uint32_t)(j / S) & 1u;
        if (!wait(&kv_empty[s], ph ^ 1u, abort_flag, a.err, 0x1100u + s)) {
          ok = false;
          break;
        }
        const bool hist = j < NH;
        const CUtensorMap* mk = hist ? &maps.kh : &maps.kself;
        const CUtensorMap* mv = hist ? &maps.vh : &maps.vself;
        const int row = hist ? j * 128 : (j - NH) * 128;
        mbar_arrive_expect_tx(&k_full[s], 32768u);
        tma_load(Kt(s), mk, h * 128, row, &k_full[s], pol_kv);
        tma_load(Kt(s) + 16384, mk, h * 128 + 64, row, &k_full[s], pol_kv);
        mbar_arrive_expect_tx(&v_full[s], 32768u);
        tma_load(Vt(s), mv, h * 128, row, &v_full[s], pol_kv);
        tma_load(Vt(s) + 16384, mv, h * 128 + 64, row, &v_full[s], pol_kv);
        issued[s] = 1;
        issued_ph[s] = ph;
      }
      if (*abort_flag) {
        // every load this thread issued lands before the CTA can leave
        auto drain = [&](uint64_t* bar, uint32_t parity) {
          const long long w0 = clock64();
          while (!mbar_test(bar, parity) && clock64() - w0 < kWaitBudget) {
          }
        };
        drain(q_full, 0);
        for (int i = 0; i < S; ++i)
          if (issued[i]) {
            drain(&k_full[i], issued_ph[i]);
            drain(&v_full[i], issued_ph[i]);
          }
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint32_t id128 = idesc_bf16(128, 128);
      const uint32_t idv = idesc_bf16_bmn(128, 128);
      bool ok = wait(q_tmem, 0, abort_flag, a.err, 0x1310u);
      if (JC && ok) ok = wait(qx_full, 0, abort_flag, a.err, 0x1311u);
      for (int j = 0; j <= NT && ok; ++j) {
        if (j < NT) {
          const int s = j % S, b = j & 1;
          const uint32_t ph = (uint32_t)(j / S) & 1u;
          if (!wait(&k_full[s], ph, abort_flag, a.err, 0x1320u + s)) break;
          if (JC && j < NH && !wait(&x_full[s], ph, abort_flag, a.err, 0x1328u + s)) break;
          tc_fence_after();
          // S(j) = Q K(j)^T into slot b, which last held P(j-2), read by PV(j-2) issued before
          const uint64_t kd = desc_sw128(smem_u32(Kt(s)));
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t off = (k >> 2) * (16384 >> 4) + (k & 3) * 2;
            umma_ts(SC(b), QC + k * 8, kd + off, id128, k == 0 ? 0u : 1u);
          }
          if (JC && j < NH) {  // the Jensen term of the history keys: one K = 16 step (slices 0 and 1 + s)
            const uint64_t xd = desc_sw128(smem_u32(X));
            umma(SC(b), xd, xd + 2 * (s + 1), id128, 1u);
          }
          umma_commit(&s_full[b]);
        }
        if (j >= 1) {
          // O += P(t) V(t), P from TMEM
          const int t = j - 1, st = t % S, b = t & 1;
          if (!wait(&p_full[b], (uint32_t)(t >> 1) & 1u, abort_flag, a.err, 0x1330u + b)) break;
          if (!wait(&v_full[st], (uint32_t)(t / S) & 1u, abort_flag, a.err, 0x1340u + st)) break;
          tc_fence_after();
          const uint64_t vd = desc_mn_sw128(smem_u32(Vt(st)), 16384);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            umma_ts(OC, SC(b) + k * 8, vd + (uint64_t)k * (2048 >> 4), idv, (t == 0 && k == 0) ? 0u : 1u);
          umma_commit(pv_done);
          umma_commit(&kv_empty[st]);
        }
      }
      umma_commit(o_done);
      umma_commit(mma_done);
      const long long w0 = clock64();
      while (!mbar_test(mma_done, 0) && clock64() - w0 < kWaitBudget) {
      }
    }
  } else if (warp < 6) {
    // ================================================================ softmax (warps 2-5)
    const int qd = warp & 3;
    const int row = qd * 32 + lane;  // query row
    const uint32_t lane_addr = tmem + ((uint32_t)(qd * 32) << 16);
    const float c = a.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    // this thread's Q row, from the 128-byte-swizzled tile, into tensor memory
    wait(q_full, 0, abort_flag, a.err, 0x1505u);
    {
      uint32_t qw[64];
#pragma unroll
      for (int k = 0; k < 16; ++k) {  // 16-byte chunk k of the row: elements 8k .. 8k + 7
        const uint4 u = *reinterpret_cast<const uint4*>(Qs + (k / 8) * 16384 + sw128_off(row, k % 8));
        qw[4 * k] = u.x;
        qw[4 * k + 1] = u.y;
        qw[4 * k + 2] = u.z;
        qw[4 * k + 3] = u.w;
      }
      uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&qw[0]);
      uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&qw[32]);
      tmem_st32u(lane_addr + (QC - tmem), lo);
      tmem_st32u(lane_addr + (QC - tmem) + 32, hi);
    }
    tc_fence_before();
    mbar_arrive(q_tmem);
    for (int j = 0; j < NT; ++j) {
      const int b = j & 1;
      const uint32_t sc = lane_addr + (SC(b) - tmem);
      const bool hist = j < NH;
      wait(&s_full[b], (uint32_t)(j >> 1) & 1u, abort_flag, a.err, 0x1500u + b);
      tc_fence_after();
      const int64_t kbase = hist ? (int64_t)j * 128 : (int64_t)(j - NH) * 128;
      const int64_t klim = hist ? a.T : a.n_self;
      const int nvalid = klim - kbase < 128 ? (int)(klim - kbase) : 128;
      // the whole S row in registers: four loads, one wait
      float sv[4][32];
      tmem_ld32_async(sc, sv[0]);
      tmem_ld32_async(sc + 32, sv[1]);
      tmem_ld32_async(sc + 64, sv[2]);
      tmem_ld32_async(sc + 96, sv[3]);
      tmem_ld_wait(sv[0], sv[1], sv[2], sv[3]);
      if (nvalid < 128) {
#pragma unroll
        for (int pc = 0; pc < 4; ++pc)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (pc * 32 + i >= nvalid) sv[pc][i] = -INFINITY;
      }
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int pc = 0; pc < 4; ++pc)
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
      // P over S: the 16 packed columns of pass pc land on S columns already read
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          // a quarter of the weights on the FMA pipe balances its issue slots
          // against the exponential unit's throughput
          const float x0 = fmaf(sv[pc][2 * i], c, -m_used), x1 = fmaf(sv[pc][2 * i + 1], c, -m_used);
          const bool fma_pipe = (i & 3) == 3;
          const float p0 = fma_pipe ? ex2_cubic(x0) : ex2_approx(x0);
          const float p1 = fma_pipe ? ex2_cubic(x1) : ex2_approx(x1);
          ls[i & 3] += p0 + p1;
          w[i] = pack_bf16x2(p0, p1);
        }
        tmem_st16(sc + pc * 16, w);
      }
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      // O is rescaled before P(j) is handed over (PV(j) follows p_full)
      if (__any_sync(0xffffffffu, need && j > 0)) {
        wait(pv_done, (uint32_t)(j - 1) & 1u, abort_flag, a.err, 0x1502u);  // O holds PV(j-1)
        tc_fence_after();
#pragma unroll
        for (int pc = 0; pc < 4; ++pc) {
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
    wait(o_done, 0, abort_flag, a.err, 0x1503u);
    tc_fence_after();
    const int64_t qrow = (int64_t)q0 + row;
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int pc = 0; pc < 4; ++pc) {
      float ov[32];
      tmem_ld32(lane_addr + (OC - tmem) + pc * 32, ov);
      if (qrow < a.n_q) {
        uint4* dst = reinterpret_cast<uint4*>(a.O + (qrow * a.Hq + hq) * 128 + pc * 32);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) w[i] = pack_bf16x2(ov[ch * 8 + 2 * i] * inv, ov[ch * 8 + 2 * i + 1] * inv);
          dst[ch] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
  } else if (JC) {
    // ================================================================ Jensen operands (warp 6)
    // A (once, slice 0): row r, logical column g < NG holds -|q_g|^2 * 0.5 scale / 12;
    // B (per history tile, slice 1 + stage): key row k, column g holds s_g^2.
    // Logical columns NG .. 15 of a slice are zero; the MMA reads the slice's
    // 16 columns of the 128-byte-swizzled rows.  The tile lies over Q's first
    // sub-tile, so it is written once the softmax warps have moved Q to tensor
    // memory (and this warp has read the rows it needs).
    constexpr int GQ = 128 / NG;  // channels per group
    if (!wait(q_full, 0, abort_flag, a.err, 0x1600u)) {
      // the MMA warp gives up as well
    } else {
      float qn[4][NG];  // rows lane + 32 i
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = lane + 32 * i;
#pragma unroll
        for (int g = 0; g < NG; ++g) qn[i][g] = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) {  // 16-byte chunk k of the row: elements 8k .. 8k + 7
          const uint4 u = *reinterpret_cast<const uint4*>(Qs + (k / 8) * 16384 + sw128_off(r, k % 8));
          float x[8];
          unpack_bf16x8(u, x, 0);
#pragma unroll
          for (int e = 0; e < 8; ++e) qn[i][(8 * k) / GQ] = fmaf(x[e], x[e], qn[i][(8 * k) / GQ]);
        }
      }
      wait(q_tmem, 0, abort_flag, a.err, 0x1601u);  // after an abort the MMA warp issues nothing
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = lane + 32 * i;
        float v[16];
#pragma unroll
        for (int g = 0; g < 16; ++g) v[g] = g < NG ? qn[i][g] * a.jensen_a : 0.f;
#pragma unroll
        for (int ch = 0; ch < 2; ++ch)
          *reinterpret_cast<uint4*>(X + sw128_off(r, ch)) =
              make_uint4(pack_bf16x2(v[8 * ch], v[8 * ch + 1]), pack_bf16x2(v[8 * ch + 2], v[8 * ch + 3]),
                         pack_bf16x2(v[8 * ch + 4], v[8 * ch + 5]), pack_bf16x2(v[8 * ch + 6], v[8 * ch + 7]));
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(qx_full);
      // the (scale, zero) pairs of this lane's four keys of a tile, one load per key
      // (NG pairs are 8 or 16 contiguous bytes); the next tile's are in flight
      // while this one waits for its stage
      using PR = typename std::conditional<NG == 4, uint4, uint2>::type;
      auto load_params = [&](int j, PR (&pr)[4]) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int64_t t = (int64_t)j * 128 + lane + 32 * i;
          pr[i] = t < a.T ? __ldg(reinterpret_cast<const PR*>(a.kparams + (t * a.H + h) * NG)) : PR{};
        }
      };
      PR cur[4], nxt[4];
      if (NH > 0) load_params(0, nxt);
      for (int j = 0; j < NH; ++j) {
        const int s = j % S;
        const uint32_t ph = (uint32_t)(j / S) & 1u;
#pragma unroll
        for (int i = 0; i < 4; ++i) cur[i] = nxt[i];
        if (j + 1 < NH) load_params(j + 1, nxt);
        // the stage's previous tile is done (its S, and so its Jensen MMA, completed before its PV)
        if (!wait(&kv_empty[s], ph ^ 1u, abort_flag, a.err, 0x1610u + s)) break;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = lane + 32 * i;
          const __half2* pr = reinterpret_cast<const __half2*>(&cur[i]);
          float v[16];
#pragma unroll
          for (int g = 0; g < 16; ++g) v[g] = 0.f;
#pragma unroll
          for (int g = 0; g < NG; ++g) {
            const float sg = __low2float(pr[g]);
            v[g] = sg * sg;
          }
#pragma unroll
          for (int ch = 0; ch < 2; ++ch)
            *reinterpret_cast<uint4*>(X + sw128_off(r, 2 * (s + 1) + ch)) =
                make_uint4(pack_bf16x2(v[8 * ch], v[8 * ch + 1]), pack_bf16x2(v[8 * ch + 2], v[8 * ch + 3]),
                           pack_bf16x2(v[8 * ch + 4], v[8 * ch + 5]), pack_bf16x2(v[8 * ch + 6], v[8 * ch + 7]));
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&x_full[s]);
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

template <bool JC, int NG>
static cudaError_t launch(const Maps& m, const Args& a, cudaStream_t st) {
  using L = Cfg<JC>;
  auto k = attend_kernel<JC, NG>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
  if (e != cudaSuccess) return e;
  const unsigned nqt = (unsigned)((a.n_q + 127) / 128);
  k<<<dim3(nqt, (unsigned)a.Hq), L::kThreads, L::kSmem, st>>>(m, a);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace flash
}  // namespace tc

bool tc_flash_supported(const kvc_layer_desc* d) { return d->dtype == KVC_BF16 && d->head_dim == 128; }

bool tc_flash_debiased_supported(const kvc_layer_desc* d, const kvc_predictor* p) {
  return tc_flash_supported(d) && p->kind == KVC_PRED_XLAYER_DPLR && d->residual_codec == KVC_RESIDUAL_RTN &&
         d->param_dtype == KVC_F16 && (d->group == 32 || d->group == 64);
}

cudaError_t tc_flash(const kvc_layer_desc* d, const void* Q, int64_t n_q, const void* Kh, const void* Vh,
                     const void* K_self, const void* V_self, int64_t n_self, float scale, void* O,
                     const void* k_params, cudaStream_t st) {
  const uint64_t T = (uint64_t)d->n_tokens, H = d->n_heads, C = H * 128;
  const uint64_t Hq = d->q_heads > 0 ? (uint64_t)d->q_heads : H;
  tc::flash::Maps m;
  memset(&m, 0, sizeof(m));
  // maps need a non-empty extent: a map over no rows points at Q and is never read
  bool ok = tc::map2d(&m.q, Q, (uint64_t)n_q, Hq * 128, 128) && tc::map2d(&m.kh, T ? Kh : Q, T ? T : 1, C, 128) &&
            tc::map2d(&m.vh, T ? Vh : Q, T ? T : 1, C, 128) &&
            tc::map2d(&m.kself, n_self ? K_self : Q, n_self ? (uint64_t)n_self : 1, C, 128) &&
            tc::map2d(&m.vself, n_self ? V_self : Q, n_self ? (uint64_t)n_self : 1, C, 128);
  if (!ok) return cudaErrorInvalidValue;
  unsigned* err = tc_error_word();
  if (!err) return cudaErrorInvalidDevice;
  const float log2e = 1.4426950408889634f;
  tc::flash::Args a{err, n_q, (int64_t)T, n_self, (int)H, (int)Hq, d->group, scale * log2e,
                    (const __half2*)k_params, -0.5f * scale / 12.f, (__nv_bfloat16*)O};
  if (!k_params) return tc::flash::launch<false, 1>(m, a, st);
  return d->group == 32 ? tc::flash::launch<true, 4>(m, a, st) : tc::flash::launch<true, 2>(m, a, st);
}

}  // namespace kvc
