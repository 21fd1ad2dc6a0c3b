// Attention over a compressed cross-layer history (tcgen05 + TMEM + TMA,
// thread-block clusters).
//
//   O = softmax(scale Q [K^_hist ; K_self]^T) [V^_hist ; V_self]
//
// ("NanoKV: High-Ratio KV Cache Compression for Autoregressive Video
// Generation", abstract: attention over the compressed history is the
// bottleneck; "CORAL-KV ...", Fig. 3: the history of layer l is decoded from
// its codes and the reconstruction of layer l-1.)  The history is decoded tile
// by tile on chip and never written to device memory: for a 128-key tile the
// block-DPLR prediction runs on the tensor cores (the layer's low-rank latents
// come precomputed, as bf16 hi / lo pairs, from the latent-only codec kernel),
// the dequantized codes are added and the bf16 K^ / V^ tile is kept in shared
// memory.  A cluster of CTAs (consecutive query tiles of one head) shares that
// work: each CTA decodes every CQ-th key tile and pushes it into the others'
// shared memory, so a key tile is decoded once per cluster instead of once per
// query tile.  S = Q K^T and O += P V^ run on tcgen05; P stays in tensor memory.
// When the caller asks for the decoded history as well (K_rec_opt / V_rec_opt),
// the first cluster of each head also stores every tile it decodes with TMA
// stores of the same shared-memory tile it pushes to its peers.
//
// Warp roles: 0 TMA producer, 1 MMA issuer (and TMEM owner), 2-5 decode
// epilogue (TMEM -> K^ / V^ tiles, pushed to the cluster), 6-9 softmax (S -> P,
// running max / sum, lazy rescaling of O, final normalisation).  TMEM: decode
// accumulator, S / P slots [2], O (128 columns each).
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
#ifndef KVC_ATTN_CLUSTER
#define KVC_ATTN_CLUSTER 4
#endif
// CTAs per cluster (even, at most 8): consecutive query tiles of one head share the decoded history
constexpr int CQ = KVC_ATTN_CLUSTER;
static_assert(CQ % 2 == 0 && CQ <= 8, "cluster of an even size up to 8");
constexpr int kStages = 2;
constexpr int kStage = 32768;
// shared memory (offsets from a 1024-aligned base)
constexpr int kQ = 0;                        // Q tile, 2 sub-tiles
constexpr int kK = kQ + 32768;               // K^ slots [2]
constexpr int kV = kK + 2 * 32768;           // V^ slots [2]
constexpr int kSt = kV + 2 * 32768;          // decode operand stages
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
  CUtensorMap kr, vr;              // optional decoded-history outputs [T][C]
};

struct Args {
  unsigned* err;
  int64_t n_q, T, n_self;
  int H, bits, group;
  int Hq;  // query heads (a multiple of H); query head h reads KV head h / (Hq / H)
  float scale_log2;  // softmax scale * log2(e)
  const uint8_t* kcodes;
  const __half2* kparams;
  const uint8_t* vcodes;
  const __half2* vparams;
  __nv_bfloat16* O;  // [n_q][H][128]
  int store_k, store_v;  // write the decoded history through maps.kr / maps.vr
  float jensen_log2;     // JC: 0.5 scale^2 log2(e) / 12 (Jensen term per |q_g|^2 s_g^2, in log2 units)
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

// ---------------------------------------------------------------- cluster primitives

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared-memory location in cluster CTA `rank`
__device__ __forceinline__ uint32_t peer_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// bulk copy of `bytes` from this CTA's shared memory into a peer's, completing on the peer's mbarrier
__device__ __forceinline__ void push_to_peer(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "r"(smem_u32(src)), "r"(bytes), "r"(bar)
               : "memory");
}
// commit whose arrival lands on the mbarrier at the same offset in the CTAs of `mask`
__device__ __forceinline__ void umma_commit_mc(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
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
__device__ __forceinline__ void tmem_ld_wait2(float (&a)[32], float (&b)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  tie32(a);
  tie32(b);
}
// 2^x by the hardware approximation (flush-to-zero; softmax weights only)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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
// Cluster of CQ CTAs = CQ consecutive 128-query tiles of one head.  History key
// tile j is decoded by cluster rank j mod CQ and pushed, as bf16 K^ / V^ tiles,
// into the same double-buffered tile slots of every CTA of the cluster; the
// chunk's own keys (K_self, V_self) are loaded by each CTA.  Per key tile j
// (slot b = j mod 2) every CTA runs S(j) = Q K^(j)^T into TMEM S[b], the softmax
// writes P(j) over S[b] as bf16 pairs, and O += P(j) V^(j) takes P from TMEM.
//
// Slot reuse across the cluster: the decoder of tile j writes slot b only after
// every CTA has finished with tile j-2 in that slot (kfree / vfree gather CQ
// arrivals, sent by tcgen05.commit multicast after S(j-2) / PV(j-2)); the
// decoder announces the bytes on each peer's kfull / vfull and pushes the tile
// with a bulk copy that completes there.

template <int RC, int G, int BITS, bool JC>
__global__ void __launch_bounds__(kThreads, 1) attend_cluster_kernel(const __grid_constant__ Maps maps, const Args a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBar);
  uint64_t* full = bars;               // [kStages] decode operands landed
  uint64_t* empty = full + kStages;    // [kStages]
  uint64_t* q_full = empty + kStages;
  uint64_t* d_full = q_full + 1;       // decode accumulator ready
  uint64_t* kfull = d_full + 1;        // [2] K^ slot holds tile j
  uint64_t* vfull = kfull + 2;         // [2] V^ slot holds tile j
  uint64_t* kfree = vfull + 2;         // cluster gather: K^ slot free for this CTA's next decoded tile
  uint64_t* vfree = kfree + 1;         // cluster gather: V^ slot free
  uint64_t* kt_free = vfree + 1;       // [2] local: K^ slot free for a chunk tile
  uint64_t* vt_free = kt_free + 2;     // [2] local: V^ slot free for a chunk tile
  uint64_t* s_full = vt_free + 2;      // [2]
  uint64_t* p_full = s_full + 2;       // [2]
  uint64_t* pv_done = p_full + 2;
  uint64_t* o_done = pv_done + 1;
  uint64_t* mma_done = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hq = blockIdx.y;           // query head
  const int h = hq / (a.Hq / a.H);     // its KV head (grouped-query attention when Hq > H)
  const int q0 = blockIdx.x * 128;
  const bool has_q = q0 < a.n_q;  // the last cluster of a head may hold CTAs past the queries
  const int rank = (int)cluster_rank();
  const int NH = (int)((a.T + 127) / 128);       // history key tiles
  const int NS = (int)((a.n_self + 127) / 128);  // chunk key tiles
  const int NT = NH + NS;
  auto own = [&](int j) { return j < NH && j % CQ == rank; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(d_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&vfull[i], 1);
      mbar_init(&kt_free[i], 1);
      mbar_init(&vt_free[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
    }
    mbar_init(kfree, CQ);
    mbar_init(vfree, CQ);
    mbar_init(pv_done, 1);
    mbar_init(o_done, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    // slots of history tiles 0 and 1 decoded elsewhere expect their pushed bytes
    for (int j = 0; j < 2 && j < NH; ++j)
      if (j % CQ != rank) {
        mbar_arrive_expect_tx(&kfull[j], 32768u);
        mbar_arrive_expect_tx(&vfull[j], 32768u);
      }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // every CTA's barriers exist before any remote arrival or push
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t DC = tmem, OC = tmem + 384;
  auto SC = [&](int b) { return tmem + 128 + 128 * b; };

  auto stA = [&](int s) { return smem + kSt + s * kStage; };
  auto stB = [&](int s) { return smem + kSt + s * kStage + 16384; };
  uint8_t* Qs = smem + kQ;
  auto Kt = [&](int b) { return smem + kK + b * 32768; };
  auto Vt = [&](int b) { return smem + kV + b * 32768; };

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      // the last phase armed on each barrier this thread loads into (drained after an abort)
      int st_issued[kStages] = {}, self_issued[2][2] = {};
      uint32_t st_ph[kStages] = {}, self_ph[2][2] = {};
      auto load = [&](const CUtensorMap* ma, int ax, int ay, const CUtensorMap* mb, int bx, int by) {
        if (!ok) return;
        if (!wait(&empty[s], ph ^ 1, abort_flag, a.err, 0x1100u + s)) {
          ok = false;
          return;
        }
        mbar_arrive_expect_tx(&full[s], (ma ? 16384u : 0u) + 16384u);
        if (ma) tma_load(stA(s), ma, ax, ay, &full[s], pol_stream);
        tma_load(stB(s), mb, bx, by, &full[s], pol_keep);
        st_issued[s] = 1;
        st_ph[s] = ph;
        if (++s == kStages) {
          s = 0;
          ph ^= 1;
        }
      };
      if (has_q) {
        mbar_arrive_expect_tx(q_full, 32768u);
        tma_load(Qs, &maps.q, hq * 128, q0, q_full, pol_stream);
        tma_load(Qs + 16384, &maps.q, hq * 128 + 64, q0, q_full, pol_stream);
      }
      // decode operands of this CTA's history tiles, in the order the MMA warp takes them
      for (int j = rank; j < NH && ok; j += CQ) {
        const int t0 = j * 128;
        constexpr int rbytes = 128 * BITS / 8;
        tma_prefetch(&maps.ck, h * rbytes, t0);
        tma_prefetch(&maps.cv, h * rbytes, t0);
        if (G == 32) {
          tma_prefetch(&maps.pk, h * 16, t0);
          tma_prefetch(&maps.pv, h * 16, t0);
        }
        // K: K^_{l-1,h} B_h^T + [Z_K hi | lo] U_h^T
        for (int c = 0; c < 2; ++c) load(&maps.ks, h * 128 + c * 64, t0, &maps.bk, c * 64, h * 128);
        for (int c = 0; c < RC; ++c) {
          load(&maps.zkh, c * 64, t0, &maps.uk, c * 64, h * 128);
          load(&maps.zkl, c * 64, t0, &maps.uk, c * 64, h * 128);
        }
        // V: [K^_{l,h} (resident) | V^_{l-1,h}] BV_h^T + [Z_V hi | lo] UV_h^T, the V^_{l-1,h}
        // half first as in the codec kernel, so that the sums round the same way
        for (int c = 0; c < 2; ++c) load(&maps.vs, h * 128 + c * 64, t0, &maps.bv, 128 + c * 64, h * 128);
        for (int c = 0; c < 2; ++c) load(nullptr, 0, 0, &maps.bv, c * 64, h * 128);
        for (int c = 0; c < RC; ++c) {
          load(&maps.zvh, c * 64, t0, &maps.uv, c * 64, h * 128);
          load(&maps.zvl, c * 64, t0, &maps.uv, c * 64, h * 128);
        }
      }
      // the chunk's own key tiles, into the slots once this CTA is done with them
      int ktf[2] = {0, 0}, vtf[2] = {0, 0};
      for (int j = NH; j < NT && ok && has_q; ++j) {
        const int b = j & 1;
        const int s0 = (j - NH) * 128;
        if (j >= 2 && !wait(&kt_free[b], ktf[b]++ & 1, abort_flag, a.err, 0x1200u + b)) ok = false;
        if (!ok) break;
        mbar_arrive_expect_tx(&kfull[b], 32768u);
        tma_load(Kt(b), &maps.kself, h * 128, s0, &kfull[b], pol_stream);
        tma_load(Kt(b) + 16384, &maps.kself, h * 128 + 64, s0, &kfull[b], pol_stream);
        self_issued[0][b] = 1;
        self_ph[0][b] = (j >> 1) & 1;
        if (j >= 2 && !wait(&vt_free[b], vtf[b]++ & 1, abort_flag, a.err, 0x1210u + b)) ok = false;
        if (!ok) break;
        mbar_arrive_expect_tx(&vfull[b], 32768u);
        tma_load(Vt(b), &maps.vself, h * 128, s0, &vfull[b], pol_stream);
        tma_load(Vt(b) + 16384, &maps.vself, h * 128 + 64, s0, &vfull[b], pol_stream);
        self_issued[1][b] = 1;
        self_ph[1][b] = (j >> 1) & 1;
      }
      if (*abort_flag) {
        // every load this thread issued lands before the CTA can leave
        auto drain = [&](uint64_t* bar, uint32_t parity) {
          const long long w0 = clock64();
          while (!mbar_test(bar, parity) && clock64() - w0 < kWaitBudget) {
          }
        };
        if (has_q) drain(q_full, 0);
        for (int i = 0; i < kStages; ++i)
          if (st_issued[i]) drain(&full[i], st_ph[i]);
        for (int b = 0; b < 2; ++b) {
          if (self_issued[0][b]) drain(&kfull[b], self_ph[0][b]);
          if (self_issued[1][b]) drain(&vfull[b], self_ph[1][b]);
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
        for (int c = 0; c < 2; ++c) chunk(DC, c == 0, nullptr);
        for (int c = 0; c < 2 * RC; ++c) chunk(DC, false, nullptr);
        umma_commit(d_full);
      };
      auto dec_v = [&](int b) {
        for (int c = 0; c < 2; ++c) chunk(DC, c == 0, nullptr);  // V^_{l-1,h} half
        for (int c = 0; c < 2; ++c) chunk(DC, false, Kt(b) + c * 16384);
        for (int c = 0; c < 2 * RC; ++c) chunk(DC, false, nullptr);
        umma_commit(d_full);
      };
      // slot of tile t released (S(t) / PV(t) issued): to the decoder of tile t+2, or locally
      auto release = [&](int t, uint64_t* gather, uint64_t* local) {
        const int j2 = t + 2;
        if (j2 < NH)
          umma_commit_mc(gather, (uint16_t)(1u << (j2 % CQ)));
        else if (j2 < NT && has_q)
          umma_commit(&local[t & 1]);
      };
      if (has_q && !wait(q_full, 0, abort_flag, a.err, 0x1310u)) ok = false;
      if (own(rank)) dec_k();
      if (own(0)) {  // tile 0 has no earlier iteration to take its V decode
        wait(&kfull[0], 0, abort_flag, a.err, 0x1324u);
        tc_fence_after();
        dec_v(0);
      }
      const int NE = has_q ? NT : NH;  // key tiles this CTA takes part in
      for (int j = 0; j <= NE; ++j) {
        if (j < NE) {
          const int b = j & 1;
          wait(&kfull[b], (j >> 1) & 1, abort_flag, a.err, 0x1320u + b);
          // the slot's next history tile, if a peer decodes it, will be pushed here
          if (j + 2 < NH && (j + 2) % CQ != rank) mbar_arrive_expect_tx(&kfull[b], 32768u);
          tc_fence_after();
          if (has_q) {
            // S(j) = Q K^(j)^T into S[b]; S[b] last held P(j-2), read by PV(j-2) issued before
            const uint64_t qd = desc_sw128(smem_u32(Qs));
            const uint64_t kd = desc_sw128(smem_u32(Kt(b)));
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint32_t off = (k >> 2) * (16384 >> 4) + (k & 3) * 2;
              umma(SC(b), qd + off, kd + off, id128, k == 0 ? 0u : 1u);
            }
            umma_commit(&s_full[b]);
          }
          release(j, kfree, kt_free);
        }
        if (j >= 1) {
          const int t = j - 1, b = t & 1;
          if (has_q) {
            // O += P(t) V^(t), P from TMEM
            wait(&p_full[b], (t >> 1) & 1, abort_flag, a.err, 0x1330u + b);
            wait(&vfull[b], (t >> 1) & 1, abort_flag, a.err, 0x1340u + b);
            if (t + 2 < NH && (t + 2) % CQ != rank) mbar_arrive_expect_tx(&vfull[b], 32768u);
            tc_fence_after();
            const uint64_t vd = desc_mn_sw128(smem_u32(Vt(b)), 16384);
            const uint32_t idv = idesc_bf16_bmn(128, 128);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              umma_ts(OC, SC(b) + k * 8, vd + (uint64_t)k * (2048 >> 4), idv, (t == 0 && k == 0) ? 0u : 1u);
            umma_commit(pv_done);
          } else {
            wait(&vfull[b], (t >> 1) & 1, abort_flag, a.err, 0x1341u + b);
            if (t + 2 < NH && (t + 2) % CQ != rank) mbar_arrive_expect_tx(&vfull[b], 32768u);
          }
          release(t, vfree, vt_free);
          // the decode accumulator is free once V^(t) is out: start this CTA's next tile
          if (own(t) && t + CQ < NH) dec_k();
        }
        // V decode of this CTA's tile j+1 one iteration early, as soon as its K^ is
        // published here (that also means the decode accumulator was drained)
        if (j + 1 < NH && own(j + 1)) {
          const int b1 = (j + 1) & 1;
          wait(&kfull[b1], ((j + 1) >> 1) & 1, abort_flag, a.err, 0x1325u);
          tc_fence_after();
          dec_v(b1);
        }
      }
      if (has_q) umma_commit(o_done);
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
    constexpr int LEVELS = (1 << BITS) - 1;
    constexpr int RB = 128 * BITS / 8;  // code bytes of a row
    constexpr int NW = RB / 4;          // code words of a row
    constexpr int NG = 128 / G;
    const bool elected = warp == 2 && lane == 0;
    int dfu = 0, kfu = 0, vfu = 0;
    // the codes and (scale, zero) pairs of one row of one tile
    struct RowIn {
      uint32_t cw[NW];
      __half2 pr[NG];
    };
    auto fetch = [&](const uint8_t* codes, const __half2* params, bool valid, RowIn& in) {
#pragma unroll
      for (int i = 0; i < NW / 4; ++i) {
        const uint4 w = valid ? __ldcs(reinterpret_cast<const uint4*>(codes) + i) : make_uint4(0, 0, 0, 0);
        in.cw[4 * i] = w.x;
        in.cw[4 * i + 1] = w.y;
        in.cw[4 * i + 2] = w.z;
        in.cw[4 * i + 3] = w.w;
      }
#pragma unroll
      for (int g = 0; g < NG; ++g) in.pr[g] = valid ? params[g] : __floats2half2_rn(0.f, 0.f);
    };
    // TMEM accumulator + dequantized codes -> bf16 row of a K^ / V^ tile
    auto emit = [&](const RowIn& in, uint8_t* tile) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float p[2][32];
        tmem_ld32_async(lane_addr + (DC - tmem) + half * 64, p[0]);
        tmem_ld32_async(lane_addr + (DC - tmem) + half * 64 + 32, p[1]);
        tmem_ld_wait2(p[0], p[1]);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            const int e = (half * 2 + q) * 32 + ch * 8;  // element of the row
            const float2 f = __half22float2(in.pr[e / G]);
            float r[8];
            dequant8<BITS>(in.cw[BITS == 2 ? e / 16 : e / 8], e, f.x, f.y, &p[q][ch * 8], r);
            *reinterpret_cast<uint4*>(tile + (e / 64) * 16384 + sw128_off(row, (e % 64) / 8)) =
                make_uint4(pack_bf16x2(r[0], r[1]), pack_bf16x2(r[2], r[3]), pack_bf16x2(r[4], r[5]),
                           pack_bf16x2(r[6], r[7]));
          }
        }
      }
      tc_fence_before();
      fence_async_smem();
      asm volatile("bar.sync 1, 128;" ::: "memory");
    };
    // the first cluster of the first query head of each KV head writes the
    // decoded history when asked to
    const bool first_cluster = blockIdx.x < (unsigned)CQ && hq % (a.Hq / a.H) == 0;
    const bool st_k = first_cluster && a.store_k, st_v = first_cluster && a.store_v;
    // the tile is complete here: announce it to every peer, push it, and mark it locally
    auto publish = [&](uint8_t* tile, uint64_t* bar, const CUtensorMap* out, int j) {
      if (!elected) return;
      // each peer armed its slot barrier for these bytes (see the MMA warp)
      for (int p = 1; p < CQ; ++p) {
        const uint32_t peer = (uint32_t)((rank + p) % CQ);
        push_to_peer(peer_addr(tile, peer), tile, 32768u, peer_addr(bar, peer));
      }
      if (out) {  // rows past T are clipped by the map
        tma_store(out, h * 128, j * 128, tile);
        tma_store(out, h * 128 + 64, j * 128, tile + 16384);
      }
      bulk_commit();
      mbar_arrive(bar);
    };
    // a slot that a TMA store still reads is not rewritten (the peers' pushes are
    // known to be complete once the slot's free barrier has gathered them)
    auto slot_stored = [&](bool stored) {
      if (!stored) return;
      if (elected) bulk_wait_read0();
      asm volatile("bar.sync 1, 128;" ::: "memory");
    };
    for (int j = rank; j < NH; j += CQ) {
      const int b = j & 1;
      const int64_t t = (int64_t)j * 128 + row;
      const bool valid = t < a.T;
      const int64_t rowi = t * a.H + h;
      RowIn kin, vin;
      fetch(a.kcodes + rowi * RB, a.kparams + rowi * NG, valid, kin);
      wait(d_full, dfu++ & 1, abort_flag, a.err, 0x1400u);
      if (j >= 2) wait(kfree, kfu++ & 1, abort_flag, a.err, 0x1401u);
      slot_stored(st_k && j >= 2);
      tc_fence_after();
      emit(kin, Kt(b));
      publish(Kt(b), &kfull[b], st_k ? &maps.kr : nullptr, j);
      fetch(a.vcodes + rowi * RB, a.vparams + rowi * NG, valid, vin);
      wait(d_full, dfu++ & 1, abort_flag, a.err, 0x1402u);
      if (j >= 2) wait(vfree, vfu++ & 1, abort_flag, a.err, 0x1403u);
      slot_stored(st_v && j >= 2);
      tc_fence_after();
      emit(vin, Vt(b));
      publish(Vt(b), &vfull[b], st_v ? &maps.vr : nullptr, j);
    }
    if (elected) bulk_wait_all();
  } else if (has_q) {
    // ================================================================ softmax (warps 6-9)
    const int qd = warp & 3;
    const int row = qd * 32 + lane;  // query row
    const uint32_t lane_addr = tmem + ((uint32_t)(qd * 32) << 16);
    const float c = a.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    // Jensen correction: |q_g|^2 of this thread's query row, from the Q tile
    constexpr int NGQ = 128 / G;
    float qn[JC ? NGQ : 1];
    if (JC) {
      wait(q_full, 0, abort_flag, a.err, 0x1504u);
#pragma unroll
      for (int g = 0; g < NGQ; ++g) qn[g] = 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) {  // 16-byte chunk k of the row: elements 8k .. 8k + 7
        const uint4 u = *reinterpret_cast<const uint4*>(Qs + (k / 8) * 16384 + sw128_off(row, k % 8));
        float x[8];
        unpack_bf16x8(u, x, 0);
#pragma unroll
        for (int i = 0; i < 8; ++i) qn[(8 * k) / G] = fmaf(x[i], x[i], qn[(8 * k) / G]);
      }
    }
    for (int j = 0; j < NT; ++j) {
      const int b = j & 1;
      const uint32_t sc = lane_addr + (SC(b) - tmem);
      const bool hist = j < NH;
      // JC: lane l holds the Jensen weights w_g = s_g^2 jensen_log2 of keys l, l + 32,
      // l + 64, l + 96 of a history tile (loaded before the S wait hides their latency)
      float w[JC ? 4 : 1][JC ? NGQ : 1];
      if (JC && hist) {
#pragma unroll
        for (int pc = 0; pc < 4; ++pc) {
          const int64_t t = (int64_t)j * 128 + pc * 32 + lane;
          const __half2* pr = a.kparams + (t * a.H + h) * NGQ;
#pragma unroll
          for (int g = 0; g < NGQ; ++g) {
            const float sg = t < a.T ? __low2float(pr[g]) : 0.f;
            w[pc][g] = sg * sg * a.jensen_log2;
          }
        }
      }
      wait(&s_full[b], (j >> 1) & 1, abort_flag, a.err, 0x1500u + b);
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
      if (JC) {
        // scores in log2 units, history keys lowered by their Jensen term
        // sum_g |q_g|^2 w_g (key pc * 32 + i's weights come from lane i)
#pragma unroll
        for (int pc = 0; pc < 4; ++pc)
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float corr = 0.f;
            if (hist) {
#pragma unroll
              for (int g = 0; g < NGQ; ++g) corr = fmaf(qn[g], __shfl_sync(0xffffffffu, w[pc][g], i), corr);
            }
            sv[pc][i] = fmaf(sv[pc][i], c, -corr);
          }
      }
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
      const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * (JC ? 1.f : c);
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
          const float p0 = ex2_approx(JC ? sv[pc][2 * i] - m_used : fmaf(sv[pc][2 * i], c, -m_used));
          const float p1 = ex2_approx(JC ? sv[pc][2 * i + 1] - m_used : fmaf(sv[pc][2 * i + 1], c, -m_used));
          ls[i & 3] += p0 + p1;
          w[i] = pack_bf16x2(p0, p1);
        }
        tmem_st16(sc + pc * 16, w);
      }
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      // O is rescaled before P(j) is handed over (PV(j) follows p_full)
      if (__any_sync(0xffffffffu, need && j > 0)) {
        wait(pv_done, (j - 1) & 1, abort_flag, a.err, 0x1502u);  // O holds PV(j-1)
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
  }

  tc_fence_before();
  __syncthreads();
  // no CTA leaves while a peer may still push into it or arrive on its barriers
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int RC, int G, int BITS, bool JC>
static cudaError_t launch(const Maps& m, const Args& a, cudaStream_t st) {
  auto k = attend_cluster_kernel<RC, G, BITS, JC>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  const unsigned nqt = (unsigned)((a.n_q + 127) / 128);
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((nqt + CQ - 1) / CQ * CQ, (unsigned)a.Hq);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CQ;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, k, m, a);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int RC, bool JC>
static cudaError_t dispatch_gb(int group, int bits, const Maps& m, const Args& a, cudaStream_t st) {
  if (group == 32) return bits == 2 ? launch<RC, 32, 2, JC>(m, a, st) : launch<RC, 32, 4, JC>(m, a, st);
  return bits == 2 ? launch<RC, 64, 2, JC>(m, a, st) : launch<RC, 64, 4, JC>(m, a, st);
}
template <bool JC>
static cudaError_t dispatch(int rc, int group, int bits, const Maps& m, const Args& a, cudaStream_t st) {
  if (rc == 0) return dispatch_gb<0, JC>(group, bits, m, a, st);
  if (rc == 1) return dispatch_gb<1, JC>(group, bits, m, a, st);
  return dispatch_gb<2, JC>(group, bits, m, a, st);
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
                      float scale, void* O, void* K_rec, void* V_rec, void* ws, size_t ws_bytes, cudaStream_t st,
                      bool jensen) {
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
  const uint64_t Hq = d->q_heads > 0 ? (uint64_t)d->q_heads : H;
  const uint64_t Th = T > 0 ? T : 1;  // maps need a non-empty extent; no history tile is read when T = 0
  bool ok = tc::map2d(&m.q, Q, (uint64_t)n_q, Hq * 128, 128) && tc::map2d(&m.ks, T ? Ks : Q, Th, C, 128) &&
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
  const bool sk = K_rec && T > 0, sv = V_rec && T > 0;
  if (ok && sk) ok = tc::map2d(&m.kr, K_rec, T, C, 128);
  if (ok && sv) ok = tc::map2d(&m.vr, V_rec, T, C, 128);
  if (!ok) return cudaErrorInvalidValue;
  unsigned* err = tc_error_word();
  if (!err) return cudaErrorInvalidDevice;
  tc::attn::Args a{err, n_q, (int64_t)T, n_self, (int)H, d->bits, d->group, (int)Hq, scale * 1.4426950408889634f,
                   (const uint8_t*)c->k_codes, (const __half2*)c->k_params, (const uint8_t*)c->v_codes,
                   (const __half2*)c->v_params, (__nv_bfloat16*)O, sk ? 1 : 0, sv ? 1 : 0,
                   0.5f * scale * scale * 1.4426950408889634f / 12.f};
  const int rc = r == 0 ? 0 : r == 64 ? 1 : 2;
  return jensen ? tc::attn::dispatch<true>(rc, d->group, d->bits, m, a, st)
                : tc::attn::dispatch<false>(rc, d->group, d->bits, m, a, st);
}

}  // namespace kvc
