// Tensor-core kernels (tcgen05 + TMEM + TMA) of the bf16 / head_dim 128 hot path.
//
// Cross-layer block-DPLR codec, persistent CTAs (one per SM) looping over
// 128-token tiles, all heads fused ("CORAL-KV: Compact Cross-Layer Prediction
// and Residual Coding for Autoregressive Video KV Caches", Fig. 3: K_l from the
// reconstructed K_{l-1}; V_l from the reconstructed [K_l, V_{l-1}];
// block-diagonal per-head maps plus a global rank-r term).  Per tile:
//
//   Z_K  = K^_{l-1} W_K^T                         (TMEM, 64-channel chunks)
//   for each head h (K):  acc = K^_{l-1,h} B_h^T + [Z_K hi | lo] U_h^T
//        epilogue: residual, group min/max, fp16 (scale, zero), codes, packing,
//        reconstruction K^_{l,h} -> shared memory -> TMA store, and
//        Z_V += K^_{l,h} W_V[:, h]^T (the V latent grows head by head)
//        Z_V += V^_{l-1,h} W_V[:, C + h]^T (the other half, interleaved)
//   for each head h (V):  acc = [K^_{l,h} | V^_{l-1,h}] BV_h^T + [Z_V hi | lo] UV_h^T
//        epilogue as above, writing V^_{l,h}
//
// The latent GEMMs are spread over the head loops so the tensor pipe and the
// epilogue warps stay busy while the latent's operands stream in; at rank 64
// the next tile's Z_K is accumulated in a second TMEM slot during the V heads.
// The latent is carried to the second factor as a pair of bf16 values whose
// sum is within 2^-16 of the fp32 accumulator, so no rounding decision is taken
// on it.  Warp roles: warp 0 issues TMA loads, warp 1 allocates TMEM and one
// thread issues every tcgen05.mma, warps 2..9 run the epilogue as two groups of
// four warps (one TMEM lane quarter each) taking alternate heads.  Every wait is
// bounded: a wait that runs out records an error word, raises an abort flag
// seen by all roles, and the CTA drains what it issued and returns.
#include <cuda.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <vector>

#include "../../include/kvc_testing.h"
#include "tc.h"
#include "tc_ptx.cuh"

namespace kvc {

// First error recorded by a bounded device-side wait (0 = none).
__device__ unsigned int g_device_error = 0;

unsigned int* tc_error_word() {
  static unsigned int* ptr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    ptr[dev] = static_cast<unsigned int*>(p);
  }
  return ptr[dev];
}

cudaError_t tc_read_and_clear_error(unsigned int* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  const unsigned int zero = 0;
  return *value ? cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) : cudaSuccess;
}

namespace tc {

// One-shot test hook of kvc_testing_inject_stall (read and cleared by the next
// cross-layer codec launch).
static std::atomic<int> g_inject_stall{0};

constexpr int kThreads = 352;     // 11 warps: producer, MMA, two epilogue groups of 4, MMA sync
constexpr int kSyncWarp = 10;
constexpr int kGroupThreads = 128;

enum Mode { kEncode = 0, kDecode = 1 };

// ---------------------------------------------------------------- kernel arguments

struct Maps {
  CUtensorMap ks, vs;  // reconstructions of layer l-1, [T][C]
  CUtensorMap ko, vo;  // reconstructions of layer l (written; K also read back), [T][C]
  CUtensorMap wk, wv;  // [r][C], [r][2C]
  CUtensorMap bk, bv;  // [H*128][128], [H*128][256]
  CUtensorMap uk, uv;  // [C][r]
  // L2 prefetch only: clean inputs [T][C] (encode), codes [T][H*row_bytes] and
  // params [T][H*16] as bytes (decode)
  CUtensorMap xk, xv, ck, cv, pk, pv;
};

// the per-layer buffers of a call
struct Ptrs {
  const __nv_bfloat16* xk;  // clean K (encode)
  const __nv_bfloat16* xv;  // clean V (encode)
  uint8_t* kcodes;
  __half2* kparams;
  uint8_t* vcodes;
  __half2* vparams;
};

// one layer of a multi-layer call, in device memory (tensor maps 64-byte aligned)
struct alignas(64) LayerDev {
  Maps maps;
  Ptrs p;
};

struct Args {
  unsigned* err;  // device error word
  int64_t T;
  int H, bits;
  Ptrs p;
  int store_v;  // V^_l is written (always for decode)
  // multi-layer calls: the layers' maps and buffers, and one counter per
  // (layer, tile) that the tile's epilogue groups raise once its reconstruction
  // is stored (the next layer's tile waits for it)
  const LayerDev* layers;
  int n_layers;
  unsigned* flags;
  // test hook (kvc_testing_inject_stall): 1 = CTA 0's producer leaves its first
  // stage unarmed, so that the consumer's bounded wait runs out
  int inject;
  // H64 / EDEN-2 residuals: the 16 two-dimensional codebook points (32 fp32)
  const float* codebook;
};

// SLIM: a paired decode of 2-bit codes in 32-value groups stages only 48 bytes a
// thread (two chunks of code words, one of (scale, zero) pairs), so its input
// slots are 64 bytes and the 16 KB this frees hold a sixth pipeline stage
template <int MODE, int G, int BITS, bool PAIR, bool EDEN>
constexpr bool kSlim = PAIR && MODE == kDecode && !EDEN && BITS == 2 && G == 32;

template <int RC, bool PAIR, bool SLIM = false>
struct Layout {
  // pipeline stages (the latent lives in TMEM, not here); a CTA of a pair holds
  // half of every B operand, so its stages are smaller and there are more of them
  static constexpr int S = PAIR ? (SLIM ? 6 : 5) : 4;
  static constexpr int kStage = PAIR ? 24576 : 32768;  // A 16 KB + B 16 KB (pair: B 8 KB)
  static constexpr int kRecon = 32768;  // [128][128] bf16 as two 64-column sub-tiles
  static constexpr int kIn = SLIM ? 64 : 128;  // staged epilogue inputs: bytes per epilogue thread
  static constexpr int kStageOff = 0;
  static constexpr int kReconOff = S * kStage;
  static constexpr int kInOff = kReconOff + 2 * kRecon;
  static constexpr int kBarOff = kInOff + 256 * kIn;
  static constexpr int kBytes = kBarOff + 1024;
};

// Orthonormal Walsh-Hadamard transform of one thread's 64 values (Sylvester
// order: entry (i, j) = (-1)^popcount(i & j) / 8), six butterfly stages in registers.
// Entries e and e + 2 (bit 1 of e clear) travel as one packed pair, so every
// stage but the one over bit 1 does two butterflies an instruction; each entry
// still takes one rounded addition a stage, in the same order.  The pairing
// also puts the first coordinates of the point pairs 2m and 2m + 1 side by side
// (entries 4m and 4m + 2), as the EDEN-2 search wants them.
__device__ __forceinline__ void walsh64_thread(float (&v)[64]) {
#pragma unroll
  for (int b = 1; b < 64; b <<= 1) {
#pragma unroll
    for (int e = 0; e < 64; ++e) {
      if ((e & b) || (e & 2)) continue;
      if (b == 2) {
        const float x = v[e], y = v[e + 2];
        v[e] = x + y;
        v[e + 2] = x - y;
      } else {
        const float2 x = make_float2(v[e], v[e + 2]), y = make_float2(v[e + b], v[e + b + 2]);
        const float2 s = add2(x, y), d = sub2(x, y);
        v[e] = s.x;
        v[e + 2] = s.y;
        v[e + b] = d.x;
        v[e + b + 2] = d.y;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 64; ++e) {
    if (e & 2) continue;
    const float2 s = mul2(make_float2(v[e], v[e + 2]), make_float2(0.125f, 0.125f));
    v[e] = s.x;
    v[e + 2] = s.y;
  }
}

// ---------------------------------------------------------------- the kernel

template <int MODE, int G, int RC, int BITS, bool PAIR, bool EDEN, bool MULTI>
__global__ void __launch_bounds__(kThreads, 1) xlayer_tc_kernel(const __grid_constant__ Maps maps, const Args a) {
  constexpr bool ENC = MODE == kEncode;
  static_assert(!EDEN || (G == 64 && BITS == 2), "EDEN-2 codes 64-value groups at 4 bits a pair");
  constexpr bool SLIM = kSlim<MODE, G, BITS, PAIR, EDEN>;
  using L = Layout<RC, PAIR, SLIM>;
  constexpr int S = L::S;
  constexpr int R = RC * 64;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* full = bars;                 // [S]
  uint64_t* empty = bars + S;            // [S]
  uint64_t* acc_full = bars + 2 * S;     // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint64_t* rec_full = acc_empty + 2;    // [2]
  uint64_t* rec_free = rec_full + 2;     // [2]
  uint64_t* zk_full = rec_free + 2;
  uint64_t* zv_full = zk_full + 1;
  uint64_t* z_ready = zv_full + 1;
  uint64_t* khat_stored = z_ready + 1;
  uint64_t* mma_done = khat_stored + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_cb = reinterpret_cast<float*>(smem + L::kBarOff + 512);  // EDEN-2 codebook [16][2]
  // the search's form of point j, each term twice (one per lane of a packed
  // pair): (-2 c_j0, -2 c_j0, -2 c_j1, -2 c_j1) and (|c_j|^2, |c_j|^2)
  float4* s_cxy = reinterpret_cast<float4*>(smem + L::kBarOff + 640);  // [16]
  float2* s_cz = reinterpret_cast<float2*>(smem + L::kBarOff + 896);   // [16]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = a.H;
  const int C = H * 128;
  const int NCH = C / 64;
  // persistent CTAs: this CTA codes items blockIdx.x, blockIdx.x + gridDim.x, ...
  // An item is a tile of one layer; a multi-layer call orders them layer by
  // layer, and the tile of layer l waits for the same tile of layer l-1.
  // A pair (cluster of two) codes 256-token tiles: the even CTA (the leader,
  // which issues the MMAs) its first 128 tokens, the odd one the rest.
  const uint32_t crank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = crank == 0;
  const int unit = (int)(PAIR ? blockIdx.x >> 1 : blockIdx.x);
  const int nunits = (int)(PAIR ? gridDim.x >> 1 : gridDim.x);
  const int span = PAIR ? 256 : 128;
  const int ntiles = (int)((a.T + span - 1) / span);
  const int nitems = (MULTI ? a.n_layers : 1) * ntiles;
  const int my_tiles = unit < nitems ? (nitems - 1 - unit) / nunits + 1 : 0;  // items of this CTA
  auto item_of = [&](int it) { return unit + it * nunits; };  // the static order
  auto tile_t0 = [&](int i) { return (i % ntiles) * span + (int)crank * 128; };
  auto layer_of = [&](int i) { return MULTI ? i / ntiles : 0; };
  // the maps and buffers of a layer (a single-layer launch has them as arguments)
  auto LM = [&](int l) -> const Maps* {
    if constexpr (MULTI) return &a.layers[l].maps;
    else return &maps;
  };
  auto LP = [&](int l) -> const Ptrs& {
    if constexpr (MULTI) return a.layers[l].p;
    else return a.p;
  };
  // a tile's counter reaches flag_full once every epilogue group coding it has
  // stored its reconstruction
  constexpr unsigned flag_full = PAIR ? 4u : 2u;
  auto flag_of = [&](int l, int i) { return a.flags + (size_t)l * ntiles + i % ntiles; };
  // the leader's barriers, as shared::cluster addresses (a pair's arrivals and TMA bytes land there)
  auto lead_bar = [&](uint64_t* b) { return PAIR ? mapa_rank(b, crank & ~1u) : smem_u32(b); };
  // With rank 64 the TMEM has room for two latent slots, so the next tile's K
  // latent streams in during this tile's V heads.
  constexpr bool OVL = RC == 1;
  // The next item's K latent is loaded during this item's V heads.  In a
  // multi-layer call that needs the next item's own dependency first; it is an
  // earlier item (no cycle of waits) only while the grid has fewer units than a
  // layer has tiles, so with more the overlap is off (each item loads its latent).
  const bool ovl = OVL && (!MULTI || nunits < ntiles);
  const int HH = 2 * H;  // heads per tile (K then V)

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      // a pair's epilogue groups arrive once each, by an elected thread, on the leader's barriers
      mbar_init(&acc_empty[i], PAIR ? 2 : kGroupThreads);
      mbar_init(&rec_full[i], PAIR ? 2 : 1);
      mbar_init(&rec_free[i], 1);
    }
    mbar_init(zk_full, 1);
    mbar_init(zv_full, 1);
    mbar_init(z_ready, PAIR ? 2 : kGroupThreads);
    mbar_init(khat_stored, 2);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    if (EDEN) {
      for (int i = 0; i < 32; ++i) s_cb[i] = a.codebook[i];
      for (int j = 0; j < 16; ++j) {
        const float c0 = a.codebook[2 * j], c1 = a.codebook[2 * j + 1];
        s_cxy[j] = make_float4(-2.f * c0, -2.f * c0, -2.f * c1, -2.f * c1);
        const float cc = fmaf(c0, c0, c1 * c1);
        s_cz[j] = make_float2(cc, cc);
      }
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_async_smem();
  }
  if (warp == 1) {
    if constexpr (PAIR) {  // the same columns in both CTAs of the pair (a kernel uses one CTA group)
      tmem_alloc_pair(tmem_slot, 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, 512);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_arrive_wait();  // both CTAs' barriers exist before any remote arrival or TMA byte
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: accumulators [0,128) and [128,256); latent slot k of Z_K / Z_V
  auto zk_col = [&](int it) { return tmem + 256 + (OVL ? (it & 1) * 128 : 0); };
  auto zv_col = [&](int it) { return tmem + 256 + (OVL ? (it & 1) * 128 + 64 : R); };

  auto stageA = [&](int s) { return smem + L::kStageOff + s * L::kStage; };
  auto stageB = [&](int s) { return smem + L::kStageOff + s * L::kStage + 16384; };
  auto recon = [&](int b) { return smem + L::kReconOff + b * L::kRecon; };
  const uint32_t in_base = smem_u32(smem + L::kInOff);

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      int s = 0;
      uint32_t ph = 0;
      int issued[S];          // a load was issued into stage i ...
      uint32_t issued_ph[S];  // ... in this phase of full[i]
      for (int i = 0; i < S; ++i) issued[i] = 0, issued_ph[i] = 0;
      bool ok = true;
      bool stall = a.inject == 1 && blockIdx.x == 0;  // test hook: one stage is never armed
      auto load = [&](const CUtensorMap* ma, int ax, int ay, uint64_t pa, const CUtensorMap* mb, int bx, int by,
                      uint32_t bbytes) {
        if (!ok) return;
        if (!wait(&empty[s], ph ^ 1, abort_flag, a.err, 0x100u + s)) {
          ok = false;
          return;
        }
        if (stall) {  // neither armed nor loaded: the MMA side's wait on full[s] runs out
          stall = false;
          if (++s == S) {
            s = 0;
            ph ^= 1;
          }
          return;
        }
        if (PAIR) {
          // this CTA's 128 rows of A and half of B's rows (a box of bbytes / 128 rows,
          // 128 bytes each); the leader expects the bytes of both CTAs
          if (leader) mbar_arrive_expect_tx(&full[s], (ma ? 2u * 16384u : 0u) + bbytes);
          const uint32_t fb = lead_bar(&full[s]);
          if (ma) tma_load_pair(stageA(s), ma, ax, ay, fb, pa);
          tma_load_pair(stageB(s), mb, bx, by + (int)(crank * (bbytes / 256)), fb, pol_keep);
        } else {
          mbar_arrive_expect_tx(&full[s], (ma ? 16384u : 0u) + bbytes);
          if (ma) tma_load(stageA(s), ma, ax, ay, &full[s], pa);
          tma_load(stageB(s), mb, bx, by, &full[s], pol_keep);
        }
        issued[s] = 1;
        issued_ph[s] = ph;
        if (++s == S) {
          s = 0;
          ph ^= 1;
        }
      };
      // two B boxes of the same map in one stage (first in the A half, second in the B half)
      auto load2 = [&](const CUtensorMap* mb, int bx0, int bx1, int by, uint32_t bbytes) {
        if (!ok) return;
        if (!wait(&empty[s], ph ^ 1, abort_flag, a.err, 0x100u + s)) {
          ok = false;
          return;
        }
        if (PAIR) {
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * bbytes);
          const uint32_t fb = lead_bar(&full[s]);
          const int hy = by + (int)(crank * (bbytes / 256));
          tma_load_pair(stageA(s), mb, bx0, hy, fb, pol_keep);
          tma_load_pair(stageB(s), mb, bx1, hy, fb, pol_keep);
        } else {
          mbar_arrive_expect_tx(&full[s], 2 * bbytes);
          tma_load(stageA(s), mb, bx0, by, &full[s], pol_keep);
          tma_load(stageB(s), mb, bx1, by, &full[s], pol_keep);
        }
        issued[s] = 1;
        issued_ph[s] = ph;
        if (++s == S) {
          s = 0;
          ph ^= 1;
        }
      };
      const uint32_t wbytes = R * 128;
      constexpr int rbytes = 128 * BITS / 8;
      // Multi-layer calls: before the first load of an item that reads layer
      // l-1's reconstruction, the same tile of layer l-1 must be stored (bounded
      // wait on its counter, then a proxy fence for the TMA loads that follow)
      auto dep_wait = [&](int i) {
        if constexpr (MULTI) {
          const int l = layer_of(i);
          if (l == 0 || !ok) return;
          const unsigned* f = flag_of(l - 1, i);
          const long long w0 = clock64();
          unsigned v;
          while (true) {
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
            if (v >= flag_full) break;
            if (*abort_flag) {
              ok = false;
              return;
            }
            if (clock64() - w0 > kWaitBudget) {
              *abort_flag = 1;
              atomicCAS(a.err, 0u, 0xB00u);
              ok = false;
              return;
            }
          }
          fence_async_global();
        }
      };
      int cur = my_tiles > 0 ? item_of(0) : -1;
      bool cur_pf = false;  // the current item's K latent was loaded during the previous item
      for (int it = 0; cur >= 0 && ok; ++it) {
        const int t0 = tile_t0(cur);
        const int nxt = it + 1 < my_tiles ? item_of(it + 1) : -1;
        bool nxt_pf = false;
        const Maps& mp = *LM(layer_of(cur));
        // the epilogue of head h reads its clean inputs (encode) or codes (decode)
        // from global memory: bring them into L2 as the head's operands stream in
        auto prefetch_head = [&](bool is_v, int h) {
          if (t0 >= a.T) return;  // a pair's odd CTA past the last token
          if (ENC) {
            const CUtensorMap* m = is_v ? &mp.xv : &mp.xk;
            tma_prefetch(m, h * 128, t0);
            tma_prefetch(m, h * 128 + 64, t0);
          } else {
            tma_prefetch(is_v ? &mp.cv : &mp.ck, h * rbytes, t0);
            if (G == 32) tma_prefetch(is_v ? &mp.pv : &mp.pk, h * 16, t0);
          }
        };
        if (!cur_pf) dep_wait(cur);  // (else the previous item checked it)
        if (RC && !cur_pf)
          for (int c = 0; c < NCH; ++c) load(&mp.ks, c * 64, t0, pol_keep, &mp.wk, c * 64, 0, wbytes);
        for (int h = 0; h < H && ok; ++h) {
          prefetch_head(false, h);
          for (int j = 0; j < 2; ++j)
            load(&mp.ks, h * 128 + j * 64, t0, pol_stream, &mp.bk, j * 64, h * 128, 16384);
          for (int j = 0; j < RC; ++j) load(nullptr, 0, 0, 0, &mp.uk, j * 64, h * 128, 16384);
          if (RC && h >= 2) load2(&mp.wv, (h - 2) * 128, (h - 2) * 128 + 64, 0, wbytes);
          if (RC)  // the V latent's V^_{l-1} half, interleaved with the K heads
            for (int c = 2 * h; c < 2 * h + 2; ++c)
              load(&mp.vs, c * 64, t0, pol_keep, &mp.wv, C + c * 64, 0, wbytes);
        }
        if (RC)
          for (int g = H >= 2 ? H - 2 : 0; g < H; ++g) load2(&mp.wv, g * 128, g * 128 + 64, 0, wbytes);
        for (int h = 0; h < H && ok; ++h) {
          prefetch_head(true, h);
          for (int j = 0; j < 2; ++j)
            load(&mp.vs, h * 128 + j * 64, t0, pol_stream, &mp.bv, 128 + j * 64, h * 128, 16384);
          if (h == 0) {  // K^_l is read back once both epilogue groups have stored it
            if (ok && !wait(khat_stored, it & 1, abort_flag, a.err, 0x200u)) ok = false;
            if (ok) fence_async_global();
          }
          for (int j = 0; j < 2; ++j)
            load(&mp.ko, h * 128 + j * 64, t0, pol_stream, &mp.bv, j * 64, h * 128, 16384);
          for (int j = 0; j < RC; ++j) load(nullptr, 0, 0, 0, &mp.uv, j * 64, h * 128, 16384);
          if (h == 0) {  // whether the next item's K latent streams in now
            nxt_pf = ovl && nxt >= 0;
            if (nxt_pf) dep_wait(nxt);
          }
          if (nxt_pf) {  // the next item's K latent, interleaved with the V heads
            const Maps& nm = *LM(layer_of(nxt));
            const int nt0 = tile_t0(nxt);
            for (int c = 2 * h; c < 2 * h + 2; ++c)
              load(&nm.ks, c * 64, nt0, pol_keep, &nm.wk, c * 64, 0, wbytes);
          }
        }
        cur = nxt;
        cur_pf = nxt_pf;
      }
      if (!ok && (!PAIR || leader)) {
        // drain: the loads already issued must land before the CTA exits
        for (int i = 0; i < S; ++i) {
          if (!issued[i]) continue;
          const long long w0 = clock64();
          while (!mbar_test(&full[i], issued_ph[i]) && clock64() - w0 < kWaitBudget) {
          }
        }
      }
      if (PAIR) {
        // This CTA's bytes complete on the leader's barriers.  Without an abort the
        // leader's MMAs release every stage, so each load has landed once its stage
        // is released.  After an abort some stages are never consumed: the CTA then
        // waits a fixed grace period (about 0.5 ms; a TMA load lands in microseconds)
        // before it meets the closing cluster barrier.
        for (int i = 0; i < S; ++i) {
          if (!issued[i]) continue;
          const long long w0 = clock64();
          while (!mbar_test(&empty[i], issued_ph[i]) && !*abort_flag && clock64() - w0 < kWaitBudget) {
          }
        }
        if (!ok || *abort_flag) {
          const long long w0 = clock64();
          while (clock64() - w0 < (1ll << 20)) {
          }
        }
      }
    }
  } else if (warp == 1 || warp == kSyncWarp) {
    // ================================================================ MMA issue and its waits
    // The MMA schedule is walked by two warps in lock step.  The sync warp waits
    // on every mbarrier a group of chunks needs (operands landed, accumulator
    // drained, latent converted ...) and hands the group to the MMA warp through
    // named barrier 3; the MMA warp, converged, issues the group's MMAs and
    // commits from one lane.  The MMA warp never polls shared memory: a poll
    // from the issuing warp waits for that warp's in-flight MMA operand reads,
    // which leaves the tensor pipe idle between chunks.
    // a pair's leader issues M = 256 MMAs over both CTAs' rows and commits to both
    constexpr int MM = PAIR ? 256 : 128;
    auto mma_ss = [](uint32_t lead, uint32_t d, uint64_t ad, uint64_t bd, uint32_t id, uint32_t acc) {
      if constexpr (PAIR)
        umma_pair_if(lead, d, ad, bd, id, acc);
      else
        umma_if(lead, d, ad, bd, id, acc);
    };
    auto mma_ts = [](uint32_t lead, uint32_t d, uint32_t at, uint64_t bd, uint32_t id, uint32_t acc) {
      if constexpr (PAIR)
        umma_pair_ts_if(lead, d, at, bd, id, acc);
      else
        umma_ts_if(lead, d, at, bd, id, acc);
    };
    auto walk = [&](auto issue_tag) {
      constexpr bool ISSUE = decltype(issue_tag)::value;
      const uint32_t lead = lane == 0;
      const uint32_t acc_col[2] = {tmem, tmem + 128};
      int s = 0;
      uint32_t ph = 0;
      int use[2] = {0, 0};   // uses of each accumulator
      int recf[2] = {0, 0};  // rec_full completions consumed per reconstruction tile
      int zr = 0;            // z_ready completions consumed
      auto wt = [&](uint64_t* bar, uint32_t parity, unsigned where) {
        if (!ISSUE && lane == 0) wait(bar, parity, abort_flag, a.err, where);
      };
      auto commit = [&](uint64_t* bar) {
        if constexpr (PAIR) {
          if (ISSUE) umma_commit_pair_if(lead, bar, 3);
        } else {
          if (ISSUE) umma_commit_if(lead, bar);
        }
      };
      // one 64-wide K chunk from stage st: A from the stage (resA == 0) or resident smem
      auto issue = [&](int st, uint32_t d, int N, bool first, const uint8_t* resA, const uint8_t* resA2) {
        if (!ISSUE) return;
        const uint32_t idesc = idesc_bf16(MM, N);
        const uint64_t bd = desc_sw128(smem_u32(stageB(st)));
        const uint64_t ad = desc_sw128(smem_u32(resA ? resA : stageA(st)));
#pragma unroll
        for (int k = 0; k < 4; ++k) mma_ss(lead, d, ad + 2 * k, bd + 2 * k, idesc, (first && k == 0) ? 0u : 1u);
        if (resA2) {
          const uint64_t ad2 = desc_sw128(smem_u32(resA2));
#pragma unroll
          for (int k = 0; k < 4; ++k) mma_ss(lead, d, ad2 + 2 * k, bd + 2 * k, idesc, 1u);
        }
      };
      // n chunks from the next n stages, after the waits in pre(): one hand-off a
      // stage, so that a stage's MMAs are issued as soon as it has landed
      auto group = [&](int n, auto&& pre, auto&& body) {
        for (int i = 0; i < n; ++i) {
          if (!ISSUE) {
            if (i == 0) pre();
            wt(&full[s], ph, 0x300u + s);
            __syncwarp();
          }
          asm volatile("bar.sync 3, 64;" ::: "memory");
          if (ISSUE) tc_fence_after();
          body(i, s);
          commit(&empty[s]);
          if (++s == S) {
            s = 0;
            ph ^= 1;
          }
        }
      };
      auto nop = [] {};
      auto acq = [&](int b) {
        if (use[b] >= 1) wt(&acc_empty[b], (use[b] - 1) & 1, 0x400u + b);
      };
      // the k-th item's state: 0 none, 1 an item, 2 an item whose K latent was
      // loaded during item k-1
      auto item_state = [&](int k) -> int { return k < my_tiles ? (ovl && k > 0 ? 2 : 1) : 0; };
      int st_cur = item_state(0);
      for (int it = 0; st_cur; ++it) {
        const uint32_t zk = zk_col(it), zv = zv_col(it);
        int st_next = 0;
        if (RC && st_cur != 2) {
          for (int c = 0; c < NCH; c += 2)
            group(2, nop, [&](int i, int st) { issue(st, zk, R, c + i == 0, nullptr, nullptr); });
          commit(zk_full);
        }
        // Z_V += K^_{l,g} W_V[:, g]^T from the reconstruction tile of K head g
        auto zva = [&](int g) {
          const int rb = (it * HH + g) & 1;
          // both 64-channel halves of the head from one stage (W_V boxes in its A and B halves)
          group(
              1, [&] { wt(&rec_full[rb], recf[rb] & 1, 0x500u + rb); },
              [&](int, int st) {
                if (!ISSUE) return;
                const uint32_t idesc = idesc_bf16(MM, R);
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                  const uint64_t bd = desc_sw128(smem_u32(j ? stageB(st) : stageA(st)));
                  const uint64_t ad = desc_sw128(smem_u32(recon(rb) + j * 16384));
#pragma unroll
                  for (int k = 0; k < 4; ++k) mma_ss(lead, zv, ad + 2 * k, bd + 2 * k, idesc, 1u);
                }
              });
          recf[rb]++;
          commit(&rec_free[rb]);
        };
        // the latent factor of a head: acc += [Z hi | Z lo] U^T, Z as bf16 pairs in TMEM
        // (64 rank columns per chunk i: hi pairs at +0, lo pairs at +32)
        auto lowrank = [&](int b, uint32_t zcol, bool first_head, unsigned where) {
          group(
              RC, [&] { if (first_head) wt(z_ready, zr & 1, where); },
              [&](int i, int st) {
                if (!ISSUE) return;
                const uint32_t idesc = idesc_bf16(MM, 128);
                const uint64_t bd = desc_sw128(smem_u32(stageB(st)));
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  mma_ts(lead, acc_col[b], zcol + i * 64 + k * 8, bd + 2 * k, idesc, 1u);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  mma_ts(lead, acc_col[b], zcol + i * 64 + 32 + k * 8, bd + 2 * k, idesc, 1u);
              });
          if (first_head) zr++;
        };
        for (int h = 0; h < H; ++h) {
          const int b = (it * HH + h) & 1;
          group(2, [&] { acq(b); }, [&](int i, int st) { issue(st, acc_col[b], 128, i == 0, nullptr, nullptr); });
          if (RC) lowrank(b, zk, h == 0, 0x600u);
          commit(&acc_full[b]);
          use[b]++;
          // two heads behind, so that the epilogue of head h-2 is long done
          if (RC && h >= 2) zva(h - 2);
          if (RC)  // V^_{l-1} half of the V latent; its first chunk initialises Z_V
            group(2, nop, [&](int i, int st) { issue(st, zv, R, 2 * h + i == 0, nullptr, nullptr); });
        }
        if (RC) {
          for (int g = H >= 2 ? H - 2 : 0; g < H; ++g) zva(g);
          commit(zv_full);
        }
        for (int h = 0; h < H; ++h) {
          const int b = (it * HH + H + h) & 1;
          // V^_{l-1,h} part first (chunks 2, 3 of BV_h), then K^_{l,h} (chunks 0, 1)
          group(2, [&] { acq(b); }, [&](int i, int st) { issue(st, acc_col[b], 128, i == 0, nullptr, nullptr); });
          group(2, nop, [&](int i, int st) { issue(st, acc_col[b], 128, false, nullptr, nullptr); });
          if (RC) lowrank(b, zv, h == 0, 0x601u);
          commit(&acc_full[b]);
          use[b]++;
          if (h == 0) st_next = item_state(it + 1);
          if (st_next == 2)
            group(2, nop, [&](int i, int st) { issue(st, zk_col(it + 1), R, 2 * h + i == 0, nullptr, nullptr); });
        }
        if (st_next == 2) commit(zk_full);
        st_cur = st_next;
      }
      if (ISSUE) {
        // every issued MMA completes before TMEM is released
        if constexpr (PAIR)
          umma_commit_pair_if(lead, mma_done, 1);
        else
          commit(mma_done);
        if (lane == 0) {
          const long long w0 = clock64();
          while (!mbar_test(mma_done, 0) && clock64() - w0 < kWaitBudget) {
          }
        }
        __syncwarp();
      }
    };
    if (PAIR && !leader) {
      // the leader issues the pair's MMAs
    } else if (warp == 1) {
      walk(Tag<true>{});
    } else {
      walk(Tag<false>{});
    }
  } else {
    // ================================================================ epilogue: two groups of 4 warps
    // Group g owns TMEM accumulator g and reconstruction tile g, i.e. the heads
    // whose running index (over tiles, K heads then V heads) is congruent to g
    // mod 2; each warp of a group covers one TMEM lane quarter (32 tokens) and
    // all 128 channels.
    const int grp = (warp - 2) >> 2;
    const int ew = (warp - 2) & 3;
    const int q = warp & 3;  // TMEM lane quarter of this warp
    const int row = q * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16);
    const bool elected = ew == 0 && lane == 0;
    constexpr int LEVELS = (1 << BITS) - 1;
    constexpr int NG = 128 / G;          // groups in a row
    constexpr int NP = G / 32;           // 32-column passes per group
    constexpr int RB = 128 * BITS / 8;   // code bytes of a row
    constexpr int GW = G * BITS / 32;    // code words of a group
    constexpr int XQ = G / 8;            // 16-byte words of x in a group
    constexpr bool KEEP = ENC && NP == 1;  // encode of a one-pass group keeps its prediction
    int use = 0;                 // uses of this group's accumulator
    int recfree = 0;             // rec_free completions consumed
    bool prev_k = false;         // the previous use of this group's tile fed Z_V
    int zk_use = 0, zv_use = 0;
    auto gsync = [&]() {
      if (grp == 0)
        asm volatile("bar.sync 1, 128;" ::: "memory");
      else
        asm volatile("bar.sync 2, 128;" ::: "memory");
    };

    // fp32 latent in TMEM -> bf16 hi / lo pairs written back over it (per 64 rank
    // columns: 32 columns of hi pairs, then 32 of lo pairs), the A operand of the
    // low-rank MMAs
    auto convert_latent = [&](uint32_t col) {
      for (int j = 0; j < RC; ++j) {
        const uint32_t base = lane_addr + (col - tmem) + j * 64;
        float v[2][32];
        tmem_ld32(base, v[0]);
        tmem_ld32(base + 32, v[1]);
        uint32_t wh[32], wl[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float x0 = v[i / 16][(2 * i) % 32], x1 = v[i / 16][(2 * i + 1) % 32];
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(x0, x1);
          const float2 hf = __bfloat1622float2(h2);
          wh[i] = *reinterpret_cast<const uint32_t*>(&h2);
          wl[i] = pack_bf16x2(x0 - hf.x, x1 - hf.y);
        }
        tmem_st32u(base, wh);
        tmem_st32u(base + 32, wl);
      }
      tc_fence_before();
      if constexpr (PAIR) {  // both CTAs' conversions gate the leader's low-rank MMAs
        gsync();
        if (elected) mbar_arrive_remote(lead_bar(z_ready));
      } else {
        mbar_arrive(z_ready);
      }
    };

    // Global inputs of a head reach a per-thread slot of shared memory by the
    // thread's own asynchronous copies, issued before the accumulator wait, so
    // their latency overlaps the MMAs.  A slot is 8 chunks of 16 bytes, swizzled
    // by row so that a warp's 16-byte reads are free of bank conflicts.  Decode:
    // the row's code words (chunks 0 ..) and its (scale, zero) pairs (chunk 4).
    // Encode with 32-element groups: x of two groups in flight (chunks 0-3 and
    // 4-7, group g in half g & 1); wider groups fetch x into registers.
    constexpr bool STX = ENC && G == 32;
    constexpr bool STE = ENC && EDEN;  // EDEN-2 encode: x of the next 64-value group in the slot
    const uint32_t slot = in_base + (uint32_t)(grp * 128 + row) * L::kIn;
    auto chunk = [&](int c) { return slot + (((uint32_t)c ^ (uint32_t)(row & (L::kIn / 16 - 1))) << 4); };
    constexpr int PCH = SLIM ? 2 : 4;  // the chunk of the (scale, zero) pairs (decode)

    // one head of this group: h its index, is_v K or V, t0 the tile.  The
    // groups of the row are processed by a rolled loop (the kernel's code must
    // stay small enough for the instruction caches).
    auto head = [&](int h, bool is_v, int t0, int l) {
      const int b = grp;
      const int64_t t = (int64_t)t0 + row;
      const bool valid = t < a.T;
      const int64_t rowi = t * H + h;
      const Ptrs& pp = LP(l);
      uint32_t* codes = reinterpret_cast<uint32_t*>((is_v ? pp.vcodes : pp.kcodes) + rowi * RB);
      __half2* params = (is_v ? pp.vparams : pp.kparams) + rowi * NG;
      const uint4* X = reinterpret_cast<const uint4*>((is_v ? pp.xv : pp.xk) + t * C + h * 128);
      // inputs of the current group: x (encode) or code words and (scale, zero)
      uint4 xc[ENC ? XQ : 1];
      uint32_t cc[ENC ? 1 : GW];
      __half2 pc = __floats2half2_rn(0.f, 0.f);
      auto stage_x = [&](int g) {
#pragma unroll
        for (int i = 0; i < XQ; ++i)
          cp_async16(chunk((g & 1) * XQ + i), valid ? (const void*)(X + g * XQ + i) : (const void*)pp.xk,
                     valid ? 16u : 0u);
        cp_async_commit();
      };
      auto stage_xe = [&](int g) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          cp_async16(chunk(i), valid ? (const void*)(X + g * 8 + i) : (const void*)pp.xk, valid ? 16u : 0u);
        cp_async_commit();
      };
      if (STX) {
        stage_x(0);
        if (NG > 1) stage_x(1);
      }
      if (STE) stage_xe(0);
      if (!ENC) {  // rows past T copy nothing and read zeros (source: the buffers' first bytes)
        const uint8_t* src = reinterpret_cast<const uint8_t*>(codes);
        const void* c0 = is_v ? pp.vcodes : pp.kcodes;
        const __half2* p0 = is_v ? pp.vparams : pp.kparams;
#pragma unroll
        for (int i = 0; i < RB / 16; ++i) cp_async16(chunk(i), valid ? (const void*)(src + 16 * i) : c0, valid ? 16u : 0u);
        if (EDEN) {  // the row's two fp16 scales
          const __half* es = reinterpret_cast<const __half*>(is_v ? pp.vparams : pp.kparams) + rowi * 2;
          cp_async4(chunk(PCH), valid ? (const void*)es : (const void*)p0, valid ? 4u : 0u);
        } else if (G == 32) {
          cp_async16(chunk(PCH), valid ? params : p0, valid ? 16u : 0u);
        } else {
#pragma unroll
          for (int i = 0; i < NG; ++i) cp_async4(chunk(PCH) + 4 * i, valid ? params + i : p0, valid ? 4u : 0u);
        }
        cp_async_commit();
      }
      // group g's inputs into registers (from the slot, or from global memory)
      auto fetch = [&](int g, uint4 (&xo)[ENC ? XQ : 1], uint32_t (&co)[ENC ? 1 : GW], __half2& po) {
        if (STX) {
#pragma unroll
          for (int i = 0; i < XQ; ++i) xo[i] = lds128(chunk((g & 1) * XQ + i));
        } else if (ENC) {
#pragma unroll
          for (int i = 0; i < XQ; ++i) xo[i] = valid ? __ldcs(X + g * XQ + i) : make_uint4(0, 0, 0, 0);
        } else {
#pragma unroll
          for (int i = 0; i < GW; i += 2) {
            const int wi = g * GW + i;  // code word of the row
            const uint2 w = lds64(chunk(wi / 4) + (wi % 4) * 4);
            co[i] = w.x;
            co[i + 1] = w.y;
          }
          const uint32_t pw = lds32(chunk(PCH) + 4 * g);
          po = *reinterpret_cast<const __half2*>(&pw);
        }
      };
      if (ENC && !STX && !STE) fetch(0, xc, cc, pc);
      // the reconstruction tile is free once its previous TMA store has read it
      // and, if it held a K head, the MMA of Z_V has consumed it
      if (elected) bulk_wait_read0();
      gsync();
      wait(&acc_full[b], use & 1, abort_flag, a.err, 0x800u + b);
      use++;
      if (RC && prev_k) wait(&rec_free[b], recfree++ & 1, abort_flag, a.err, 0x700u + b);
      prev_k = !is_v && RC;
      tc_fence_after();
      if (!ENC) {
        cp_async_wait<0>();
        fetch(0, xc, cc, pc);
      }
      const uint32_t acc = lane_addr + b * 128;
#pragma unroll 1
      for (int g = 0; g < NG; ++g) {
        uint4 xn[ENC ? XQ : 1];
        uint32_t cn[ENC ? 1 : GW];
        __half2 pn = pc;
        if (STX) {
          if (g + 1 < NG)
            cp_async_wait<1>();
          else
            cp_async_wait<0>();
          fetch(g, xc, cc, pc);
        } else if (!STE && g + 1 < NG) {
          fetch(g + 1, xn, cn, pn);
        }
        if constexpr (EDEN) {
          // H64 / EDEN-2: y = H r / 8 over the group's 64 residuals; each pair of y / sigma
          // takes its nearest codebook point (ties to the lower index); scale
          // S = |y|^2 / <y, c>; r^ = H (S c) / 8.  u = y / sigma replaces y in place.
          float y[64], sf;
          uint32_t gw[4] = {0u, 0u, 0u, 0u};  // pair p of the group at bits [4 (p % 8), +4) of word p / 8
          if constexpr (ENC) {
            cp_async_wait<0>();  // x of group g is in the slot
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              float p[32];
              tmem_ld32(acc + g * 64 + q * 32, p);
#pragma unroll
              for (int ch = 0; ch < 4; ++ch) {
                float x[8];
                unpack_bf16x8(lds128(chunk(q * 4 + ch)), x, 0);
#pragma unroll
                for (int i = 0; i < 8; ++i) y[q * 32 + ch * 8 + i] = x[i] - p[ch * 8 + i];
              }
            }
            if (g + 1 < NG) stage_xe(g + 1);  // the slot's x is in registers now
            walsh64_thread(y);
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 64; ++e) ss = fmaf(y[e], y[e], ss);
            const float sigma = sqrtf(ss * (1.f / 64.f));
            const float inv_sigma = ss > 0.f ? 1.f / sigma : 0.f;
#pragma unroll
            for (int e = 0; e < 64; ++e) {
              if (e & 2) continue;
              const float2 u = mul2(make_float2(y[e], y[e + 2]), make_float2(inv_sigma, inv_sigma));
              y[e] = u.x;
              y[e + 2] = u.y;
            }
            // |u - c|^2 = |u|^2 + |c|^2 - 2 <u, c>: per pair the point with the least
            // |c|^2 - 2 <u, c> (two FMAs, here packed over pairs 2m and 2m + 1:
            // entries (4m, 4m + 2) and (4m + 1, 4m + 3)); the index goes into the
            // pair's nibble of gw with one three-input logic op (j replicated over
            // all nibbles)
            float bd[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) bd[i] = INFINITY;
#pragma unroll 2  // two points in flight (one measured 1.5% slower, four 6%)
            for (int j = 0; j < 16; ++j) {  // points in index order: a strict < keeps the lowest
              const float4 cxy = s_cxy[j];
              const float2 cz = s_cz[j];
              const uint32_t jr = (uint32_t)j * 0x11111111u;
#pragma unroll
              for (int m = 0; m < 16; ++m) {
                const float2 d2 = fma2(make_float2(y[4 * m], y[4 * m + 2]), make_float2(cxy.x, cxy.y),
                                       fma2(make_float2(y[4 * m + 1], y[4 * m + 3]), make_float2(cxy.z, cxy.w), cz));
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  const int i = 2 * m + h;
                  const float d = h ? d2.y : d2.x;
                  if (d < bd[i]) {
                    bd[i] = d;
                    const uint32_t msk = 15u << (4 * (i % 8));
                    gw[i / 8] = (gw[i / 8] & ~msk) | (jr & msk);
                  }
                }
              }
            }
            float dot = 0.f;  // <u, c>
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int k = (int)((gw[i / 8] >> (4 * (i % 8))) & 15u);
              const float2 c = reinterpret_cast<const float2*>(s_cb)[k];
              dot = fmaf(y[2 * i], c.x, fmaf(y[2 * i + 1], c.y, dot));
            }
            const float yc = dot * sigma;  // <y, c>
            const __half sh = __float2half_rn(ss > 0.f && yc > 0.f ? ss / yc : 0.f);
            sf = __half2float(sh);
            if (valid) {
              reinterpret_cast<__half*>(is_v ? pp.vparams : pp.kparams)[rowi * 2 + g] = sh;
              *reinterpret_cast<uint4*>(codes + g * 4) = make_uint4(gw[0], gw[1], gw[2], gw[3]);
            }
          } else {
            const uint32_t sw = lds32(chunk(PCH));
            sf = __half2float(__ushort_as_half((unsigned short)(g ? sw >> 16 : sw & 0xffffu)));
#pragma unroll
            for (int i = 0; i < 4; ++i) gw[i] = cc[i];
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int k = (int)((gw[i / 8] >> (4 * (i % 8))) & 15u);
            const float2 c = reinterpret_cast<const float2*>(s_cb)[k];
            y[2 * i] = sf * c.x;
            y[2 * i + 1] = sf * c.y;
          }
          walsh64_thread(y);
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            float p[32];
            tmem_ld32(acc + g * 64 + q * 32, p);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
              uint32_t w[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int e = q * 32 + ch * 8 + 2 * i;
                w[i] = pack_bf16x2(p[ch * 8 + 2 * i] + y[e], p[ch * 8 + 2 * i + 1] + y[e + 1]);
              }
              const int e = g * 64 + q * 32 + ch * 8;  // element of the row
              *reinterpret_cast<uint4*>(recon(b) + (e >> 6) * 16384 + sw128_off(row, (e & 63) >> 3)) =
                  make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        } else {
        float pk[KEEP ? 32 : 1];  // prediction of a one-pass group, kept for the second pass
        float sf, zf;
        if (ENC) {
          // group min / max of the residual over its NP passes of 32 columns
          float mn0 = INFINITY, mx0 = -INFINITY, mn1 = INFINITY, mx1 = -INFINITY;
#pragma unroll
          for (int q = 0; q < NP; ++q) {
            float p[32];
            tmem_ld32(acc + g * G + q * 32, p);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
              float x[8];
              unpack_bf16x8(xc[q * 4 + ch], x, 0);
#pragma unroll
              for (int i = 0; i < 8; i += 2) {
                const float2 r = sub2(make_float2(x[i], x[i + 1]), make_float2(p[ch * 8 + i], p[ch * 8 + i + 1]));
                mn0 = fminf(mn0, r.x);
                mx0 = fmaxf(mx0, r.x);
                mn1 = fminf(mn1, r.y);
                mx1 = fmaxf(mx1, r.y);
              }
            }
            if (KEEP) {
#pragma unroll
              for (int i = 0; i < 32; ++i) pk[i] = p[i];
            }
          }
          const float mn = fminf(mn0, mn1), mx = fmaxf(mx0, mx1);
          const __half sh = __float2half_rn((mx - mn) / (float)LEVELS);
          const __half zh = __float2half_rn(mn);
          sf = __half2float(sh);
          zf = __half2float(zh);
          if (valid) params[g] = __halves2half2(sh, zh);
          // x of group g is in registers (the pass above consumed it): its half
          // of the slot takes group g + 2
          if (STX && g + 2 < NG) stage_x(g + 2);
        } else {
          const float2 f = __half22float2(pc);
          sf = f.x;
          zf = f.y;
        }
        const float inv = sf > 0.f ? 1.f / sf : 0.f;
        uint32_t gw[GW];  // packed codes of the group (encode)
#pragma unroll
        for (int q = 0; q < NP; ++q) {
          float p[32];
          if (KEEP) {
#pragma unroll
            for (int i = 0; i < 32; ++i) p[i] = pk[i];
          } else {
            tmem_ld32(acc + g * G + q * 32, p);
          }
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {  // 8 elements: codes, packing, reconstruction
            const int eg = q * 32 + ch * 8;  // element within the group
            float r[8];  // reconstruction
            if (ENC) {
              float x[8];
              unpack_bf16x8(xc[eg / 8], x, 0);
              const uint32_t v = quant8<BITS>(x, &p[ch * 8], sf, zf, inv, r);
              if (BITS == 2) {
                if ((eg % 16) == 0)
                  gw[eg / 16] = v;
                else
                  gw[eg / 16] |= v << 16;
              } else {
                gw[eg / 8] = v;
              }
            } else {
              dequant8<BITS>(BITS == 2 ? cc[eg / 16] : cc[eg / 8], eg, sf, zf, &p[ch * 8], r);
            }
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) w[i] = pack_bf16x2(r[2 * i], r[2 * i + 1]);
            const int e = g * G + eg;  // element of the row
            *reinterpret_cast<uint4*>(recon(b) + (e >> 6) * 16384 + sw128_off(row, (e & 63) >> 3)) =
                make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
        if (ENC && valid) {
#pragma unroll
          for (int i = 0; i < GW; i += 2) *reinterpret_cast<uint2*>(codes + g * GW + i) = make_uint2(gw[i], gw[i + 1]);
        }
        }  // RTN
        if (!STX && !STE && g + 1 < NG) {
#pragma unroll
          for (int i = 0; i < (ENC ? XQ : 1); ++i) xc[i] = xn[i];
#pragma unroll
          for (int i = 0; i < (ENC ? 1 : GW); ++i) cc[i] = cn[i];
          pc = pn;
        }
      }
      tc_fence_before();
      if (!PAIR) mbar_arrive(&acc_empty[b]);
      fence_async_smem();
      gsync();
      if (elected) {
        if (PAIR) mbar_arrive_remote(lead_bar(&acc_empty[b]));
        if ((!is_v || a.store_v) && t0 < a.T) {  // (a pair's odd CTA may be past the last token)
          if (is_v) {
            tma_store(&LM(l)->vo, h * 128, t0, recon(b));
            tma_store(&LM(l)->vo, h * 128 + 64, t0, recon(b) + 16384);
          } else {  // K^_l is read back by this tile's V heads: kept in L2 until then
            const uint64_t keep = policy_evict_last();
            tma_store_hint(&LM(l)->ko, h * 128, t0, recon(b), keep);
            tma_store_hint(&LM(l)->ko, h * 128 + 64, t0, recon(b) + 16384, keep);
          }
        }
        bulk_commit();
        if (!is_v && RC) {
          if (PAIR)
            mbar_arrive_remote(lead_bar(&rec_full[b]));
          else
            mbar_arrive(&rec_full[b]);
        }
      }
    };

    // After an abort every wait returns at once; the loops still run to the end
    // so that all threads of a group meet at every named barrier.
    for (int it = 0;; ++it) {
      const int cur = it < my_tiles ? item_of(it) : -1;
      if (cur < 0) break;
      const int t0 = tile_t0(cur), l = layer_of(cur);
      // the item's K latent (loaded at its start, or during the previous item's V heads)
      if (RC && grp == 0) {
        wait(zk_full, zk_use++ & 1, abort_flag, a.err, 0x900u);
        tc_fence_after();
        convert_latent(zk_col(it));
      }
      // K heads u < H, then V heads; head u of the tile goes to group (it*2H + u) mod 2
      const int nu = 2 * H;
#pragma unroll 1
      for (int u = 0; u < nu; ++u) {
        if (u == H) {  // between the K and the V heads
          if (elected) {
            bulk_wait_all();
            fence_async_global();
            mbar_arrive(khat_stored);
          }
          if (RC && grp == 0) {
            wait(zv_full, zv_use++ & 1, abort_flag, a.err, 0x901u);
            tc_fence_after();
            convert_latent(zv_col(it));
          }
        }
        if (((it * HH + u) & 1) == grp) head(u < H ? u : u - H, u >= H, t0, l);
      }
      if constexpr (MULTI) {
        // this group's reconstruction of the item is in memory: release it to the
        // next layer's tile (the async-proxy stores complete, then a proxy fence
        // before the generic release)
        if (elected) {
          bulk_wait_all();
          fence_async_global();
          asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(flag_of(l, cur)) : "memory");
        }
      }
    }
    if (elected) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  // a pair: the leader's last MMAs (into this CTA's TMEM, from its shared memory)
  // and every remote arrival are complete before either CTA frees or leaves
  if (PAIR) cluster_arrive_wait();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem, 512);
    else
      tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D byte tensor [rows][cols] for L2 prefetches of box_rows x box_cols bytes.
bool map2d_bytes(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                 uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same byte tensor in boxes of box_rows x 64 bytes with the 64-byte
// swizzle: in shared memory, 16-byte chunk c of box row r sits at chunk
// c ^ ((r >> 1) & 3) of the row (for a box that starts on a 512-byte boundary).
bool map2d_bytes_sw64(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 tensor [rows][cols] (row-major) read or written in boxes of
// box_rows x 64 columns with the 128-byte swizzle.
bool map2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [frames][rows][cols] view of a row-major [frames * rows][cols] tensor,
// boxes of box_rows x 64 columns of one frame with the 128-byte swizzle: a box
// that reaches past a frame's last row is clipped there.
bool map3d_frames(CUtensorMap* m, const void* base, uint64_t frames, uint64_t rows, uint64_t cols,
                  uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {cols, rows, frames};
  cuuint64_t strides[2] = {cols * 2, rows * cols * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Streaming multiprocessors of the current device (0 on error).
static int sm_count() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev] = n;
  }
  return cached[dev];
}

// Decode runs as CTA pairs (each SM streams half of every weight box; measured
// 7% faster).  A one-layer encode runs as single CTAs, whose heavier epilogue
// gains nothing from the pair's lock step; a multi-layer encode, whose items
// fill each other's wave tails, runs as pairs (29 layers: 6.1 -> 5.8 ms).
template <int MODE, bool MULTI>
constexpr bool kPaired = MODE == kDecode || MULTI;

// Multi-layer launches wait across CTAs (a tile of layer l on the same tile of
// layer l-1), so their grid is at most what is resident at once.
template <int MODE, int G, int RC, int BITS, bool EDEN = false, bool MULTI = false>
static cudaError_t launch(const Maps& m, const Args& a, cudaStream_t st) {
  const int sms = sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const int64_t nl = MULTI ? a.n_layers : 1;
  if constexpr (!kPaired<MODE, MULTI>) {
    auto k = xlayer_tc_kernel<MODE, G, RC, BITS, false, EDEN, MULTI>;
    const int smem = Layout<RC, false>::kBytes + 1024;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 1;
    if (MULTI && ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kThreads, smem)) != cudaSuccess))
      return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    // persistent: at most one CTA per SM, each looping over token tiles (of each layer)
    const int64_t nitems = (a.T + 127) / 128 * nl;
    const int grid = (int)(nitems < sms ? nitems : sms);
    k<<<grid, kThreads, smem, st>>>(m, a);
    count_launches(1);
    return cudaGetLastError();
  } else {
    // pairs: clusters of two CTAs, each pair looping over 256-token tiles (of each layer)
    auto k = xlayer_tc_kernel<MODE, G, RC, BITS, true, EDEN, MULTI>;
    const int smem = Layout<RC, true, kSlim<MODE, G, BITS, true, EDEN>>::kBytes + 1024;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int max_pairs = sms / 2;
    if (MULTI) {
      cfg.gridDim = dim3((unsigned)(2 * max_pairs));
      int active = 0;
      if ((e = cudaOccupancyMaxActiveClusters(&active, k, &cfg)) != cudaSuccess) return e;
      if (active < 1) return cudaErrorInvalidConfiguration;
      max_pairs = active < max_pairs ? active : max_pairs;
    }
    const int64_t npairs = (a.T + 255) / 256 * nl;
    const int grid = 2 * (int)(npairs < max_pairs ? npairs : max_pairs);
    cfg.gridDim = dim3((unsigned)grid);
    e = cudaLaunchKernelEx(&cfg, k, m, a);
    count_launches(1);
    return e != cudaSuccess ? e : cudaGetLastError();
  }
}

template <int MODE, int BITS, bool MULTI = false>
static cudaError_t dispatch_bits(int group, int rc, const Maps& m, const Args& a, cudaStream_t st) {
  if (group == 32) {
    if (rc == 0) return launch<MODE, 32, 0, BITS, false, MULTI>(m, a, st);
    if (rc == 1) return launch<MODE, 32, 1, BITS, false, MULTI>(m, a, st);
    return launch<MODE, 32, 2, BITS, false, MULTI>(m, a, st);
  }
  if (rc == 0) return launch<MODE, 64, 0, BITS, false, MULTI>(m, a, st);
  if (rc == 1) return launch<MODE, 64, 1, BITS, false, MULTI>(m, a, st);
  return launch<MODE, 64, 2, BITS, false, MULTI>(m, a, st);
}

// H64 / EDEN-2 residuals: 64-value groups, 4 bits a pair
template <int MODE>
static cudaError_t dispatch_eden(int rc, const Maps& m, const Args& a, cudaStream_t st) {
  if (rc == 0) return launch<MODE, 64, 0, 2, true>(m, a, st);
  if (rc == 1) return launch<MODE, 64, 1, 2, true>(m, a, st);
  return launch<MODE, 64, 2, 2, true>(m, a, st);
}

template <int MODE, bool MULTI = false>
static cudaError_t dispatch(int group, int rc, const Maps& m, const Args& a, cudaStream_t st) {
  return a.bits == 2 ? dispatch_bits<MODE, 2, MULTI>(group, rc, m, a, st)
                     : dispatch_bits<MODE, 4, MULTI>(group, rc, m, a, st);
}

// The weight maps: a pair's CTA loads half of each box's rows.
static bool weight_maps(Maps& m, const kvc_layer_desc* d, const kvc_predictor* p, bool pair) {
  const uint64_t H = d->n_heads, C = H * 128, r = p->rank;
  const uint32_t hb = pair ? 64 : 128, hr = pair ? (uint32_t)r / 2 : (uint32_t)r;
  bool ok = map2d(&m.bk, p->k_block, H * 128, 128, hb) && map2d(&m.bv, p->v_block, H * 128, 256, hb);
  if (ok && r > 0)
    ok = map2d(&m.wk, p->k_w, r, C, hr) && map2d(&m.wv, p->v_w, r, 2 * C, hr) && map2d(&m.uk, p->k_u, C, r, hb) &&
         map2d(&m.uv, p->v_u, C, r, hb);
  return ok;
}

}  // namespace tc

bool tc_codec_supported(const kvc_layer_desc* d, const kvc_predictor* p) {
  if (p->kind != KVC_PRED_XLAYER_DPLR) return false;
  if (d->residual_codec != KVC_RESIDUAL_RTN &&
      (d->residual_codec != KVC_RESIDUAL_H64_EDEN2 || d->bits != 2 || d->group != 64 || !p->residual_codebook))
    return false;
  if (d->dtype != KVC_BF16 || d->head_dim != 128 || d->param_dtype != KVC_F16) return false;
  if (d->bits != 2 && d->bits != 4) return false;
  if (d->group != 32 && d->group != 64) return false;
  if (p->rank != 0 && p->rank != 64 && p->rank != 128) return false;
  if (d->n_tokens < 1 || (int64_t)d->n_heads * 128 * 2 > (1 << 20)) return false;
  return tc::encode_fn() != nullptr;
}

size_t tc_workspace(int op, const kvc_layer_desc* d, const kvc_predictor* p, int64_t n_q) {
  if (op != KVC_OP_ATTEND) return 0;
  if (tc_mixed_supported(d, p)) return tc_mixed_workspace(d, n_q);
  return 0;
}

namespace tc {
// the tensor maps of one layer's call
// pair: the maps of a CTA-pair launch (half weight boxes), which decode and
// multi-layer calls use
static bool layer_maps(Maps& m, const kvc_layer_desc* d, const kvc_predictor* p, bool pair, bool enc,
                       const void* K, const void* V, const void* Ks, const void* Vs, const kvc_codes* c, void* Kr,
                       void* Vr) {
  const uint64_t T = (uint64_t)d->n_tokens, H = d->n_heads, C = H * 128;
  memset(&m, 0, sizeof(m));
  bool ok = map2d(&m.ks, Ks, T, C, 128) && map2d(&m.vs, Vs, T, C, 128) && map2d(&m.ko, Kr, T, C, 128) &&
            map2d(&m.vo, Vr ? Vr : Kr, T, C, 128) && weight_maps(m, d, p, pair);
  const uint64_t rb = 128 * (uint64_t)d->bits / 8;
  if (ok && enc) ok = map2d(&m.xk, K, T, C, 128) && map2d(&m.xv, V, T, C, 128);
  if (ok && !enc)
    ok = map2d_bytes(&m.ck, c->k_codes, T, H * rb, (uint32_t)rb, 128) &&
         map2d_bytes(&m.cv, c->v_codes, T, H * rb, (uint32_t)rb, 128) &&
         (d->group != 32 || (map2d_bytes(&m.pk, c->k_params, T, H * 16, 16, 128) &&
                             map2d_bytes(&m.pv, c->v_params, T, H * 16, 16, 128)));
  return ok;
}
static Ptrs layer_ptrs(const void* K, const void* V, const kvc_codes* c) {
  return Ptrs{(const __nv_bfloat16*)K, (const __nv_bfloat16*)V, (uint8_t*)c->k_codes, (__half2*)c->k_params,
              (uint8_t*)c->v_codes, (__half2*)c->v_params};
}
}  // namespace tc

cudaError_t tc_codec_layer(const kvc_layer_desc* d, const kvc_predictor* p, bool enc, const void* K, const void* V,
                           const void* Ks, const void* Vs, const kvc_codes* c, void* Kr, void* Vr, void*, size_t,
                           cudaStream_t st) {
  const uint64_t H = d->n_heads, r = p->rank;
  tc::Maps m;
  if (!tc::layer_maps(m, d, p, !enc, enc, K, V, Ks, Vs, c, Kr, Vr)) return cudaErrorInvalidValue;
  unsigned* err = tc_error_word();
  if (!err) return cudaErrorInvalidDevice;
  tc::Args a{err, (int64_t)d->n_tokens, (int)H, d->bits, tc::layer_ptrs(K, V, c), (enc && !Vr) ? 0 : 1,
             nullptr, 0, nullptr, tc::g_inject_stall.exchange(0), (const float*)p->residual_codebook};
  const int rc = (int)(r / 64);
  if (d->residual_codec == KVC_RESIDUAL_H64_EDEN2)
    return enc ? tc::dispatch_eden<tc::kEncode>(rc, m, a, st) : tc::dispatch_eden<tc::kDecode>(rc, m, a, st);
  return enc ? tc::dispatch<tc::kEncode>(d->group, rc, m, a, st)
             : tc::dispatch<tc::kDecode>(d->group, rc, m, a, st);
}



// ---------------------------------------------------------------- multi-layer calls

static size_t align256u(size_t x) { return (x + 255) & ~size_t(255); }

bool tc_codec_layers_supported(const kvc_layer_desc* d, const kvc_predictor* preds, int n) {
  if (n < 1 || d->residual_codec != KVC_RESIDUAL_RTN) return false;
  for (int i = 0; i < n; ++i)
    if (!tc_codec_supported(d, &preds[i]) || preds[i].rank != preds[0].rank) return false;
  return true;
}

size_t tc_codec_layers_workspace(const kvc_layer_desc* d, int n) {
  const size_t ntiles = ((size_t)d->n_tokens + 127) / 128;
  // the layer table, then a counter per (layer, 128-token tile)
  return align256u((size_t)n * sizeof(tc::LayerDev)) + align256u((size_t)n * ntiles * sizeof(unsigned));
}

cudaError_t tc_codec_layers(const kvc_layer_desc* d, const kvc_predictor* preds, int n, bool enc,
                            const void* const* K, const void* const* V, const void* Ks0, const void* Vs0,
                            const kvc_codes* c, void* const* Kr, void* const* Vr, void* ws, size_t ws_bytes,
                            cudaStream_t st) {
  if (ws_bytes < tc_codec_layers_workspace(d, n) || !ws) return cudaErrorInvalidValue;
  // layer i of the call reads the reconstruction of layer i-1 (Ks0 / Vs0 for i = 0)
  std::vector<tc::LayerDev> host((size_t)n);
  for (int i = 0; i < n; ++i) {
    const void* ks = i ? Kr[i - 1] : Ks0;
    const void* vs = i ? Vr[i - 1] : Vs0;
    const void* k = enc ? K[i] : nullptr;
    const void* v = enc ? V[i] : nullptr;
    if (!tc::layer_maps(host[i].maps, d, &preds[i], true, enc, k, v, ks, vs, &c[i], Kr[i], Vr[i]))
      return cudaErrorInvalidValue;
    host[i].p = tc::layer_ptrs(k, v, &c[i]);
  }
  char* w = static_cast<char*>(ws);
  tc::LayerDev* dev = reinterpret_cast<tc::LayerDev*>(w);
  unsigned* flags = reinterpret_cast<unsigned*>(w + align256u((size_t)n * sizeof(tc::LayerDev)));
  const size_t ntiles = ((size_t)d->n_tokens + 127) / 128;
  cudaError_t e = cudaMemcpyAsync(dev, host.data(), (size_t)n * sizeof(tc::LayerDev), cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(flags, 0, (size_t)n * ntiles * sizeof(unsigned), st)) != cudaSuccess) return e;
  unsigned* err = tc_error_word();
  if (!err) return cudaErrorInvalidDevice;
  tc::Maps none;
  memset(&none, 0, sizeof(none));
  tc::Args a{err, (int64_t)d->n_tokens, (int)d->n_heads, d->bits, tc::Ptrs{}, 1, dev, n, flags,
             tc::g_inject_stall.exchange(0), nullptr};
  const int rc = (int)(preds[0].rank / 64);
  return enc ? tc::dispatch<tc::kEncode, true>(d->group, rc, none, a, st)
             : tc::dispatch<tc::kDecode, true>(d->group, rc, none, a, st);
}

}  // namespace kvc

extern "C" void kvc_testing_inject_stall(int what) { kvc::tc::g_inject_stall.store(what == 1 ? 1 : 0); }
