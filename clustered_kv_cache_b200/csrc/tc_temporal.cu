// Temporal predictive codec on tcgen05 ("TempoKV: Predictive KV Cache
// Quantization for Autoregressive Video Generation", Fig. 2(b): K of frame f is
// predicted from the reconstructed K of frames f-1 and f-2 at the same spatial
// position, V of frame f from the aligned reconstructed K of frame f and V of
// frame f-1; only the low-bit residual is stored).
//
// One CTA per (128-position tile, head) walks every frame of the call in order.
// The head's two 128x256 maps stay in shared memory; the reconstructed state
// (K of frames f and f-1, V of frame f-1) lives in tensor memory as bf16 pairs
// and is the A operand of the prediction MMAs: each new reconstruction
// overwrites the slot that its own prediction was the last to read.  Per frame
// the MMA of V(f) and of K(f+1) are issued together once K^_f exists, and two
// epilogue groups quantize V(f) and K(f+1) side by side.  A three-slot ring of
// shared-memory tiles moved by TMA carries x to the encode epilogues about a
// frame ahead, the reconstruction out of the decode epilogues, and the supplied
// history of a continuation call into tensor memory.
//
// Warp roles: 0 TMA (maps, history, x), 1 MMA + TMEM, 2-9 K epilogue, 10-17 V
// epilogue.  An epilogue group is eight warps: two per TMEM lane quarter, one
// for each 64-column half of the row, so that the per-frame chain (prediction
// MMA, then the epilogue that writes the state the next MMA reads) runs each
// row's quantization on two warps.
#include <cuda.h>
#include <string.h>

#include "tc.h"
#include "tc_ptx.cuh"

namespace kvc {
namespace tc {

bool map2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);
bool map3d_frames(CUtensorMap* m, const void* base, uint64_t frames, uint64_t rows, uint64_t cols,
                  uint32_t box_rows);

namespace temporal {

constexpr int kThreads = 576;
constexpr int kGroup = 256;  // threads of an epilogue group
constexpr int kAK = 0;                   // AK_h as 4 sub-tiles [128 out][64 in]
constexpr int kAV = kAK + 65536;         // AV_h
constexpr int kX = kAV + 65536;          // three staged [128][128] bf16 tiles: x of K(f), V(f) in turn
                                         // (encode); the supplied history at the start (continuation)
constexpr int kBar = kX + 3 * 32768;
constexpr int kSmem = kBar + 1024 + 1024;

struct Maps {
  CUtensorMap ak, av;      // [H*128][256]
  CUtensorMap ksrc, vsrc;  // history: [2F][C], [F][C] (continuation only)
  CUtensorMap xk, xv;      // clean K, V [T][C] (encode)
  // reconstructions written by decode: whole frames as [frames][F][C], the
  // partial last frame as [rows][C]
  CUtensorMap kr3, vr3, krt, vrt;
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

__device__ __forceinline__ void tma_store3(const CUtensorMap* m, int x, int y, int z, const void* src) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(x), "r"(y), "r"(z), "r"(smem_u32(src))
               : "memory");
}

// 16 consecutive 32-bit TMEM columns of this thread's lane (no wait)
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&w)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]), "r"(w[8]), "r"(w[9]),
      "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15])
      : "memory");
}

// 16 consecutive fp32 TMEM columns of this thread's lane
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// 16 or 32 consecutive fp32 TMEM columns of this thread's lane
template <int W>
__device__ __forceinline__ void tmem_ldw(uint32_t taddr, float (&v)[W]) {
  static_assert(W == 16 || W == 32, "16 or 32 columns");
  if constexpr (W == 16)
    tmem_ld16(taddr, v);
  else
    tmem_ld32(taddr, v);
}
// 8 consecutive 32-bit TMEM columns of this thread's lane (no wait)
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&w)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(w[0]),
               "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

template <bool ENC, int G>
__global__ void __launch_bounds__(kThreads, 1) temporal_kernel(const __grid_constant__ Maps maps, const Args a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBar);
  uint64_t* w_full = bars;           // maps (+ history) landed
  uint64_t* kacc_full = bars + 1;    // K prediction of a frame in TMEM
  uint64_t* vacc_full = bars + 2;    // V prediction of a frame in TMEM
  uint64_t* kready = bars + 3;       // K^ of a frame in its TMEM slot (K epilogue, 256 arrivals)
  uint64_t* vready = bars + 4;       // V^ of a frame in its TMEM slot (V epilogue)
  uint64_t* mma_done = bars + 5;
  uint64_t* h_ready = bars + 6;      // initial history in TMEM (both epilogue groups, 512 arrivals)
  // Ring item i (x of K(f) for i = 2f, of V(f) for i = 2f + 1) lands in slot
  // i % 3 and completes on x_full[slot][i & 1]: the slots alternate between K
  // and V items, and a barrier that only one group waits on shows that group
  // each of its phases in order (a parity wait cannot tell a phase from the one
  // two later).  The j-th item of a group in a slot is item i with j = i / 6.
  uint64_t* x_full = bars + 7;       // [3][2] staged tile landed, per slot and group
  uint64_t* x_free = bars + 13;      // [3] staged tile read (256 arrivals; only the producer waits)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int s0 = blockIdx.x * 128;
  const int H = a.H;
  const int64_t C = (int64_t)H * 128;
  const int64_t F = a.F;
  const int nf = (int)((a.T + F - 1) / F);
  const bool cont = a.anchor_bits == 0;
  auto xs = [&](int i) { return smem + kX + (i % 3) * 32768; };  // staged tile of ring item i

  if (threadIdx.x == 0) {
    mbar_init(w_full, 1);
    mbar_init(kacc_full, 1);
    mbar_init(vacc_full, 1);
    mbar_init(kready, kGroup);
    mbar_init(vready, kGroup);
    mbar_init(mma_done, 1);
    mbar_init(h_ready, 2 * kGroup);
    for (int i = 0; i < 3; ++i) {
      mbar_init(&x_full[2 * i], 1);
      mbar_init(&x_full[2 * i + 1], 1);
      mbar_init(&x_free[i], kGroup);
    }
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
  // TMEM columns: K accumulator [0,128), V accumulator [128,256), then the
  // reconstructed state as bf16 pairs (the A operands of the predictions): K^ of
  // frame f in [256 + 64 (f & 1), +64), V^ of the previous frame in [384, 448)
  const uint32_t KACC = tmem, VACC = tmem + 128;
  auto KH = [&](int f) { return tmem + 256 + (uint32_t)(f & 1) * 64; };
  const uint32_t VH = tmem + 384;

  if (warp == 0) {
    if (lane == 0) {
      // ================================================================ TMA: maps, history, staged x
      const uint64_t pol = policy_evict_last();
      const uint64_t pol_x = policy_evict_first();
      mbar_arrive_expect_tx(w_full, 131072u + (cont ? 98304u : 0u));
      for (int c = 0; c < 4; ++c) {
        tma_load(smem + kAK + c * 16384, &maps.ak, c * 64, h * 128, w_full, pol);
        tma_load(smem + kAV + c * 16384, &maps.av, c * 64, h * 128, w_full, pol);
      }
      if (cont) {  // K^ of frames -1 (slot 0) and -2 (slot 1), V^ of frame -1 (slot 2)
        for (int c = 0; c < 2; ++c) {
          tma_load(xs(0) + c * 16384, &maps.ksrc, h * 128 + c * 64, (int)(F + s0), w_full, pol_x);
          tma_load(xs(1) + c * 16384, &maps.ksrc, h * 128 + c * 64, s0, w_full, pol_x);
          tma_load(xs(2) + c * 16384, &maps.vsrc, h * 128 + c * 64, s0, w_full, pol_x);
        }
      }
      if (ENC) {
        // ring items: x of K(f) is item 2f, x of V(f) item 2f + 1, in slot item % 3
        bool ok = !cont || wait(h_ready, 0, abort_flag, a.err, 0x2120u);  // the history left the slots
        int last = -1;
        for (int i = 0; i < 2 * nf && ok; ++i) {
          const int use = i / 3;
          if (use >= 1 && !wait(&x_free[i % 3], (use - 1) & 1, abort_flag, a.err, 0x2121u)) {
            ok = false;
            break;
          }
          const CUtensorMap* m = (i & 1) ? &maps.xv : &maps.xk;
          const int row = (int)((i >> 1) * F + s0);
          uint64_t* xf = &x_full[2 * (i % 3) + (i & 1)];
          mbar_arrive_expect_tx(xf, 32768u);
          tma_load(xs(i), m, h * 128, row, xf, pol_x);
          tma_load(xs(i) + 16384, m, h * 128 + 64, row, xf, pol_x);
          last = i;
        }
        if (*abort_flag) {  // the loads this thread issued land before the CTA can leave
          for (int i = last - 2; i <= last; ++i) {
            if (i < 0) continue;
            const long long w0 = clock64();
            while (!mbar_test(&x_full[2 * (i % 3) + (i & 1)], (i / 6) & 1) && clock64() - w0 < kWaitBudget) {
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ================================================================ MMA
      bool ok = wait(w_full, 0, abort_flag, a.err, 0x2100u) && wait(h_ready, 0, abort_flag, a.err, 0x2101u);
      tc_fence_after();
      const uint32_t id = idesc_bf16(128, 128);
      // D = [A0 | A1] W^T over 256 inputs, A0 / A1 in TMEM (64 columns of bf16 pairs
      // each), W as 4 sub-tiles of 64 inputs
      auto mma256 = [&](uint32_t d, uint32_t A0, uint32_t A1, const uint8_t* W) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t ab = (c < 2 ? A0 : A1) + (uint32_t)(c & 1) * 32;
          const uint64_t bd = desc_sw128(smem_u32(W + c * 16384));
#pragma unroll
          for (int k = 0; k < 4; ++k) umma_ts_if(1u, d, ab + k * 8, bd + 2 * k, id, (c == 0 && k == 0) ? 0u : 1u);
        }
      };
      int kr = 0, vr = 0;  // completions of kready / vready seen
      // frame f's K prediction: [K^_{f-1} | K^_{f-2}] AK^T; K^_{f-2} sits in the slot of frame f
      auto issue_k = [&](int f) {
        mma256(KACC, KH(f - 1), KH(f), smem + kAK);
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
            mma256(VACC, KH(f), VH, smem + kAV);
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
    // ================================================================ epilogues: warps 2-9 K, 10-17 V
    const bool isv = warp >= 10;
    const int q = warp & 3;                  // TMEM lane quarter
    const int hc = ((warp - 2) >> 2) & 1;    // 64-column half of the row
    const int row = q * 32 + lane;
    const int64_t s = s0 + row;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t acc_addr = lane_off + (isv ? VACC : KACC);
    uint64_t* acc_full = isv ? vacc_full : kacc_full;
    int acc_use = 0;
    const int64_t F0 = cont ? 0 : (F < a.T ? F : a.T);
    const int arb = 128 * a.anchor_bits / 8;
    // this thread's half of row r of a staged [128][128] bf16 tile (two
    // 128-byte-swizzled 64-column sub-tiles: the half is sub-tile hc) as 32 words
    auto read_half = [&](const uint8_t* tile, uint4 (&w)[8]) {
#pragma unroll
      for (int c = 0; c < 8; ++c) w[c] = *reinterpret_cast<const uint4*>(tile + hc * 16384 + sw128_off(row, c));
    };
    auto half_to_tmem = [&](const uint4 (&w)[8], uint32_t col) {
      const uint32_t* u = reinterpret_cast<const uint32_t*>(w);
      uint32_t v[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = u[i];
      tmem_st32u(lane_off + col + hc * 32, v);
    };
    // the state before frame 0: the supplied history, or (no history) a zero
    // K^ of frame -1 as the lag-2 input of frame 1
    wait(w_full, 0, abort_flag, a.err, 0x2200u);
    if (cont) {
      uint4 w[8];
      if (!isv) {
        read_half(xs(0), w);
        half_to_tmem(w, KH(-1) - tmem);
        read_half(xs(1), w);
        half_to_tmem(w, KH(-2) - tmem);
      } else {
        read_half(xs(2), w);
        half_to_tmem(w, VH - tmem);
      }
    } else if (!isv) {
      uint4 w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = make_uint4(0, 0, 0, 0);
      half_to_tmem(w, KH(-1) - tmem);
    }
    tc_fence_before();
    fence_async_smem();  // (continuation) the history slots are read; TMA loads x into them next
    mbar_arrive(h_ready);
    // Decode writes the reconstruction through a staged tile (K: slot 0, V: slot
    // 2, idle in decode once the history is in TMEM) and TMA stores of one frame's
    // rows; encode (whose ring holds x) stores it row by row when asked for.
    __nv_bfloat16* rec = isv ? a.vrec : a.krec;
    const bool stage = !ENC && rec != nullptr;
    uint8_t* stile = xs(isv ? 2 : 0);
    const bool elected = warp == (isv ? 10 : 2) && lane == 0;
    auto gsync = [&] {
      if (isv)
        asm volatile("bar.sync 2, 256;" ::: "memory");
      else
        asm volatile("bar.sync 1, 256;" ::: "memory");
    };
    const int64_t nff = a.T / F;  // whole frames
    constexpr int NG = 128 / G;
    constexpr int NGH = NG / 2;  // groups of the half row
    // accumulator columns per TMEM round trip: encode (x not in registers) 32,
    // decode 16 (the register budget of 576 threads is 96 a thread)
    constexpr int PW = ENC ? 32 : 16;
    constexpr int NPW = G / PW;
    for (int f = 0; f < nf; ++f) {
      const int64_t n_f = (a.T - f * F) < F ? (a.T - f * F) : F;
      const bool valid = s < n_f;
      const bool anchor = f == 0 && !cont;
      const int bits = anchor ? a.anchor_bits : a.bits;
      const int levels = (1 << bits) - 1;
      const int64_t t = f * F + s;
      const int64_t rowi = t * H + h;
      const int row_bytes = 128 * bits / 8;
      const int half_bytes = row_bytes / 2;
      const int64_t cofs = rowi < F0 * H ? rowi * arb : F0 * H * arb + (rowi - F0 * H) * row_bytes;
      uint8_t* codes = (isv ? a.vcodes : a.kcodes) + cofs + hc * half_bytes;
      __half2* params = (isv ? a.vparams : a.kparams) + rowi * NG + hc * NGH;
      uint4 cin[2];
      __half2 pin[NGH];
      // encode: x of this half row is read from its staged tile in both passes
      // (x in registers would cost 32 of the 96; the tile is released at the end)
      const int xi = 2 * f + (isv ? 1 : 0);  // ring item of x
      auto xq = [&](int c8) {  // 16-byte chunk c8 (elements 8 c8 .. 8 c8 + 7) of the half row
        return *reinterpret_cast<const uint4*>(xs(xi) + hc * 16384 + sw128_off(row, c8));
      };
      if (ENC) {
        wait(&x_full[2 * (xi % 3) + (xi & 1)], (xi / 6) & 1, abort_flag, a.err, 0x2220u + isv);
      } else {
#pragma unroll
        for (int i = 0; i < 2; ++i)
          cin[i] = (valid && i * 16 < half_bytes) ? __ldcs(reinterpret_cast<const uint4*>(codes) + i)
                                                  : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int g = 0; g < NGH; ++g) pin[g] = valid ? params[g] : __floats2half2_rn(0.f, 0.f);
      }
      // V(f) reads K^_f: the V epilogue of frame f starts after the K epilogue of f
      if (!anchor) {
        wait(acc_full, acc_use & 1, abort_flag, a.err, 0x2210u + isv);
        acc_use++;
        tc_fence_after();
      }
      // the new state goes to the slot its own prediction was the last to read
      const uint32_t state = lane_off + (isv ? VH : KH(f));
      uint32_t cw[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      const uint32_t* cwin = reinterpret_cast<const uint32_t*>(cin);
      if (stage) {  // the staged tile's previous store has read it
        if (elected) bulk_wait_read0();
        gsync();
      }
#pragma unroll
      for (int gh = 0; gh < NGH; ++gh) {
        const int g = hc * NGH + gh;  // group of the row
        float sf, zf;
        if (ENC) {
          float mn = INFINITY, mx = -INFINITY;
#pragma unroll
          for (int pc = 0; pc < NPW; ++pc) {
            float p[PW];
            if (anchor) {
#pragma unroll
              for (int i = 0; i < PW; ++i) p[i] = 0.f;
            } else {
              tmem_ldw(acc_addr + g * G + pc * PW, p);
            }
#pragma unroll
            for (int ch = 0; ch < PW / 8; ++ch) {
              float x[8];
              unpack_bf16x8(xq((gh * G + pc * PW) / 8 + ch), x, 0);
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
          if (valid) params[gh] = __halves2half2(sh, zh);
        } else {
          const float2 fz = __half22float2(pin[gh]);
          sf = fz.x;
          zf = fz.y;
        }
        const float inv = sf > 0.f ? 1.f / sf : 0.f;
#pragma unroll
        for (int pc = 0; pc < NPW; ++pc) {
          const int e0 = g * G + pc * PW;   // element of the row
          const int h0 = gh * G + pc * PW;  // element of the half row
          float p[PW];
          if (anchor) {
#pragma unroll
            for (int i = 0; i < PW; ++i) p[i] = 0.f;
          } else {
            tmem_ldw(acc_addr + e0, p);
          }
          uint32_t recw[PW / 2];  // PW reconstructed values as bf16 pairs
#pragma unroll
          for (int ch = 0; ch < PW / 8; ++ch) {
            const int e = h0 + ch * 8;
            float r[8];  // reconstruction
            if (ENC) {
              float x[8];
              unpack_bf16x8(xq(e / 8), x, 0);
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
#pragma unroll
            for (int i = 0; i < 4; ++i) recw[ch * 4 + i] = pack_bf16x2(r[2 * i], r[2 * i + 1]);
          }
          // the slot was last read by this frame's prediction, which is complete (acc_full)
#pragma unroll
          for (int k = 0; k < PW / 16; ++k)
            tmem_st8(state + e0 / 2 + 8 * k, *reinterpret_cast<const uint32_t(*)[8]>(&recw[8 * k]));
          if (stage) {
#pragma unroll
            for (int ch = 0; ch < PW / 8; ++ch) {
              const int e = e0 + ch * 8;
              *reinterpret_cast<uint4*>(stile + (e / 64) * 16384 + sw128_off(row, (e % 64) / 8)) =
                  make_uint4(recw[4 * ch], recw[4 * ch + 1], recw[4 * ch + 2], recw[4 * ch + 3]);
            }
          } else if (rec && valid) {
            uint4* dst = reinterpret_cast<uint4*>(rec + t * C + h * 128 + e0);
#pragma unroll
            for (int ch = 0; ch < PW / 8; ++ch)
              dst[ch] = make_uint4(recw[4 * ch], recw[4 * ch + 1], recw[4 * ch + 2], recw[4 * ch + 3]);
          }
        }
      }
      if (ENC) {
        // x is read: the next TMA load into this slot is an async-proxy write, so
        // this thread's generic reads of the slot are ordered before it
        fence_async_smem();
        mbar_arrive(&x_free[xi % 3]);
      }
      if (ENC && valid) {
        uint4* dst = reinterpret_cast<uint4*>(codes);
#pragma unroll
        for (int i = 0; i < 2; ++i)
          if (i * 16 < half_bytes) dst[i] = make_uint4(cw[4 * i], cw[4 * i + 1], cw[4 * i + 2], cw[4 * i + 3]);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      mbar_arrive(isv ? vready : kready);
      if (stage) {  // rows past the frame's end are clipped by the maps
        fence_async_smem();
        gsync();
        if (elected && s0 < n_f) {
          if (f < nff) {
            const CUtensorMap* m = isv ? &maps.vr3 : &maps.kr3;
            tma_store3(m, h * 128, s0, f, stile);
            tma_store3(m, h * 128 + 64, s0, f, stile + 16384);
          } else {
            const CUtensorMap* m = isv ? &maps.vrt : &maps.krt;
            tma_store(m, h * 128, s0, stile);
            tma_store(m, h * 128 + 64, s0, stile + 16384);
          }
          bulk_commit();
        }
      }
    }
    if (elected) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
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
  if (ok && enc) ok = tc::map2d(&m.xk, K, (uint64_t)d->n_tokens, C, 128) && tc::map2d(&m.xv, V, (uint64_t)d->n_tokens, C, 128);
  if (ok && !enc) {
    const uint64_t T = (uint64_t)d->n_tokens, nff = T / F, tail = T - nff * F;
    auto maps_for = [&](void* r, CUtensorMap* m3, CUtensorMap* mt) {
      if (!r) return true;
      return (nff == 0 || tc::map3d_frames(m3, r, nff, F, C, 128)) &&
             (tail == 0 || tc::map2d(mt, static_cast<char*>(r) + nff * F * C * 2, tail, C, 128));
    };
    ok = maps_for(Kr, &m.kr3, &m.krt) && maps_for(Vr, &m.vr3, &m.vrt);
  }
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
