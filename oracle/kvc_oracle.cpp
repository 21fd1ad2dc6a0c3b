// Plain fp64 CPU oracle of the predict-then-quantize-residual KV-cache codec
// and of attention over the compressed history.
//
// TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the CPU
// legs of bench.py load this library (through oracle/kvc_oracle_c.py).  It
// shares no code, header or table with the CUDA library and includes none of
// its files.
//
// Everything is written as plain loops over float64 values in the order the
// pages describe; every function is single-threaded and keeps no state.  Sums
// run in index order.  Inputs that the GPU path receives in bf16 or fp32
// arrive here as doubles holding exactly those values.
//
// Sources (page title, then the figure / table followed):
//  [CORAL] "CORAL-KV: Compact Cross-Layer Prediction and Residual Coding for
//          Autoregressive Video KV Caches": abstract (per-head block-diagonal
//          maps plus a global low-rank term; the prediction residual is
//          quantized), Fig. 3 (layer l > 0 is predicted from the reconstructed
//          layer l-1: K_l from K_{l-1}, V_l from [K_l, V_{l-1}]), Fig. 5
//          (non-overlapping groups of residual channels, one shared scale per
//          group), Fig. 8 (INT4 layer-zero anchor), Table 9 (scalar INT2
//          residual codec).
//  [TEMPO] "TempoKV: Predictive KV Cache Quantization for Autoregressive Video
//          Generation": abstract and Fig. 2(b) (K predicted from the
//          reconstructed K history, V from the aligned reconstructed K plus the
//          reconstructed V history; only the low-bit residual is stored),
//          Tables 1-3 and 8 (INT2 / INT4 group quantizers, 5.33x / 3.20x),
//          appendix Table 7 (anchor precision).
//  [NANO]  "NanoKV: High-Ratio KV Cache Compression for Autoregressive Video
//          Generation": abstract (shared content in cluster centres; the joint
//          head-channel residual is encoded into low-bit coefficients; the Fast
//          variant attends on the stored coefficients without rebuilding the
//          full-dimensional keys).
//
// Readings where the pages are silent (the same as the numpy oracle's):
//  R1 asymmetric min/max round-to-nearest per group: s = (max - min) /
//     (2^b - 1), z = min, q = clamp(rint((r - z) / s), 0, 2^b - 1), value
//     z + s q.
//  R2 rint rounds half to even; s and z are rounded to the parameter format
//     first and the codes use the rounded values.
//  R3 a group whose stored scale is 0 gets all-zero codes (value z).
//  R4 groups are runs of `group` consecutive channels of one (token, head) row
//     (clustered codec: of the code_dim coefficients of a token).
//  R5 x^ = round_state(pred + (z + s q)) is what later predictions read.
//  R6 the low-rank latent x W^T is kept at full precision.
//  R7 weights are [out][in]: y = x W^T.
//  R8 temporal: frame 0 is the anchor (prediction 0, anchor bits); the lag-2
//     frame of frame 1 is zero; a partial last frame holds the first n
//     positions; a call may continue a sequence from a supplied history.
//  R9 the temporal K map reads [K^_{f-1} | K^_{f-2}] and the V map
//     [K^_f | V^_{f-1}] (2D inputs per head each).
//  R10 clustered codec: a = argmin_j (|c_j|^2 - 2 x.c_j), ties to the lowest
//     j; coef = E (x - c_a); x^ = c_a + W_dec coef^.
//  R11 mixed-dimensional attention: V is clustered and coded like K; the
//     output is sum_j m_j c^V_j + W^V_dec sum_t p_t coef^V_t, m_j the softmax
//     mass of the tokens assigned to centre j.
//  E1-E6 the H64 / EDEN-2 residual codec ("CORAL-KV ...", Fig. 5, Fig. 9,
//     Table 9): see eden2_code_group below.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

// ---------------------------------------------------------------- storage formats
//
// fmt: 0 = float64 (no rounding), 1 = float32, 2 = bfloat16, 3 = float16.

struct Format {
  int p;        // significand bits including the implicit one
  int emin;     // exponent of the smallest normal number
  double fmax;  // largest finite value
};

Format format_of(int fmt) {
  switch (fmt) {
    case 1: return {24, -126, std::ldexp(2.0 - std::ldexp(1.0, -23), 127)};
    case 2: return {8, -126, std::ldexp(2.0 - std::ldexp(1.0, -7), 127)};
    case 3: return {11, -14, 65504.0};
    default: return {53, -1022, 0.0};
  }
}

// Nearest value of the format (ties to even), with gradual underflow and
// overflow to infinity.  x = 1.f 2^E has quantum 2^(max(E, emin) - (p - 1));
// x / quantum is exact in float64 and nearbyint rounds half to even.
double round_to(double x, int fmt) {
  if (fmt == 0 || x == 0.0 || !std::isfinite(x)) return x;
  const Format f = format_of(fmt);
  int e = 0;
  std::frexp(x, &e);
  int E = e - 1;
  if (E < f.emin) E = f.emin;
  const double quantum = std::ldexp(1.0, E - (f.p - 1));
  const double y = std::nearbyint(x / quantum) * quantum;
  if (std::fabs(y) > f.fmax) return std::copysign(INFINITY, x);
  return y;
}

// ---------------------------------------------------------------- the residual quantizer
// [CORAL Fig. 5, Table 9; TEMPO Tables 1-3, 8]; readings R1-R4.

// One group of n residuals -> codes q, stored scale *s and zero *z.
void quantize_group(const double* r, int n, int bits, int pfmt, uint8_t* q, double* s, double* z) {
  const int levels = (1 << bits) - 1;
  double mn = r[0], mx = r[0];
  for (int i = 1; i < n; ++i) {
    if (r[i] < mn) mn = r[i];
    if (r[i] > mx) mx = r[i];
  }
  const double sv = round_to((mx - mn) / levels, pfmt);
  const double zv = round_to(mn, pfmt);
  for (int i = 0; i < n; ++i) {
    if (sv > 0.0) {
      double t = std::nearbyint((r[i] - zv) / sv);
      if (t < 0.0) t = 0.0;
      if (t > levels) t = levels;
      q[i] = (uint8_t)t;
    } else {
      q[i] = 0;  // R3
    }
  }
  *s = sv;
  *z = zv;
}

// Value of one code: z + s q (R1).
inline double dequant(uint8_t q, double s, double z) { return z + s * (double)q; }

// A row of n values coded against its prediction (R5): residual, groups,
// reconstruction rounded to the state format.
void code_row(const double* x, const double* pred, int n, int bits, int group, int pfmt, int sfmt, uint8_t* q,
              double* s, double* z, double* xhat) {
  std::vector<double> r(n);
  for (int i = 0; i < n; ++i) r[i] = x[i] - pred[i];
  for (int g = 0; g < n / group; ++g)
    quantize_group(&r[g * group], group, bits, pfmt, q + g * group, s + g, z + g);
  for (int i = 0; i < n; ++i) xhat[i] = round_to(pred[i] + dequant(q[i], s[i / group], z[i / group]), sfmt);
}

void decode_row(const uint8_t* q, const double* s, const double* z, const double* pred, int n, int group, int sfmt,
                double* xhat) {
  for (int i = 0; i < n; ++i) xhat[i] = round_to(pred[i] + dequant(q[i], s[i / group], z[i / group]), sfmt);
}

// ---------------------------------------------------------------- H64 / EDEN-2 residual codec
// ["CORAL-KV ...", Fig. 5 (H_n transforms each non-overlapping group of n
// residual channels; one shared scale per 64 values), Fig. 9 (16 EDEN-2
// reconstruction points over pairs of H64-transformed residuals), Table 9 (the
// H64 / EDEN-2 residual codec beside scalar INT2).]  Readings:
//  E1 a group is 64 consecutive residual channels of a (token, head) row; it
//     is transformed by the orthonormal Sylvester Walsh-Hadamard matrix,
//     y_i = (1/8) sum_j (-1)^popcount(i & j) r_j.
//  E2 the 32 pairs of a group are (y_2p, y_2p+1).
//  E3 the 16 two-dimensional points are an input (the pages picture but do not
//     print them).
//  E4 the pairs are normalised by sigma = sqrt(mean_i y_i^2) and each takes the
//     index of its nearest point (ties to the lowest index); the one stored
//     scale is EDEN's unbiased one, S = |y|^2 / <y, c>, rounded to the
//     parameter format (S = 0 when y = 0 or <y, c> <= 0).
//  E5 index of pair p at bits [4p, 4p + 4) of the row, least significant first
//     (4 bits per pair: the 2 bits per value of INT2).
//  E6 the decoded residual is the inverse transform of S c (the transform is
//     its own inverse), and x^ = round_state(pred + r^).

inline double walsh(int i, int j) { return (__builtin_popcount((unsigned)(i & j)) & 1) ? -1.0 : 1.0; }

// The transform of E1 (and its inverse, the same map).
void hadamard64(const double* in, double* out) {
  for (int i = 0; i < 64; ++i) {
    double acc = 0.0;
    for (int j = 0; j < 64; ++j) acc += walsh(i, j) * in[j];
    out[i] = acc / 8.0;
  }
}

// One group of 64 residuals r -> 32 indices, the stored scale, and the decoded
// residual rh (E1-E6).  cb: 16 points [16][2].
void eden2_code_group(const double* r, int pfmt, const double* cb, uint8_t* idx, double* S, double* rh) {
  double y[64], yh[64];
  hadamard64(r, y);
  double sumsq = 0.0;
  for (int i = 0; i < 64; ++i) sumsq += y[i] * y[i];
  double dot = 0.0;
  if (sumsq > 0.0) {
    const double sigma = std::sqrt(sumsq / 64.0);
    for (int p = 0; p < 32; ++p) {
      const double u0 = y[2 * p] / sigma, u1 = y[2 * p + 1] / sigma;
      int best = 0;
      double bd = 0.0;
      for (int k = 0; k < 16; ++k) {
        const double d0 = u0 - cb[2 * k], d1 = u1 - cb[2 * k + 1];
        const double d = d0 * d0 + d1 * d1;
        if (k == 0 || d < bd) {
          best = k;
          bd = d;
        }
      }
      idx[p] = (uint8_t)best;
      dot += y[2 * p] * cb[2 * best] + y[2 * p + 1] * cb[2 * best + 1];
    }
  } else {
    for (int p = 0; p < 32; ++p) idx[p] = 0;
  }
  *S = (sumsq > 0.0 && dot > 0.0) ? round_to(sumsq / dot, pfmt) : 0.0;
  for (int p = 0; p < 32; ++p) {
    yh[2 * p] = *S * cb[2 * idx[p]];
    yh[2 * p + 1] = *S * cb[2 * idx[p] + 1];
  }
  hadamard64(yh, rh);
}

void eden2_decode_group(const uint8_t* idx, double S, const double* cb, double* rh) {
  double yh[64];
  for (int p = 0; p < 32; ++p) {
    yh[2 * p] = S * cb[2 * idx[p]];
    yh[2 * p + 1] = S * cb[2 * idx[p] + 1];
  }
  hadamard64(yh, rh);
}

// A row of n values coded against its prediction with H64 / EDEN-2: q receives
// n / 2 pair indices, s the n / 64 scales (z is unused and set to 0).
void eden2_code_row(const double* x, const double* pred, int n, int pfmt, int sfmt, const double* cb, uint8_t* q,
                    double* s, double* z, double* xhat) {
  double r[64], rh[64];
  for (int g = 0; g < n / 64; ++g) {
    for (int i = 0; i < 64; ++i) r[i] = x[g * 64 + i] - pred[g * 64 + i];
    eden2_code_group(r, pfmt, cb, q + g * 32, s + g, rh);
    z[g] = 0.0;
    for (int i = 0; i < 64; ++i) xhat[g * 64 + i] = round_to(pred[g * 64 + i] + rh[i], sfmt);
  }
}

void eden2_decode_row(const uint8_t* q, const double* s, const double* pred, int n, int sfmt, const double* cb,
                      double* xhat) {
  double rh[64];
  for (int g = 0; g < n / 64; ++g) {
    eden2_decode_group(q + g * 32, s[g], cb, rh);
    for (int i = 0; i < 64; ++i) xhat[g * 64 + i] = round_to(pred[g * 64 + i] + rh[i], sfmt);
  }
}

// The residual codec of a layer: cb == NULL is the scalar group quantizer
// (R1-R4), otherwise H64 / EDEN-2 with codebook cb.  Codes are per element
// (scalar) or per pair (EDEN-2): `qn` entries per row of n values.
struct RowCoder {
  int bits, group, pfmt, sfmt;
  const double* cb;
  int qn(int n) const { return cb ? n / 2 : n; }
  int sn(int n) const { return cb ? n / 64 : n / group; }
  void code(const double* x, const double* pred, int n, uint8_t* q, double* s, double* z, double* xhat) const {
    if (cb)
      eden2_code_row(x, pred, n, pfmt, sfmt, cb, q, s, z, xhat);
    else
      code_row(x, pred, n, bits, group, pfmt, sfmt, q, s, z, xhat);
  }
  void decode(const uint8_t* q, const double* s, const double* z, const double* pred, int n, double* xhat) const {
    if (cb)
      eden2_decode_row(q, s, pred, n, sfmt, cb, xhat);
    else
      decode_row(q, s, z, pred, n, group, sfmt, xhat);
  }
};

// ---------------------------------------------------------------- cross-layer block-DPLR prediction
// [CORAL abstract, Fig. 3]

// Prediction of one token's K_l row (C = H D values) from its reconstructed
// K_{l-1} row: per head, B_h applied to that head's channels; globally, the
// latent u = x W^T (r values, R6) and then u U^T.
void predict_k_token(int H, int D, int r, const double* ks, const double* bk, const double* wk, const double* uk,
                     double* pred) {
  const int C = H * D;
  std::vector<double> u(r > 0 ? r : 1);
  for (int j = 0; j < r; ++j) {
    double acc = 0.0;
    for (int c = 0; c < C; ++c) acc += ks[c] * wk[(int64_t)j * C + c];
    u[j] = acc;
  }
  for (int h = 0; h < H; ++h) {
    for (int o = 0; o < D; ++o) {
      double blk = 0.0;
      for (int i = 0; i < D; ++i) blk += ks[h * D + i] * bk[((int64_t)h * D + o) * D + i];
      double low = 0.0;
      for (int j = 0; j < r; ++j) low += u[j] * uk[(int64_t)(h * D + o) * r + j];
      pred[h * D + o] = blk + low;
    }
  }
}

// Prediction of one token's V_l row from the reconstructed K_l row (kh) and
// V_{l-1} row (vs): per head, the 2D-wide input [kh_h | vs_h] through BV_h;
// globally, the 2C-wide input [kh | vs] through W_V and then U_V (Fig. 3:
// K first, then V from the reconstructed K).
void predict_v_token(int H, int D, int r, const double* kh, const double* vs, const double* bv, const double* wv,
                     const double* uv, double* pred) {
  const int C = H * D;
  std::vector<double> u(r > 0 ? r : 1);
  for (int j = 0; j < r; ++j) {
    double acc = 0.0;
    for (int c = 0; c < C; ++c) acc += kh[c] * wv[(int64_t)j * 2 * C + c];
    for (int c = 0; c < C; ++c) acc += vs[c] * wv[(int64_t)j * 2 * C + C + c];
    u[j] = acc;
  }
  for (int h = 0; h < H; ++h) {
    for (int o = 0; o < D; ++o) {
      const double* w = bv + ((int64_t)h * D + o) * 2 * D;
      double blk = 0.0;
      for (int i = 0; i < D; ++i) blk += kh[h * D + i] * w[i];
      for (int i = 0; i < D; ++i) blk += vs[h * D + i] * w[D + i];
      double low = 0.0;
      for (int j = 0; j < r; ++j) low += u[j] * uv[(int64_t)(h * D + o) * r + j];
      pred[h * D + o] = blk + low;
    }
  }
}

// ---------------------------------------------------------------- temporal prediction
// [TEMPO abstract, Fig. 2(b)]; readings R8, R9.  One head's map a [D][2D]
// applied to the inputs [x1 | x2] of one position.
void predict_temporal_head(int D, const double* a, const double* x1, const double* x2, double* pred) {
  for (int o = 0; o < D; ++o) {
    const double* w = a + (int64_t)o * 2 * D;
    double acc = 0.0;
    for (int i = 0; i < D; ++i) acc += x1[i] * w[i];
    for (int i = 0; i < D; ++i) acc += x2[i] * w[D + i];
    pred[o] = acc;
  }
}

// ---------------------------------------------------------------- clustered prediction
// [NANO abstract]; R10: the nearest centre by |c_j|^2 - 2 x.c_j (the |x|^2
// term is common to all j), ties to the lowest j.  norm[j] = |c_j|^2.
int nearest_centre(int C, int nc, const double* x, const double* cent, const double* norm) {
  int best = 0;
  double best_d = 0.0;
  for (int j = 0; j < nc; ++j) {
    double dot = 0.0;
    for (int c = 0; c < C; ++c) dot += x[c] * cent[(int64_t)j * C + c];
    const double d = norm[j] - 2.0 * dot;
    if (j == 0 || d < best_d) {
      best = j;
      best_d = d;
    }
  }
  return best;
}

void centre_norms(int C, int nc, const double* cent, double* norm) {
  for (int j = 0; j < nc; ++j) {
    double acc = 0.0;
    for (int c = 0; c < C; ++c) acc += cent[(int64_t)j * C + c] * cent[(int64_t)j * C + c];
    norm[j] = acc;
  }
}

}  // namespace

extern "C" {

// ---------------------------------------------------------------- building blocks (exported for the pins)

double kvo_round(double x, int fmt) { return round_to(x, fmt); }

void kvo_round_array(const double* x, int64_t n, int fmt, double* y) {
  for (int64_t i = 0; i < n; ++i) y[i] = round_to(x[i], fmt);
}

// rows x n residuals -> codes [rows][n], s, z [rows][n / group].
void kvo_quantize_groups(const double* r, int64_t rows, int n, int bits, int group, int pfmt, uint8_t* q, double* s,
                         double* z) {
  const int ng = n / group;
  for (int64_t t = 0; t < rows; ++t)
    for (int g = 0; g < ng; ++g)
      quantize_group(r + t * n + g * group, group, bits, pfmt, q + t * n + g * group, s + t * ng + g, z + t * ng + g);
}

// Values z + s q of rows x n codes (R1).
void kvo_dequantize_groups(const uint8_t* q, const double* s, const double* z, int64_t rows, int n, int group,
                           double* out) {
  const int ng = n / group;
  for (int64_t t = 0; t < rows; ++t)
    for (int j = 0; j < n; ++j) out[t * n + j] = dequant(q[t * n + j], s[t * ng + j / group], z[t * ng + j / group]);
}

// Element j of a row of n codes sits at bits [j b, (j + 1) b) of the row,
// least significant bit first (the layout the pages' byte accounting implies).
void kvo_pack(const uint8_t* q, int64_t rows, int n, int bits, uint8_t* out) {
  const int64_t rb = (int64_t)n * bits / 8;
  for (int64_t t = 0; t < rows; ++t) {
    uint8_t* o = out + t * rb;
    for (int64_t i = 0; i < rb; ++i) o[i] = 0;
    for (int j = 0; j < n; ++j) {
      const int64_t bit = (int64_t)j * bits;
      o[bit / 8] = (uint8_t)(o[bit / 8] | (q[t * n + j] << (bit % 8)));
    }
  }
}

void kvo_unpack(const uint8_t* packed, int64_t rows, int n, int bits, uint8_t* q) {
  const int64_t rb = (int64_t)n * bits / 8;
  const int mask = (1 << bits) - 1;
  for (int64_t t = 0; t < rows; ++t)
    for (int j = 0; j < n; ++j) {
      const int64_t bit = (int64_t)j * bits;
      q[t * n + j] = (uint8_t)((packed[t * rb + bit / 8] >> (bit % 8)) & mask);
    }
}

// The predictions alone, [T][H][D] each (pins of the predictor structure).
void kvo_predict_xlayer_k(int64_t T, int H, int D, int r, const double* Ks, const double* bk, const double* wk,
                          const double* uk, double* pred) {
  const int C = H * D;
  for (int64_t t = 0; t < T; ++t) predict_k_token(H, D, r, Ks + t * C, bk, wk, uk, pred + t * C);
}

void kvo_predict_xlayer_v(int64_t T, int H, int D, int r, const double* Kh, const double* Vs, const double* bv,
                          const double* wv, const double* uv, double* pred) {
  const int C = H * D;
  for (int64_t t = 0; t < T; ++t) predict_v_token(H, D, r, Kh + t * C, Vs + t * C, bv, wv, uv, pred + t * C);
}

// ---------------------------------------------------------------- one layer, null predictor (anchor)
// [CORAL Fig. 8; TEMPO appendix Table 7]: every row coded against 0.  cb:
// NULL for the scalar group quantizer, else the 16 EDEN-2 points ([16][2]);
// q then holds D / 2 pair indices per row and s D / 64 scales.

void kvo_encode_none(int64_t T, int H, int D, int bits, int group, int pfmt, int sfmt, const double* X, uint8_t* q,
                     double* s, double* z, double* xhat, const double* cb) {
  const RowCoder rc{bits, group, pfmt, sfmt, cb};
  const int qn = rc.qn(D), sn = rc.sn(D);
  std::vector<double> zero(D, 0.0);
  for (int64_t t = 0; t < T; ++t)
    for (int h = 0; h < H; ++h) {
      const int64_t row = t * H + h;
      rc.code(X + row * D, zero.data(), D, q + row * qn, s + row * sn, z + row * sn, xhat + row * D);
    }
}

void kvo_decode_none(int64_t T, int H, int D, int group, int sfmt, const uint8_t* q, const double* s, const double* z,
                     double* xhat, const double* cb) {
  const RowCoder rc{0, group, 0, sfmt, cb};
  const int qn = rc.qn(D), sn = rc.sn(D);
  std::vector<double> zero(D, 0.0);
  for (int64_t t = 0; t < T; ++t)
    for (int h = 0; h < H; ++h) {
      const int64_t row = t * H + h;
      rc.decode(q + row * qn, s + row * sn, z + row * sn, zero.data(), D, xhat + row * D);
    }
}

// ---------------------------------------------------------------- one cross-layer layer l > 0
// [CORAL Fig. 3]: per token, K first (its prediction needs only layer l-1),
// then V, whose prediction reads the reconstructed K_l.  Tokens do not
// interact.  K, V, Ks, Vs, kh, vh: [T][H][D]; bk [H][D][D], wk [r][C],
// uk [C][r], bv [H][D][2D], wv [r][2C], uv [C][r].  `pk`, `pv` (optional,
// may be NULL) receive the predictions.  cb as for kvo_encode_none.

void kvo_encode_xlayer(int64_t T, int H, int D, int r, int bits, int group, int pfmt, int sfmt, const double* K,
                       const double* V, const double* Ks, const double* Vs, const double* bk, const double* wk,
                       const double* uk, const double* bv, const double* wv, const double* uv, uint8_t* qk, double* sk,
                       double* zk, uint8_t* qv, double* sv, double* zv, double* kh, double* vh, double* pk,
                       double* pv, const double* cb) {
  const RowCoder rc{bits, group, pfmt, sfmt, cb};
  const int C = H * D, qn = rc.qn(D), sn = rc.sn(D);
  std::vector<double> pred(C);
  for (int64_t t = 0; t < T; ++t) {
    const int64_t o = t * C, oq = t * H * qn, og = t * H * sn;
    predict_k_token(H, D, r, Ks + o, bk, wk, uk, pred.data());
    if (pk) std::memcpy(pk + o, pred.data(), sizeof(double) * C);
    for (int h = 0; h < H; ++h)
      rc.code(K + o + h * D, pred.data() + h * D, D, qk + oq + h * qn, sk + og + h * sn, zk + og + h * sn,
              kh + o + h * D);
    predict_v_token(H, D, r, kh + o, Vs + o, bv, wv, uv, pred.data());
    if (pv) std::memcpy(pv + o, pred.data(), sizeof(double) * C);
    for (int h = 0; h < H; ++h)
      rc.code(V + o + h * D, pred.data() + h * D, D, qv + oq + h * qn, sv + og + h * sn, zv + og + h * sn,
              vh + o + h * D);
  }
}

// The decoder replays the encoder's prediction chain from the codes.
void kvo_decode_xlayer(int64_t T, int H, int D, int r, int group, int sfmt, const uint8_t* qk, const double* sk,
                       const double* zk, const uint8_t* qv, const double* sv, const double* zv, const double* Ks,
                       const double* Vs, const double* bk, const double* wk, const double* uk, const double* bv,
                       const double* wv, const double* uv, double* kh, double* vh, const double* cb) {
  const RowCoder rc{0, group, 0, sfmt, cb};
  const int C = H * D, qn = rc.qn(D), sn = rc.sn(D);
  std::vector<double> pred(C);
  for (int64_t t = 0; t < T; ++t) {
    const int64_t o = t * C, oq = t * H * qn, og = t * H * sn;
    predict_k_token(H, D, r, Ks + o, bk, wk, uk, pred.data());
    for (int h = 0; h < H; ++h)
      rc.decode(qk + oq + h * qn, sk + og + h * sn, zk + og + h * sn, pred.data() + h * D, D, kh + o + h * D);
    predict_v_token(H, D, r, kh + o, Vs + o, bv, wv, uv, pred.data());
    for (int h = 0; h < H; ++h)
      rc.decode(qv + oq + h * qn, sv + og + h * sn, zv + og + h * sn, pred.data() + h * D, D, vh + o + h * D);
  }
}

// The H64 / EDEN-2 transform of E1 on rows of 64 values (exported for the pins).
void kvo_hadamard64(const double* in, int64_t rows, double* out) {
  for (int64_t t = 0; t < rows; ++t) hadamard64(in + t * 64, out + t * 64);
}

// ---------------------------------------------------------------- one temporal layer
// [TEMPO Fig. 2(b)]; R8, R9.  Frames in time order; token t = f F + s.  The
// frame-0 rows are the anchor (prediction 0, anchor_bits) unless the call
// continues a sequence (khist [2][F][H][D]: frames f0-2, f0-1; vhist
// [F][H][D]: frame f0-1), in which case every frame is predicted and coded at
// `bits`.  Heads and positions do not interact.  ak, av: [H][D][2D].
// `decode` replays the chain from q, s, z instead of coding K, V.

void kvo_temporal(int decode, int64_t T, int H, int D, int F, int bits, int anchor_bits, int group, int pfmt,
                  int sfmt, const double* K, const double* V, const double* khist, const double* vhist,
                  const double* ak, const double* av, uint8_t* qk, double* sk, double* zk, uint8_t* qv, double* sv,
                  double* zv, double* kh, double* vh) {
  const int C = H * D, ng = D / group;
  const bool cont = khist != nullptr;
  const int64_t n_frames = (T + F - 1) / F;
  std::vector<double> zero(D, 0.0), pred(D);
  // reconstructed K row of frame f (f may be -1 or -2: the supplied history, else zeros)
  auto krow = [&](int64_t f, int64_t s, int h) -> const double* {
    if (f >= 0) return kh + (f * F + s) * C + h * D;
    if (!cont) return zero.data();
    return khist + ((f + 2) * F + s) * C + h * D;
  };
  auto vrow = [&](int64_t f, int64_t s, int h) -> const double* {
    if (f >= 0) return vh + (f * F + s) * C + h * D;
    if (!cont) return zero.data();
    return vhist + (s * C) + h * D;
  };
  for (int64_t f = 0; f < n_frames; ++f) {
    const int64_t n = (f + 1) * F <= T ? F : T - f * F;
    const bool anchor = f == 0 && !cont;
    const int b = anchor ? anchor_bits : bits;
    for (int64_t s = 0; s < n; ++s) {
      const int64_t t = f * F + s;
      for (int h = 0; h < H; ++h) {
        const int64_t o = t * C + h * D, og = (t * H + h) * ng;
        // K_f from [K^_{f-1} | K^_{f-2}]
        if (anchor)
          std::memcpy(pred.data(), zero.data(), sizeof(double) * D);
        else
          predict_temporal_head(D, ak + (int64_t)h * D * 2 * D, krow(f - 1, s, h), krow(f - 2, s, h), pred.data());
        if (decode)
          decode_row(qk + o, sk + og, zk + og, pred.data(), D, group, sfmt, kh + o);
        else
          code_row(K + o, pred.data(), D, b, group, pfmt, sfmt, qk + o, sk + og, zk + og, kh + o);
      }
      for (int h = 0; h < H; ++h) {
        const int64_t o = t * C + h * D, og = (t * H + h) * ng;
        // V_f from [K^_f | V^_{f-1}]
        if (anchor)
          std::memcpy(pred.data(), zero.data(), sizeof(double) * D);
        else
          predict_temporal_head(D, av + (int64_t)h * D * 2 * D, kh + o, vrow(f - 1, s, h), pred.data());
        if (decode)
          decode_row(qv + o, sv + og, zv + og, pred.data(), D, group, sfmt, vh + o);
        else
          code_row(V + o, pred.data(), D, b, group, pfmt, sfmt, qv + o, sv + og, zv + og, vh + o);
      }
    }
  }
}

// ---------------------------------------------------------------- clustered codec, one tensor
// Nearest-centre assignment of T rows of X [T][C] (R10).
void kvo_cluster_assign(int64_t T, int C, int nc, const double* X, const double* cent, int64_t* assign) {
  std::vector<double> norm(nc);
  centre_norms(C, nc, cent, norm.data());
  for (int64_t t = 0; t < T; ++t) assign[t] = nearest_centre(C, nc, X + t * C, cent, norm.data());
}

// [NANO abstract]; R10.  X [T][C]; cent [nc][C]; enc [m][C]; dec [C][m].
// Writes the assignment, the m coefficient codes with their (s, z) pairs and
// the reconstruction rounded to the state format (unrounded if sfmt is 0).

void kvo_cluster_encode(int64_t T, int C, int m, int nc, int bits, int group, int pfmt, int sfmt, const double* X,
                        const double* cent, const double* enc, const double* dec, int64_t* assign, uint8_t* q,
                        double* s, double* z, double* xhat) {
  const int ng = m / group;
  std::vector<double> norm(nc), coef(m), res(C);
  centre_norms(C, nc, cent, norm.data());
  for (int64_t t = 0; t < T; ++t) {
    const double* x = X + t * C;
    const int best = nearest_centre(C, nc, x, cent, norm.data());
    assign[t] = best;
    const double* ca = cent + (int64_t)best * C;
    for (int c = 0; c < C; ++c) res[c] = x[c] - ca[c];
    for (int k = 0; k < m; ++k) {
      double acc = 0.0;
      for (int c = 0; c < C; ++c) acc += res[c] * enc[(int64_t)k * C + c];
      coef[k] = acc;
    }
    for (int g = 0; g < ng; ++g)
      quantize_group(&coef[g * group], group, bits, pfmt, q + t * m + g * group, s + t * ng + g, z + t * ng + g);
    if (xhat) {
      for (int c = 0; c < C; ++c) {
        double acc = 0.0;
        for (int k = 0; k < m; ++k) acc += dequant(q[t * m + k], s[t * ng + k / group], z[t * ng + k / group]) *
                                           dec[(int64_t)c * m + k];
        xhat[t * C + c] = round_to(ca[c] + acc, sfmt);
      }
    }
  }
}

void kvo_cluster_decode(int64_t T, int C, int m, int group, int sfmt, const int64_t* assign, const uint8_t* q,
                        const double* s, const double* z, const double* cent, const double* dec, double* xhat) {
  const int ng = m / group;
  for (int64_t t = 0; t < T; ++t) {
    const double* ca = cent + assign[t] * C;
    for (int c = 0; c < C; ++c) {
      double acc = 0.0;
      for (int k = 0; k < m; ++k)
        acc += dequant(q[t * m + k], s[t * ng + k / group], z[t * ng + k / group]) * dec[(int64_t)c * m + k];
      xhat[t * C + c] = round_to(ca[c] + acc, sfmt);
    }
  }
}

// ---------------------------------------------------------------- attention
// Naive two-pass softmax attention over the decoded history (and any
// uncompressed keys appended to it by the caller): for each query row and
// head, s_t = scale q.k_t, m = max_t s_t, p_t = exp(s_t - m),
// o = sum_t p_t v_t / sum_t p_t.  Q [nq][H][D]; K, V [nk][H][D].

// Jensen-bias correction (the abstract on the "Jensen bias" of INT2 key caches,
// among the related papers listed on the CORAL-KV page): quantization noise e on a cached key raises
// E[exp(scale q.(k + e))] above exp(scale q.k); to second order (the
// log-moment of a uniform rounding error of step s is x^2 s^2 / 24 + O(x^4))
// the excess is exp(0.5 scale^2 sum_g |q_g|^2 s_g^2 / 12), g over the key's
// quantization groups.  Subtracting that exponent from the score of every
// quantized key removes the bias in expectation; uncompressed keys are left
// alone.  q: one head's query row (D values); sk: the key's group scales.
static double jensen_term(const double* q, const double* sk, int D, int group, double scale) {
  double acc = 0.0;
  for (int g = 0; g < D / group; ++g) {
    double qn = 0.0;
    for (int i = 0; i < group; ++i) qn += q[g * group + i] * q[g * group + i];
    acc += qn * sk[g] * sk[g] / 12.0;
  }
  return 0.5 * scale * scale * acc;
}

void kvo_attention_corrected(int64_t nq, int64_t nk, int Hq, int H, int D, double scale, const double* Q,
                             const double* K, const double* V, int64_t n_hist, const double* s_hist, int group,
                             double* O);

void kvo_attention(int64_t nq, int64_t nk, int H, int D, double scale, const double* Q, const double* K,
                   const double* V, double* O) {
  kvo_attention_corrected(nq, nk, H, H, D, scale, Q, K, V, 0, nullptr, 1, O);
}

// As kvo_attention, with Hq query heads over H key / value heads (Hq a multiple
// of H: query head hq reads head hq / (Hq / H), grouped-query attention); the
// first n_hist keys are quantized history whose group scales
// s_hist [n_hist][H][D / group] give each one's Jensen correction (s_hist
// NULL: no correction).  Q, O [nq][Hq][D]; K, V [nk][H][D].
void kvo_attention_corrected(int64_t nq, int64_t nk, int Hq, int H, int D, double scale, const double* Q,
                             const double* K, const double* V, int64_t n_hist, const double* s_hist, int group,
                             double* O) {
  const int C = H * D, Cq = Hq * D, ng = D / group, g = Hq / H;
  std::vector<double> sc(nk > 0 ? nk : 1), acc(D);
  for (int64_t i = 0; i < nq; ++i)
    for (int hq = 0; hq < Hq; ++hq) {
      const int h = hq / g;
      const double* q = Q + i * Cq + hq * D;
      double m = -INFINITY;
      for (int64_t t = 0; t < nk; ++t) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += q[d] * K[t * C + h * D + d];
        sc[t] = dot * scale;
        if (s_hist && t < n_hist) sc[t] -= jensen_term(q, s_hist + (t * H + h) * ng, D, group, scale);
        if (sc[t] > m) m = sc[t];
      }
      double l = 0.0;
      for (int64_t t = 0; t < nk; ++t) {
        sc[t] = std::exp(sc[t] - m);
        l += sc[t];
      }
      // o[d] = sum_t p_t v_t[d] in key order (keys outer, so V is read row by row)
      for (int d = 0; d < D; ++d) acc[d] = 0.0;
      for (int64_t t = 0; t < nk; ++t) {
        const double* v = V + t * C + h * D;
        for (int d = 0; d < D; ++d) acc[d] += sc[t] * v[d];
      }
      double* o = O + i * Cq + hq * D;
      for (int d = 0; d < D; ++d) o[d] = acc[d] / l;
    }
}

// Mixed-dimensional attention on the stored coefficients ([NANO abstract], the
// Fast variant; R11).  Per query row and head h:
//   s_t = scale (q_h . c_{a(t),h} + (W_dec,h^T q_h) . coef^_t)
//   p = softmax(s);  m_j = sum_{t: a_v(t) = j} p_t;  cbar = sum_t p_t coef^V_t
//   o_h = sum_j m_j c^V_{j,h} + W^V_dec,h cbar
// ck, cv: dequantized coefficients [T][m]; ak, av: assignments [T];
// cent_k, cent_v [nc][C]; dec_k, dec_v [C][m]; Q, O [nq][H][D].

void kvo_mixed_attention(int64_t nq, int64_t T, int H, int D, int m, int nc, double scale, const double* Q,
                         const double* ck, const int64_t* ak, const double* cent_k, const double* dec_k,
                         const double* cv, const int64_t* av, const double* cent_v, const double* dec_v, double* O) {
  const int C = H * D;
  std::vector<double> table(nc), qt(m), sc(T > 0 ? T : 1), mass(nc), cbar(m), cacc(D);
  for (int64_t i = 0; i < nq; ++i)
    for (int h = 0; h < H; ++h) {
      const double* q = Q + i * C + h * D;
      for (int j = 0; j < nc; ++j) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d) acc += q[d] * cent_k[(int64_t)j * C + h * D + d];
        table[j] = acc;
      }
      // qt[k] = sum_d q[d] W_dec[h D + d][k] in channel order (channels outer)
      for (int k = 0; k < m; ++k) qt[k] = 0.0;
      for (int d = 0; d < D; ++d)
        for (int k = 0; k < m; ++k) qt[k] += q[d] * dec_k[(int64_t)(h * D + d) * m + k];
      double mx = -INFINITY;
      for (int64_t t = 0; t < T; ++t) {
        double acc = 0.0;
        for (int k = 0; k < m; ++k) acc += qt[k] * ck[t * m + k];
        sc[t] = scale * (table[ak[t]] + acc);
        if (sc[t] > mx) mx = sc[t];
      }
      double l = 0.0;
      for (int64_t t = 0; t < T; ++t) {
        sc[t] = std::exp(sc[t] - mx);
        l += sc[t];
      }
      for (int j = 0; j < nc; ++j) mass[j] = 0.0;
      for (int k = 0; k < m; ++k) cbar[k] = 0.0;
      for (int64_t t = 0; t < T; ++t) {
        const double p = sc[t] / l;
        mass[av[t]] += p;
        for (int k = 0; k < m; ++k) cbar[k] += p * cv[t * m + k];
      }
      // sum_j m_j c^V_j[d] in centre order (centres outer), plus W^V_dec cbar
      for (int d = 0; d < D; ++d) cacc[d] = 0.0;
      for (int j = 0; j < nc; ++j)
        for (int d = 0; d < D; ++d) cacc[d] += mass[j] * cent_v[(int64_t)j * C + h * D + d];
      double* o = O + i * C + h * D;
      for (int d = 0; d < D; ++d) {
        double acc2 = 0.0;
        for (int k = 0; k < m; ++k) acc2 += dec_v[(int64_t)(h * D + d) * m + k] * cbar[k];
        o[d] = cacc[d] + acc2;
      }
    }
}

// ---------------------------------------------------------------- video-adapted block-DPLR refit
// ["CORAL-KV ...", Fig. 4: the video-adapted block-DPLR keeps its low-rank
// factors fixed and refits the block-diagonal terms for each filled cache
// block.]  Reading V1: the refit is a ridge least-squares fit of each head's
// block on the block's tokens, against the target left after the fixed
// low-rank term:
//   B_h^T = (X_h^T X_h + ridge I)^{-1} X_h^T (Y_h - LR_h),
// X_h the head's predictor input (K: K^_{l-1,h}; V: [K^_{l,h} | V^_{l-1,h}]),
// Y_h the clean values, LR = (X_flat W^T) U^T the fixed low-rank prediction.
// Solved by a Cholesky factorisation G = L L^T and two triangular solves.
// X0, X1 [T][H][D] (X1 NULL for K); Y [T][H][D]; w [r][Cin], u [C][r];
// block [H][D][din] with din = D (K) or 2 D (V).
void kvo_refit_block_diag(int64_t T, int H, int D, int r, const double* X0, const double* X1, const double* Y,
                          const double* w, const double* u, double ridge, double* block) {
  const int C = H * D, din = X1 ? 2 * D : D, cin = X1 ? 2 * C : C;
  // the fixed low-rank prediction of every token, all heads
  std::vector<double> lat(r > 0 ? r : 1), lr((size_t)T * C, 0.0);
  for (int64_t t = 0; t < T; ++t) {
    for (int j = 0; j < r; ++j) {
      double acc = 0.0;
      for (int c = 0; c < C; ++c) acc += X0[t * C + c] * w[(int64_t)j * cin + c];
      if (X1)
        for (int c = 0; c < C; ++c) acc += X1[t * C + c] * w[(int64_t)j * cin + C + c];
      lat[j] = acc;
    }
    for (int o = 0; o < C; ++o) {
      double acc = 0.0;
      for (int j = 0; j < r; ++j) acc += lat[j] * u[(int64_t)o * r + j];
      lr[t * C + o] = acc;
    }
  }
  std::vector<double> G((size_t)din * din), Rhs((size_t)din * D), x(din), L((size_t)din * din);
  for (int h = 0; h < H; ++h) {
    std::fill(G.begin(), G.end(), 0.0);
    std::fill(Rhs.begin(), Rhs.end(), 0.0);
    for (int64_t t = 0; t < T; ++t) {
      for (int i = 0; i < D; ++i) x[i] = X0[t * C + h * D + i];
      if (X1)
        for (int i = 0; i < D; ++i) x[D + i] = X1[t * C + h * D + i];
      for (int i = 0; i < din; ++i) {
        for (int j = 0; j < din; ++j) G[(size_t)i * din + j] += x[i] * x[j];
        for (int o = 0; o < D; ++o) Rhs[(size_t)i * D + o] += x[i] * (Y[t * C + h * D + o] - lr[t * C + h * D + o]);
      }
    }
    for (int i = 0; i < din; ++i) G[(size_t)i * din + i] += ridge;
    // Cholesky: G = L L^T (lower triangular L)
    for (int j = 0; j < din; ++j) {
      double d = G[(size_t)j * din + j];
      for (int k = 0; k < j; ++k) d -= L[(size_t)j * din + k] * L[(size_t)j * din + k];
      const double ljj = std::sqrt(d);
      L[(size_t)j * din + j] = ljj;
      for (int i = j + 1; i < din; ++i) {
        double v = G[(size_t)i * din + j];
        for (int k = 0; k < j; ++k) v -= L[(size_t)i * din + k] * L[(size_t)j * din + k];
        L[(size_t)i * din + j] = v / ljj;
      }
    }
    // for each output channel o: L z = rhs_o, then L^T b = z; block[h][o][i] = b_i
    std::vector<double> z(din), b(din);
    for (int o = 0; o < D; ++o) {
      for (int i = 0; i < din; ++i) {
        double v = Rhs[(size_t)i * D + o];
        for (int k = 0; k < i; ++k) v -= L[(size_t)i * din + k] * z[k];
        z[i] = v / L[(size_t)i * din + i];
      }
      for (int i = din - 1; i >= 0; --i) {
        double v = z[i];
        for (int k = i + 1; k < din; ++k) v -= L[(size_t)k * din + i] * b[k];
        b[i] = v / L[(size_t)i * din + i];
      }
      for (int i = 0; i < din; ++i) block[((int64_t)h * D + o) * din + i] = b[i];
    }
  }
}

// ---------------------------------------------------------------- storage accounting
// [TEMPO Tables 1-3 (5.33x), Table 8 (3.20x), appendix Table 7]: bytes of
// codes + (scale, zero) pairs (+ one-byte centre indices) of one layer's K and
// V.  kind: 0 none / cross-layer, 1 temporal, 2 clustered.

int64_t kvo_codes_bytes(int kind, int64_t T, int H, int D, int bits, int group, int param_bytes, int F,
                        int anchor_bits, int m) {
  const int64_t pair = 2 * (int64_t)param_bytes;
  // H64 / EDEN-2 (kind 3): a 4-bit index per pair of values and one scale per 64 values
  if (kind == 3) return 2 * T * H * ((int64_t)(D / 2) * 4 / 8 + (D / 64) * (int64_t)param_bytes);
  if (kind == 2) return 2 * T * ((int64_t)m * bits / 8 + (m / group) * pair + 1);
  const int64_t row_params = (D / group) * pair;
  if (kind == 1) {
    const int64_t n0 = anchor_bits ? (F < T ? F : T) : 0;
    const int64_t one = n0 * H * ((int64_t)D * anchor_bits / 8) + (T - n0) * H * ((int64_t)D * bits / 8) +
                        T * H * row_params;
    return 2 * one;
  }
  return 2 * T * H * ((int64_t)D * bits / 8 + row_params);
}

}  // extern "C"
