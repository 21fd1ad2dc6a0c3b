"""fp64 CPU oracle of the predict-then-quantize-residual KV-cache codec and of
attention over the compressed history.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The product package (``clustered_kv_cache_b200``) never imports it and
has no CPU fallback; the two share no code.

Everything here is plain numpy in float64 over whole tensors, in the order the
pages describe, with library matmuls as the only building block.  Inputs that
the GPU path receives in bf16 or fp32 arrive here as float64 arrays holding
exactly those values.

Sources (page title, then the figure / table / section followed):

* [CORAL] "CORAL-KV: Compact Cross-Layer Prediction and Residual Coding for
  Autoregressive Video KV Caches": abstract (block-diagonal per-head maps plus a
  global low-rank term; prediction residual quantized), Fig. 3 (at layer l>0 the
  reconstructed states of layer l-1 feed the predictors; K_l from K_{l-1}, V_l
  from [K_l, V_{l-1}]), Fig. 5 (non-overlapping groups of residual channels, one
  shared scale per group), Fig. 8 (INT4 layer-zero anchor), Table 9 (scalar
  INT2 residual codec).
* [TEMPO] "TempoKV: Predictive KV Cache Quantization for Autoregressive Video
  Generation": abstract and Fig. 2(b) (K predicted from the reconstructed K
  history, V from the aligned reconstructed K plus reconstructed V history,
  only the low-bit residual stored), Tables 1-3 and 8 (INT2 / INT4 group
  quantizers at 5.33x / 3.20x), appendix Table 7 (anchor precision).
* [NANO] "NanoKV: High-Ratio KV Cache Compression for Autoregressive Video
  Generation": abstract (shared content in cluster centres, joint head-channel
  residual encoded into low-bit coefficients; the Fast variant attends on the
  stored coefficients without rebuilding full-dimensional keys).

Readings taken where the pages are silent (each restated at its function):

R1  quantizer: asymmetric min/max round-to-nearest per group, s = (max-min) /
    (2^b-1), z = min, code q = clamp(rint((r-z)/s), 0, 2^b-1), value z + s*q.
R2  rint is round-half-to-even; s and z are rounded to the parameter dtype
    (fp16 for bf16 data, fp32 for fp32 data) before the codes are computed.
R3  a group whose stored scale is 0 gets all-zero codes and decodes to z.
R4  groups are runs of `group` consecutive channels inside one (token, head) row
    (for the clustered codec: inside the 128 coefficients of a token).
R5  the reconstruction x_hat = round_state(pred + (z + s*q)) is what later
    predictions consume (closed loop); state dtype is bf16 or fp32.
R6  the low-rank latent z = x_hat @ W^T is kept at full precision (the pages
    give no rounding for it) before the second factor is applied.
R7  weights use the [out][in] convention: y = x @ W^T.
R8  temporal: frame 0 of a layer is coded with the null predictor at
    `anchor_bits`; at frame 1 the missing lag-2 frame is taken as zero; a
    partial last frame uses the first n spatial positions of earlier frames.
    A sequence may also be continued from a supplied reconstructed history
    (the two previous K frames, the previous V frame); no frame is then an
    anchor.
R9  the temporal K map takes [K_{f-1} | K_{f-2}] (2D inputs per head); the V map
    takes [K_f | V_{f-1}] (2D inputs per head).
R10 clustered codec: a(t) = argmin_j (|c_j|^2 - 2 x_t.c_j), ties to the lowest
    j; coefficients = E (x_t - c_a); decode x_hat = c_a + W_dec coef_hat.
R11 mixed-dimensional attention: the value side is clustered and coded the same
    way as keys; its output is sum_j m_j c^V_j + W^V_dec sum_t p_t coef_hat^V_t
    with m_j the softmax mass of the tokens assigned to centre j.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

# --------------------------------------------------------------------------
# Rounding to storage formats (exact, direct from float64)
# --------------------------------------------------------------------------

_FORMATS = {
    # name: (significand bits incl. the implicit one, min normal exponent, max finite)
    "bf16": (8, -126, float.fromhex("0x1.fep127")),
    "f16": (11, -14, 65504.0),
    "f32": (24, -126, float.fromhex("0x1.fffffep127")),
}


def round_to(x, fmt: str) -> np.ndarray:
    """Round float64 values to the nearest value of format `fmt` (ties to even),
    with gradual underflow and overflow to +-inf.  `fmt` == "f64" is identity.

    The value x = 1.f * 2^E has quantum 2^(max(E, Emin) - (p-1)); x / quantum is
    exact in float64, np.rint rounds half to even, and the product is exact.
    """
    x = np.asarray(x, dtype=np.float64)
    if fmt == "f64":
        return x.copy()
    p, emin, fmax = _FORMATS[fmt]
    _, e = np.frexp(x)
    E = np.maximum(e - 1, emin)
    quantum = np.ldexp(1.0, E - (p - 1))
    y = np.rint(x / quantum) * quantum
    return np.where(np.abs(y) > fmax, np.copysign(np.inf, x), y)


# --------------------------------------------------------------------------
# Layer description
# --------------------------------------------------------------------------


@dataclass
class Desc:
    n_tokens: int
    n_heads: int
    head_dim: int
    state: str = "bf16"  # dtype of K/V and of every reconstruction ("bf16" | "f32")
    bits: int = 2
    group: int = 32
    param: str = "f16"  # dtype of the stored (scale, zero) pair ("f16" | "f32")
    frame_tokens: int = 0  # temporal codec only
    anchor_bits: int = 4  # temporal codec: bits of frame 0
    codec: str = "rtn"  # residual codec: "rtn" (scalar group quantizer) | "eden2" (H64 / EDEN-2)

    @property
    def channels(self) -> int:
        return self.n_heads * self.head_dim


# --------------------------------------------------------------------------
# Residual group quantizer [CORAL Fig. 5, Table 9; TEMPO Tables 1-3, 8]
# --------------------------------------------------------------------------


def quantize_groups(r, bits: int, group: int, param: str):
    """Asymmetric round-to-nearest group quantizer (readings R1-R4).

    r: float64 [..., n] with n % group == 0.
    Returns (q uint8 [..., n], s [..., n//group], z [..., n//group]); s and z
    hold the values of the parameter dtype.
    """
    r = np.asarray(r, dtype=np.float64)
    n = r.shape[-1]
    if n % group:
        raise ValueError("group must divide the row length")
    levels = (1 << bits) - 1
    rg = r.reshape(r.shape[:-1] + (n // group, group))
    mn = rg.min(axis=-1)
    mx = rg.max(axis=-1)
    s = round_to((mx - mn) / levels, param)
    z = round_to(mn, param)
    live = s > 0
    safe_s = np.where(live, s, 1.0)
    t = (rg - z[..., None]) / safe_s[..., None]
    q = np.clip(np.rint(t), 0, levels)
    q = np.where(live[..., None], q, 0.0)
    return q.reshape(r.shape).astype(np.uint8), s, z


def dequantize_groups(q, s, z, group: int) -> np.ndarray:
    """Value of each code, z + s*q, in float64 (reading R1)."""
    q = np.asarray(q, dtype=np.float64)
    n = q.shape[-1]
    qg = q.reshape(q.shape[:-1] + (n // group, group))
    v = z[..., None] + s[..., None] * qg
    return v.reshape(q.shape)


# --------------------------------------------------------------------------
# Bit packing, element j of a row at bits [j*b, (j+1)*b), LSB first
# --------------------------------------------------------------------------


def pack_codes(q, bits: int) -> np.ndarray:
    """Pack b-bit codes along the last axis into bytes, LSB first."""
    q = np.asarray(q, dtype=np.uint16)
    per = 8 // bits
    n = q.shape[-1]
    if (n * bits) % 8:
        raise ValueError("row does not fill whole bytes")
    qq = q.reshape(q.shape[:-1] + (n // per, per))
    shifts = (np.arange(per, dtype=np.uint16) * bits).astype(np.uint16)
    return (qq << shifts).sum(axis=-1).astype(np.uint8)


def unpack_codes(packed, bits: int, n: int) -> np.ndarray:
    """Inverse of pack_codes: bytes [..., n*b/8] -> codes uint8 [..., n]."""
    packed = np.asarray(packed, dtype=np.uint8)
    per = 8 // bits
    mask = (1 << bits) - 1
    shifts = np.arange(per) * bits
    q = (packed[..., None] >> shifts) & mask
    return q.reshape(packed.shape[:-1] + (n,)).astype(np.uint8)


# --------------------------------------------------------------------------
# Storage accounting [TEMPO Tables 1-3 (5.33x), Table 8 (3.20x), Table 7]
# --------------------------------------------------------------------------

_PARAM_BYTES = {"f16": 2, "f32": 4}


def bits_per_element(bits: int, group: int, param: str = "f16") -> float:
    """Stored bits per residual element: the code plus a (scale, zero) pair
    shared by `group` elements."""
    return bits + 2 * 8 * _PARAM_BYTES[param] / group


def codes_bytes(desc: Desc, kind: str = "none", code_dim: int = 0) -> int:
    """Bytes of codes + parameters (+ assignments) that one layer's K *and* V
    occupy, for the layouts the codec writes.

    kind "none"/"xlayer": every row at desc.bits.  "temporal": the rows of frame
    0 at desc.anchor_bits, the rest at desc.bits.  "cluster": one row of
    `code_dim` coefficients per token plus a one-byte centre index.
    """
    T, H, D = desc.n_tokens, desc.n_heads, desc.head_dim
    pb = 2 * _PARAM_BYTES[desc.param]
    if desc.codec == "eden2":  # a 4-bit index per pair of values, one scale per 64 values
        return 2 * T * H * ((D // 2) * 4 // 8 + (D // 64) * _PARAM_BYTES[desc.param])
    if kind == "cluster":
        per_tok = code_dim * desc.bits // 8 + (code_dim // desc.group) * pb + 1
        return 2 * T * per_tok
    row_params = (D // desc.group) * pb
    if kind == "temporal":
        n0 = min(desc.frame_tokens, T) if desc.anchor_bits else 0
        rows_anchor = n0 * H
        rows_rest = (T - n0) * H
        one = rows_anchor * (D * desc.anchor_bits // 8) + rows_rest * (D * desc.bits // 8)
        one += T * H * row_params
        return 2 * one
    return 2 * T * H * (D * desc.bits // 8 + row_params)


# --------------------------------------------------------------------------
# H64 / EDEN-2 residual codec [CORAL Fig. 5, Fig. 9, Table 9]
# --------------------------------------------------------------------------
#
# E1 groups of 64 consecutive residual channels are transformed by the
#    orthonormal Sylvester Walsh-Hadamard matrix H64 / 8;
# E2 the 32 pairs of a group are (y_2p, y_2p+1);
# E3 the 16 two-dimensional points are an input (pictured, not printed);
# E4 pairs normalised by sigma = sqrt(mean y^2) take the nearest point's index
#    (ties to the lowest); the stored scale is EDEN's S = |y|^2 / <y, c>,
#    rounded to the parameter dtype (0 when y = 0 or <y, c> <= 0);
# E5 pair p's 4-bit index at bits [4p, 4p+4) of the row;
# E6 the decoded residual is H64 / 8 applied to S c.


def hadamard_matrix(n: int = 64) -> np.ndarray:
    """Sylvester's construction H_2n = [[H, H], [H, -H]] from H_1 = [1]."""
    Hm = np.ones((1, 1))
    while Hm.shape[0] < n:
        Hm = np.block([[Hm, Hm], [Hm, -Hm]])
    return Hm


def eden2_code(r, param: str, codebook):
    """r [..., 64] -> (indices [..., 32], scale [...], decoded residual [..., 64])."""
    Hn = hadamard_matrix(64) / 8.0
    cb = np.asarray(codebook, np.float64).reshape(16, 2)
    y = np.asarray(r, np.float64) @ Hn.T
    sumsq = (y * y).sum(-1)
    pairs = y.reshape(y.shape[:-1] + (32, 2))
    sigma = np.sqrt(sumsq / 64.0)
    u = pairs / np.where(sigma > 0, sigma, 1.0)[..., None, None]
    d = ((u[..., :, None, :] - cb) ** 2).sum(-1)  # [..., 32, 16]
    idx = np.where((sumsq > 0)[..., None], d.argmin(-1), 0)
    dot = (pairs * cb[idx]).sum((-1, -2))
    S = np.where((sumsq > 0) & (dot > 0), round_to(sumsq / np.where(dot > 0, dot, 1.0), param), 0.0)
    return idx.astype(np.uint8), S, eden2_decode(idx, S, cb)


def eden2_decode(idx, S, codebook) -> np.ndarray:
    Hn = hadamard_matrix(64) / 8.0
    cb = np.asarray(codebook, np.float64).reshape(16, 2)
    yh = np.asarray(S, np.float64)[..., None, None] * cb[np.asarray(idx, np.int64)]
    return yh.reshape(yh.shape[:-2] + (64,)) @ Hn.T


# --------------------------------------------------------------------------
# One coded tensor: residual -> codes -> reconstruction (closed loop)
# --------------------------------------------------------------------------


def code_residual(x, pred, bits: int, group: int, param: str, state: str, codec: str = "rtn", codebook=None):
    """r = x - pred is quantized; the reconstruction pred + deq(r) is rounded to
    the state dtype (readings R1-R5).  Returns (q, s, z, x_hat); with the
    H64 / EDEN-2 codec q holds pair indices and s the per-64 scales."""
    r = np.asarray(x, dtype=np.float64) - pred
    if codec == "eden2":
        n = r.shape[-1]
        rg = r.reshape(r.shape[:-1] + (n // 64, 64))
        idx, S, rh = eden2_code(rg, param, codebook)
        q = idx.reshape(r.shape[:-1] + (n // 2,))
        return q, S, np.zeros_like(S), round_to(pred + rh.reshape(r.shape), state)
    q, s, z = quantize_groups(r, bits, group, param)
    x_hat = round_to(pred + dequantize_groups(q, s, z, group), state)
    return q, s, z, x_hat


def decode_residual(q, s, z, pred, group: int, state: str, codec: str = "rtn", codebook=None) -> np.ndarray:
    if codec == "eden2":
        q = np.asarray(q)
        idx = q.reshape(q.shape[:-1] + (q.shape[-1] // 32, 32))
        rh = eden2_decode(idx, s, codebook)
        return round_to(pred + rh.reshape(np.shape(pred)), state)
    return round_to(pred + dequantize_groups(q, s, z, group), state)


# --------------------------------------------------------------------------
# Cross-layer block-DPLR predictors [CORAL abstract, Fig. 3]
# --------------------------------------------------------------------------


def _blockdiag(x, block) -> np.ndarray:
    """Per-head map: x [T,H,Din], block [H,Dout,Din] -> [T,H,Dout]."""
    out = np.matmul(x.transpose(1, 0, 2), block.transpose(0, 2, 1))  # [H,T,Dout]
    return out.transpose(1, 0, 2)


def _lowrank(flat_in, w, u, T: int, H: int, D: int) -> np.ndarray:
    """Global low-rank term: (flat_in @ w^T) @ u^T (reading R6)."""
    if w is None or w.shape[0] == 0:
        return np.zeros((T, H, D))
    z = flat_in @ w.T
    return (z @ u.T).reshape(T, H, D)


def xlayer_predict_k(K_src, k_block, k_w, k_u) -> np.ndarray:
    """K~_l = blockdiag_h(K^_{l-1,h} B_h^T) + (K^_{l-1} W^T) U^T.

    K_src [T,H,D] reconstructed layer l-1; k_block [H,D,D]; k_w [r,C]; k_u [C,r].
    """
    T, H, D = K_src.shape
    pred = _blockdiag(K_src, k_block)
    return pred + _lowrank(K_src.reshape(T, H * D), k_w, k_u, T, H, D)


def xlayer_predict_v(K_rec, V_src, v_block, v_w, v_u) -> np.ndarray:
    """V~_l from the reconstructed pair [K^_l, V^_{l-1}]: per head the 2D-wide
    input [K^_{l,h} | V^_{l-1,h}] through v_block [H,D,2D]; globally the 2C-wide
    input [K^_l | V^_{l-1}] through v_w [r,2C] and v_u [C,r]."""
    T, H, D = K_rec.shape
    pred = _blockdiag(np.concatenate([K_rec, V_src], axis=-1), v_block)
    flat = np.concatenate([K_rec.reshape(T, H * D), V_src.reshape(T, H * D)], axis=-1)
    return pred + _lowrank(flat, v_w, v_u, T, H, D)


@dataclass
class Coded:
    """Codes of one tensor (K or V) of one layer, unpacked, plus parameters."""

    q: np.ndarray  # uint8 [T,H,D] (or [T,m] for the clustered codec)
    s: np.ndarray  # [T,H,D/G] (or [T,m/G])
    z: np.ndarray
    assign: np.ndarray | None = None  # clustered codec: centre index per token


def encode_layer_none(desc: Desc, K, V, codebook=None):
    """Anchor / RTN: the null predictor, every row coded directly
    [CORAL Fig. 8 INT4 anchor]."""
    zero = np.zeros(np.shape(K))
    out = []
    for x in (K, V):
        q, s, z, xh = code_residual(x, zero, desc.bits, desc.group, desc.param, desc.state, desc.codec, codebook)
        out.append((Coded(q, s, z), xh))
    return out[0][0], out[1][0], out[0][1], out[1][1]


def decode_layer_none(desc: Desc, ck: Coded, cv: Coded, codebook=None):
    T, H = ck.q.shape[:2]
    zero = np.zeros((T, H, desc.head_dim))
    K = decode_residual(ck.q, ck.s, ck.z, zero, desc.group, desc.state, desc.codec, codebook)
    V = decode_residual(cv.q, cv.s, cv.z, zero, desc.group, desc.state, desc.codec, codebook)
    return K, V


def encode_layer_xlayer(desc: Desc, w: dict, K, V, K_src, V_src, codebook=None):
    """One Coral layer l>0: K first (its prediction needs only layer l-1), then V,
    whose prediction needs the reconstructed K^_l [CORAL Fig. 3].

    w holds k_block, k_w, k_u, v_block, v_w, v_u (float64 copies of the weights).
    Returns (coded K, coded V, K^_l, V^_l).
    """
    pk = xlayer_predict_k(K_src, w["k_block"], w["k_w"], w["k_u"])
    qk, sk, zk, K_hat = code_residual(K, pk, desc.bits, desc.group, desc.param, desc.state, desc.codec, codebook)
    pv = xlayer_predict_v(K_hat, V_src, w["v_block"], w["v_w"], w["v_u"])
    qv, sv, zv, V_hat = code_residual(V, pv, desc.bits, desc.group, desc.param, desc.state, desc.codec, codebook)
    return Coded(qk, sk, zk), Coded(qv, sv, zv), K_hat, V_hat


def decode_layer_xlayer(desc: Desc, w: dict, ck: Coded, cv: Coded, K_src, V_src, codebook=None):
    """Replays the encoder's prediction chain from the codes."""
    pk = xlayer_predict_k(K_src, w["k_block"], w["k_w"], w["k_u"])
    K_hat = decode_residual(ck.q, ck.s, ck.z, pk, desc.group, desc.state, desc.codec, codebook)
    pv = xlayer_predict_v(K_hat, V_src, w["v_block"], w["v_w"], w["v_u"])
    V_hat = decode_residual(cv.q, cv.s, cv.z, pv, desc.group, desc.state, desc.codec, codebook)
    return K_hat, V_hat


# --------------------------------------------------------------------------
# Temporal predictor [TEMPO abstract, Fig. 2(b), appendix Table 7]
# --------------------------------------------------------------------------


def _frame_rows(desc: Desc):
    F = desc.frame_tokens
    T = desc.n_tokens
    n_frames = (T + F - 1) // F
    return [(f * F, min(T, (f + 1) * F)) for f in range(n_frames)]


def _history(hist, F, H, D, n_back):
    """Reconstructed frames before the first one of this call, oldest first,
    as a [n_back*F, H, D] block (zeros where absent)."""
    if hist is None:
        return np.zeros((n_back * F, H, D))
    return np.asarray(hist, dtype=np.float64).reshape(n_back * F, H, D)


def encode_layer_temporal(desc: Desc, w: dict, K, V, k_hist=None, v_hist=None):
    """Frame by frame in time order (readings R8, R9).

    w: ak [H,D,2D] over [K^_{f-1} | K^_{f-2}], av [H,D,2D] over [K^_f | V^_{f-1}].
    k_hist [2,F,H,D] (frames f0-2, f0-1) and v_hist [F,H,D] (frame f0-1), when
    given, continue an earlier sequence: frame 0 of this call is then predicted
    and coded at desc.bits.  Without them the codes of frame 0 are the anchor at
    desc.anchor_bits.  Returns (coded K, coded V, K^, V^) over all T tokens.
    """
    T, H, D = K.shape
    F = desc.frame_tokens
    cont = k_hist is not None
    K_hat = np.concatenate([_history(k_hist, F, H, D, 2), np.zeros((T, H, D))])
    V_hat = np.concatenate([_history(v_hist, F, H, D, 1), np.zeros((T, H, D))])
    ko, vo = 2 * F, F  # offsets of this call's frame 0 in K_hat / V_hat
    qk = np.zeros((T, H, D), np.uint8)
    qv = np.zeros((T, H, D), np.uint8)
    ng = D // desc.group
    sk, zk, sv, zv = (np.zeros((T, H, ng)) for _ in range(4))
    for f, (a, b) in enumerate(_frame_rows(desc)):
        n = b - a
        anchor = f == 0 and not cont
        bits = desc.anchor_bits if anchor else desc.bits
        if anchor:
            pk = np.zeros((n, H, D))
        else:
            k1 = K_hat[ko + a - F : ko + a - F + n]
            k2 = K_hat[ko + a - 2 * F : ko + a - 2 * F + n]  # zeros before frame 0 of a sequence
            pk = _blockdiag(np.concatenate([k1, k2], axis=-1), w["ak"])
        qk[a:b], sk[a:b], zk[a:b], K_hat[ko + a:ko + b] = code_residual(
            K[a:b], pk, bits, desc.group, desc.param, desc.state)
        if anchor:
            pv = np.zeros((n, H, D))
        else:
            v1 = V_hat[vo + a - F : vo + a - F + n]
            pv = _blockdiag(np.concatenate([K_hat[ko + a:ko + b], v1], axis=-1), w["av"])
        qv[a:b], sv[a:b], zv[a:b], V_hat[vo + a:vo + b] = code_residual(
            V[a:b], pv, bits, desc.group, desc.param, desc.state)
    return Coded(qk, sk, zk), Coded(qv, sv, zv), K_hat[ko:], V_hat[vo:]


def decode_layer_temporal(desc: Desc, w: dict, ck: Coded, cv: Coded, k_hist=None, v_hist=None):
    """Replays the frame chain of encode_layer_temporal from the codes."""
    T, H, D = ck.q.shape
    F = desc.frame_tokens
    cont = k_hist is not None
    K_hat = np.concatenate([_history(k_hist, F, H, D, 2), np.zeros((T, H, D))])
    V_hat = np.concatenate([_history(v_hist, F, H, D, 1), np.zeros((T, H, D))])
    ko, vo = 2 * F, F
    for f, (a, b) in enumerate(_frame_rows(desc)):
        n = b - a
        anchor = f == 0 and not cont
        if anchor:
            pk = np.zeros((n, H, D))
        else:
            k1 = K_hat[ko + a - F : ko + a - F + n]
            k2 = K_hat[ko + a - 2 * F : ko + a - 2 * F + n]
            pk = _blockdiag(np.concatenate([k1, k2], axis=-1), w["ak"])
        K_hat[ko + a:ko + b] = decode_residual(ck.q[a:b], ck.s[a:b], ck.z[a:b], pk, desc.group, desc.state)
        if anchor:
            pv = np.zeros((n, H, D))
        else:
            v1 = V_hat[vo + a - F : vo + a - F + n]
            pv = _blockdiag(np.concatenate([K_hat[ko + a:ko + b], v1], axis=-1), w["av"])
        V_hat[vo + a:vo + b] = decode_residual(cv.q[a:b], cv.s[a:b], cv.z[a:b], pv, desc.group, desc.state)
    return K_hat[ko:], V_hat[vo:]


# --------------------------------------------------------------------------
# Clustered predictor [NANO abstract]
# --------------------------------------------------------------------------


def cluster_scores(X, centroids) -> np.ndarray:
    """Assignment scores |c_j|^2 - 2 x.c_j (the |x|^2 term is common to all j)."""
    return (centroids * centroids).sum(axis=1)[None, :] - 2.0 * (X @ centroids.T)


def cluster_assign(X, centroids) -> np.ndarray:
    """Nearest centre, ties to the lowest index (reading R10)."""
    return np.argmin(cluster_scores(X, centroids), axis=1)


def encode_tensor_cluster(desc: Desc, X, centroids, enc, dec):
    """X [T,H,D] -> (Coded with assign, x_hat [T,H,D]).

    enc [m,C] maps the residual x - c_a to m coefficients, dec [C,m] maps the
    dequantized coefficients back; groups run over the m coefficients.
    """
    T, H, D = X.shape
    flat = X.reshape(T, H * D)
    a = cluster_assign(flat, centroids)
    coef = (flat - centroids[a]) @ enc.T
    q, s, z = quantize_groups(coef, desc.bits, desc.group, desc.param)
    coef_hat = dequantize_groups(q, s, z, desc.group)
    x_hat = round_to(centroids[a] + coef_hat @ dec.T, desc.state).reshape(T, H, D)
    return Coded(q, s, z, a.astype(np.int64)), x_hat


def decode_tensor_cluster(desc: Desc, c: Coded, centroids, dec, exact: bool = False):
    """x_hat = c_a + W_dec coef_hat, rounded to the state dtype unless `exact`."""
    coef_hat = dequantize_groups(c.q, c.s, c.z, desc.group)
    x = centroids[c.assign] + coef_hat @ dec.T
    T = c.q.shape[0]
    x = x if exact else round_to(x, desc.state)
    return x.reshape(T, desc.n_heads, desc.head_dim)


# --------------------------------------------------------------------------
# Attention over the decoded history [NANO abstract: attention over history]
# --------------------------------------------------------------------------


def _gqa(Q, X):
    """Key / value heads repeated for the query heads that read them."""
    g = Q.shape[1] // X.shape[1]
    return X if g == 1 else np.repeat(np.asarray(X), g, axis=1)


def attention(Q, K, V, scale: float) -> np.ndarray:
    """Naive two-pass softmax attention, fp64.

    Q [Nq,Hq,D], K [Nk,H,D], V [Nk,H,D] -> O [Nq,Hq,D];
    m = max_k s, p = exp(s - m), o = sum p v / sum p.  Hq a multiple of H:
    query head j reads head j // (Hq // H) (grouped-query attention).
    """
    K, V = _gqa(Q, K), _gqa(Q, V)
    S = np.matmul(Q.transpose(1, 0, 2), K.transpose(1, 2, 0)) * scale  # [H,Nq,Nk]
    m = S.max(axis=-1, keepdims=True)
    p = np.exp(S - m)
    O = np.matmul(p, V.transpose(1, 0, 2)) / p.sum(axis=-1, keepdims=True)  # [H,Nq,D]
    return O.transpose(1, 0, 2)


def jensen_correction(Q, s_hist, group: int, scale: float) -> np.ndarray:
    """Jensen-bias term of every (head, query, quantized key): [H, Nq, T].

    (The abstract on the "Jensen bias" of INT2 key caches, among the related
    papers listed on the CORAL-KV page.)  Uniform rounding noise of step s
    on a key raises E[exp(scale q.k^)] by exp(0.5 scale^2 sum_g |q_g|^2 s_g^2/12)
    to second order; this is that exponent."""
    Nq, H, D = Q.shape
    qn = (Q.reshape(Nq, H, D // group, group) ** 2).sum(-1)  # [Nq,H,NG]
    var = np.asarray(s_hist, np.float64) ** 2 / 12.0  # [T,H,NG]
    return 0.5 * scale * scale * np.einsum("qhg,thg->hqt", qn, var)


def attention_corrected(Q, K, V, scale: float, n_hist: int, s_hist, group: int) -> np.ndarray:
    """Naive attention whose first n_hist (quantized) keys have their scores
    lowered by the Jensen-bias term; the remaining keys are uncompressed."""
    K, V, s_hist = _gqa(Q, K), _gqa(Q, V), _gqa(Q, s_hist)
    S = np.matmul(Q.transpose(1, 0, 2), K.transpose(1, 2, 0)) * scale  # [H,Nq,Nk]
    S[:, :, :n_hist] -= jensen_correction(Q, s_hist, group, scale)
    m = S.max(axis=-1, keepdims=True)
    p = np.exp(S - m)
    O = np.matmul(p, V.transpose(1, 0, 2)) / p.sum(axis=-1, keepdims=True)
    return O.transpose(1, 0, 2)


def mixed_attention(Q, ck: Coded, cent_k, dec_k, cv: Coded, cent_v, dec_v,
                    desc: Desc, scale: float) -> np.ndarray:
    """Attention computed on the stored coefficients (reading R11).

    score(q,h,t) = scale * (q_h . c_{a(t),h} + (W_dec,h^T q_h) . coef_hat_t)
    o_h = sum_j m_j c^V_{j,h} + W^V_dec,h (sum_t p_t coef_hat^V_t).
    """
    H, D = desc.n_heads, desc.head_dim
    Nq = Q.shape[0]
    ck_hat = dequantize_groups(ck.q, ck.s, ck.z, desc.group)  # [T,m]
    cv_hat = dequantize_groups(cv.q, cv.s, cv.z, desc.group)
    n_c = cent_v.shape[0]
    O = np.zeros((Nq, H, D))
    for h in range(H):
        sl = slice(h * D, (h + 1) * D)
        qh = Q[:, h, :]  # [Nq,D]
        table = qh @ cent_k[:, sl].T  # [Nq,n_centres]
        qt = qh @ dec_k[sl, :]  # [Nq,m]
        S = scale * (table[:, ck.assign] + qt @ ck_hat.T)  # [Nq,T]
        m = S.max(axis=-1, keepdims=True)
        p = np.exp(S - m)
        p = p / p.sum(axis=-1, keepdims=True)
        onehot = np.zeros((ck.q.shape[0], n_c))
        onehot[np.arange(ck.q.shape[0]), cv.assign] = 1.0
        mass = p @ onehot  # [Nq,n_centres]
        cbar = p @ cv_hat  # [Nq,m]
        O[:, h, :] = mass @ cent_v[:, sl] + cbar @ dec_v[sl, :].T
    return O


# --------------------------------------------------------------------------
# Full-layer helpers used by the tests and the timed baseline
# --------------------------------------------------------------------------


def attend_compressed_xlayer(desc: Desc, w: dict, Q, ck: Coded, cv: Coded, K_src, V_src,
                             K_self, V_self, scale: float) -> np.ndarray:
    """Softmax attention of Q over [decoded history ; uncompressed chunk]."""
    K_hist, V_hist = decode_layer_xlayer(desc, w, ck, cv, K_src, V_src)
    if K_self is not None and len(K_self):
        K_all = np.concatenate([K_hist, K_self], axis=0)
        V_all = np.concatenate([V_hist, V_self], axis=0)
    else:
        K_all, V_all = K_hist, V_hist
    return attention(Q, K_all, V_all, scale)


# --------------------------------------------------------------------------
# Video-adapted block-DPLR refit [CORAL Fig. 4]
# --------------------------------------------------------------------------


def refit_block_diag(X0, X1, Y, w_lr, u_lr, ridge: float) -> np.ndarray:
    """Each head's block refitted on a filled cache block with the low-rank
    factors fixed (reading V1): B_h^T = (X_h^T X_h + ridge I)^-1 X_h^T (Y_h - LR_h)
    with X_h = X0_h (K) or [X0_h | X1_h] (V) and LR the fixed low-rank term."""
    X0 = np.asarray(X0, np.float64)
    T, H, D = X0.shape
    flat = X0.reshape(T, H * D) if X1 is None else np.concatenate(
        [X0.reshape(T, H * D), np.asarray(X1, np.float64).reshape(T, H * D)], axis=1)
    lr = _lowrank(flat, None if w_lr is None else np.asarray(w_lr, np.float64),
                  None if u_lr is None else np.asarray(u_lr, np.float64), T, H, D)
    R = np.asarray(Y, np.float64) - lr
    Xh = X0 if X1 is None else np.concatenate([X0, np.asarray(X1, np.float64)], axis=-1)  # [T,H,din]
    din = Xh.shape[-1]
    out = np.empty((H, D, din))
    for h in range(H):
        G = Xh[:, h, :].T @ Xh[:, h, :] + ridge * np.eye(din)
        out[h] = np.linalg.solve(G, Xh[:, h, :].T @ R[:, h, :]).T
    return out


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


