"""Pins of the fp64 oracles against what the pages and the mathematics fix.

Each test checks an oracle against something other than itself: a library
routine, a value printed on the pages (tests/golden), a hand-worked example, a
closed form, an invariant, or brute force on tiny inputs.  Every test runs on
both oracles: the plain single-threaded C++ one (oracle/kvc_oracle.cpp, the
parity reference of the GPU tests) and the numpy one (oracle/kvc_oracle.py).
None needs a GPU.
"""

import json
import os

import numpy as np
import pytest
import torch

from oracle import kvc_oracle as O_NUMPY
from oracle import kvc_oracle_c as O_CPP

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(20261202)


@pytest.fixture(params=["cpp", "numpy"])
def O(request):
    return O_CPP if request.param == "cpp" else O_NUMPY


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- rounding


def test_round_to_f16_f32_match_numpy_casts(O):
    x = RNG.standard_normal(200_000) * np.exp2(RNG.integers(-30, 20, 200_000))
    # exact ties of both formats
    ties = np.array([1 + 2.0**-11, 1 + 3 * 2.0**-11, 2049.0, 2051.0, 1 + 2.0**-24, 1 + 3 * 2.0**-24,
                     65519.99, 65520.0, 2.0**-25, 3 * 2.0**-25, 6e-8])
    x = np.concatenate([x, ties, -ties])
    with np.errstate(over="ignore"):
        ref16 = x.astype(np.float16).astype(np.float64)
    np.testing.assert_array_equal(O.round_to(x, "f16"), ref16)
    np.testing.assert_array_equal(O.round_to(x, "f32"), x.astype(np.float32).astype(np.float64))


def test_round_to_bf16_matches_torch_on_float32_inputs(O):
    x32 = (RNG.standard_normal(200_000) * np.exp2(RNG.integers(-40, 40, 200_000))).astype(np.float32)
    ties = np.array([1 + 2.0**-8, 1 + 3 * 2.0**-8, 257.0, 259.0, -(1 + 2.0**-8)], np.float32)
    x32 = np.concatenate([x32, ties])
    ref = torch.from_numpy(x32).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(O.round_to(x32.astype(np.float64), "bf16"), ref)


# ---------------------------------------------------------------- quantizer


@pytest.mark.parametrize("bits,group,param", [(2, 32, "f16"), (4, 32, "f16"), (4, 64, "f16"),
                                              (4, 32, "f32"), (8, 16, "f16")])
def test_quantizer_matches_brute_force_nearest_level(O, bits, group, param):
    r = RNG.standard_normal((64, 4 * group)) * np.exp2(RNG.integers(-3, 4, (64, 1)))
    q, s, z = O.quantize_groups(r, bits, group, param)
    L = (1 << bits) - 1
    rg = r.reshape(64, 4, group)
    levels = z[..., None, None] + s[..., None, None] * np.arange(L + 1)  # [64,4,1,L+1]
    dist = np.abs(rg[..., None] - levels)
    best = dist.argmin(-1)
    qg = q.reshape(64, 4, group)
    srt = np.sort(dist, axis=-1)
    tie = (srt[..., 1] - srt[..., 0]) < 1e-12 * (1 + np.abs(rg))
    assert np.all((best == qg) | tie)
    # error bound: half a step, plus what fp rounding of s and z moved the grid
    mn, mx = rg.min(-1), rg.max(-1)
    s_exact = (mx - mn) / L
    bound = s / 2 + np.abs(z - mn) + L * np.abs(s - s_exact) + 1e-12
    err = np.abs(rg - O.dequantize_groups(q, s, z, group).reshape(64, 4, group))
    assert np.all(err <= bound[..., None])
    assert np.all(q <= L)


def test_quantizer_degenerate_group_and_exact_grid(O):
    r = np.full((3, 32), 0.3)
    q, s, z = O.quantize_groups(r, 2, 32, "f16")
    assert np.all(q == 0) and np.all(s == 0)
    np.testing.assert_array_equal(z, np.float16(0.3).astype(np.float64))
    # values exactly on a representable grid with both ends present: lossless
    grid = -1.5 + 1.0 * RNG.integers(0, 4, (5, 32))
    grid[:, 0], grid[:, 1] = -1.5, 1.5
    q, s, z = O.quantize_groups(grid, 2, 32, "f16")
    np.testing.assert_array_equal(O.dequantize_groups(q, s, z, 32), grid)


# ---------------------------------------------------------------- packing


def test_pack_hand_worked_examples(O):
    for case in _golden("pack_worked_example.json")["cases"]:
        codes = np.array(case["codes"], np.uint8)
        got = O.pack_codes(codes, case["bits"])
        assert got.tolist() == case["bytes"], case
        np.testing.assert_array_equal(O.unpack_codes(got, case["bits"], len(codes)), codes)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_pack_matches_numpy_unpackbits(O, bits):
    codes = RNG.integers(0, 1 << bits, (17, 128)).astype(np.uint8)
    packed = O.pack_codes(codes, bits)
    assert packed.shape == (17, 128 * bits // 8)
    bitstr = np.unpackbits(packed, axis=-1, bitorder="little").reshape(17, 128, bits)
    rebuilt = (bitstr * (1 << np.arange(bits))).sum(-1)
    np.testing.assert_array_equal(rebuilt, codes)


# ---------------------------------------------------------------- storage accounting


def test_group_quantizer_ratios_printed_on_pages(O):
    g = _golden("page_compression_ratios.json")
    for key in ("int2_group_quantizer", "int4_group_quantizer"):
        e = g[key]
        d = O.Desc(n_tokens=1000, n_heads=12, head_dim=128, bits=e["bits"], group=32)
        elems = 2 * 1000 * 12 * 128
        ratio = 16.0 * elems / (8 * O.codes_bytes(d))
        assert round(ratio, e["printed_decimals"]) == pytest.approx(e["ratio"]), key
        assert ratio == pytest.approx(16.0 / O_NUMPY.bits_per_element(e["bits"], 32, "f16"))


def test_tempokv_anchor_sweep_slope(O):
    """One anchor latent frame among ~180 (717 video frames): each extra anchor
    bit costs 1/180 bit per element; the printed ratios give the same slope."""
    e = _golden("page_compression_ratios.json")["tempokv_anchor_sweep"]
    printed_bits = 16.0 / np.array(e["ratio"])
    n_lat = (e["video_frames"] - 1) // 4 + 1
    F, H, D = 16, 2, 64
    model = []
    for ab in e["anchor_bits"]:
        d = O.Desc(n_tokens=n_lat * F, n_heads=H, head_dim=D, bits=2, group=32, frame_tokens=F, anchor_bits=ab)
        model.append(O.codes_bytes(d, "temporal") * 8 / (2 * n_lat * F * H * D))
    model = np.array(model)
    tol = 2 * 16.0 * 0.5 * 10.0 ** -e["printed_decimals"] / np.array(e["ratio"]) ** 2
    np.testing.assert_array_less(np.abs(np.diff(printed_bits) - np.diff(model)), tol[1:] + tol[:-1])


# ---------------------------------------------------------------- cross-layer predictor


def _dense_dplr(block, w, u, H, D, Din_head, Cin_order):
    """Dense Cin x C matrix of a block-DPLR map, built entry by entry."""
    Cin = w.shape[1]
    C = H * D
    M = np.zeros((Cin, C))
    for h in range(H):
        for o in range(D):
            for i in range(Din_head):
                M[Cin_order(h, i), h * D + o] += block[h, o, i]
    M += w.T @ u.T
    return M


def test_dplr_prediction_equals_dense_map(O):
    H, D, r, T = 3, 8, 2, 11
    rng = np.random.default_rng(1)
    Ks, Vs = rng.standard_normal((T, H, D)), rng.standard_normal((T, H, D))
    kb, vb = rng.standard_normal((H, D, D)), rng.standard_normal((H, D, 2 * D))
    kw, ku = rng.standard_normal((r, H * D)), rng.standard_normal((H * D, r))
    vw, vu = rng.standard_normal((r, 2 * H * D)), rng.standard_normal((H * D, r))
    Mk = _dense_dplr(kb, kw, ku, H, D, D, lambda h, i: h * D + i)
    got = O.xlayer_predict_k(Ks, kb, kw, ku).reshape(T, -1)
    np.testing.assert_allclose(got, Ks.reshape(T, -1) @ Mk, rtol=1e-12, atol=1e-12)
    # V's per-head input is [K_h | V_h]; its global input is [K (all heads) | V (all heads)]
    Mv = _dense_dplr(vb, vw, vu, H, D, 2 * D,
                     lambda h, i: h * D + i if i < D else H * D + h * D + (i - D))
    flat = np.concatenate([Ks.reshape(T, -1), Vs.reshape(T, -1)], axis=1)
    got = O.xlayer_predict_v(Ks, Vs, vb, vw, vu).reshape(T, -1)
    np.testing.assert_allclose(got, flat @ Mv, rtol=1e-12, atol=1e-12)
    # rank 0 is the pure block-diagonal map
    got0 = O.xlayer_predict_k(Ks, kb, kw[:0], ku[:, :0]).reshape(T, -1)
    np.testing.assert_allclose(got0, Ks.reshape(T, -1) @ _dense_dplr(kb, kw[:0], ku[:, :0], H, D, D,
                                                                      lambda h, i: h * D + i), rtol=1e-12)


def test_low_rank_latent_is_not_rounded(O):
    """The latent passes to the second factor at full precision: with U = I
    the first r outputs of a zero-block map are x W^T exactly."""
    H, D, r, T = 2, 4, 3, 5
    rng = np.random.default_rng(2)
    Ks = rng.standard_normal((T, H, D))
    kb = np.zeros((H, D, D))
    kw, ku = rng.standard_normal((r, H * D)), np.eye(H * D, r)
    got = O.xlayer_predict_k(Ks, kb, kw, ku).reshape(T, -1)[:, :r]
    ref = np.einsum("tc,jc->tj", Ks.reshape(T, -1), kw)
    np.testing.assert_allclose(got, ref, rtol=1e-14, atol=1e-14)
    assert not np.array_equal(got, O.round_to(got, "bf16"))


def _grid_values(rng, shape):
    """Values in {-1.5,-0.5,0.5,1.5} with both ends in every 32-group: INT2 lossless."""
    v = -1.5 + rng.integers(0, 4, shape).astype(np.float64)
    v[..., 0::32] = -1.5
    v[..., 1::32] = 1.5
    return v


def test_exact_predictor_gives_zero_residual(O):
    H, D, r, T = 2, 64, 4, 40
    rng = np.random.default_rng(3)
    K0, V0 = _grid_values(rng, (T, H, D)), _grid_values(rng, (T, H, D))
    d0 = O.Desc(T, H, D, state="bf16", bits=2, group=32)
    ck0, cv0, K0h, V0h = O.encode_layer_none(d0, K0, V0)
    np.testing.assert_array_equal(K0h, K0)  # anchor lossless on its grid

    def sparse(shape, nnz_per_row):
        m = np.zeros(shape)
        for idx in np.ndindex(*shape[:-1]):
            cols = rng.choice(shape[-1], nnz_per_row, replace=False)
            m[idx + (cols,)] = rng.choice([-1.0, 1.0], nnz_per_row)
        return m

    w = dict(k_block=sparse((H, D, D), 3), k_w=sparse((r, H * D), 3), k_u=sparse((H * D, r), 2),
             v_block=sparse((H, D, 2 * D), 3), v_w=sparse((r, 2 * H * D), 3), v_u=sparse((H * D, r), 2))
    Mk = _dense_dplr(w["k_block"], w["k_w"], w["k_u"], H, D, D, lambda h, i: h * D + i)
    K1 = (K0.reshape(T, -1) @ Mk).reshape(T, H, D)
    Mv = _dense_dplr(w["v_block"], w["v_w"], w["v_u"], H, D, 2 * D,
                     lambda h, i: h * D + i if i < D else H * D + h * D + (i - D))
    V1 = (np.concatenate([K1.reshape(T, -1), V0.reshape(T, -1)], 1) @ Mv).reshape(T, H, D)
    assert np.array_equal(O.round_to(K1, "bf16"), K1) and np.array_equal(O.round_to(V1, "bf16"), V1)
    ck, cv, K1h, V1h = O.encode_layer_xlayer(d0, w, K1, V1, K0h, V0h)
    for c in (ck, cv):
        assert np.all(c.q == 0) and np.all(c.s == 0)
    np.testing.assert_array_equal(K1h, K1)
    np.testing.assert_array_equal(V1h, V1)


def _chain_workload(O, L=6, T=300, H=2, D=64, r=4, seed=5):
    rng = np.random.default_rng(seed)
    C = H * D
    K = [rng.standard_normal((T, H, D))]
    V = [rng.standard_normal((T, H, D))]
    W = [None]
    for _ in range(1, L):
        w = dict(k_block=0.9 * np.stack([np.linalg.qr(rng.standard_normal((D, D)))[0] for _ in range(H)]),
                 k_w=rng.standard_normal((r, C)) / np.sqrt(C), k_u=0.1 * rng.standard_normal((C, r)),
                 v_block=0.5 * rng.standard_normal((H, D, 2 * D)) / np.sqrt(2 * D),
                 v_w=rng.standard_normal((r, 2 * C)) / np.sqrt(2 * C), v_u=0.1 * rng.standard_normal((C, r)))
        w = {k: O.round_to(v, "bf16") for k, v in w.items()}
        W.append(w)
        K.append(O.round_to(O.xlayer_predict_k(K[-1], w["k_block"], w["k_w"], w["k_u"])
                            + 0.3 * rng.standard_normal((T, H, D)), "bf16"))
        V.append(O.round_to(O.xlayer_predict_v(K[-1], V[-1], w["v_block"], w["v_w"], w["v_u"])
                            + 0.3 * rng.standard_normal((T, H, D)), "bf16"))
    K[0], V[0] = O.round_to(K[0], "bf16"), O.round_to(V[0], "bf16")
    return K, V, W


def test_closed_loop_error_does_not_accumulate_and_decode_replays_encode(O):
    K, V, W = _chain_workload(O)
    T, H, D = K[0].shape
    d_anchor = O.Desc(T, H, D, bits=4, group=32)
    d = O.Desc(T, H, D, bits=2, group=32)
    ck, cv, Kh, Vh = O.encode_layer_none(d_anchor, K[0], V[0])
    Kd, Vd = O.decode_layer_none(d_anchor, ck, cv)
    np.testing.assert_array_equal(Kd, Kh)
    open_K = Kh  # decoder-side state of an open-loop encoder
    open_err = []
    for l in range(1, len(K)):
        Ks, Vs = Kh, Vh
        ck, cv, Kh, Vh = O.encode_layer_xlayer(d, W[l], K[l], V[l], Ks, Vs)
        Kd, Vd = O.decode_layer_xlayer(d, W[l], ck, cv, Ks, Vs)
        np.testing.assert_array_equal(Kd, Kh)
        np.testing.assert_array_equal(Vd, Vh)
        # closed loop: the error of every layer is its own quantization error only
        for x, xh, c in ((K[l], Kh, ck), (V[l], Vh, cv)):
            s = np.repeat(c.s, 32, axis=-1)
            assert np.all(np.abs(x - xh) <= 0.5 * s + 2.0 ** -7 * np.abs(x) + 1e-3 * s + 1e-30)
        # open loop: predict from clean K_{l-1}; the decoder only has its own state
        pk_clean = O.xlayer_predict_k(K[l - 1], W[l]["k_block"], W[l]["k_w"], W[l]["k_u"])
        qo, so, zo = O.quantize_groups(K[l] - pk_clean, 2, 32, "f16")
        pk_dec = O.xlayer_predict_k(open_K, W[l]["k_block"], W[l]["k_w"], W[l]["k_u"])
        open_K = O.round_to(pk_dec + O.dequantize_groups(qo, so, zo, 32), "bf16")
        open_err.append(np.abs(open_K - K[l]).max() / np.repeat(so, 32, -1).max())
    assert open_err[-1] > 0.75  # drift beyond the half-step bound the closed loop keeps


# ---------------------------------------------------------------- temporal predictor


def test_temporal_exact_predictor_and_ragged_frame(O):
    H, D, F = 2, 64, 10
    T = 4 * F + 3  # ragged last frame
    rng = np.random.default_rng(7)
    ak = np.zeros((H, D, 2 * D))
    av = np.zeros((H, D, 2 * D))
    for h in range(H):
        ak[h, :, :D] = 0.5 * np.eye(D)  # K_f = 0.5 K_{f-1} + 0.5 K_{f-2}
        ak[h, :, D:] = 0.5 * np.eye(D)
        av[h, :, :D] = np.eye(D)[rng.permutation(D)]  # V_f = P K_f + 0.5 V_{f-1}
        av[h, :, D:] = 0.5 * np.eye(D)
    K = np.zeros((T, H, D))
    V = np.zeros((T, H, D))
    K[:F] = _grid_values(rng, (F, H, D))
    V[:F] = _grid_values(rng, (F, H, D))
    for f in range(1, 5):
        a, b = f * F, min(T, (f + 1) * F)
        n = b - a
        k1 = K[a - F:a - F + n]
        k2 = K[a - 2 * F:a - 2 * F + n] if f >= 2 else 0.0
        K[a:b] = 0.5 * k1 + 0.5 * k2
        V[a:b] = np.einsum("thi,hoi->tho", K[a:b], av[:, :, :D]) + 0.5 * V[a - F:a - F + n]
    assert np.array_equal(O.round_to(K, "bf16"), K) and np.array_equal(O.round_to(V, "bf16"), V)
    d = O.Desc(T, H, D, bits=2, group=32, frame_tokens=F, anchor_bits=2)
    ck, cv, Kh, Vh = O.encode_layer_temporal(d, dict(ak=ak, av=av), K, V)
    np.testing.assert_array_equal(Kh, K)
    np.testing.assert_array_equal(Vh, V)
    assert np.all(ck.s[F:] == 0) and np.all(cv.s[F:] == 0)
    Kd, Vd = O.decode_layer_temporal(d, dict(ak=ak, av=av), ck, cv)
    np.testing.assert_array_equal(Kd, K)
    np.testing.assert_array_equal(Vd, V)


def test_temporal_lag_order_with_asymmetric_maps(O):
    """The K map's first D inputs read frame f-1 and its last D read frame f-2
    (reading R9).  Frames built exactly as K_f = K_{f-1} + 0.5 P K_{f-2} (P a
    permutation) code to zero residuals; a coder with the two lags swapped
    would predict 0.5 P K_{f-1} + K_{f-2} and leave non-zero residuals."""
    H, D, F = 2, 64, 8
    T = 3 * F + 3  # few enough frames for every value to stay exact in bf16
    rng = np.random.default_rng(15)
    ak = np.zeros((H, D, 2 * D))
    av = np.zeros((H, D, 2 * D))
    for h in range(H):
        ak[h, :, :D] = np.eye(D)  # lag 1
        ak[h, :, D:] = 0.5 * np.eye(D)[rng.permutation(D)]  # lag 2
        av[h, :, :D] = np.eye(D)[rng.permutation(D)]
        av[h, :, D:] = 0.5 * np.eye(D)
    K = np.zeros((T, H, D))
    V = np.zeros((T, H, D))
    K[:F] = _grid_values(rng, (F, H, D))
    V[:F] = _grid_values(rng, (F, H, D))
    for f in range(1, 4):
        a, b = f * F, min(T, (f + 1) * F)
        n = b - a
        k2 = K[a - 2 * F:a - 2 * F + n] if f >= 2 else np.zeros((n, H, D))
        K[a:b] = K[a - F:a - F + n] + np.einsum("thi,hoi->tho", k2, ak[:, :, D:])
        V[a:b] = np.einsum("thi,hoi->tho", K[a:b], av[:, :, :D]) + 0.5 * V[a - F:a - F + n]
    assert np.array_equal(O_NUMPY.round_to(K, "bf16"), K) and np.array_equal(O_NUMPY.round_to(V, "bf16"), V)
    d = O.Desc(T, H, D, bits=2, group=32, frame_tokens=F, anchor_bits=2)
    ck, cv, Kh, Vh = O.encode_layer_temporal(d, dict(ak=ak, av=av), K, V)
    np.testing.assert_array_equal(Kh, K)
    np.testing.assert_array_equal(Vh, V)
    assert np.all(ck.s[F:] == 0) and np.all(cv.s[F:] == 0)
    swapped = np.concatenate([ak[:, :, D:], ak[:, :, :D]], axis=-1)
    ck2, _, _, _ = O.encode_layer_temporal(d, dict(ak=swapped, av=av), K, V)
    assert np.any(ck2.s[2 * F:] > 0)


def test_cluster_storage_closed_form(O):
    """Per token and tensor: code_dim b-bit codes, one (scale, zero) pair of
    two fp16 values per group, and a one-byte centre index (256 centres fit in
    8 bits); for the 128 INT4 g32 coefficients that is 64 + 16 + 1 = 81 bytes."""
    for T, m, bits, group, param in ((32768, 128, 4, 32, "f16"), (1000, 128, 2, 32, "f16"),
                                     (7, 64, 8, 16, "f32")):
        d = O.Desc(T, 16, 128, bits=bits, group=group, param=param)
        pair = 2 * (2 if param == "f16" else 4)
        per_token = m * bits // 8 + (m // group) * pair + 1
        assert O.codes_bytes(d, "cluster", m) == 2 * T * per_token
    assert O.codes_bytes(O.Desc(1, 16, 128, bits=4, group=32), "cluster", 128) == 2 * 81


def test_temporal_continuation_equals_one_sequence(O):
    """Coding frames [0, 3) and then [3, 5) from the reconstructed history
    (K of frames 1 and 2, V of frame 2) gives the codes of one 5-frame call."""
    H, D, F = 2, 64, 12
    rng = np.random.default_rng(14)
    T = 5 * F
    K = O.round_to(rng.standard_normal((T, H, D)), "bf16")
    V = O.round_to(rng.standard_normal((T, H, D)), "bf16")
    w = dict(ak=rng.standard_normal((H, D, 2 * D)) * 0.05, av=rng.standard_normal((H, D, 2 * D)) * 0.05)
    d = O.Desc(T, H, D, bits=2, group=32, frame_tokens=F, anchor_bits=4)
    ck, cv, Kh, Vh = O.encode_layer_temporal(d, w, K, V)
    d1 = O.Desc(3 * F, H, D, bits=2, group=32, frame_tokens=F, anchor_bits=4)
    ck1, cv1, Kh1, Vh1 = O.encode_layer_temporal(d1, w, K[:3 * F], V[:3 * F])
    d2 = O.Desc(2 * F, H, D, bits=2, group=32, frame_tokens=F, anchor_bits=0)
    kh = Kh1[F:3 * F].reshape(2, F, H, D)
    ck2, cv2, Kh2, Vh2 = O.encode_layer_temporal(d2, w, K[3 * F:], V[3 * F:], kh, Vh1[2 * F:])
    np.testing.assert_array_equal(np.concatenate([ck1.q, ck2.q]), ck.q)
    np.testing.assert_array_equal(np.concatenate([cv1.q, cv2.q]), cv.q)
    np.testing.assert_array_equal(np.concatenate([Vh1, Vh2]), Vh)
    Kd, Vd = O.decode_layer_temporal(d2, w, ck2, cv2, kh, Vh1[2 * F:])
    np.testing.assert_array_equal(Kd, Kh2)
    # a continued call stores every frame at `bits`
    assert O.codes_bytes(d2, "temporal") == 2 * 2 * F * H * (D * 2 // 8 + 2 * 2 * 2)


def test_temporal_frame_zero_is_plain_group_rtn_at_anchor_bits(O):
    H, D, F, T = 2, 64, 8, 20
    rng = np.random.default_rng(8)
    K = O.round_to(rng.standard_normal((T, H, D)), "bf16")
    V = O.round_to(rng.standard_normal((T, H, D)), "bf16")
    w = dict(ak=rng.standard_normal((H, D, 2 * D)) * 0.05, av=rng.standard_normal((H, D, 2 * D)) * 0.05)
    d = O.Desc(T, H, D, bits=2, group=32, frame_tokens=F, anchor_bits=4)
    ck, _, Kh, _ = O.encode_layer_temporal(d, w, K, V)
    assert ck.q[:F].max() > 3  # anchor rows use 4-bit codes
    assert ck.q[F:].max() <= 3
    # frame 0 against brute-force nearest level at 4 bits
    q, s, z = ck.q[:F], ck.s[:F], ck.z[:F]
    lv = z[..., None] + s[..., None] * np.arange(16)
    dist = np.abs(K[:F].reshape(F, H, 2, 32)[..., None] - lv[:, :, :, None, :])
    assert np.mean(dist.argmin(-1) == q.reshape(F, H, 2, 32)) > 0.999


# ---------------------------------------------------------------- clustered predictor


def test_cluster_assignment_is_nearest_centre_by_euclidean_distance(O):
    rng = np.random.default_rng(9)
    cent = rng.standard_normal((16, 64))
    X = cent[rng.integers(0, 16, 200)] + 0.3 * rng.standard_normal((200, 64))
    a = O.cluster_assign(X, cent)
    brute = np.array([min(range(16), key=lambda j: float(np.sum((x - cent[j]) ** 2))) for x in X])
    np.testing.assert_array_equal(a, brute)
    # ties go to the lowest index
    cent2 = np.stack([cent[0], cent[0], cent[1]])
    assert O.cluster_assign(cent[:1], cent2)[0] == 0


def test_cluster_codec_is_exact_when_residual_is_on_grid_in_decoder_span(O):
    H, D, m, T, nc = 2, 32, 32, 24, 4
    C = H * D
    rng = np.random.default_rng(10)
    E, _ = np.linalg.qr(rng.standard_normal((C, m)))
    # an orthonormal basis made of signed unit vectors keeps every product exact
    E = np.zeros((C, m))
    E[rng.permutation(C)[:m], np.arange(m)] = rng.choice([-1.0, 1.0], m)
    cent = np.round(rng.standard_normal((nc, C)) * 4) * 4.0  # far apart, integers
    coef = _grid_values(rng, (T, m))  # on the INT2 grid of each 32-group
    a = rng.integers(0, nc, T)
    X = (cent[a] + coef @ E.T).reshape(T, H, D)
    d = O.Desc(T, H, D, bits=2, group=32)
    c, xh = O.encode_tensor_cluster(d, X, cent, E.T, E)
    np.testing.assert_array_equal(c.assign, a)
    np.testing.assert_array_equal(xh, X)
    np.testing.assert_array_equal(O.decode_tensor_cluster(d, c, cent, E), X)


# ---------------------------------------------------------------- attention


def test_attention_matches_torch_sdpa_in_float64(O):
    rng = np.random.default_rng(11)
    Q, K, V = rng.standard_normal((7, 3, 16)), rng.standard_normal((29, 3, 16)), rng.standard_normal((29, 3, 16))
    got = O.attention(Q, K, V, 0.37)
    t = lambda x: torch.from_numpy(x).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(t(Q), t(K), t(V), scale=0.37)[0].permute(1, 0, 2)
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-13)


def test_attention_special_cases(O):
    rng = np.random.default_rng(12)
    Q = rng.standard_normal((4, 2, 8))
    K1 = np.repeat(rng.standard_normal((1, 2, 8)), 9, axis=0)
    V = rng.standard_normal((9, 2, 8))
    np.testing.assert_allclose(O.attention(Q, K1, V, 1.0), np.broadcast_to(V.mean(0), (4, 2, 8)), atol=1e-13)
    np.testing.assert_allclose(O.attention(Q, K1[:1], V[:1], 1.0), np.broadcast_to(V[0], (4, 2, 8)), atol=1e-14)
    K = rng.standard_normal((9, 2, 8))
    shift = np.zeros_like(K) + rng.standard_normal((1, 2, 8))  # q.shift is constant over keys
    np.testing.assert_allclose(O.attention(Q, K + shift, V, 0.5), O.attention(Q, K, V, 0.5), atol=1e-12)


def test_mixed_attention_equals_attention_on_reconstructed_keys(O):
    H, D, m, T, nc = 2, 32, 16, 50, 8
    C = H * D
    rng = np.random.default_rng(13)
    E, _ = np.linalg.qr(rng.standard_normal((C, m)))
    cent_k, cent_v = rng.standard_normal((nc, C)), rng.standard_normal((nc, C))
    K = (cent_k[rng.integers(0, nc, T)] + 0.2 * rng.standard_normal((T, C))).reshape(T, H, D)
    V = (cent_v[rng.integers(0, nc, T)] + 0.2 * rng.standard_normal((T, C))).reshape(T, H, D)
    d = O.Desc(T, H, D, bits=4, group=16)
    ck, _ = O.encode_tensor_cluster(d, K, cent_k, E.T, E)
    cv, _ = O.encode_tensor_cluster(d, V, cent_v, E.T, E)
    Q = rng.standard_normal((6, H, D))
    fast = O.mixed_attention(Q, ck, cent_k, E, cv, cent_v, E, d, 0.25)
    Kx = O.decode_tensor_cluster(d, ck, cent_k, E, exact=True)
    Vx = O.decode_tensor_cluster(d, cv, cent_v, E, exact=True)
    np.testing.assert_allclose(fast, O.attention(Q, Kx, Vx, 0.25), rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- Jensen-bias correction


def test_jensen_correction_is_the_second_order_log_moment_of_rounding_noise(O):
    """A key rounded with step s carries noise e ~ U(-s/2, s/2) per element, and
    log E[exp(a e)] = log(sinh(a s / 2) / (a s / 2)) exactly; its second-order
    term a^2 s^2 / 24 summed over the channels is the correction.  One quantized
    history key and one chunk key with the same k: the ratio of their weights
    is exp(-correction)."""
    rng = np.random.default_rng(16)
    D, group, scale = 64, 32, 0.3
    q = rng.standard_normal((1, 1, D)) * np.exp2(rng.integers(-1, 2, (1, 1, D)))
    k = rng.standard_normal((1, 1, D))
    s = np.array([[[0.04, 0.11]]])  # unequal group scales: a swapped or shared group would show
    K = np.concatenate([k, k])
    V = np.zeros((2, 1, D))
    V[0, 0, 0] = V[1, 0, 1] = 1.0
    out = O.attention_corrected(q, K, V, scale, 1, s, group)
    c = np.log(out[0, 0, 1] / out[0, 0, 0])
    a = scale * q[0, 0]
    x = a * np.repeat(s[0, 0], group) / 2
    exact = np.sum(np.log(np.sinh(x) / x))
    assert c > 0 and abs(c - exact) <= 1e-3 * exact, (c, exact)
    # with no quantized keys, or lossless ones, it is plain attention
    Q = rng.standard_normal((3, 2, D))
    Kr, Vr = rng.standard_normal((9, 2, D)), rng.standard_normal((9, 2, D))
    np.testing.assert_allclose(O.attention_corrected(Q, Kr, Vr, 0.4, 0, np.zeros((0, 2, 2)), group),
                               O.attention(Q, Kr, Vr, 0.4), atol=1e-14)
    np.testing.assert_allclose(O.attention_corrected(Q, Kr, Vr, 0.4, 9, np.zeros((9, 2, 2)), group),
                               O.attention(Q, Kr, Vr, 0.4), atol=1e-14)


def test_jensen_correction_removes_the_bias_in_expectation(O):
    """Monte Carlo: keys k + e with e uniform of step s in each group; the mean
    over noise draws of exp(score - correction) matches exp(score) of the
    clean key, while the uncorrected mean is biased upward."""
    rng = np.random.default_rng(17)
    D, group, scale, n = 64, 32, 0.5, 200_000
    q = rng.standard_normal(D)
    k = rng.standard_normal(D)
    s = np.array([0.3, 0.6])
    e = (rng.random((n, D)) - 0.5) * np.repeat(s, group)
    raw = scale * (k + e) @ q
    # the oracle's correction for this query and key, read off a two-key attention
    K = np.stack([k, k])[:, None, :]
    V = np.zeros((2, 1, D))
    V[0, 0, 0] = V[1, 0, 1] = 1.0
    out = O.attention_corrected(q[None, None, :], K, V, scale, 1, s[None, None, :], group)
    c = np.log(out[0, 0, 1] / out[0, 0, 0])
    clean = np.exp(scale * k @ q)
    biased = np.mean(np.exp(raw)) / clean - 1
    fixed = np.mean(np.exp(raw - c)) / clean - 1
    se = np.std(np.exp(raw)) / clean / np.sqrt(n)
    assert biased > 10 * se
    assert abs(fixed) < 4 * se + 0.02 * biased, (fixed, biased, se)


# ---------------------------------------------------------------- H64 / EDEN-2 residual codec


def _cb():
    from clustered_kv_cache_b200 import synth

    return synth.eden2_codebook().double().numpy()


def test_h64_is_the_orthonormal_sylvester_hadamard_transform(O):
    """The transform matches scipy's Hadamard matrix (Sylvester order) / 8,
    and applying it twice gives the identity."""
    from scipy.linalg import hadamard

    rng = np.random.default_rng(18)
    x = rng.standard_normal((5, 64))
    Hs = hadamard(64).astype(np.float64) / 8.0
    y = O.hadamard64(x) if O is O_CPP else x @ (O.hadamard_matrix(64) / 8.0).T
    np.testing.assert_allclose(y, x @ Hs.T, rtol=1e-13, atol=1e-13)
    back = O.hadamard64(y) if O is O_CPP else y @ (O.hadamard_matrix(64) / 8.0).T
    np.testing.assert_allclose(back, x, rtol=1e-13, atol=1e-13)


def _eden_rows(O, x, cb, param="f16", state="f64"):
    """One tensor [T, 1, D] coded by the anchor path with the EDEN-2 codec."""
    T, D = x.shape
    d = O.Desc(T, 1, D, state, 2, 64, param, codec="eden2")
    c, _, xh, _ = O.encode_layer_none(d, x[:, None, :], x[:, None, :], codebook=cb)
    return c, xh[:, 0, :]


def test_eden2_is_lossless_on_scaled_codebook_points(O):
    """Residuals whose transform is exactly S times codebook points (a 4 x 4
    grid codebook, dyadic S) come back exactly: indices, scale (EDEN's
    |y|^2 / <y, c> = S) and values."""
    g1 = np.array([-1.5, -0.5, 0.5, 1.5])
    cb = np.array([[a, b] for a in g1 for b in g1])
    rng = np.random.default_rng(19)
    k = rng.integers(0, 16, (6, 64))  # 32 pairs per group, 2 groups per row
    S = np.array([0.5, 0.25, 2.0, 1.0, 0.125, 4.0])
    y = S[:, None, None] * cb[k]  # [6, 64, 2] = 6 rows x 128 values
    y = y.reshape(6, 2, 64)
    x = (y @ (np.asarray(__import__("scipy.linalg", fromlist=["hadamard"]).hadamard(64), float).T / 8.0)).reshape(6, 128)
    c, xh = _eden_rows(O, x, cb)
    np.testing.assert_array_equal(c.q.reshape(6, 64), k)
    np.testing.assert_array_equal(c.s.reshape(6, 2), np.repeat(S[:, None], 2, 1))
    np.testing.assert_allclose(xh, x, rtol=0, atol=1e-14)


def test_eden2_indices_are_the_nearest_points_and_the_scale_is_unbiased(O):
    """Brute force over the 16 points on the sigma-normalised pairs, the scale
    satisfies <S c, y> = |y|^2 up to its fp16 rounding, a zero residual codes
    to zeros, and the bits per value are those of INT2."""
    cb = _cb()
    rng = np.random.default_rng(20)
    x = rng.standard_normal((40, 128)) * np.exp2(rng.integers(-3, 3, (40, 1)))
    x[3] = 0.0
    c, xh = _eden_rows(O, x, cb)
    from scipy.linalg import hadamard

    Hs = hadamard(64).astype(float) / 8.0
    y = x.reshape(40, 2, 64) @ Hs.T
    sig = np.sqrt((y * y).mean(-1))
    u = (y / np.where(sig > 0, sig, 1)[..., None]).reshape(40, 2, 32, 2)
    d = ((u[..., None, :] - cb) ** 2).sum(-1)
    best = d.argmin(-1)
    srt = np.sort(d, -1)
    tie = (srt[..., 1] - srt[..., 0]) < 1e-12
    q = c.q.reshape(40, 2, 32)
    assert np.all((q == best) | tie)
    assert np.all(q[3] == 0) and np.all(c.s.reshape(40, 2)[3] == 0) and np.all(xh[3] == 0)
    yh = c.s.reshape(40, 2)[..., None, None] * cb[q]
    lhs = (yh * y.reshape(40, 2, 32, 2)).sum((-1, -2))
    rhs = (y * y).sum(-1)
    live = rhs > 0
    np.testing.assert_allclose(lhs[live], rhs[live], rtol=2.0 ** -10)
    dd = O.Desc(1000, 12, 128, "bf16", 2, 64, "f16", codec="eden2")
    assert O.codes_bytes(dd) * 8 / (2 * 1000 * 12 * 128) == pytest.approx(2 + 16 / 64)


def test_eden2_beats_scalar_int2_on_gaussian_residuals(O):
    """The point of the transform and the 2-D points: on Gaussian residuals the
    H64 / EDEN-2 codec (2.25 bits per value) has lower error than scalar INT2
    with fp16 (scale, zero) per 64 values (2.5 bits per value)."""
    cb = _cb()
    rng = np.random.default_rng(21)
    x = rng.standard_normal((200, 128))
    _, xe = _eden_rows(O, x, cb)
    d = O.Desc(200, 1, 128, "f64", 2, 64, "f16")
    _, _, xs, _ = O.encode_layer_none(d, x[:, None, :], x[:, None, :])
    assert np.mean((xe - x) ** 2) < 0.8 * np.mean((xs[:, 0] - x) ** 2)


# ---------------------------------------------------------------- video-adapted refit


def test_refit_recovers_an_exact_block_and_satisfies_the_normal_equations(O):
    """Targets made exactly by a block-DPLR map: with a vanishing ridge the
    refit returns that map's blocks; with a ridge the result satisfies the
    normal equations X^T (Y - LR - X B^T) = ridge B^T; rank 0 without a ridge
    is plain per-head least squares (numpy lstsq)."""
    rng = np.random.default_rng(22)
    T, H, D, r = 300, 2, 16, 3
    X0, X1 = rng.standard_normal((T, H, D)), rng.standard_normal((T, H, D))
    Bv = rng.standard_normal((H, D, 2 * D)) * 0.3
    w, u = rng.standard_normal((r, 2 * H * D)) * 0.1, rng.standard_normal((H * D, r))
    flat = np.concatenate([X0.reshape(T, -1), X1.reshape(T, -1)], 1)
    lr = ((flat @ w.T) @ u.T).reshape(T, H, D)
    Xh = np.concatenate([X0, X1], -1)
    Y = np.einsum("thi,hoi->tho", Xh, Bv) + lr
    np.testing.assert_allclose(O.refit_block_diag(X0, X1, Y, w, u, 1e-12), Bv, atol=1e-9)
    Yn = Y + 0.5 * rng.standard_normal(Y.shape)
    ridge = 7.0
    B = O.refit_block_diag(X0, X1, Yn, w, u, ridge)
    for h in range(H):
        res = Yn[:, h] - lr[:, h] - Xh[:, h] @ B[h].T
        np.testing.assert_allclose(Xh[:, h].T @ res, ridge * B[h].T, atol=1e-9)
    B0 = O.refit_block_diag(X0, None, Yn, None, None, 0.0)
    for h in range(H):
        ref = np.linalg.lstsq(X0[:, h], Yn[:, h], rcond=None)[0].T
        np.testing.assert_allclose(B0[h], ref, atol=1e-10)


def test_grouped_query_attention_matches_torch_sdpa(O):
    """Query head j reads KV head j // (Hq / H): torch's SDPA with enable_gqa
    (fp64) gives the same outputs."""
    rng = np.random.default_rng(23)
    Q = rng.standard_normal((9, 6, 16))
    K, V = rng.standard_normal((31, 2, 16)), rng.standard_normal((31, 2, 16))
    got = O.attention(Q, K, V, 0.3)
    t = lambda x: torch.from_numpy(x).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(t(Q), t(K), t(V), scale=0.3, enable_gqa=True)
    np.testing.assert_allclose(got, ref[0].permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-13)
