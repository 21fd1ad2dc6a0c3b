"""The two fp64 oracles against each other.

The plain C++ oracle (loops, single-threaded functions, sums in index order)
and the numpy oracle (library matmuls over whole tensors) are written
independently; on the same seeded inputs their codes, (scale, zero) pairs and
rounded reconstructions must be identical and their unrounded outputs equal to
1e-12 relative.  The only difference between them is the fp64 summation order,
which moves a discrete decision only when a value lies within ~1e-15 of a
rounding boundary: none of these inputs has one.  Also checks that the C++
oracle's thread driver gives the same result for any thread count.  CPU only.
"""

import numpy as np
import pytest

from oracle import kvc_oracle as N
from oracle import kvc_oracle_c as C

RNG = np.random.default_rng(424242)


def _bf16(x):
    return N.round_to(x, "bf16")


def _same_coded(a, b, what):
    np.testing.assert_array_equal(a.q, b.q, err_msg=what + " codes")
    np.testing.assert_array_equal(a.s, b.s, err_msg=what + " scales")
    np.testing.assert_array_equal(a.z, b.z, err_msg=what + " zeros")
    if a.assign is not None or b.assign is not None:
        np.testing.assert_array_equal(a.assign, b.assign, err_msg=what + " assignments")


def _close(a, b, rtol=1e-12):
    scale = max(np.abs(b).max(), 1e-300)
    assert np.abs(a - b).max() <= rtol * scale


def _xlayer_inputs(T, H, D, r, state, seed):
    rng = np.random.default_rng(seed)
    Cc = H * D
    rnd = (lambda x: N.round_to(x, state)) if state != "f64" else (lambda x: x)
    w = dict(k_block=rnd(rng.standard_normal((H, D, D)) / np.sqrt(D)),
             k_w=rnd(rng.standard_normal((r, Cc)) / np.sqrt(Cc)), k_u=rnd(0.2 * rng.standard_normal((Cc, r))),
             v_block=rnd(rng.standard_normal((H, D, 2 * D)) / np.sqrt(2 * D)),
             v_w=rnd(rng.standard_normal((r, 2 * Cc)) / np.sqrt(2 * Cc)), v_u=rnd(0.2 * rng.standard_normal((Cc, r))))
    Ks, Vs = rnd(rng.standard_normal((T, H, D))), rnd(rng.standard_normal((T, H, D)))
    K = rnd(N.xlayer_predict_k(Ks, w["k_block"], w["k_w"], w["k_u"]) + 0.3 * rng.standard_normal((T, H, D)))
    V = rnd(0.5 * rng.standard_normal((T, H, D)) + 0.5 * Vs)
    return w, K, V, Ks, Vs


@pytest.mark.parametrize("T,H,D,r,bits,group,state,param", [
    (150, 4, 128, 16, 2, 32, "bf16", "f16"),
    (97, 3, 64, 0, 4, 32, "bf16", "f16"),
    (64, 2, 64, 8, 4, 32, "f32", "f32"),
    (40, 2, 128, 4, 8, 16, "bf16", "f16"),
])
def test_cross_layer_layer(T, H, D, r, bits, group, state, param):
    w, K, V, Ks, Vs = _xlayer_inputs(T, H, D, r, state, T + r)
    d = N.Desc(T, H, D, state, bits, group, param)
    a = N.encode_layer_xlayer(d, w, K, V, Ks, Vs)
    b = C.encode_layer_xlayer(d, w, K, V, Ks, Vs, threads=3)
    _same_coded(a[0], b[0], "K")
    _same_coded(a[1], b[1], "V")
    np.testing.assert_array_equal(a[2], b[2])
    np.testing.assert_array_equal(a[3], b[3])
    kd, vd = C.decode_layer_xlayer(d, w, b[0], b[1], Ks, Vs, threads=2)
    np.testing.assert_array_equal(kd, b[2])
    np.testing.assert_array_equal(vd, b[3])
    # predictions alone, to 1e-12
    _close(C.xlayer_predict_k(Ks, w["k_block"], w["k_w"], w["k_u"]),
           N.xlayer_predict_k(Ks, w["k_block"], w["k_w"], w["k_u"]))


def test_anchor_layer():
    K = _bf16(RNG.standard_normal((70, 3, 128)) * np.exp2(RNG.integers(-2, 3, (1, 1, 128))))
    V = _bf16(RNG.standard_normal((70, 3, 128)))
    d = N.Desc(70, 3, 128, "bf16", 4, 32, "f16")
    a = N.encode_layer_none(d, K, V)
    b = C.encode_layer_none(d, K, V)
    for i in range(2):
        _same_coded(a[i], b[i], "anchor")
        np.testing.assert_array_equal(a[2 + i], b[2 + i])
    kd, vd = C.decode_layer_none(d, b[0], b[1])
    np.testing.assert_array_equal(kd, b[2])
    np.testing.assert_array_equal(vd, b[3])


@pytest.mark.parametrize("T,F,ab,cont", [(3 * 20 + 7, 20, 4, False), (2 * 16, 16, 0, True), (11, 16, 2, False)])
def test_temporal_layer(T, F, ab, cont):
    H, D = 3, 64
    rng = np.random.default_rng(T + F)
    w = dict(ak=_bf16(rng.standard_normal((H, D, 2 * D)) * 0.08), av=_bf16(rng.standard_normal((H, D, 2 * D)) * 0.08))
    K = _bf16(rng.standard_normal((T, H, D)))
    V = _bf16(rng.standard_normal((T, H, D)))
    kh = _bf16(rng.standard_normal((2, F, H, D))) if cont else None
    vh = _bf16(rng.standard_normal((F, H, D))) if cont else None
    d = N.Desc(T, H, D, "bf16", 2, 32, "f16", F, ab)
    a = N.encode_layer_temporal(d, w, K, V, kh, vh)
    b = C.encode_layer_temporal(d, w, K, V, kh, vh, threads=2)
    _same_coded(a[0], b[0], "K")
    _same_coded(a[1], b[1], "V")
    np.testing.assert_array_equal(a[2], b[2])
    np.testing.assert_array_equal(a[3], b[3])
    kd, vd = C.decode_layer_temporal(d, w, b[0], b[1], kh, vh)
    np.testing.assert_array_equal(kd, b[2])
    np.testing.assert_array_equal(vd, b[3])


def test_cluster_codec():
    T, H, D, nc, m = 300, 4, 64, 16, 64
    Cc = H * D
    rng = np.random.default_rng(7)
    cent = _bf16(rng.standard_normal((nc, Cc)))
    X = _bf16(cent[rng.integers(0, nc, T)] + 0.2 * rng.standard_normal((T, Cc))).reshape(T, H, D)
    E = np.linalg.qr(rng.standard_normal((Cc, m)))[0]
    enc, dec = _bf16(E.T), _bf16(E)
    d = N.Desc(T, H, D, "bf16", 4, 32, "f16")
    ca, xa = N.encode_tensor_cluster(d, X, cent, enc, dec)
    cb, xb = C.encode_tensor_cluster(d, X, cent, enc, dec, threads=4)
    _same_coded(ca, cb, "cluster")
    np.testing.assert_array_equal(xa, xb)
    np.testing.assert_array_equal(C.decode_tensor_cluster(d, cb, cent, dec), xb)
    _close(C.decode_tensor_cluster(d, cb, cent, dec, exact=True), N.decode_tensor_cluster(d, ca, cent, dec, exact=True))
    np.testing.assert_array_equal(C.cluster_assign(X.reshape(T, -1), cent), N.cluster_assign(X.reshape(T, -1), cent))


def test_attention_and_mixed_attention():
    Q = RNG.standard_normal((33, 3, 32))
    K, V = RNG.standard_normal((200, 3, 32)), RNG.standard_normal((200, 3, 32))
    _close(C.attention(Q, K, V, 0.2, threads=5), N.attention(Q, K, V, 0.2))
    T, H, D, nc, m = 120, 2, 32, 8, 32
    Cc = H * D
    E = np.linalg.qr(RNG.standard_normal((Cc, m)))[0]
    ck_c, cv_c = RNG.standard_normal((nc, Cc)), RNG.standard_normal((nc, Cc))
    Kx = (ck_c[RNG.integers(0, nc, T)] + 0.2 * RNG.standard_normal((T, Cc))).reshape(T, H, D)
    Vx = (cv_c[RNG.integers(0, nc, T)] + 0.2 * RNG.standard_normal((T, Cc))).reshape(T, H, D)
    d = N.Desc(T, H, D, "bf16", 4, 16, "f16")
    ck, _ = N.encode_tensor_cluster(d, Kx, ck_c, E.T, E)
    cv, _ = N.encode_tensor_cluster(d, Vx, cv_c, E.T, E)
    q = RNG.standard_normal((9, H, D))
    _close(C.mixed_attention(q, ck, ck_c, E, cv, cv_c, E, d, 0.3, threads=3),
           N.mixed_attention(q, ck, ck_c, E, cv, cv_c, E, d, 0.3))


def test_thread_count_does_not_change_results():
    w, K, V, Ks, Vs = _xlayer_inputs(131, 2, 64, 8, "bf16", 99)
    d = N.Desc(131, 2, 64, "bf16", 2, 32, "f16")
    one = C.encode_layer_xlayer(d, w, K, V, Ks, Vs, threads=1)
    many = C.encode_layer_xlayer(d, w, K, V, Ks, Vs, threads=7)
    for x, y in zip(one, many):
        if isinstance(x, np.ndarray):
            np.testing.assert_array_equal(x, y)
        else:
            _same_coded(x, y, "threads")
    Q = RNG.standard_normal((17, 2, 64))
    np.testing.assert_array_equal(C.attention(Q, K, V, 0.1, threads=1), C.attention(Q, K, V, 0.1, threads=6))


def test_eden2_codec_layers():
    """The H64 / EDEN-2 codec through an anchor layer and a cross-layer layer."""
    from clustered_kv_cache_b200 import synth

    cb = synth.eden2_codebook().double().numpy()
    w, K, V, Ks, Vs = _xlayer_inputs(90, 3, 128, 16, "bf16", 77)
    d = N.Desc(90, 3, 128, "bf16", 2, 64, "f16", codec="eden2")
    a = N.encode_layer_none(d, K, V, codebook=cb)
    b = C.encode_layer_none(d, K, V, threads=2, codebook=cb)
    for i in range(2):
        _same_coded(a[i], b[i], "anchor eden2")
        np.testing.assert_array_equal(a[2 + i], b[2 + i])
    a = N.encode_layer_xlayer(d, w, K, V, Ks, Vs, codebook=cb)
    b = C.encode_layer_xlayer(d, w, K, V, Ks, Vs, threads=3, codebook=cb)
    _same_coded(a[0], b[0], "K")
    _same_coded(a[1], b[1], "V")
    np.testing.assert_array_equal(a[2], b[2])
    np.testing.assert_array_equal(a[3], b[3])
    kd, vd = C.decode_layer_xlayer(d, w, b[0], b[1], Ks, Vs, codebook=cb)
    np.testing.assert_array_equal(kd, b[2])
    np.testing.assert_array_equal(vd, b[3])
    nk, nv = N.decode_layer_xlayer(d, w, b[0], b[1], Ks, Vs, codebook=cb)
    np.testing.assert_array_equal(nk, kd)
    assert C.codes_bytes(d) == N.codes_bytes(d)
