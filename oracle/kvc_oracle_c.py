"""Python face of the plain single-threaded fp64 C++ oracle (kvc_oracle.cpp).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__`` and the CPU legs
of ``bench.py`` may import this module.  It compiles ``kvc_oracle.cpp`` with the
host C++ compiler into ``liboracle.so`` beside it (``build()``), loads it with
ctypes and marshals numpy float64 arrays in and out.  It shares no code with
the CUDA library.  The containers ``Desc`` and ``Coded`` are the plain
dataclasses of the numpy oracle (no arithmetic).

Every C function is single-threaded.  The thread driver here only splits a call
into disjoint runs of units that do not interact (tokens of the cross-layer and
clustered codecs, heads of the temporal codec, query rows of attention), calls
the C function on each run from its own Python thread (ctypes releases the
interpreter lock during the call) and puts the pieces back together, so the
result is the same for any thread count.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from oracle.kvc_oracle import Coded, Desc  # plain containers

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kvc_oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")
CXXFLAGS = ["-O2", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]

_FMT = {"f64": 0, "f32": 1, "bf16": 2, "f16": 3}
_PARAM_BYTES = {"f16": 2, "f32": 4}
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle library if it is missing or older than its source."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".{os.getpid()}.tmp"
        cxx = os.environ.get("CXX", "g++")
        r = subprocess.run([cxx, *CXXFLAGS, SRC, "-o", tmp], capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"building the C++ oracle failed:\n{r.stdout}{r.stderr}")
        os.replace(tmp, LIB)
    return LIB


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(LIB)
            L.kvo_round.restype = ctypes.c_double
            L.kvo_round.argtypes = [ctypes.c_double, ctypes.c_int]
            L.kvo_codes_bytes.restype = ctypes.c_int64
            _lib = L
    return _lib


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count() or 1)


# ---------------------------------------------------------------- marshalling

_D = ctypes.POINTER(ctypes.c_double)
_U8 = ctypes.POINTER(ctypes.c_uint8)
_I64 = ctypes.POINTER(ctypes.c_int64)


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a):
    """ctypes pointer to a contiguous numpy array (None -> NULL)."""
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as({np.dtype(np.float64): _D, np.dtype(np.uint8): _U8, np.dtype(np.int64): _I64}[a.dtype])


def _i(x) -> ctypes.c_int64:
    return ctypes.c_int64(int(x))


def _runs(n: int, threads: int | None, min_run: int = 1):
    """Disjoint [a, b) runs covering range(n), one per worker."""
    k = max(1, min(threads or default_threads(), max(1, n // max(1, min_run))))
    edges = np.linspace(0, n, k + 1).round().astype(int)
    return [(int(a), int(b)) for a, b in zip(edges[:-1], edges[1:]) if b > a]


def _drive(runs, fn):
    if len(runs) <= 1:
        for a, b in runs:
            fn(a, b)
        return
    with ThreadPoolExecutor(len(runs)) as ex:
        for f in [ex.submit(fn, a, b) for a, b in runs]:
            f.result()


# ---------------------------------------------------------------- building blocks


def round_to(x, fmt: str) -> np.ndarray:
    x = _f64(x)
    y = np.empty_like(x)
    lib().kvo_round_array(_p(x), _i(x.size), _FMT[fmt], _p(y))
    return y


def quantize_groups(r, bits: int, group: int, param: str):
    r = _f64(r)
    n = r.shape[-1]
    rows = r.size // n if n else 0
    q = np.empty(r.shape, np.uint8)
    s = np.empty(r.shape[:-1] + (n // group,))
    z = np.empty_like(s)
    lib().kvo_quantize_groups(_p(r), _i(rows), n, bits, group, _FMT[param], _p(q), _p(s), _p(z))
    return q, s, z


def dequantize_groups(q, s, z, group: int) -> np.ndarray:
    """z + s q per element (reading R1)."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    n = q.shape[-1]
    out = np.empty(q.shape)
    lib().kvo_dequantize_groups(_p(q), _p(_f64(s)), _p(_f64(z)), _i(q.size // n if n else 0), n, group, _p(out))
    return out


def pack_codes(q, bits: int) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    n = q.shape[-1]
    rows = q.size // n
    out = np.empty(q.shape[:-1] + (n * bits // 8,), np.uint8)
    lib().kvo_pack(_p(q), _i(rows), n, bits, _p(out))
    return out


def unpack_codes(packed, bits: int, n: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    rb = packed.shape[-1]
    rows = packed.size // rb
    q = np.empty(packed.shape[:-1] + (n,), np.uint8)
    lib().kvo_unpack(_p(packed), _i(rows), n, bits, _p(q))
    return q


def codes_bytes(desc: Desc, kind: str = "none", code_dim: int = 0) -> int:
    k = {"none": 0, "xlayer": 0, "temporal": 1, "cluster": 2}[kind]
    if getattr(desc, "codec", "rtn") == "eden2":
        k = 3
    return int(lib().kvo_codes_bytes(k, _i(desc.n_tokens), desc.n_heads, desc.head_dim, desc.bits, desc.group,
                                     _PARAM_BYTES[desc.param], desc.frame_tokens, desc.anchor_bits, code_dim))


# ---------------------------------------------------------------- layers


def _empty_coded(T, H, D, group, eden=False):
    """Codes of a [T, H, D] tensor: per element (scalar quantizer) or per pair
    (H64 / EDEN-2: D / 2 indices, D / 64 scales, zeros unused)."""
    if eden:
        return (np.empty((T, H, D // 2), np.uint8), np.empty((T, H, D // 64)), np.zeros((T, H, D // 64)))
    return (np.empty((T, H, D), np.uint8), np.empty((T, H, D // group)), np.empty((T, H, D // group)))


def _cb(desc: Desc, codebook):
    """The EDEN-2 points as a contiguous float64 [16, 2] array (None: scalar codec)."""
    if getattr(desc, "codec", "rtn") != "eden2":
        return None
    assert codebook is not None, "the H64 / EDEN-2 codec needs its 16 points"
    cb = _f64(codebook).reshape(16, 2)
    return cb


def encode_layer_none(desc: Desc, K, V, threads=None, codebook=None):
    """Anchor: both tensors coded against prediction 0 [CORAL Fig. 8]."""
    cb = _cb(desc, codebook)
    out = []
    for X in (K, V):
        X = _f64(X)
        T, H, D = X.shape
        q, s, z = _empty_coded(T, H, D, desc.group, cb is not None)
        xh = np.empty_like(X)

        def run(a, b):
            lib().kvo_encode_none(_i(b - a), H, D, desc.bits, desc.group, _FMT[desc.param], _FMT[desc.state],
                                  _p(X[a:b]), _p(q[a:b]), _p(s[a:b]), _p(z[a:b]), _p(xh[a:b]), _p(cb))

        _drive(_runs(T, threads, 64), run)
        out.append((Coded(q, s, z), xh))
    return out[0][0], out[1][0], out[0][1], out[1][1]


def decode_layer_none(desc: Desc, ck: Coded, cv: Coded, threads=None, codebook=None):
    cb = _cb(desc, codebook)
    res = []
    for c in (ck, cv):
        q, s, z = np.ascontiguousarray(c.q), _f64(c.s), _f64(c.z)
        T, H = q.shape[:2]
        D = desc.head_dim
        xh = np.empty((T, H, D))
        lib().kvo_decode_none(_i(T), H, D, desc.group, _FMT[desc.state], _p(q), _p(s), _p(z), _p(xh), _p(cb))
        res.append(xh)
    return res[0], res[1]


def hadamard64(x) -> np.ndarray:
    """The orthonormal Sylvester Walsh-Hadamard transform of rows of 64 values."""
    x = _f64(x)
    out = np.empty_like(x)
    lib().kvo_hadamard64(_p(x), _i(x.size // 64), _p(out))
    return out


def _xw(w: dict):
    r = w["k_w"].shape[0] if w.get("k_w") is not None else 0
    f = lambda k: _f64(w[k]) if r or k in ("k_block", "v_block") else np.zeros(1)
    return r, f("k_block"), f("k_w"), f("k_u"), f("v_block"), f("v_w"), f("v_u")


def xlayer_predict_k(K_src, k_block, k_w, k_u) -> np.ndarray:
    """K~_l = blockdiag_h(K^_{l-1,h} B_h^T) + (K^_{l-1} W^T) U^T [CORAL Fig. 3]."""
    Ks = _f64(K_src)
    T, H, D = Ks.shape
    r = int(np.shape(k_w)[0])
    out = np.empty_like(Ks)
    f = lambda x: _f64(x) if r else np.zeros(1)
    lib().kvo_predict_xlayer_k(_i(T), H, D, r, _p(Ks), _p(_f64(k_block)), _p(f(k_w)), _p(f(k_u)), _p(out))
    return out


def xlayer_predict_v(K_rec, V_src, v_block, v_w, v_u) -> np.ndarray:
    """V~_l from the reconstructed pair [K^_l, V^_{l-1}] [CORAL Fig. 3]."""
    Kh, Vs = _f64(K_rec), _f64(V_src)
    T, H, D = Kh.shape
    r = int(np.shape(v_w)[0])
    out = np.empty_like(Kh)
    f = lambda x: _f64(x) if r else np.zeros(1)
    lib().kvo_predict_xlayer_v(_i(T), H, D, r, _p(Kh), _p(Vs), _p(_f64(v_block)), _p(f(v_w)), _p(f(v_u)), _p(out))
    return out


def encode_layer_xlayer(desc: Desc, w: dict, K, V, K_src, V_src, threads=None, with_pred: bool = False,
                        codebook=None):
    """One Coral layer l > 0 [CORAL Fig. 3]; returns (coded K, coded V, K^_l,
    V^_l) and, with `with_pred`, the two predictions as well."""
    K, V, Ks, Vs = _f64(K), _f64(V), _f64(K_src), _f64(V_src)
    T, H, D = K.shape
    cb = _cb(desc, codebook)
    r, bk, wk, uk, bv, wv, uv = _xw(w)
    qk, sk, zk = _empty_coded(T, H, D, desc.group, cb is not None)
    qv, sv, zv = _empty_coded(T, H, D, desc.group, cb is not None)
    kh, vh = np.empty_like(K), np.empty_like(V)
    pk = np.empty_like(K) if with_pred else None
    pv = np.empty_like(V) if with_pred else None

    def run(a, b):
        lib().kvo_encode_xlayer(_i(b - a), H, D, r, desc.bits, desc.group, _FMT[desc.param], _FMT[desc.state],
                                _p(K[a:b]), _p(V[a:b]), _p(Ks[a:b]), _p(Vs[a:b]), _p(bk), _p(wk), _p(uk), _p(bv),
                                _p(wv), _p(uv), _p(qk[a:b]), _p(sk[a:b]), _p(zk[a:b]), _p(qv[a:b]), _p(sv[a:b]),
                                _p(zv[a:b]), _p(kh[a:b]), _p(vh[a:b]), _p(pk[a:b]) if with_pred else None,
                                _p(pv[a:b]) if with_pred else None, _p(cb))

    _drive(_runs(T, threads, 16), run)
    out = (Coded(qk, sk, zk), Coded(qv, sv, zv), kh, vh)
    return out + (pk, pv) if with_pred else out


def decode_layer_xlayer(desc: Desc, w: dict, ck: Coded, cv: Coded, K_src, V_src, threads=None, codebook=None):
    Ks, Vs = _f64(K_src), _f64(V_src)
    T, H, D = Ks.shape
    cb = _cb(desc, codebook)
    r, bk, wk, uk, bv, wv, uv = _xw(w)
    qk, sk, zk = np.ascontiguousarray(ck.q), _f64(ck.s), _f64(ck.z)
    qv, sv, zv = np.ascontiguousarray(cv.q), _f64(cv.s), _f64(cv.z)
    kh, vh = np.empty_like(Ks), np.empty_like(Vs)

    def run(a, b):
        lib().kvo_decode_xlayer(_i(b - a), H, D, r, desc.group, _FMT[desc.state], _p(qk[a:b]), _p(sk[a:b]),
                                _p(zk[a:b]), _p(qv[a:b]), _p(sv[a:b]), _p(zv[a:b]), _p(Ks[a:b]), _p(Vs[a:b]), _p(bk),
                                _p(wk), _p(uk), _p(bv), _p(wv), _p(uv), _p(kh[a:b]), _p(vh[a:b]), _p(cb))

    _drive(_runs(T, threads, 16), run)
    return kh, vh


def _temporal(decode: bool, desc: Desc, w: dict, K, V, ck, cv, k_hist, v_hist, threads):
    """Frame chain of one temporal layer [TEMPO Fig. 2(b)]; the thread driver
    splits the heads (each head has its own maps and its own history)."""
    ak, av = _f64(w["ak"]), _f64(w["av"])
    T, H, D = (ck.q.shape if decode else np.shape(K))
    F = desc.frame_tokens
    if decode:
        qk, sk, zk = np.ascontiguousarray(ck.q), _f64(ck.s), _f64(ck.z)
        qv, sv, zv = np.ascontiguousarray(cv.q), _f64(cv.s), _f64(cv.z)
        K = V = None
    else:
        K, V = _f64(K), _f64(V)
        qk, sk, zk = _empty_coded(T, H, D, desc.group)
        qv, sv, zv = _empty_coded(T, H, D, desc.group)
    kh, vh = np.empty((T, H, D)), np.empty((T, H, D))
    kh_all = None if k_hist is None else _f64(k_hist).reshape(2, F, H, D)
    vh_all = None if v_hist is None else _f64(v_hist).reshape(F, H, D)

    def run(a, b):
        sl = lambda x: None if x is None else np.ascontiguousarray(x[..., a:b, :])
        q_k, s_k, z_k, q_v, s_v, z_v = (np.ascontiguousarray(x[:, a:b]) for x in (qk, sk, zk, qv, sv, zv))
        k_h, v_h = np.empty((T, b - a, D)), np.empty((T, b - a, D))
        lib().kvo_temporal(int(decode), _i(T), b - a, D, F, desc.bits, desc.anchor_bits, desc.group,
                           _FMT[desc.param], _FMT[desc.state], _p(sl(K)), _p(sl(V)), _p(sl(kh_all)), _p(sl(vh_all)),
                           _p(np.ascontiguousarray(ak[a:b])), _p(np.ascontiguousarray(av[a:b])), _p(q_k), _p(s_k),
                           _p(z_k), _p(q_v), _p(s_v), _p(z_v), _p(k_h), _p(v_h))
        if not decode:
            qk[:, a:b], sk[:, a:b], zk[:, a:b], qv[:, a:b], sv[:, a:b], zv[:, a:b] = q_k, s_k, z_k, q_v, s_v, z_v
        kh[:, a:b], vh[:, a:b] = k_h, v_h

    _drive(_runs(H, threads), run)
    if decode:
        return kh, vh
    return Coded(qk, sk, zk), Coded(qv, sv, zv), kh, vh


def encode_layer_temporal(desc: Desc, w: dict, K, V, k_hist=None, v_hist=None, threads=None):
    return _temporal(False, desc, w, K, V, None, None, k_hist, v_hist, threads)


def decode_layer_temporal(desc: Desc, w: dict, ck: Coded, cv: Coded, k_hist=None, v_hist=None, threads=None):
    return _temporal(True, desc, w, None, None, ck, cv, k_hist, v_hist, threads)


def cluster_assign(X, centroids) -> np.ndarray:
    """Nearest centre of each row of X [T,C], ties to the lowest index (R10)."""
    X, cent = _f64(X), _f64(centroids)
    T, C = X.shape
    a = np.empty(T, np.int64)
    lib().kvo_cluster_assign(_i(T), C, cent.shape[0], _p(X), _p(cent), _p(a))
    return a


def encode_tensor_cluster(desc: Desc, X, centroids, enc, dec, threads=None, reconstruct: bool = True):
    """X [T,H,D] -> (Coded with assign, x_hat [T,H,D]) [NANO abstract]."""
    X = _f64(X)
    T, H, D = X.shape
    C = H * D
    cent, E, W = _f64(centroids), _f64(enc), _f64(dec)
    m, nc = E.shape[0], cent.shape[0]
    a = np.empty(T, np.int64)
    q = np.empty((T, m), np.uint8)
    s = np.empty((T, m // desc.group))
    z = np.empty_like(s)
    xh = np.empty((T, C)) if reconstruct else None
    Xf = X.reshape(T, C)

    def run(lo, hi):
        lib().kvo_cluster_encode(_i(hi - lo), C, m, nc, desc.bits, desc.group, _FMT[desc.param], _FMT[desc.state],
                                 _p(Xf[lo:hi]), _p(cent), _p(E), _p(W), _p(a[lo:hi]), _p(q[lo:hi]), _p(s[lo:hi]),
                                 _p(z[lo:hi]), _p(xh[lo:hi]) if reconstruct else None)

    _drive(_runs(T, threads, 16), run)
    return Coded(q, s, z, a), (xh.reshape(T, H, D) if reconstruct else None)


def decode_tensor_cluster(desc: Desc, c: Coded, centroids, dec, exact: bool = False, threads=None):
    T, m = c.q.shape
    cent, W = _f64(centroids), _f64(dec)
    C = cent.shape[1]
    q, s, z = np.ascontiguousarray(c.q), _f64(c.s), _f64(c.z)
    a = np.ascontiguousarray(c.assign, dtype=np.int64)
    xh = np.empty((T, C))

    def run(lo, hi):
        lib().kvo_cluster_decode(_i(hi - lo), C, m, desc.group, 0 if exact else _FMT[desc.state], _p(a[lo:hi]),
                                 _p(q[lo:hi]), _p(s[lo:hi]), _p(z[lo:hi]), _p(cent), _p(W), _p(xh[lo:hi]))

    _drive(_runs(T, threads, 16), run)
    return xh.reshape(T, desc.n_heads, desc.head_dim)


# ---------------------------------------------------------------- attention


def attention(Q, K, V, scale: float, threads=None) -> np.ndarray:
    """Naive two-pass softmax attention; query rows split over threads.  Q may
    have a multiple of K's heads (grouped-query attention)."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    nq, Hq, D = Q.shape
    nk, H = K.shape[:2]
    O = np.empty((nq, Hq, D))

    def run(a, b):
        lib().kvo_attention_corrected(_i(b - a), _i(nk), Hq, H, D, ctypes.c_double(scale), _p(Q[a:b]), _p(K), _p(V),
                                      _i(0), None, 1, _p(O[a:b]))

    _drive(_runs(nq, threads), run)
    return O


def attention_corrected(Q, K, V, scale: float, n_hist: int, s_hist, group: int, threads=None) -> np.ndarray:
    """Softmax attention in which each of the first n_hist (quantized) keys'
    scores is lowered by its Jensen-bias term 0.5 scale^2 sum_g |q_g|^2 s_g^2 / 12
    (the abstract on the "Jensen bias" of INT2 key caches, CORAL-KV page);
    s_hist [n_hist, H, D/group]."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    nq, Hq, D = Q.shape
    nk, H = K.shape[:2]
    sh = _f64(s_hist)
    O = np.empty((nq, Hq, D))

    def run(a, b):
        lib().kvo_attention_corrected(_i(b - a), _i(nk), Hq, H, D, ctypes.c_double(scale), _p(Q[a:b]), _p(K), _p(V),
                                      _i(n_hist), _p(sh), group, _p(O[a:b]))

    _drive(_runs(nq, threads), run)
    return O


def attend_compressed_xlayer(desc: Desc, w: dict, Q, ck: Coded, cv: Coded, K_src, V_src, K_self, V_self,
                             scale: float, threads=None, jensen: bool = False, codebook=None) -> np.ndarray:
    """Softmax attention of Q over [decoded history ; uncompressed chunk]."""
    K_hist, V_hist = decode_layer_xlayer(desc, w, ck, cv, K_src, V_src, threads, codebook)
    T = K_hist.shape[0]
    if K_self is not None and len(K_self):
        K_hist = np.concatenate([K_hist, _f64(K_self)], axis=0)
        V_hist = np.concatenate([V_hist, _f64(V_self)], axis=0)
    if jensen:
        return attention_corrected(Q, K_hist, V_hist, scale, T, ck.s, desc.group, threads)
    return attention(Q, K_hist, V_hist, scale, threads)


def mixed_attention(Q, ck: Coded, cent_k, dec_k, cv: Coded, cent_v, dec_v, desc: Desc, scale: float,
                    threads=None) -> np.ndarray:
    """Attention on the stored coefficients [NANO abstract, Fast variant]."""
    Q = _f64(Q)
    nq, H, D = Q.shape
    ckh = _f64(dequantize_groups(ck.q, ck.s, ck.z, desc.group))
    cvh = _f64(dequantize_groups(cv.q, cv.s, cv.z, desc.group))
    T, m = ckh.shape
    ak = np.ascontiguousarray(ck.assign, dtype=np.int64)
    av = np.ascontiguousarray(cv.assign, dtype=np.int64)
    Ck, Wk, Cv, Wv = _f64(cent_k), _f64(dec_k), _f64(cent_v), _f64(dec_v)
    nc = Ck.shape[0]
    O = np.empty((nq, H, D))

    def run(a, b):
        lib().kvo_mixed_attention(_i(b - a), _i(T), H, D, m, nc, ctypes.c_double(scale), _p(Q[a:b]), _p(ckh), _p(ak),
                                  _p(Ck), _p(Wk), _p(cvh), _p(av), _p(Cv), _p(Wv), _p(O[a:b]))

    _drive(_runs(nq, threads), run)
    return O


# ---------------------------------------------------------------- video-adapted refit


def refit_block_diag(X0, X1, Y, w_lr, u_lr, ridge: float) -> np.ndarray:
    """Ridge least-squares refit of every head's block-diagonal map with the
    low-rank factors fixed ("CORAL-KV ...", Fig. 4, video-adapted block-DPLR):
    returns block [H, D, din] (din = D for K, 2 D for V with X1 given)."""
    X0, Y = _f64(X0), _f64(Y)
    T, H, D = X0.shape
    X1 = None if X1 is None else _f64(X1)
    r = int(np.shape(w_lr)[0]) if w_lr is not None else 0
    din = 2 * D if X1 is not None else D
    w = _f64(w_lr) if r else np.zeros(1)
    u = _f64(u_lr) if r else np.zeros(1)
    out = np.empty((H, D, din))
    lib().kvo_refit_block_diag(_i(T), H, D, r, _p(X0), _p(X1), _p(Y), _p(w), _p(u), ctypes.c_double(ridge), _p(out))
    return out
