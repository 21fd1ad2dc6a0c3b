"""Parity of the CUDA codec (through the C ABI) with the fp64 oracle.

The reference is the plain single-threaded C++ oracle (oracle/kvc_oracle.cpp,
driven over disjoint tokens / heads / query rows by its thread driver); the
numpy oracle is used only for the score margins of the clustered assignment.
Each test feeds the GPU and the oracle the same seeded inputs; where a layer's
prediction source is a reconstruction, both receive the oracle's (teacher
forcing), so each call is checked on its own.  Tolerances: tests/kvc_testutil.
"""

import numpy as np
import pytest
import torch

from clustered_kv_cache_b200 import kvc, synth
from oracle import kvc_oracle as ON
from oracle import kvc_oracle_c as O

import kvc_testutil as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from clustered_kv_cache_b200 import build

    build.build()
    kvc.lib()


def _sync_ok():
    torch.cuda.synchronize()
    assert kvc.kvc_get_device_error() == 0


def _desc(T, H, D, dtype, bits, group, param, F=0, ab=4):
    return kvc.make_desc(T, H, D, dtype, bits, group, param, F, ab)


def _odesc(T, H, D, dtype, bits, group, param, F=0, ab=4):
    return O.Desc(T, H, D, U.np_state(dtype), bits, group, U.np_param(param), F, ab)


def _gpu_coded(buf: kvc.CodeBuffers, T, H, D, bits, group, param, which="k"):
    codes = getattr(buf, which + "_codes")
    params = getattr(buf, which + "_params")
    q = U.codes_from_gpu(codes, (T, H, D), bits)
    s, z = U.params_from_gpu(params, (T, H, D // group), param)
    return O.Coded(q, s, z)


def _compare(gc: O.Coded, oc: O.Coded, rec_gpu, rec_ref, exact, x, state, group, what, param="f16", err=None,
             skip_tokens=None):
    """Codes, parameters and reconstructions of one coded tensor [T,H,D].
    err: per-element bound of the GPU prediction's accumulation error;
    skip_tokens: tokens whose prediction inputs already differ (a flipped code
    or reconstruction upstream), checked for validity and against the budgets
    only.  Returns the per-token mask of tokens whose codes, (scale, zero) or
    reconstruction differ in any element."""
    keep = slice(None) if skip_tokens is None else ~skip_tokens  # tokens with the same inputs on both sides
    U.assert_codes_close(gc.q[keep], oc.q[keep], what + " codes")
    skip = None
    if skip_tokens is not None:
        skip = np.broadcast_to(skip_tokens.reshape((-1,) + (1,) * (oc.s.ndim - 1)), oc.s.shape)
    levels = int(max(3, oc.q.max()))
    pdiff = U.assert_params_close(gc.s, gc.z, oc.s, oc.z, param, what + " params", levels=levels, err=err,
                                  group=group, skip=skip)
    flip = gc.q != oc.q
    if param == "f16":  # a different fp16 (scale, zero) moves the whole group
        flip = flip | np.repeat(pdiff, group, axis=-1)
    if skip_tokens is not None:
        flip = flip | skip_tokens.reshape((-1,) + (1,) * (flip.ndim - 1))
    # the GPU's own code around the oracle's prediction (validity of flipped elements)
    pred_ref = exact - O.dequantize_groups(oc.q, oc.s, oc.z, group)
    alt = pred_ref + O.dequantize_groups(gc.q, gc.s, gc.z, group)
    if skip_tokens is not None:
        alt = np.where(skip_tokens.reshape((-1,) + (1,) * (flip.ndim - 1)), rec_gpu, alt)
    U.assert_recon_close(rec_gpu, rec_ref, exact, x, flip, state, what + " recon", err=err, alt=alt)
    differs = flip | (rec_gpu != rec_ref)
    return differs.reshape(differs.shape[0], -1).any(axis=1)


# ---------------------------------------------------------------- packing


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_pack_unpack_bit_exact(bits):
    rng = np.random.default_rng(bits)
    n = (128 // bits) * 16 * 37
    q = rng.integers(0, 1 << bits, n, dtype=np.uint8)
    ref = O.pack_codes(q, bits)
    out = torch.empty(n * bits // 8, dtype=torch.uint8, device="cuda")
    kvc.kvc_pack_codes(torch.from_numpy(q).cuda(), bits, out)
    back = torch.empty(n, dtype=torch.uint8, device="cuda")
    kvc.kvc_unpack_codes(torch.from_numpy(ref).cuda(), n, bits, back)
    _sync_ok()
    np.testing.assert_array_equal(out.cpu().numpy(), ref)
    np.testing.assert_array_equal(back.cpu().numpy(), q)


# ---------------------------------------------------------------- anchor / plain group RTN


@pytest.mark.parametrize("dtype,param,bits,group,T,H,D", [
    (torch.bfloat16, torch.float16, 4, 32, 300, 12, 128),
    (torch.bfloat16, torch.float16, 2, 32, 97, 3, 128),
    (torch.bfloat16, torch.float16, 2, 64, 65, 2, 64),
    (torch.bfloat16, torch.float16, 4, 64, 33, 5, 128),
    (torch.float32, torch.float32, 4, 32, 130, 2, 64),
    (torch.bfloat16, torch.float16, 8, 16, 40, 2, 128),
])
def test_anchor_codec_parity(dtype, param, bits, group, T, H, D):
    g = torch.Generator().manual_seed(T * 7 + bits)
    K = (torch.randn(T, H, D, generator=g) * torch.exp2(torch.randint(-2, 3, (1, 1, D), generator=g))).to(dtype)
    V = torch.randn(T, H, D, generator=g).to(dtype)
    desc = _desc(T, H, D, dtype, bits, group, param)
    pred = kvc.make_predictor(kvc.PRED_NONE)
    buf = kvc.alloc_codes(desc, pred)
    Kr, Vr = torch.empty_like(K, device="cuda"), torch.empty_like(V, device="cuda")
    kvc.kvc_encode_layer(desc, pred, K.cuda(), V.cuda(), None, None, buf, Kr, Vr)
    Kd, Vd = torch.empty_like(Kr), torch.empty_like(Vr)
    kvc.kvc_decode_layer(desc, pred, buf, None, None, Kd, Vd)
    _sync_ok()
    assert torch.equal(Kd, Kr) and torch.equal(Vd, Vr)
    od = _odesc(T, H, D, dtype, bits, group, param)
    ck, cv, Kh, Vh = O.encode_layer_none(od, U.to64(K), U.to64(V))
    for which, oc, rec, ref, x in (("k", ck, Kr, Kh, K), ("v", cv, Vr, Vh, V)):
        gc = _gpu_coded(buf, T, H, D, bits, group, U.np_param(param), which)
        _compare(gc, oc, U.to64(rec), ref, U.exact_none(oc, group), U.to64(x), od.state, group, which,
                 U.np_param(param))


def test_empty_layer_is_a_no_op():
    desc = _desc(0, 2, 128, torch.bfloat16, 2, 32, torch.float16)
    pred = kvc.make_predictor(kvc.PRED_NONE)
    buf = kvc.alloc_codes(desc, pred)
    e = torch.empty(0, 2, 128, dtype=torch.bfloat16, device="cuda")
    kvc.kvc_encode_layer(desc, pred, e, e, None, None, buf, e, e)
    _sync_ok()


# ---------------------------------------------------------------- cross-layer block-DPLR


def _xlayer_gpu(desc, pred, K, V, Ks, Vs):
    buf = kvc.alloc_codes(desc, pred)
    Kr, Vr = torch.empty_like(K), torch.empty_like(V)
    ws = kvc.alloc_workspace(kvc.OP_ENCODE, desc, pred)
    kvc.kvc_encode_layer(desc, pred, K, V, Ks, Vs, buf, Kr, Vr, ws)
    Kd, Vd = torch.empty_like(K), torch.empty_like(V)
    wsd = kvc.alloc_workspace(kvc.OP_DECODE, desc, pred)
    kvc.kvc_decode_layer(desc, pred, buf, Ks, Vs, Kd, Vd, wsd)
    _sync_ok()
    assert torch.equal(Kd, Kr) and torch.equal(Vd, Vr), "decode must replay encode exactly"
    return buf, Kr, Vr


def _check_xlayer_layer(w, K, V, Ks, Vs, dtype, param, bits, group, rank):
    """GPU vs oracle on one predicted layer, both fed the same K_src / V_src."""
    T, H, D = K.shape
    wg = {k: v.cuda() for k, v in w.items()}
    desc = _desc(T, H, D, dtype, bits, group, param)
    pred = kvc.make_predictor(kvc.PRED_XLAYER_DPLR, wg, rank=rank)
    buf, Kr, Vr = _xlayer_gpu(desc, pred, K.cuda(), V.cuda(), Ks.cuda(), Vs.cuda())
    od = _odesc(T, H, D, dtype, bits, group, param)
    w64 = {k: U.to64(v) for k, v in w.items()}
    Ks64, Vs64 = U.to64(Ks), U.to64(Vs)
    ck, cv, Kh, Vh = O.encode_layer_xlayer(od, w64, U.to64(K), U.to64(V), Ks64, Vs64)
    ek, ev = U.exact_xlayer(od, w64, ck, cv, Ks64, Vs64, Kh)
    errk, errv = U.err_xlayer(od, w64, Ks64, Vs64, Kh)
    p = U.np_param(param)
    # V is predicted from the GPU's own K_rec: tokens with a flipped K code feed it other values
    kflip = _compare(_gpu_coded(buf, T, H, D, bits, group, p, "k"), ck, U.to64(Kr), Kh, ek, U.to64(K), od.state,
                     group, "K", p, errk)
    _compare(_gpu_coded(buf, T, H, D, bits, group, p, "v"), cv, U.to64(Vr), Vh, ev, U.to64(V), od.state, group, "V",
             p, errv, kflip)
    return Kh, Vh


def test_tiny_fp32_cross_layer_chain():
    """The tiny fp32 case: INT4 g32 anchor, then the true block-DPLR maps."""
    wl = synth.tiny_xlayer()
    T, H, D = wl.K[0].shape
    f32 = torch.float32
    # layer 0 (anchor)
    desc0 = _desc(T, H, D, f32, 4, 32, f32)
    p0 = kvc.make_predictor(kvc.PRED_NONE)
    buf0 = kvc.alloc_codes(desc0, p0)
    K0r, V0r = torch.empty(T, H, D, device="cuda"), torch.empty(T, H, D, device="cuda")
    kvc.kvc_encode_layer(desc0, p0, wl.K[0].cuda(), wl.V[0].cuda(), None, None, buf0, K0r, V0r)
    _sync_ok()
    od0 = _odesc(T, H, D, f32, 4, 32, f32)
    ck0, cv0, K0h, V0h = O.encode_layer_none(od0, U.to64(wl.K[0]), U.to64(wl.V[0]))
    U.assert_codes_close(_gpu_coded(buf0, T, H, D, 4, 32, "f32", "k").q, ck0.q, "K0")
    # layer 1 from the oracle's layer-0 reconstruction
    _check_xlayer_layer(wl.weights[1], wl.K[1], wl.V[1], torch.from_numpy(K0h).float(),
                        torch.from_numpy(V0h).float(), f32, f32, 4, 32, wl.rank)
    # the GPU chain end to end against the oracle chain
    w = {k: v.cuda() for k, v in wl.weights[1].items()}
    desc1 = _desc(T, H, D, f32, 4, 32, f32)
    p1 = kvc.make_predictor(kvc.PRED_XLAYER_DPLR, w, rank=wl.rank)
    buf1, K1r, V1r = _xlayer_gpu(desc1, p1, wl.K[1].cuda(), wl.V[1].cuda(), K0r, V0r)
    ck1, cv1, K1h, V1h = O.encode_layer_xlayer(od0, {k: U.to64(v) for k, v in wl.weights[1].items()},
                                               U.to64(wl.K[1]), U.to64(wl.V[1]), K0h, V0h)
    U.assert_codes_close(_gpu_coded(buf1, T, H, D, 4, 32, "f32", "k").q, ck1.q, "chain K1")
    U.assert_codes_close(_gpu_coded(buf1, T, H, D, 4, 32, "f32", "v").q, cv1.q, "chain V1")
    np.testing.assert_allclose(U.to64(V1r), V1h, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("T,rank", [(3 * 128 + 57, 64), (200, 0), (131, 16)])
def test_bf16_cross_layer_parity(T, rank):
    """Wan-shaped heads (12 x 128), INT2 g32 with fp16 (scale, zero); T spans
    several 128-token tiles plus a ragged tail."""
    wl = synth.wan_xlayer(seed=synth.SEED_BASE + 101, L=3, T=T, rank=rank, calib_tokens=1024)
    bf, hf = torch.bfloat16, torch.float16
    for l in (1, 2):
        # teacher forcing: layer l-1 sources are the clean values (bf16), shared by both sides
        _check_xlayer_layer(wl.weights[l], wl.K[l], wl.V[l], wl.K[l - 1], wl.V[l - 1], bf, hf, 2, 32, rank)


def _exact_xlayer_chain(L, T, H, D, r, seed):
    """Layers whose K / V are exact bf16 images of sparse +-1 block-DPLR maps of
    the previous (reconstructed) layer, with an INT2-grid anchor: every residual
    of layers >= 1 is exactly 0 and no rounding decision is near a tie."""
    rng = np.random.default_rng(seed)
    C = H * D

    def sparse(shape, nnz):
        m = np.zeros(shape)
        for idx in np.ndindex(*shape[:-1]):
            m[idx + (rng.choice(shape[-1], nnz, replace=False),)] = rng.choice([-1.0, 1.0], nnz)
        return m

    grid = -1.5 + rng.integers(0, 4, (T, H, D)).astype(np.float64)
    grid[..., 0::32], grid[..., 1::32] = -1.5, 1.5
    K = [grid]
    g2 = -1.5 + rng.integers(0, 4, (T, H, D)).astype(np.float64)
    g2[..., 0::32], g2[..., 1::32] = -1.5, 1.5
    V = [g2]
    W = [None]
    for _ in range(1, L):
        w = dict(k_block=sparse((H, D, D), 1), k_w=sparse((r, C), 1) if r else np.zeros((0, C)),
                 k_u=sparse((C, r), 1) * 0.5 if r else np.zeros((C, 0)),
                 v_block=sparse((H, D, 2 * D), 1), v_w=sparse((r, 2 * C), 1) if r else np.zeros((0, 2 * C)),
                 v_u=sparse((C, r), 1) * 0.5 if r else np.zeros((C, 0)))
        Kl = O.xlayer_predict_k(K[-1], w["k_block"], w["k_w"], w["k_u"])
        Vl = O.xlayer_predict_v(Kl, V[-1], w["v_block"], w["v_w"], w["v_u"])
        assert np.array_equal(O.round_to(Kl, "bf16"), Kl) and np.array_equal(O.round_to(Vl, "bf16"), Vl)
        K.append(Kl)
        V.append(Vl)
        W.append(w)
    t = lambda x: torch.from_numpy(x).float().to(torch.bfloat16).contiguous()
    return [t(k) for k in K], [t(v) for v in V], [None] + [{k: t(v) for k, v in w.items()} for w in W[1:]]


@pytest.mark.parametrize("rank", [64, 0])
def test_cross_layer_chain_exact_predictor(rank):
    """The GPU's own closed-loop chain over several layers (each layer
    predicted from the GPU's reconstruction of the previous one) stays
    bit-identical to the exact values when every prediction is exact."""
    L, T, H, D = 3, 2 * 128 + 40, 12, 128
    K, V, W = _exact_xlayer_chain(L, T, H, D, rank, 31 + rank)
    bf, hf = torch.bfloat16, torch.float16
    desc0 = _desc(T, H, D, bf, 2, 32, hf)
    p0 = kvc.make_predictor(kvc.PRED_NONE)
    buf = kvc.alloc_codes(desc0, p0)
    Kr, Vr = torch.empty(T, H, D, dtype=bf, device="cuda"), torch.empty(T, H, D, dtype=bf, device="cuda")
    kvc.kvc_encode_layer(desc0, p0, K[0].cuda(), V[0].cuda(), None, None, buf, Kr, Vr)
    for l in range(1, L):
        pred = kvc.make_predictor(kvc.PRED_XLAYER_DPLR, {k: v.cuda() for k, v in W[l].items()}, rank=rank)
        b2, Kn, Vn = _xlayer_gpu(desc0, pred, K[l].cuda(), V[l].cuda(), Kr, Vr)
        assert torch.equal(Kn.cpu(), K[l]) and torch.equal(Vn.cpu(), V[l]), f"layer {l}"
        assert int(b2.k_codes.count_nonzero()) == 0 and int(b2.v_codes.count_nonzero()) == 0
        s_, z_ = U.params_from_gpu(b2.k_params, (T, H, D // 32), "f16")
        assert np.all(s_ == 0) and np.all(z_ == 0)
        Kr, Vr = Kn, Vn


@pytest.mark.parametrize("rank", [64, 128])
def test_bf16_cross_layer_full_size_sampled(rank):
    """Full Wan-shaped layer (32760 tokens, so every CTA of the persistent
    kernel codes two tiles); the oracle checks sampled tokens, which are
    independent of one another through the whole layer."""
    dev = "cuda"
    wl = synth.wan_xlayer(seed=synth.SEED_BASE + 1, device=dev, L=3, rank=rank, layers_needed=[2])
    T, H, D = wl.K[2].shape
    bf, hf = torch.bfloat16, torch.float16
    w = wl.weights[2]
    desc = _desc(T, H, D, bf, 2, 32, hf)
    pred = kvc.make_predictor(kvc.PRED_XLAYER_DPLR, w, rank=wl.rank)
    buf, Kr, Vr = _xlayer_gpu(desc, pred, wl.K[2], wl.V[2], wl.K[1], wl.V[1])
    idx = torch.cat([torch.arange(0, 64), torch.randint(64, T - 64, (320,), generator=torch.Generator().manual_seed(3)),
                     torch.arange(T - 64, T)]).sort().values
    sub = lambda t: U.to64(t[idx.to(t.device)])
    od = _odesc(len(idx), H, D, bf, 2, 32, hf)
    w64 = {k: U.to64(v) for k, v in w.items()}
    ck, cv, Kh, Vh = O.encode_layer_xlayer(od, w64, sub(wl.K[2]), sub(wl.V[2]), sub(wl.K[1]), sub(wl.V[1]))
    ek, ev = U.exact_xlayer(od, w64, ck, cv, sub(wl.K[1]), sub(wl.V[1]), Kh)
    errk, errv = U.err_xlayer(od, w64, sub(wl.K[1]), sub(wl.V[1]), Kh)
    ii = idx.numpy()
    kflip = None
    for which, oc, rec, ref, ex, x, er in (("k", ck, Kr, Kh, ek, wl.K[2], errk), ("v", cv, Vr, Vh, ev, wl.V[2], errv)):
        q = U.codes_from_gpu(getattr(buf, which + "_codes"), (T, H, D), 2)[ii]
        s_, z_ = U.params_from_gpu(getattr(buf, which + "_params"), (T, H, D // 32), "f16")
        gc = O.Coded(q, s_[ii], z_[ii])
        f = _compare(gc, oc, sub(rec), ref, ex, sub(x), "bf16", 32, which + " (sampled tokens)", "f16", er, kflip)
        kflip = f


# ---------------------------------------------------------------- temporal


def _temporal_gpu_coded(buf, T, H, D, F, bits, ab, group, param, which):
    F0 = min(F, T) if ab else 0
    raw = getattr(buf, which + "_codes")
    n0 = F0 * H * D * ab // 8
    q0 = U.codes_from_gpu(raw[:n0], (F0, H, D), ab) if F0 else np.zeros((0, H, D), np.uint8)
    q1 = U.codes_from_gpu(raw[n0:], (T - F0, H, D), bits) if T > F0 else np.zeros((0, H, D), np.uint8)
    s, z = U.params_from_gpu(getattr(buf, which + "_params"), (T, H, D // group), param)
    return O.Coded(np.concatenate([q0, q1]), s, z)


def _temporal_call(tw_ak, tw_av, K, V, F, bits, group, param, ab, k_hist=None, v_hist=None):
    """One temporal encode + decode through the ABI; history tensors continue a sequence (ab == 0)."""
    T, H, D = K.shape
    desc = _desc(T, H, D, K.dtype, bits, group, param, F, ab)
    pred = kvc.make_predictor(kvc.PRED_TEMPORAL, {"k_block": tw_ak.cuda(), "v_block": tw_av.cuda()})
    buf = kvc.alloc_codes(desc, pred)
    K, V = K.cuda(), V.cuda()
    kh = None if k_hist is None else k_hist.cuda().contiguous()
    vh = None if v_hist is None else v_hist.cuda().contiguous()
    Kr, Vr = torch.empty_like(K), torch.empty_like(V)
    kvc.kvc_encode_layer(desc, pred, K, V, kh, vh, buf, Kr, Vr)
    Kd, Vd = torch.empty_like(K), torch.empty_like(V)
    kvc.kvc_decode_layer(desc, pred, buf, kh, vh, Kd, Vd)
    _sync_ok()
    assert torch.equal(Kd, Kr) and torch.equal(Vd, Vr), "decode must replay encode exactly"
    return buf, Kr, Vr


@pytest.mark.parametrize("T,H,D,F,bits,group,ab,dtype", [
    (4 * 100 + 16, 4, 128, 100, 4, 64, 4, torch.bfloat16),
    (3 * 50 + 7, 2, 64, 50, 2, 32, 8, torch.float32),
    (37, 2, 128, 64, 4, 64, 4, torch.bfloat16),  # a single partial frame
])
def test_temporal_parity_frame_by_frame(T, H, D, F, bits, group, ab, dtype):
    """Frame 0 (the anchor) from one call of the whole sequence; every later
    frame from a call that continues from the oracle's reconstructed history,
    so each frame's prediction, quantization and packing is checked on its own."""
    tw = synth.temporal_layer(seed=synth.SEED_BASE + 103, T=T, H=H, D=D, F=F, dtype=dtype)
    param = torch.float16 if dtype == torch.bfloat16 else torch.float32
    p = U.np_param(param)
    od = _odesc(T, H, D, dtype, bits, group, param, F, ab)
    w64 = dict(ak=U.to64(tw.ak), av=U.to64(tw.av))
    ck, cv, Kh, Vh = O.encode_layer_temporal(od, w64, U.to64(tw.K), U.to64(tw.V))
    ek, ev = U.exact_temporal(od, w64, ck, cv, Kh, Vh)
    errk, errv = U.err_temporal(od, w64, Kh, Vh)
    buf, Kr, Vr = _temporal_call(tw.ak, tw.av, tw.K, tw.V, F, bits, group, param, ab)
    n0 = min(F, T)
    gk = _temporal_gpu_coded(buf, T, H, D, F, bits, ab, group, p, "k")
    gv = _temporal_gpu_coded(buf, T, H, D, F, bits, ab, group, p, "v")
    sl = slice(0, n0)
    cut = lambda c: O.Coded(c.q[sl], c.s[sl], c.z[sl])
    kf = _compare(cut(gk), cut(ck), U.to64(Kr)[sl], Kh[sl], ek[sl], U.to64(tw.K)[sl], od.state, group, "K frame 0", p)
    _compare(cut(gv), cut(cv), U.to64(Vr)[sl], Vh[sl], ev[sl], U.to64(tw.V)[sl], od.state, group, "V frame 0", p,
             None, kf)
    tdt = torch.float32
    for f in range(1, (T + F - 1) // F):
        a, b = f * F, min(T, (f + 1) * F)
        k_hist = np.zeros((2, F, H, D))
        k_hist[1] = Kh[a - F:a]
        if f >= 2:
            k_hist[0] = Kh[a - 2 * F:a - F]
        v_hist = Vh[a - F:a]
        to_t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(tdt).to(dtype)
        fb, fK, fV = _temporal_call(tw.ak, tw.av, tw.K[a:b], tw.V[a:b], F, bits, group, param, 0,
                                    to_t(k_hist), to_t(v_hist))
        n = b - a
        ofs = O.Desc(n, H, D, od.state, bits, group, p, F, 0)
        fk, fv, fKh, fVh = O.encode_layer_temporal(ofs, w64, U.to64(tw.K[a:b]), U.to64(tw.V[a:b]), k_hist, v_hist)
        fek, fev = U.exact_temporal(ofs, w64, fk, fv, fKh, fVh, k_hist, v_hist)
        erk, erv = U.err_temporal(ofs, w64, fKh, fVh, k_hist, v_hist)
        gk = _temporal_gpu_coded(fb, n, H, D, F, bits, 0, group, p, "k")
        gv = _temporal_gpu_coded(fb, n, H, D, F, bits, 0, group, p, "v")
        kf = _compare(gk, fk, U.to64(fK), fKh, fek, U.to64(tw.K[a:b]), od.state, group, f"K frame {f}", p, erk)
        _compare(gv, fv, U.to64(fV), fVh, fev, U.to64(tw.V[a:b]), od.state, group, f"V frame {f}", p, erv, kf)


def _exact_temporal_workload(T, H, D, F, seed):
    """A sequence whose frames are exact bf16 images of the temporal maps of
    the previous ones (the anchor on the INT2 grid): every residual is 0."""
    rng = np.random.default_rng(seed)
    ak = np.zeros((H, D, 2 * D))
    av = np.zeros((H, D, 2 * D))
    for h in range(H):
        ak[h, :, :D] = 0.5 * np.eye(D)
        ak[h, :, D:] = 0.5 * np.eye(D)
        av[h, :, :D] = np.eye(D)[rng.permutation(D)]
        av[h, :, D:] = 0.5 * np.eye(D)
    grid = lambda shape: np.where(np.arange(D) % 32 == 0, -1.5, np.where(np.arange(D) % 32 == 1, 1.5,
                                                                          -1.5 + rng.integers(0, 4, shape)))
    K = np.zeros((T, H, D))
    V = np.zeros((T, H, D))
    K[:F] = grid((F, H, D))
    V[:F] = grid((F, H, D))
    for f in range(1, (T + F - 1) // F):
        a, b = f * F, min(T, (f + 1) * F)
        n = b - a
        k2 = K[a - 2 * F:a - 2 * F + n] if f >= 2 else 0.0
        K[a:b] = 0.5 * K[a - F:a - F + n] + 0.5 * k2
        V[a:b] = np.einsum("thi,hoi->tho", K[a:b], av[:, :, :D]) + 0.5 * V[a - F:a - F + n]
    assert np.array_equal(O.round_to(K, "bf16"), K) and np.array_equal(O.round_to(V, "bf16"), V)
    t = lambda x: torch.from_numpy(x).float().to(torch.bfloat16)
    return t(K), t(V), t(ak), t(av)


def test_temporal_whole_chain_exact_predictor():
    """Through a whole multi-frame call the GPU chain must stay bit-identical to
    the oracle when no rounding decision is near a tie (exact predictions)."""
    T, H, D, F = 5 * 64 + 9, 2, 128, 64
    K, V, ak, av = _exact_temporal_workload(T, H, D, F, 21)
    buf, Kr, Vr = _temporal_call(ak, av, K, V, F, 2, 32, torch.float16, 2)
    assert torch.equal(Kr.cpu(), K) and torch.equal(Vr.cpu(), V)
    q = _temporal_gpu_coded(buf, T, H, D, F, 2, 2, 32, "f16", "k")
    od = _odesc(T, H, D, torch.bfloat16, 2, 32, torch.float16, F, 2)
    ck, cv, _, _ = O.encode_layer_temporal(od, dict(ak=U.to64(ak), av=U.to64(av)), U.to64(K), U.to64(V))
    np.testing.assert_array_equal(q.q, ck.q)
    np.testing.assert_array_equal(q.s, ck.s)


def _per_head(c: "O.Coded") -> "O.Coded":
    """A coded [n, H, ...] tensor viewed as n*H single-head rows (each head's
    temporal chain is independent of the others)."""
    f = lambda a: a.reshape((a.shape[0] * a.shape[1], 1) + a.shape[2:])
    return O.Coded(f(c.q), f(c.s), f(c.z))


def test_temporal_continued_call_full_shape():
    """A continued call of three 1560-token frames of the large-backbone case
    (40 heads, INT4 g64) from a supplied history (the clean frames 18 and 19,
    bf16 values shared by both sides), against the oracle at sampled
    positions, frame by frame.  Each (position, head) chain whose earlier frames
    differ anywhere is only checked for validity from there on.  (The
    whole-layer call is checked in test_gpu_full_size.py.)"""
    tw = synth.temporal_layer(seed=synth.SEED_BASE + 3, device="cuda")
    T, H, D = tw.K.shape
    F = tw.frame_tokens
    hf = torch.float16
    n_last = T - (T // F) * F
    pos = np.sort(np.concatenate([np.arange(0, 4), np.arange(n_last - 2, n_last + 2), [F - 1],
                                  np.random.default_rng(5).choice(np.arange(n_last + 2, F - 1), 15, replace=False)]))
    w64 = dict(ak=U.to64(tw.ak), av=U.to64(tw.av))
    f0, nf = 20, 3
    a, b = f0 * F, (f0 + nf) * F
    k_hist = tw.K[(f0 - 2) * F:f0 * F].reshape(2, F, H, D)
    v_hist = tw.V[(f0 - 1) * F:f0 * F]
    fb, fK, fV = _temporal_call(tw.ak, tw.av, tw.K[a:b], tw.V[a:b], F, 4, 64, hf, 0, k_hist, v_hist)
    rows_b = np.array([f * F + s for f in range(nf) for s in pos])
    hist_rows = np.array([f * F + s for f in range(2) for s in pos])
    sb = lambda t: U.to64(t[torch.from_numpy(rows_b).to(t.device)])
    kh64 = U.to64(k_hist.reshape(2 * F, H, D)[torch.from_numpy(hist_rows).cuda()]).reshape(2, len(pos), H, D)
    vh64 = U.to64(v_hist[torch.from_numpy(pos).cuda()])
    ofs = _odesc(len(rows_b), H, D, torch.bfloat16, 4, 64, hf, len(pos), 0)
    fk, fv, fKh, fVh = O.encode_layer_temporal(ofs, w64, sb(tw.K[a:b]), sb(tw.V[a:b]), kh64, vh64)
    fek, fev = U.exact_temporal(ofs, w64, fk, fv, fKh, fVh, kh64, vh64)
    erk, erv = U.err_temporal(ofs, w64, fKh, fVh, kh64, vh64)
    npos = len(pos)
    diverged = np.zeros(npos * H, bool)  # per (position, head)
    gq = {w: U.codes_from_gpu(getattr(fb, w + "_codes"), (nf * F, H, D), 4)[rows_b] for w in "kv"}
    gp = {w: U.params_from_gpu(getattr(fb, w + "_params"), (nf * F, H, D // 64), "f16") for w in "kv"}
    flat = lambda x: x.reshape(x.shape[0] * x.shape[1], 1, x.shape[2])
    for f in range(nf):
        sl = slice(f * npos, (f + 1) * npos)
        cut = lambda c: _per_head(O.Coded(c.q[sl], c.s[sl], c.z[sl]))
        kf = diverged.copy()
        for which, oc, rec, ref, ex, x, er in (("k", fk, fK, fKh, fek, tw.K[a:b], erk),
                                              ("v", fv, fV, fVh, fev, tw.V[a:b], erv)):
            s_, z_ = gp[which]
            g = _per_head(O.Coded(gq[which][sl], s_[rows_b][sl], z_[rows_b][sl]))
            kf = kf | _compare(g, cut(oc), flat(sb(rec)[sl]), flat(ref[sl]), flat(ex[sl]), flat(sb(x)[sl]), "bf16",
                               64, f"{which} continued frame {f}", "f16", flat(er[sl]), kf)
        diverged |= kf


# ---------------------------------------------------------------- clustered


def _cluster_pred(cw: synth.ClusterWorkload, n_c):
    w = dict(k_centroids=cw.k_centroids.cuda(), k_enc=cw.k_enc.cuda(), k_dec=cw.k_dec.cuda(),
             v_centroids=cw.v_centroids.cuda(), v_enc=cw.v_enc.cuda(), v_dec=cw.v_dec.cuda())
    return kvc.make_predictor(kvc.PRED_CLUSTER, w, n_clusters=n_c, code_dim=cw.k_enc.shape[0])


def _check_cluster(cw, buf, Kr, Vr, T, H, D, dtype, param, n_c):
    """Assignments, coefficient codes, (scale, zero) pairs and reconstructions
    of both tensors against the C++ oracle."""
    od = _odesc(T, H, D, dtype, 4, 32, param)
    p = U.np_param(param)
    for which, X, cent, enc, dec, rec in (("k", cw.K, cw.k_centroids, cw.k_enc, cw.k_dec, Kr),
                                          ("v", cw.V, cw.v_centroids, cw.v_enc, cw.v_dec, Vr)):
        X64, c64 = U.to64(X), U.to64(cent)
        oc, xh = O.encode_tensor_cluster(od, X64, c64, U.to64(enc), U.to64(dec))
        a_gpu = getattr(buf, which + "_assign")[:T].cpu().numpy().astype(np.int64)
        # the assignment is unique where the best and second-best scores are apart
        sc = ON.cluster_scores(X64.reshape(T, -1), c64)
        srt = np.sort(sc, axis=1)
        margin = srt[:, 1] - srt[:, 0]
        clear = margin > 1e-4 * np.abs(srt[:, 0]) + 1e-3
        np.testing.assert_array_equal(a_gpu[clear], oc.assign[clear])
        assert np.all(sc[np.arange(T), a_gpu] <= srt[:, 0] + 1e-4 * np.abs(srt[:, 0]) + 1e-3)
        assert clear.mean() > 0.99
        q = U.codes_from_gpu(getattr(buf, which + "_codes"), (T, 128), 4)
        s, z = U.params_from_gpu(getattr(buf, which + "_params"), (T, 4), p)
        U.assert_codes_close(q, oc.q, which + " coefficient codes")
        ecoef = U.err_cluster(X64.reshape(T, -1), c64, oc.assign, U.to64(enc))
        pdiff = U.assert_params_close(s[clear], z[clear], oc.s[clear], oc.z[clear], p, which + " params",
                                      levels=15, err=ecoef[clear], group=32)
        exact = (c64[oc.assign] + ON.dequantize_groups(oc.q, oc.s, oc.z, 32) @ U.to64(dec).T).reshape(T, H, D)
        # a token whose centre, any code or any (scale, zero) differs has every channel moved
        tok_flip = (q != oc.q).any(axis=1) | ~clear
        tok_flip[np.flatnonzero(clear)[pdiff.any(axis=1)]] = True
        flip = np.repeat(tok_flip, H * D).reshape(T, H, D)
        coef_hat = ON.dequantize_groups(oc.q, oc.s, oc.z, 32)
        erec = (128 * U.U32 * (np.abs(coef_hat) @ np.abs(U.to64(dec)).T) + U.U32 * np.abs(c64[oc.assign]))
        if rec is not None:
            U.assert_recon_close(U.to64(rec), xh, exact, X64, flip, od.state, which + " recon",
                                 err=erec.reshape(T, H, D))


@pytest.mark.parametrize("T,H,n_c", [(1000, 4, 32), (300, 16, 256), (2000 - 5, 16, 256)])
def test_cluster_codec_parity(T, H, n_c):
    cw = synth.cluster_layer(seed=synth.SEED_BASE + 104, T=T, H=H, n_c=n_c, iters=5)
    D = 128
    bf, hf = torch.bfloat16, torch.float16
    desc = _desc(T, H, D, bf, 4, 32, hf)
    pred = _cluster_pred(cw, n_c)
    buf = kvc.alloc_codes(desc, pred)
    K, V = cw.K.cuda(), cw.V.cuda()
    Kr, Vr = torch.empty_like(K), torch.empty_like(V)
    ws = kvc.alloc_workspace(kvc.OP_ENCODE, desc, pred)
    kvc.kvc_encode_layer(desc, pred, K, V, None, None, buf, Kr, Vr, ws)
    Kd, Vd = torch.empty_like(K), torch.empty_like(V)
    kvc.kvc_decode_layer(desc, pred, buf, None, None, Kd, Vd, kvc.alloc_workspace(kvc.OP_DECODE, desc, pred))
    _sync_ok()
    assert torch.equal(Kd, Kr) and torch.equal(Vd, Vr)
    _check_cluster(cw, buf, Kr, Vr, T, H, D, bf, hf, n_c)


def test_cluster_token_equal_to_its_centre_codes_zero():
    """A token equal to a centre has the coefficients Y - P[a] = 0 exactly: P = C E^T
    comes from the token pass's own products in the same order (the P pass over the
    centre table).  Such tokens take that centre, and every (scale, zero) pair of
    theirs is exactly 0, so their reconstruction is the centre itself."""
    T, H, n_c = 333, 16, 256
    cw = synth.cluster_layer(seed=synth.SEED_BASE + 105, T=T, H=H, n_c=n_c, iters=5)
    D = 128
    bf, hf = torch.bfloat16, torch.float16
    rows = torch.arange(0, T, 7)
    js = (rows * 37) % n_c
    K, V = cw.K.clone(), cw.V.clone()
    K.view(T, H * D)[rows] = cw.k_centroids[js].to(bf)
    V.view(T, H * D)[rows] = cw.v_centroids[js].to(bf)
    desc = _desc(T, H, D, bf, 4, 32, hf)
    pred = _cluster_pred(cw, n_c)
    buf = kvc.alloc_codes(desc, pred)
    K, V = K.cuda(), V.cuda()
    Kr, Vr = torch.empty_like(K), torch.empty_like(V)
    kvc.kvc_encode_layer(desc, pred, K, V, None, None, buf, Kr, Vr, kvc.alloc_workspace(kvc.OP_ENCODE, desc, pred))
    _sync_ok()
    for which, X, rec in (("k", K, Kr), ("v", V, Vr)):
        a = getattr(buf, which + "_assign").cpu().long()
        assert torch.equal(a[rows], js), which
        params = getattr(buf, which + "_params").view(torch.uint8).view(torch.float16).view(T, -1).cpu().float()
        assert float(params[rows].abs().sum()) == 0.0, which
        assert torch.equal(rec.view(T, -1)[rows.cuda()], X.view(T, -1)[rows.cuda()]), which


@pytest.mark.parametrize("dtype,T,H,n_c", [(torch.float32, 300, 2, 16), (torch.bfloat16, 257, 3, 40)])
def test_cluster_codec_cuda_core_path(dtype, T, H, n_c):
    """fp32 data, or a joint row of 384 channels (not a multiple of 256): the
    CUDA-core kernels, against the oracle."""
    cw = synth.cluster_layer(seed=synth.SEED_BASE + 109, T=T, H=H, n_c=n_c, iters=3, dtype=dtype)
    D = 128
    param = torch.float32 if dtype == torch.float32 else torch.float16
    desc = _desc(T, H, D, dtype, 4, 32, param)
    pred = _cluster_pred(cw, n_c)
    buf = kvc.alloc_codes(desc, pred)
    K, V = cw.K.cuda(), cw.V.cuda()
    Kr, Vr = torch.empty_like(K), torch.empty_like(V)
    kvc.kvc_encode_layer(desc, pred, K, V, None, None, buf, Kr, Vr, kvc.alloc_workspace(kvc.OP_ENCODE, desc, pred))
    Kd, Vd = torch.empty_like(K), torch.empty_like(V)
    kvc.kvc_decode_layer(desc, pred, buf, None, None, Kd, Vd, kvc.alloc_workspace(kvc.OP_DECODE, desc, pred))
    _sync_ok()
    assert torch.equal(Kd, Kr) and torch.equal(Vd, Vr)
    _check_cluster(cw, buf, Kr, Vr, T, H, D, dtype, param, n_c)


def test_cluster_static_entry_against_the_oracle():
    """The clustered encode that allocates nothing, against the oracle."""
    T, H, D, n_c = 700, 4, 128, 64
    cw = synth.cluster_layer(seed=synth.SEED_BASE + 110, T=T, H=H, n_c=n_c, iters=3)
    bf, hf = torch.bfloat16, torch.float16
    desc = _desc(T, H, D, bf, 4, 32, hf)
    pred = _cluster_pred(cw, n_c)
    buf = kvc.alloc_codes(desc, pred)
    K, V = cw.K.cuda(), cw.V.cuda()
    Kr, Vr = torch.empty_like(K), torch.empty_like(V)
    kvc.kvc_encode_layer_cluster_static(desc, pred, K, V, buf, Kr, Vr)
    _sync_ok()
    _check_cluster(cw, buf, Kr, Vr, T, H, D, bf, hf, n_c)


# ---------------------------------------------------------------- attention


def _oracle_codes_to_gpu(ck, cv, bits, param, assign=False):
    t = lambda q: U.pad16(U.codes_to_gpu(q, bits))
    p = lambda c: U.pad16(U.params_to_gpu(c.s, c.z, param))
    buf = kvc.CodeBuffers(t(ck.q), p(ck), t(cv.q), p(cv))
    if assign:
        buf.k_assign = U.pad16(torch.from_numpy(ck.assign.astype(np.uint8)).cuda())
        buf.v_assign = U.pad16(torch.from_numpy(cv.assign.astype(np.uint8)).cuda())
    return buf


@pytest.mark.parametrize("n_q,n_self,T,rank", [(300, 130, 3 * 128 + 5, 64), (129, 0, 256, 16), (64, 128, 100, 0),
                                               (700, 300, 16 * 128 - 7, 64), (1100, 0, 9 * 128, 128)])
def test_compressed_attention_cross_layer(n_q, n_self, T, rank):
    """Attention over a decoded cross-layer history plus uncompressed chunk
    tokens, history codes written by the oracle."""
    wl = synth.wan_xlayer(seed=synth.SEED_BASE + 102, L=2, T=T, rank=rank, calib_tokens=1024)
    H, D = 12, 128
    bf, hf = torch.bfloat16, torch.float16
    od = _odesc(T, H, D, bf, 2, 32, hf)
    w64 = {k: U.to64(v) for k, v in wl.weights[1].items()}
    Ks, Vs = U.to64(wl.K[0]), U.to64(wl.V[0])
    ck, cv, _, _ = O.encode_layer_xlayer(od, w64, U.to64(wl.K[1]), U.to64(wl.V[1]), Ks, Vs)
    buf = _oracle_codes_to_gpu(ck, cv, 2, "f16")
    Q = synth.queries(11, n_q, H, D)
    Kself = synth.queries(12, n_self, H, D)
    Vself = synth.queries(13, n_self, H, D)
    desc = _desc(T, H, D, bf, 2, 32, hf)
    pred = kvc.make_predictor(kvc.PRED_XLAYER_DPLR, {k: v.cuda() for k, v in wl.weights[1].items()}, rank=rank)
    Og = torch.empty(n_q, H, D, dtype=bf, device="cuda")
    ws = kvc.alloc_workspace(kvc.OP_ATTEND, desc, pred, n_q)
    kvc.kvc_attend_compressed(desc, pred, Q.cuda(), buf, wl.K[0].cuda(), wl.V[0].cuda(),
                              Kself.cuda() if n_self else None, Vself.cuda() if n_self else None,
                              D ** -0.5, Og, ws)
    _sync_ok()
    ref = O.attend_compressed_xlayer(od, w64, U.to64(Q), ck, cv, Ks, Vs, U.to64(Kself) if n_self else None,
                                     U.to64(Vself) if n_self else None, D ** -0.5)
    err = U.rel_l2(U.to64(Og), ref)
    assert err <= U.ATT_TOL[bf], err


@pytest.mark.parametrize("rank", [64, 128])
def test_compressed_attention_full_size(rank):
    """256 queries over a full Wan-shaped history (32760 tokens, 21 latent
    frames) plus 130 chunk tokens: the latent pass codes two tiles per CTA."""
    wl = synth.wan_xlayer(seed=synth.SEED_BASE + 106, L=2, rank=rank, calib_tokens=1024)
    T, H, D = wl.K[1].shape
    n_q, n_self = 256, 130
    bf, hf = torch.bfloat16, torch.float16
    od = _odesc(T, H, D, bf, 2, 32, hf)
    w64 = {k: U.to64(v) for k, v in wl.weights[1].items()}
    Ks, Vs = U.to64(wl.K[0]), U.to64(wl.V[0])
    ck, cv, _, _ = O.encode_layer_xlayer(od, w64, U.to64(wl.K[1]), U.to64(wl.V[1]), Ks, Vs)
    buf = _oracle_codes_to_gpu(ck, cv, 2, "f16")
    Q = synth.queries(21, n_q, H, D)
    Kself = synth.queries(22, n_self, H, D)
    Vself = synth.queries(23, n_self, H, D)
    desc = _desc(T, H, D, bf, 2, 32, hf)
    pred = kvc.make_predictor(kvc.PRED_XLAYER_DPLR, {k: v.cuda() for k, v in wl.weights[1].items()}, rank=rank)
    Og = torch.empty(n_q, H, D, dtype=bf, device="cuda")
    ws = kvc.alloc_workspace(kvc.OP_ATTEND, desc, pred, n_q)
    kvc.kvc_attend_compressed(desc, pred, Q.cuda(), buf, wl.K[0].cuda(), wl.V[0].cuda(), Kself.cuda(),
                              Vself.cuda(), D ** -0.5, Og, ws)
    _sync_ok()
    ref = O.attend_compressed_xlayer(od, w64, U.to64(Q), ck, cv, Ks, Vs, U.to64(Kself), U.to64(Vself), D ** -0.5)
    err = U.rel_l2(U.to64(Og), ref)
    assert err <= U.ATT_TOL[bf], err


def test_tiny_fp32_attention():
    """64 fp32 queries over the decoded 512-token tiny history (both layers)."""
    wl = synth.tiny_xlayer()
    T, H, D = wl.K[0].shape
    f32 = torch.float32
    od = _odesc(T, H, D, f32, 4, 32, f32)
    ck0, cv0, K0h, V0h = O.encode_layer_none(od, U.to64(wl.K[0]), U.to64(wl.V[0]))
    w64 = {k: U.to64(v) for k, v in wl.weights[1].items()}
    ck1, cv1, _, _ = O.encode_layer_xlayer(od, w64, U.to64(wl.K[1]), U.to64(wl.V[1]), K0h, V0h)
    Q = synth.queries(7, 64, H, D, dtype=f32)
    desc = _desc(T, H, D, f32, 4, 32, f32)
    for layer, (ck, cv) in enumerate(((ck0, cv0), (ck1, cv1))):
        buf = _oracle_codes_to_gpu(ck, cv, 4, "f32")
        if layer == 0:
            pred = kvc.make_predictor(kvc.PRED_NONE)
            src = (None, None)
            ref = O.attention(U.to64(Q), *O.decode_layer_none(od, ck, cv), 0.125)
        else:
            pred = kvc.make_predictor(kvc.PRED_XLAYER_DPLR, {k: v.cuda() for k, v in wl.weights[1].items()},
                                      rank=wl.rank)
            src = (torch.from_numpy(K0h).float().cuda(), torch.from_numpy(V0h).float().cuda())
            ref = O.attend_compressed_xlayer(od, w64, U.to64(Q), ck, cv, K0h, V0h, None, None, 0.125)
        Og = torch.empty(64, H, D, device="cuda")
        ws = kvc.alloc_workspace(kvc.OP_ATTEND, desc, pred, 64)
        kvc.kvc_attend_compressed(desc, pred, Q.cuda(), buf, *src, None, None, 0.125, Og, ws)
        _sync_ok()
        assert U.rel_l2(U.to64(Og), ref) <= U.ATT_TOL[f32]


# T = 60 is one key tile, so the kernel runs unsplit; the others run as two key
# splits merged by the combine kernel
@pytest.mark.parametrize("n_q,T,H,n_c", [(100, 1000, 4, 32), (33, 300, 16, 256), (300, 2000 - 9, 16, 256),
                                         (70, 60, 4, 16)])
def test_mixed_dimensional_attention(n_q, T, H, n_c):
    cw = synth.cluster_layer(seed=synth.SEED_BASE + 105, T=T, H=H, n_c=n_c, iters=3)
    D = 128
    od = _odesc(T, H, D, torch.bfloat16, 4, 32, torch.float16)
    ck, _ = O.encode_tensor_cluster(od, U.to64(cw.K), U.to64(cw.k_centroids), U.to64(cw.k_enc), U.to64(cw.k_dec))
    cv, _ = O.encode_tensor_cluster(od, U.to64(cw.V), U.to64(cw.v_centroids), U.to64(cw.v_enc), U.to64(cw.v_dec))
    buf = _oracle_codes_to_gpu(ck, cv, 4, "f16", assign=True)
    Q = synth.queries(17, n_q, H, D)
    desc = _desc(T, H, D, torch.bfloat16, 4, 32, torch.float16)
    pred = _cluster_pred(cw, n_c)
    Og = torch.empty(n_q, H, D, dtype=torch.bfloat16, device="cuda")
    kvc.kvc_attend_compressed(desc, pred, Q.cuda(), buf, None, None, None, None, D ** -0.5, Og,
                              kvc.alloc_workspace(kvc.OP_ATTEND, desc, pred, n_q))
    _sync_ok()
    ref = O.mixed_attention(U.to64(Q), ck, U.to64(cw.k_centroids), U.to64(cw.k_dec), cv, U.to64(cw.v_centroids),
                            U.to64(cw.v_dec), od, D ** -0.5)
    assert U.rel_l2(U.to64(Og), ref) <= U.ATT_TOL[torch.bfloat16]


# ---------------------------------------------------------------- decoded history out of the attention


def _history_outputs_case(desc, pred, buf, Q, Ks, Vs, Kself, Vself, scale, T, H, D, dtype):
    """kvc_attend_compressed with K_rec_opt / V_rec_opt: the outputs equal
    kvc_decode_layer's bit for bit, and O equals the call without them."""
    n_q = Q.shape[0]
    ws = kvc.alloc_workspace(kvc.OP_ATTEND, desc, pred, n_q)
    O1 = torch.empty(n_q, H, D, dtype=dtype, device="cuda")
    O2 = torch.empty_like(O1)
    kvc.kvc_attend_compressed(desc, pred, Q, buf, Ks, Vs, Kself, Vself, scale, O1, ws)
    Kh = torch.full((T, H, D), float("nan"), dtype=dtype, device="cuda")
    Vh = torch.full_like(Kh, float("nan"))
    kvc.kvc_attend_compressed(desc, pred, Q, buf, Ks, Vs, Kself, Vself, scale, O2, ws, K_rec=Kh, V_rec=Vh)
    Kd, Vd = torch.empty_like(Kh), torch.empty_like(Vh)
    kvc.kvc_decode_layer(desc, pred, buf, Ks, Vs, Kd, Vd, kvc.alloc_workspace(kvc.OP_DECODE, desc, pred))
    _sync_ok()
    assert torch.equal(Kh, Kd) and torch.equal(Vh, Vd), "decoded history differs from kvc_decode_layer"
    assert torch.equal(O1, O2), "asking for the history changed the attention output"
    # only one of the two
    Kh1 = torch.full_like(Kh, float("nan"))
    kvc.kvc_attend_compressed(desc, pred, Q, buf, Ks, Vs, Kself, Vself, scale, O2, ws, K_rec=Kh1)
    _sync_ok()
    assert torch.equal(Kh1, Kd)


@pytest.mark.parametrize("n_q,n_self,T,rank", [(700, 130, 16 * 128 - 7, 64), (129, 0, 300, 0), (1100, 0, 9 * 128, 128)])
def test_attention_history_outputs_cross_layer(n_q, n_self, T, rank):
    """Tensor-core path: 700 queries are two clusters of query tiles per head;
    the first cluster stores the tiles it decodes (ragged T clips the last)."""
    wl = synth.wan_xlayer(seed=synth.SEED_BASE + 107, L=2, T=T, rank=rank, calib_tokens=1024)
    H, D = 12, 128
    bf, hf = torch.bfloat16, torch.float16
    desc = _desc(T, H, D, bf, 2, 32, hf)
    pred = kvc.make_predictor(kvc.PRED_XLAYER_DPLR, {k: v.cuda() for k, v in wl.weights[1].items()}, rank=rank)
    buf, _, _ = _xlayer_gpu(desc, pred, wl.K[1].cuda(), wl.V[1].cuda(), wl.K[0].cuda(), wl.V[0].cuda())
    Q = synth.queries(31, n_q, H, D).cuda()
    Ks = synth.queries(32, n_self, H, D).cuda() if n_self else None
    Vs = synth.queries(33, n_self, H, D).cuda() if n_self else None
    _history_outputs_case(desc, pred, buf, Q, wl.K[0].cuda(), wl.V[0].cuda(), Ks, Vs, D ** -0.5, T, H, D, bf)


def test_attention_history_outputs_fp32_and_clustered():
    """CUDA-core path (fp32 tiny layer) and the clustered history."""
    wl = synth.tiny_xlayer()
    T, H, D = wl.K[0].shape
    f32 = torch.float32
    desc = _desc(T, H, D, f32, 4, 32, f32)
    pred = kvc.make_predictor(kvc.PRED_XLAYER_DPLR, {k: v.cuda() for k, v in wl.weights[1].items()}, rank=wl.rank)
    buf, _, _ = _xlayer_gpu(desc, pred, wl.K[1].cuda(), wl.V[1].cuda(), wl.K[0].cuda(), wl.V[0].cuda())
    Q = synth.queries(7, 64, H, D, dtype=f32).cuda()
    _history_outputs_case(desc, pred, buf, Q, wl.K[0].cuda(), wl.V[0].cuda(), None, None, 0.125, T, H, D, f32)
    cw = synth.cluster_layer(seed=synth.SEED_BASE + 108, T=500, H=16, n_c=64, iters=3)
    bf, hf = torch.bfloat16, torch.float16
    cdesc = _desc(500, 16, 128, bf, 4, 32, hf)
    cpred = _cluster_pred(cw, 64)
    cbuf = kvc.alloc_codes(cdesc, cpred)
    kvc.kvc_encode_layer(cdesc, cpred, cw.K.cuda(), cw.V.cuda(), None, None, cbuf, None, None,
                         kvc.alloc_workspace(kvc.OP_ENCODE, cdesc, cpred))
    Qc = synth.queries(8, 90, 16, 128).cuda()
    _history_outputs_case(cdesc, cpred, cbuf, Qc, None, None, None, None, 128 ** -0.5, 500, 16, 128, bf)


# ---------------------------------------------------------------- Jensen-bias-corrected attention


@pytest.mark.parametrize("n_q,n_self,T,rank,group", [(300, 130, 3 * 128 + 5, 64, 32), (700, 256, 16 * 128 - 7, 64, 32),
                                                     (129, 64, 256, 0, 64)])
def test_debiased_attention_cross_layer(n_q, n_self, T, rank, group):
    """kvc_attend_compressed_debiased against the oracle's corrected softmax
    (history codes by the oracle).  Queries are scaled so that the correction
    moves the output well beyond the tolerance: the GPU result must be close to
    the corrected reference and not to the plain one."""
    wl = synth.wan_xlayer(seed=synth.SEED_BASE + 112, L=2, T=T, rank=rank, calib_tokens=1024)
    H, D = 12, 128
    bf, hf = torch.bfloat16, torch.float16
    od = _odesc(T, H, D, bf, 2, group, hf)
    w64 = {k: U.to64(v) for k, v in wl.weights[1].items()}
    Ks, Vs = U.to64(wl.K[0]), U.to64(wl.V[0])
    ck, cv, _, _ = O.encode_layer_xlayer(od, w64, U.to64(wl.K[1]), U.to64(wl.V[1]), Ks, Vs)
    buf = _oracle_codes_to_gpu(ck, cv, 2, "f16")
    Q = (synth.queries(41, n_q, H, D).float() * 3).to(bf)
    Kself, Vself = synth.queries(42, n_self, H, D), synth.queries(43, n_self, H, D)
    desc = _desc(T, H, D, bf, 2, group, hf)
    pred = kvc.make_predictor(kvc.PRED_XLAYER_DPLR, {k: v.cuda() for k, v in wl.weights[1].items()}, rank=rank)
    Og = torch.empty(n_q, H, D, dtype=bf, device="cuda")
    ws = kvc.alloc_workspace(kvc.OP_ATTEND, desc, pred, n_q)
    kvc.kvc_attend_compressed_debiased(desc, pred, Q.cuda(), buf, wl.K[0].cuda(), wl.V[0].cuda(), Kself.cuda(),
                                       Vself.cuda(), D ** -0.5, Og, ws)
    _sync_ok()
    args = (od, w64, U.to64(Q), ck, cv, Ks, Vs, U.to64(Kself), U.to64(Vself), D ** -0.5)
    ref = O.attend_compressed_xlayer(*args, jensen=True)
    plain = O.attend_compressed_xlayer(*args)
    err = U.rel_l2(U.to64(Og), ref)
    moved = U.rel_l2(plain, ref)
    U.OBSERVED.append({"check": f"debiased attention T={T}", "rel_l2": err, "correction_moves": moved})
    assert err <= U.ATT_TOL[bf], err
    assert err < 0.25 * moved, (err, moved)


# ---------------------------------------------------------------- H64 / EDEN-2 residual codec


def _eden_from_gpu(codes, params, T, H, D, param):
    """Pair indices [T, H, D/2] and scales [T, H, D/64] from the GPU buffers."""
    raw = codes[: T * H * D // 4].cpu().numpy().reshape(T, H, D // 4)
    idx = np.stack([raw & 15, raw >> 4], axis=-1).reshape(T, H, D // 2)
    n = T * H * (D // 64)
    dt = torch.float16 if param == "f16" else torch.float32
    s = params[: n * (2 if param == "f16" else 4)].view(dt).reshape(T, H, D // 64).cpu().double().numpy()
    return idx, s


def _check_eden(idx_g, s_g, rec_g, oc, rec_ref, pred_ref, x, cb, state, param, what, skip=None, perr=0.0):
    """Indices, scales and reconstructions of one tensor coded with H64 /
    EDEN-2.  A group whose index or scale differs (a near tie of the nearest
    point, or an fp16 rounding boundary) must reconstruct its own codes; the
    fraction of such groups is bounded like the scalar codec's parameters.
    Returns the per-token mask of tokens that differ anywhere."""
    from scipy.linalg import hadamard

    T, H, D = x.shape
    keep = np.ones(T, bool) if skip is None else ~skip
    U.assert_codes_close(idx_g[keep], oc.q[keep], what + " pair indices")
    gi = (idx_g != oc.q).reshape(T, H, D // 64, 32).any(-1)
    # fp16 scales either agree or sit on two sides of a rounding boundary; fp32
    # scales of the same indices differ only in their last bits (fp32 sums)
    gs = s_g != oc.s if param == "f16" else np.abs(s_g - oc.s) > 1e-5 * np.abs(oc.s)
    gdiff = (gi | gs) & keep[:, None, None]
    n_ok = int(keep.sum()) * H * (D // 64)
    rate = gdiff.sum() / max(n_ok, 1)
    U.OBSERVED.append({"check": what + " groups differing", "param": param, "param_groups_differing": float(rate),
                       "groups": n_ok})
    assert rate <= U.PARAM_FLIP_RATE + U.PARAM_FLIP_SLACK_GROUPS / max(n_ok, 1), (what, rate)
    # scales of agreeing groups: one rounding step of the parameter format plus the fp32 error
    same = ~gi & keep[:, None, None]
    ulp = U.param_ulp(oc.s, param)
    assert np.all(np.abs(s_g - oc.s)[same] <= 1.0001 * (ulp[same] + 1e-4 * np.abs(oc.s[same]))), what + " scales"
    # every group reconstructs its own codes around the oracle's prediction
    Hs = hadamard(64).astype(np.float64) / 8.0
    yh = s_g[..., None, None] * cb[idx_g.reshape(T, H, D // 64, 32)]
    own = pred_ref + (yh.reshape(T, H, D // 64, 64) @ Hs.T).reshape(T, H, D)
    tol = 1e-3 * (np.abs(x) + 1.0)
    # the GPU's fp32 prediction (perr) and its two fp32 transforms (six butterfly stages each)
    err = perr + 8 * U.U32 * (np.abs(own) + np.abs(pred_ref)) + 64 * U.U32 * np.abs(s_g).max()
    ulp_s = np.abs(O.round_to(own, state) - own) + np.spacing(np.abs(own).astype(np.float32))
    live = keep[:, None, None]
    bad = live & (np.abs(rec_g - own) > tol + err + ulp_s)
    assert not np.any(bad), f"{what}: {int(bad.sum())} values do not reconstruct their own codes"
    flip = np.repeat(gdiff, 64, axis=-1)
    # a rounding tie of the state dtype is judged with the same GPU error bound
    U.assert_recon_close(np.where(live, rec_g, rec_ref), rec_ref, own, x, flip | ~live, state, what + " recon",
                         err=err)
    return (gdiff.reshape(T, -1).any(1)) | (rec_g != rec_ref).reshape(T, -1).any(1)


@pytest.mark.parametrize("dtype,T,H,D,rank", [(torch.bfloat16, 3 * 128 + 41, 12, 128, 64),
                                              (torch.bfloat16, 2 * 128 + 7, 4, 128, 0),
                                              (torch.bfloat16, 300, 2, 128, 128),
                                              (torch.bfloat16, 97, 3, 64, 0), (torch.float32, 130, 2, 128, 8)])
def test_eden2_codec_parity(dtype, T, H, D, rank):
    """An anchor layer and a predicted cross-layer layer with the H64 / EDEN-2
    residual codec, against the oracle (teacher-forced layer-0 sources).  bf16
    with head_dim 128 and rank 0 / 64 / 128 runs the tensor-core codec (the
    epilogue transforms and codes each 64-value group in one thread); the other
    shapes run the CUDA-core kernels."""
    cbt = synth.eden2_codebook()
    cb = cbt.double().numpy()
    wl = synth.wan_xlayer(seed=synth.SEED_BASE + 113, L=2, T=T, H=H, D=D, rank=rank, calib_tokens=512, dtype=dtype)
    param_t = torch.float16 if dtype == torch.bfloat16 else torch.float32
    p = U.np_param(param_t)
    state = U.np_state(dtype)
    desc = kvc.make_desc(T, H, D, dtype, 2, 64, param_t, residual_codec=kvc.RESIDUAL_H64_EDEN2)
    od = O.Desc(T, H, D, state, 2, 64, p, codec="eden2")
    # anchor
    p0 = kvc.make_predictor(kvc.PRED_NONE, residual_codebook=cbt.cuda())
    buf0 = kvc.alloc_codes(desc, p0)
    K0, V0 = wl.K[0].cuda(), wl.V[0].cuda()
    K0r, V0r = torch.empty_like(K0), torch.empty_like(V0)
    kvc.kvc_encode_layer(desc, p0, K0, V0, None, None, buf0, K0r, V0r)
    K0d, V0d = torch.empty_like(K0), torch.empty_like(V0)
    kvc.kvc_decode_layer(desc, p0, buf0, None, None, K0d, V0d)
    _sync_ok()
    assert torch.equal(K0d, K0r) and torch.equal(V0d, V0r)
    ck0, cv0, K0h, V0h = O.encode_layer_none(od, U.to64(wl.K[0]), U.to64(wl.V[0]), codebook=cb)
    zero = np.zeros((T, H, D))
    for which, oc, rec, ref, x in (("k", ck0, K0r, K0h, wl.K[0]), ("v", cv0, V0r, V0h, wl.V[0])):
        idx, s = _eden_from_gpu(getattr(buf0, which + "_codes"), getattr(buf0, which + "_params"), T, H, D, p)
        _check_eden(idx, s, U.to64(rec), oc, ref, zero, U.to64(x), cb, state, p, f"anchor {which}")
    # a predicted layer from the clean layer-0 values (shared by both sides)
    w = {k: v.cuda() for k, v in wl.weights[1].items()}
    p1 = kvc.make_predictor(kvc.PRED_XLAYER_DPLR, w, rank=rank, residual_codebook=cbt.cuda())
    buf, Kr, Vr = _xlayer_gpu(desc, p1, wl.K[1].cuda(), wl.V[1].cuda(), K0, V0)
    w64 = {k: U.to64(v) for k, v in wl.weights[1].items()}
    Ks, Vs = U.to64(wl.K[0]), U.to64(wl.V[0])
    ck, cv, Kh, Vh, pk, pv = O.encode_layer_xlayer(od, w64, U.to64(wl.K[1]), U.to64(wl.V[1]), Ks, Vs, codebook=cb,
                                                   with_pred=True)
    errk, errv = U.err_xlayer(od, w64, Ks, Vs, Kh)
    idx, s = _eden_from_gpu(buf.k_codes, buf.k_params, T, H, D, p)
    kflip = _check_eden(idx, s, U.to64(Kr), ck, Kh, pk, U.to64(wl.K[1]), cb, state, p, "layer 1 K", perr=errk)
    idx, s = _eden_from_gpu(buf.v_codes, buf.v_params, T, H, D, p)
    _check_eden(idx, s, U.to64(Vr), cv, Vh, pv, U.to64(wl.V[1]), cb, state, p, "layer 1 V", skip=kflip, perr=errv)


# ---------------------------------------------------------------- video-adapted refit


@pytest.mark.parametrize("dtype,T,H,D,rank", [(torch.bfloat16, 1560, 12, 128, 64), (torch.float32, 300, 2, 64, 8),
                                              (torch.bfloat16, 701, 4, 128, 0)])
def test_refit_block_diag(dtype, T, H, D, rank):
    """kvc_refit_block_diag (K and V blocks) against the oracle's ridge
    least-squares fit, and the refitted block predicts the block's own tokens
    at least as well as the offline one."""
    wl = synth.wan_xlayer(seed=synth.SEED_BASE + 114, L=2, T=T, H=H, D=D, rank=rank, calib_tokens=512, dtype=dtype)
    w = {k: v.cuda() for k, v in wl.weights[1].items()}
    param = torch.float16 if dtype == torch.bfloat16 else torch.float32
    desc = _desc(T, H, D, dtype, 2, 32, param)
    pred = kvc.make_predictor(kvc.PRED_XLAYER_DPLR, w, rank=rank)
    ridge = 1e-2 * T
    w64 = {k: U.to64(v) for k, v in wl.weights[1].items()}
    state = U.np_state(dtype)
    for tensor, X0, X1, Y, wk, uk, off in ((0, wl.K[0], None, wl.K[1], "k_w", "k_u", "k_block"),
                                           (1, wl.K[1], wl.V[0], wl.V[1], "v_w", "v_u", "v_block")):
        din = D if tensor == 0 else 2 * D
        out = torch.full((H, D, din), float("nan"), dtype=dtype, device="cuda")
        ws = kvc.alloc_workspace(kvc.OP_REFIT_V if tensor else kvc.OP_REFIT_K, desc, pred)
        kvc.kvc_refit_block_diag(desc, pred, tensor, X0.cuda(), None if X1 is None else X1.cuda(), Y.cuda(), ridge,
                                 out, ws)
        _sync_ok()
        ref = O.refit_block_diag(U.to64(X0), None if X1 is None else U.to64(X1), U.to64(Y),
                                 w64[wk] if rank else None, w64[uk] if rank else None, ridge)
        got = U.to64(out)
        rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        U.OBSERVED.append({"check": f"refit tensor {tensor} T={T}", "rel_fro": float(rel)})
        # fp32 Gram sums and Cholesky against fp64, then one rounding to the layer dtype
        assert rel <= 2e-3 if state == "bf16" else rel <= 1e-4, rel
        assert np.all(np.abs(got - ref) <= 1e-3 * np.abs(ref).max() + np.abs(O.round_to(ref, state) - ref) * 2.01)
        # the refitted block fits the block's own tokens better than the offline one
        Xh = U.to64(X0) if X1 is None else np.concatenate([U.to64(X0), U.to64(X1)], -1)
        flat = Xh.reshape(T, H, 2, D).transpose(0, 2, 1, 3).reshape(T, -1) if X1 is not None else Xh.reshape(T, -1)
        lr = ((flat @ w64[wk].T) @ w64[uk].T).reshape(T, H, D) if rank else 0.0
        res = lambda B: np.linalg.norm(U.to64(Y) - lr - np.einsum("thi,hoi->tho", Xh, B))
        assert res(got) <= res(w64[off]) * 1.0001


# ---------------------------------------------------------------- grouped-query attention


@pytest.mark.parametrize("n_q,n_self,T,H,group_q,jensen", [(300, 130, 3 * 128 + 5, 4, 2, False),
                                                           (129, 0, 256, 2, 4, False), (200, 64, 300, 4, 3, True)])
def test_grouped_query_attention_cross_layer(n_q, n_self, T, H, group_q, jensen):
    """q_heads = group_q x n_heads on the tensor-core path: query head j reads
    KV head j // group_q; history codes by the oracle."""
    D = 128
    Hq = H * group_q
    wl = synth.wan_xlayer(seed=synth.SEED_BASE + 115, L=2, T=T, H=H, rank=64, calib_tokens=512)
    bf, hf = torch.bfloat16, torch.float16
    od = _odesc(T, H, D, bf, 2, 32, hf)
    w64 = {k: U.to64(v) for k, v in wl.weights[1].items()}
    Ks, Vs = U.to64(wl.K[0]), U.to64(wl.V[0])
    ck, cv, _, _ = O.encode_layer_xlayer(od, w64, U.to64(wl.K[1]), U.to64(wl.V[1]), Ks, Vs)
    buf = _oracle_codes_to_gpu(ck, cv, 2, "f16")
    Q = synth.queries(51, n_q, Hq, D)
    Kself, Vself = synth.queries(52, n_self, H, D), synth.queries(53, n_self, H, D)
    desc = kvc.make_desc(T, H, D, bf, 2, 32, hf, q_heads=Hq)
    pred = kvc.make_predictor(kvc.PRED_XLAYER_DPLR, {k: v.cuda() for k, v in wl.weights[1].items()}, rank=64)
    Og = torch.empty(n_q, Hq, D, dtype=bf, device="cuda")
    ws = kvc.alloc_workspace(kvc.OP_ATTEND, desc, pred, n_q)
    fn = kvc.kvc_attend_compressed_debiased if jensen else kvc.kvc_attend_compressed
    fn(desc, pred, Q.cuda(), buf, wl.K[0].cuda(), wl.V[0].cuda(), Kself.cuda() if n_self else None,
       Vself.cuda() if n_self else None, D ** -0.5, Og, ws)
    _sync_ok()
    ref = O.attend_compressed_xlayer(od, w64, U.to64(Q), ck, cv, Ks, Vs, U.to64(Kself) if n_self else None,
                                     U.to64(Vself) if n_self else None, D ** -0.5, jensen=jensen)
    err = U.rel_l2(U.to64(Og), ref)
    U.OBSERVED.append({"check": f"GQA attention Hq={Hq} H={H}", "rel_l2": err})
    assert err <= U.ATT_TOL[bf], err


def test_grouped_query_attention_cuda_core_path():
    """The fp32 tiny history (CUDA-core attention) with 4 query heads per KV head."""
    wl = synth.tiny_xlayer()
    T, H, D = wl.K[0].shape
    f32 = torch.float32
    od = _odesc(T, H, D, f32, 4, 32, f32)
    ck0, cv0, K0h, V0h = O.encode_layer_none(od, U.to64(wl.K[0]), U.to64(wl.V[0]))
    w64 = {k: U.to64(v) for k, v in wl.weights[1].items()}
    ck1, cv1, _, _ = O.encode_layer_xlayer(od, w64, U.to64(wl.K[1]), U.to64(wl.V[1]), K0h, V0h)
    Q = synth.queries(9, 40, 4 * H, D, dtype=f32)
    desc = kvc.make_desc(T, H, D, f32, 4, 32, f32, q_heads=4 * H)
    pred = kvc.make_predictor(kvc.PRED_XLAYER_DPLR, {k: v.cuda() for k, v in wl.weights[1].items()}, rank=wl.rank)
    buf = _oracle_codes_to_gpu(ck1, cv1, 4, "f32")
    Og = torch.empty(40, 4 * H, D, device="cuda")
    kvc.kvc_attend_compressed(desc, pred, Q.cuda(), buf, torch.from_numpy(K0h).float().cuda(),
                              torch.from_numpy(V0h).float().cuda(), None, None, 0.125, Og,
                              kvc.alloc_workspace(kvc.OP_ATTEND, desc, pred, 40))
    _sync_ok()
    ref = O.attend_compressed_xlayer(od, w64, U.to64(Q), ck1, cv1, K0h, V0h, None, None, 0.125)
    assert U.rel_l2(U.to64(Og), ref) <= U.ATT_TOL[f32]


# ---------------------------------------------------------------- the chain of layers in one call


@pytest.mark.parametrize("case", ["fp32", "rank16", "mixed_ranks", "eden2"])
def test_layer_chain_other_shapes_match_layer_calls(case):
    """Shapes the fused walk does not take (fp32 values, a rank off the
    tensor-core list, layers of different ranks, H64 / EDEN-2 residuals) run the
    layers in turn inside kvc_encode_layers / kvc_decode_layers: every code,
    parameter and reconstruction must equal the one-layer calls'."""
    L, T, H, D = 4, 2 * 128 + 19, 3, 128
    dtype = torch.float32 if case == "fp32" else torch.bfloat16
    r0 = 16 if case in ("fp32", "rank16") else 64
    wl = synth.wan_xlayer(seed=synth.SEED_BASE + 122, device="cuda", L=L, T=T, H=H, rank=r0, calib_tokens=512,
                          dtype=dtype)
    if case == "mixed_ranks":
        wl128 = synth.wan_xlayer(seed=synth.SEED_BASE + 122, device="cuda", L=L, T=T, H=H, rank=128,
                                 calib_tokens=512, layers_needed=[2])
        preds = [kvc.make_predictor(kvc.PRED_XLAYER_DPLR, wl.weights[1], rank=64),
                 kvc.make_predictor(kvc.PRED_XLAYER_DPLR, wl128.weights[2], rank=128),
                 kvc.make_predictor(kvc.PRED_XLAYER_DPLR, wl.weights[3], rank=64)]
    elif case == "eden2":
        cb = synth.eden2_codebook().cuda()
        preds = [kvc.make_predictor(kvc.PRED_XLAYER_DPLR, wl.weights[l], rank=r0, residual_codebook=cb)
                 for l in range(1, L)]
    else:
        preds = [kvc.make_predictor(kvc.PRED_XLAYER_DPLR, wl.weights[l], rank=r0) for l in range(1, L)]
    if case == "eden2":
        desc = kvc.make_desc(T, H, D, dtype, 2, 64, torch.float16, residual_codec=kvc.RESIDUAL_H64_EDEN2)
    else:
        desc = _desc(T, H, D, dtype, 2, 32, torch.float32 if case == "fp32" else torch.float16)
    n = L - 1
    ref_codes, ref_K, ref_V = [], [], []
    Ks, Vs = wl.K[0], wl.V[0]
    for i in range(n):
        buf = kvc.alloc_codes(desc, preds[i])
        Kr, Vr = torch.empty_like(Ks), torch.empty_like(Vs)
        kvc.kvc_encode_layer(desc, preds[i], wl.K[i + 1], wl.V[i + 1], Ks, Vs, buf, Kr, Vr,
                             kvc.alloc_workspace(kvc.OP_ENCODE, desc, preds[i]))
        ref_codes.append(buf), ref_K.append(Kr), ref_V.append(Vr)
        Ks, Vs = Kr, Vr
    _sync_ok()
    codes = [kvc.alloc_codes(desc, p) for p in preds]
    Kr = [torch.zeros_like(wl.K[0]) for _ in range(n)]
    Vr = [torch.zeros_like(wl.V[0]) for _ in range(n)]
    kvc.kvc_encode_layers(desc, preds, wl.K[1:], wl.V[1:], wl.K[0], wl.V[0], codes, Kr, Vr,
                          kvc.alloc_layers_workspace(kvc.OP_ENCODE, desc, preds))
    _sync_ok()
    for i in range(n):
        for name in ("k_codes", "k_params", "v_codes", "v_params"):
            assert torch.equal(getattr(codes[i], name), getattr(ref_codes[i], name)), (case, i, name)
        assert torch.equal(Kr[i], ref_K[i]) and torch.equal(Vr[i], ref_V[i]), (case, i)
    Kd = [torch.zeros_like(wl.K[0]) for _ in range(n)]
    Vd = [torch.zeros_like(wl.V[0]) for _ in range(n)]
    kvc.kvc_decode_layers(desc, preds, codes, wl.K[0], wl.V[0], Kd, Vd,
                          kvc.alloc_layers_workspace(kvc.OP_DECODE, desc, preds))
    _sync_ok()
    for i in range(n):
        assert torch.equal(Kd[i], ref_K[i]) and torch.equal(Vd[i], ref_V[i]), (case, i)  # decode replays encode


@pytest.mark.parametrize("L,T,H,rank,bits,group,pingpong", [(5, 3 * 128 + 41, 4, 64, 2, 32, False),
                                                            (5, 2 * 256 + 7, 3, 128, 4, 64, True),
                                                            (5, 300, 2, 0, 2, 64, True), (5, 128, 2, 64, 2, 32, False),
                                                            (61, 300, 2, 64, 2, 32, True),
                                                            (3, 40 * 128 + 3, 2, 64, 2, 32, True),
                                                            (2, 1, 2, 64, 2, 32, False),
                                                            (3, 129, 3, 64, 4, 64, True),
                                                            (3, 256, 2, 128, 2, 32, False)])
def test_layer_chain_in_one_call_matches_layer_calls(L, T, H, rank, bits, group, pingpong):
    """kvc_encode_layers / kvc_decode_layers (one persistent launch walking
    (layer, tile) items, each tile waiting on the same tile of the layer before)
    against kvc_encode_layer / kvc_decode_layer called layer by layer: the same
    arithmetic, so every code, parameter and reconstruction is identical.  With
    `pingpong` the chain reuses two reconstruction buffers in turn.  60 layers of
    3 tiles give more items than SMs with fewer tiles than CTAs (the latent
    overlap across items is off there); 40 tiles give CTAs several items each.
    Edges: one layer of one token (the second CTA of the pair has no rows), 129
    tokens (it has one), and exactly one 256-token pair tile."""
    D = 128
    wl = synth.wan_xlayer(seed=synth.SEED_BASE + 121, device="cuda", L=L, T=T, H=H, rank=rank, calib_tokens=512)
    bf, hf = torch.bfloat16, torch.float16
    desc = _desc(T, H, D, bf, bits, group, hf)
    preds = [kvc.make_predictor(kvc.PRED_XLAYER_DPLR, wl.weights[l], rank=rank) for l in range(1, L)]
    n = L - 1
    # the reference: layer calls in turn from layer 0's clean values
    ws = kvc.alloc_workspace(kvc.OP_ENCODE, desc, preds[0])
    wsd = kvc.alloc_workspace(kvc.OP_DECODE, desc, preds[0])
    ref_codes, ref_K, ref_V, ref_Kd, ref_Vd = [], [], [], [], []
    Ks, Vs = wl.K[0], wl.V[0]
    for i in range(n):
        buf = kvc.alloc_codes(desc, preds[i])
        Kr, Vr = torch.empty_like(Ks), torch.empty_like(Vs)
        kvc.kvc_encode_layer(desc, preds[i], wl.K[i + 1], wl.V[i + 1], Ks, Vs, buf, Kr, Vr, ws)
        ref_codes.append(buf), ref_K.append(Kr), ref_V.append(Vr)
        Ks, Vs = Kr, Vr
    Ks, Vs = wl.K[0], wl.V[0]
    for i in range(n):
        Kd, Vd = torch.empty_like(Ks), torch.empty_like(Vs)
        kvc.kvc_decode_layer(desc, preds[i], ref_codes[i], Ks, Vs, Kd, Vd, wsd)
        ref_Kd.append(Kd), ref_Vd.append(Vd)
        Ks, Vs = Kd, Vd
    # the chain in one call
    codes = [kvc.alloc_codes(desc, p) for p in preds]
    mk = lambda: torch.zeros_like(wl.K[0])
    if pingpong:
        bufs = [(mk(), mk()), (mk(), mk())]
        Kr = [bufs[i % 2][0] for i in range(n)]
        Vr = [bufs[i % 2][1] for i in range(n)]
    else:
        Kr = [mk() for _ in range(n)]
        Vr = [mk() for _ in range(n)]
    wse = kvc.alloc_layers_workspace(kvc.OP_ENCODE, desc, preds)
    kvc.kvc_encode_layers(desc, preds, wl.K[1:], wl.V[1:], wl.K[0], wl.V[0], codes, Kr, Vr, wse)
    _sync_ok()
    for i in range(n):
        for name in ("k_codes", "k_params", "v_codes", "v_params"):
            assert torch.equal(getattr(codes[i], name), getattr(ref_codes[i], name)), (i, name)
    for i in range(n - 2 if pingpong else 0, n):  # (the ping-pong buffers hold the last two layers)
        assert torch.equal(Kr[i], ref_K[i]) and torch.equal(Vr[i], ref_V[i]), i
    Kd = [mk() for _ in range(n)]
    Vd = [mk() for _ in range(n)]
    wsdl = kvc.alloc_layers_workspace(kvc.OP_DECODE, desc, preds)
    kvc.kvc_decode_layers(desc, preds, codes, wl.K[0], wl.V[0], Kd, Vd, wsdl)
    _sync_ok()
    for i in range(n):
        assert torch.equal(Kd[i], ref_Kd[i]) and torch.equal(Vd[i], ref_Vd[i]), i
        assert torch.equal(Kd[i], ref_K[i]) and torch.equal(Vd[i], ref_V[i]), i  # decode replays encode
