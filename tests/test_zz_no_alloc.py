"""The clustered-codec encode that allocates nothing.

Some callers cannot allocate device memory when they encode (allocator or pool
callbacks, runtimes that hand out pre-carved memory, plugin hosts that forbid
cudaMalloc).  kvc_encode_layer_cluster_static serves them from a static device
array inside the library.  Its results must match kvc_encode_layer's within the
tolerances of the other parity tests, on consecutive calls (the array is shared
and keeps the previous call's contents); the reconstructions may differ by one
bf16 step where the two kernels' fp32 sums round across a boundary.  This file
is collected last.
"""

import ctypes

import numpy as np
import pytest
import torch

from clustered_kv_cache_b200 import build, kvc, synth

import kvc_testutil as U


def test_static_entry_rejects_more_centres_than_its_array_holds():
    build.build()
    L = kvc.lib()
    fn = L.kvc_encode_layer_cluster_static
    fn.restype = ctypes.c_int
    desc = kvc.make_desc(100, 2, 128, torch.bfloat16, 4, 32, torch.float16)
    c = kvc.Codes(*([0x1000] * 6))
    for n_c, m in ((257, 128), (16, 64)):
        pred = kvc.Predictor(kvc.PRED_CLUSTER, 0, n_c, m, *([0x1000] * 12))
        assert fn(ctypes.byref(desc), ctypes.byref(pred), ctypes.c_void_p(0x1000), ctypes.c_void_p(0x1000),
                  ctypes.byref(c), None, None, None) == 2
    # a head_dim the library does not implement: the same status as kvc_encode_layer
    odd = kvc.make_desc(100, 2, 96, torch.bfloat16, 4, 32, torch.float16)
    pred = kvc.Predictor(kvc.PRED_CLUSTER, 0, 16, 128, *([0x1000] * 12))
    args = (ctypes.byref(odd), ctypes.byref(pred), ctypes.c_void_p(0x1000), ctypes.c_void_p(0x1000), ctypes.byref(c))
    assert fn(*args, None, None, None) == 2
    assert L.kvc_encode_layer(args[0], args[1], args[2], args[3], None, None, args[4], None, None, None,
                              ctypes.c_size_t(0), None) == 2


@pytest.mark.gpu
def test_static_scratch_encode_matches_workspace_encode_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    T, H, D, n_c = 1000, 4, 128, 64
    cw = synth.cluster_layer(seed=synth.SEED_BASE + 106, T=T, H=H, n_c=n_c, iters=5)
    w = dict(k_centroids=cw.k_centroids.cuda(), k_enc=cw.k_enc.cuda(), k_dec=cw.k_dec.cuda(),
             v_centroids=cw.v_centroids.cuda(), v_enc=cw.v_enc.cuda(), v_dec=cw.v_dec.cuda())
    pred = kvc.make_predictor(kvc.PRED_CLUSTER, w, n_clusters=n_c, code_dim=128)
    desc = kvc.make_desc(T, H, D, torch.bfloat16, 4, 32, torch.float16)
    K, V = cw.K.cuda(), cw.V.cuda()
    ref = kvc.alloc_codes(desc, pred)
    Kr, Vr = torch.empty_like(K), torch.empty_like(V)
    kvc.kvc_encode_layer(desc, pred, K, V, None, None, ref, Kr, Vr, kvc.alloc_workspace(kvc.OP_ENCODE, desc, pred))
    torch.cuda.synchronize()
    for call in range(2):
        out = kvc.alloc_codes(desc, pred)
        Ks, Vs = torch.empty_like(K), torch.empty_like(V)
        kvc.kvc_encode_layer_cluster_static(desc, pred, K, V, out, Ks, Vs)
        torch.cuda.synchronize()
        assert kvc.kvc_get_device_error() == 0
        for which, rec_s, rec_r, X in (("k", Ks, Kr, K), ("v", Vs, Vr, V)):
            a_s = getattr(out, which + "_assign")[:T].cpu().numpy()
            a_r = getattr(ref, which + "_assign")[:T].cpu().numpy()
            np.testing.assert_array_equal(a_s, a_r)
            q_s = U.codes_from_gpu(getattr(out, which + "_codes"), (T, 128), 4)
            q_r = U.codes_from_gpu(getattr(ref, which + "_codes"), (T, 128), 4)
            U.assert_codes_close(q_s, q_r, f"call {call} {which} codes")
            s_s, z_s = U.params_from_gpu(getattr(out, which + "_params"), (T, 4), "f16")
            s_r, z_r = U.params_from_gpu(getattr(ref, which + "_params"), (T, 4), "f16")
            U.assert_params_close(s_s, z_s, s_r, z_r, "f16", f"call {call} {which} params")
            r_s, r_r = U.to64(rec_s), U.to64(rec_r)
            tol = 1e-3 * (np.abs(U.to64(X)) + 1.0)
            flip = np.repeat((q_s != q_r).any(axis=1), H * D).reshape(T, H, D)
            # The static entry point runs the CUDA-core kernels and kvc_encode_layer the
            # tensor-core ones: the same products summed in another fp32 order, so where
            # the exact value sits next to a bf16 rounding boundary the two round to
            # adjacent bf16 values.  One such step is accepted, rarely.
            mag = np.maximum(np.abs(r_s), np.abs(r_r))
            ulp = np.exp2(np.floor(np.log2(np.maximum(mag, 1e-30))) - 7)
            diff = np.abs(r_s - r_r)
            one_step = (diff > tol) & (diff <= ulp * 1.0001)
            assert np.all((diff <= tol) | one_step | flip), f"call {call} {which} recon"
            assert one_step.mean() < 1e-2, f"call {call} {which} recon: {one_step.mean()} one-step differences"
