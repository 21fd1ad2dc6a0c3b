"""Failure detection without a GPU fault: a bounded device wait that runs out.

The test hook kvc_testing_inject_stall makes the next cross-layer codec launch
leave one TMA pipeline stage unarmed, so the MMA side's wait on it can never
succeed.  The wait gives up after its bounded time (about two seconds), the
kernel records KVC_ERR_DEVICE_TIMEOUT in the device error word, every role
returns and the loads already issued are drained.  The host reads the status,
and the context stays usable: the next launch codes the layer correctly.  The
multi-layer calls cover the (layer, tile) walk: the CTAs whose items wait on a
tile the stalled CTA never stores give up on that wait the same way.
"""

import time

import pytest
import torch

from clustered_kv_cache_b200 import kvc, synth

pytestmark = pytest.mark.gpu

KVC_ERR_DEVICE_TIMEOUT = 6


@pytest.mark.parametrize("op", ["encode", "decode", "encode_layers", "decode_layers"])
def test_bounded_wait_runs_out_and_reports_a_timeout(op):
    """Encode runs single CTAs, decode CTA pairs (whose loads complete on the
    pair leader's barriers): both give up, report and leave the context usable,
    in one-layer and in multi-layer calls."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from clustered_kv_cache_b200 import build

    build.build()
    T, H, D, r = 3 * 128 + 11, 12, 128, 64
    wl = synth.wan_xlayer(seed=synth.SEED_BASE + 111, L=3, T=T, rank=r, calib_tokens=1024)
    bf, hf = torch.bfloat16, torch.float16
    desc = kvc.make_desc(T, H, D, bf, 2, 32, hf)
    pred = kvc.make_predictor(kvc.PRED_XLAYER_DPLR, {k: v.cuda() for k, v in wl.weights[1].items()}, rank=r)
    if op.endswith("_layers"):
        _multi_layer_case(op, wl, desc, r)
        return
    K, V, Ks, Vs = (t.cuda() for t in (wl.K[1], wl.V[1], wl.K[0], wl.V[0]))
    ws = kvc.alloc_workspace(kvc.OP_ENCODE, desc, pred)
    ref = kvc.alloc_codes(desc, pred)
    Kr0, Vr0 = torch.empty_like(K), torch.empty_like(V)
    # a clean launch first: the reference result, and no error pending
    kvc.kvc_encode_layer(desc, pred, K, V, Ks, Vs, ref, Kr0, Vr0, ws)
    assert kvc.kvc_get_device_error() == 0

    def run():
        if op == "encode":
            buf = kvc.alloc_codes(desc, pred)
            Kr, Vr = torch.empty_like(K), torch.empty_like(V)
            kvc.kvc_encode_layer(desc, pred, K, V, Ks, Vs, buf, Kr, Vr, ws)
            return buf, Kr, Vr
        Kr, Vr = torch.empty_like(K), torch.empty_like(V)
        kvc.kvc_decode_layer(desc, pred, ref, Ks, Vs, Kr, Vr, kvc.alloc_workspace(kvc.OP_DECODE, desc, pred))
        return ref, Kr, Vr

    # the faulted launch: the launch itself succeeds, the bounded wait runs out on the device
    kvc.kvc_testing_inject_stall(1)
    t0 = time.perf_counter()
    run()
    status = kvc.kvc_get_device_error()  # synchronizes the stream
    elapsed = time.perf_counter() - t0
    assert status == KVC_ERR_DEVICE_TIMEOUT, status
    assert elapsed < 60.0, elapsed
    # read-and-clear: nothing pending now, and the hook was one-shot
    assert kvc.kvc_get_device_error() == 0
    buf, Kr, Vr = run()
    assert kvc.kvc_get_device_error() == 0
    assert torch.equal(Kr, Kr0) and torch.equal(Vr, Vr0)
    assert torch.equal(buf.k_codes, ref.k_codes) and torch.equal(buf.v_codes, ref.v_codes)


def _multi_layer_case(op, wl, desc, r):
    preds = [kvc.make_predictor(kvc.PRED_XLAYER_DPLR, {k: v.cuda() for k, v in wl.weights[l].items()}, rank=r)
             for l in (1, 2)]
    K = [wl.K[l].cuda() for l in (1, 2)]
    V = [wl.V[l].cuda() for l in (1, 2)]
    Ks, Vs = wl.K[0].cuda(), wl.V[0].cuda()
    ref = [kvc.alloc_codes(desc, p) for p in preds]
    Kr0 = [torch.empty_like(Ks) for _ in preds]
    Vr0 = [torch.empty_like(Vs) for _ in preds]
    enc_ws = kvc.alloc_layers_workspace(kvc.OP_ENCODE, desc, preds)
    kvc.kvc_encode_layers(desc, preds, K, V, Ks, Vs, ref, Kr0, Vr0, enc_ws)
    assert kvc.kvc_get_device_error() == 0
    dec_ws = kvc.alloc_layers_workspace(kvc.OP_DECODE, desc, preds)

    def run():
        Kr = [torch.empty_like(Ks) for _ in preds]
        Vr = [torch.empty_like(Vs) for _ in preds]
        if op == "encode_layers":
            codes = [kvc.alloc_codes(desc, p) for p in preds]
            kvc.kvc_encode_layers(desc, preds, K, V, Ks, Vs, codes, Kr, Vr, enc_ws)
            return codes, Kr, Vr
        kvc.kvc_decode_layers(desc, preds, ref, Ks, Vs, Kr, Vr, dec_ws)
        return ref, Kr, Vr

    kvc.kvc_testing_inject_stall(1)
    t0 = time.perf_counter()
    run()
    status = kvc.kvc_get_device_error()
    elapsed = time.perf_counter() - t0
    assert status == KVC_ERR_DEVICE_TIMEOUT, status
    assert elapsed < 60.0, elapsed
    assert kvc.kvc_get_device_error() == 0
    codes, Kr, Vr = run()
    assert kvc.kvc_get_device_error() == 0
    for i in range(len(preds)):
        assert torch.equal(Kr[i], Kr0[i]) and torch.equal(Vr[i], Vr0[i])
        assert torch.equal(codes[i].k_codes, ref[i].k_codes) and torch.equal(codes[i].v_codes, ref[i].v_codes)
