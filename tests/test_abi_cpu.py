"""Host-side checks of the C ABI: the library loads on a machine without a GPU,
exports every entry point include/*.h declares, reports the closed-form
storage the oracle computes, and rejects bad arguments before any launch."""

import ctypes
import os
import re

import pytest
import torch

from clustered_kv_cache_b200 import build as kbuild
from clustered_kv_cache_b200 import kvc
from oracle import kvc_oracle as O

INCLUDE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
HEADERS = sorted(os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h"))


@pytest.fixture(scope="module")
def L():
    kbuild.build()
    return kvc.lib()


def test_exports_every_declared_entry_point(L):
    declared = []
    for h in HEADERS:
        with open(h) as f:
            declared += re.findall(r"KVC_API\s+[\w\s\*]+?\b(kvc_\w+)\s*\(", f.read())
    assert len(declared) >= 13 and "kvc_testing_inject_stall" in declared
    assert sorted(declared) == sorted(set(declared))
    for name in declared:
        assert hasattr(L, name), name
    assert set(declared) <= set(kvc.EXPORTED) | set(declared)


@pytest.mark.parametrize("kind,bits,group,param,T,H,D,F,ab", [
    ("none", 2, 32, "f16", 32760, 12, 128, 0, 4),
    ("none", 4, 32, "f32", 512, 2, 64, 0, 4),
    ("temporal", 4, 64, "f16", 65536, 40, 128, 1560, 4),
    ("temporal", 2, 32, "f16", 1000, 2, 64, 64, 8),
    ("cluster", 4, 32, "f16", 32768, 16, 128, 0, 4),
])
def test_codes_bytes_match_oracle_accounting(L, kind, bits, group, param, T, H, D, F, ab):
    kinds = {"none": kvc.PRED_NONE, "temporal": kvc.PRED_TEMPORAL, "cluster": kvc.PRED_CLUSTER}
    dt = torch.float16 if param == "f16" else torch.float32
    desc = kvc.make_desc(T, H, D, torch.bfloat16, bits, group, dt, F, ab)
    pred = kvc.make_predictor(kinds[kind], n_clusters=256 if kind == "cluster" else 0,
                              code_dim=128 if kind == "cluster" else 0)
    od = O.Desc(T, H, D, bits=bits, group=group, param=param, frame_tokens=F, anchor_bits=ab)
    assert kvc.kvc_codes_bytes(desc, pred) == O.codes_bytes(od, kind, code_dim=128)


def _call_encode(L, desc, pred, K=0x1000, V=0x1000, Ks=0x1000, Vs=0x1000, codes=None, Kr=0x1000, Vr=0x1000,
                 ws=None, wsn=0):
    c = codes or kvc.Codes(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000)
    return L.kvc_encode_layer(ctypes.byref(desc), ctypes.byref(pred), K, V, Ks, Vs, ctypes.byref(c), Kr, Vr, ws, wsn,
                              None)


def test_validation_errors_without_launch(L):
    good = kvc.make_desc(100, 2, 128, torch.bfloat16, 2, 32)
    none = kvc.make_predictor(kvc.PRED_NONE)
    assert _call_encode(L, good, none, K=None) == 1  # NULL input
    assert _call_encode(L, good, none, K=0x1008) == 3  # misaligned
    for bad in (kvc.make_desc(100, 2, 96, torch.bfloat16, 2, 32),    # head_dim
                kvc.make_desc(100, 2, 128, torch.bfloat16, 3, 32),   # bits
                kvc.make_desc(100, 2, 128, torch.bfloat16, 2, 48),   # group does not divide D
                kvc.make_desc(100, 2, 128, torch.bfloat16, 2, 2)):   # group narrower than a lane's share
        assert _call_encode(L, bad, none) == 2
    assert _call_encode(L, kvc.make_desc(-1, 2, 128), none) == 1
    xl = kvc.make_predictor(kvc.PRED_XLAYER_DPLR, rank=8)
    assert _call_encode(L, good, xl) == 1  # missing weights
    xl = kvc.Predictor(kvc.PRED_XLAYER_DPLR, 8, 0, 0, *([0x1000] * 12))
    need = kvc.kvc_workspace_bytes(kvc.OP_ENCODE, good, xl)
    assert need >= 2 * 100 * 8 * 4
    assert _call_encode(L, good, xl, ws=0x1000, wsn=need - 1) == 4
    assert _call_encode(L, good, xl, Kr=None) == 1  # V's prediction needs K_rec
    tmp = kvc.make_predictor(kvc.PRED_TEMPORAL)
    assert _call_encode(L, kvc.make_desc(100, 2, 128, frame_tokens=0), tmp) == 2 or \
        _call_encode(L, kvc.make_desc(100, 2, 128, frame_tokens=0), tmp) == 1
    c = kvc.Codes(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000)
    q = ctypes.c_void_p(0x1000)
    # attention over a temporal history is not offered; clustered attention takes no self tokens
    tp = kvc.Predictor(kvc.PRED_TEMPORAL, 0, 0, 0, *([0x1000] * 12))
    st = L.kvc_attend_compressed(ctypes.byref(kvc.make_desc(100, 2, 128, frame_tokens=10)), ctypes.byref(tp), q, 4,
                                 ctypes.byref(c), None, None, None, None, 0, 1.0, q, None, None, None, 0, None)
    assert st == 2
    cp = kvc.Predictor(kvc.PRED_CLUSTER, 0, 16, 128, *([0x1000] * 12))
    st = L.kvc_attend_compressed(ctypes.byref(good), ctypes.byref(cp), q, 4, ctypes.byref(c), None, None, q, q, 8,
                                 1.0, q, None, None, None, 0, None)
    assert st == 2
    # a misaligned optional history output is refused before anything runs
    xp = kvc.Predictor(kvc.PRED_XLAYER_DPLR, 0, 0, 0, *([0x1000] * 12))
    st = L.kvc_attend_compressed(ctypes.byref(good), ctypes.byref(xp), q, 4, ctypes.byref(c), q, q, None, None, 0,
                                 1.0, q, ctypes.c_void_p(0x1008), None, None, 0, None)
    assert st == 3
    assert L.kvc_pack_codes(q, 100, 2, q, None) == 1  # not whole 16-byte words
    assert L.kvc_pack_codes(q, 64, 3, q, None) == 2


def test_status_strings(L):
    for s in range(7):
        assert kvc.kvc_status_string(s)
    assert kvc.kvc_status_string(99) == "unknown status"


def test_multi_layer_validation_without_launch(L):
    """kvc_encode_layers / kvc_decode_layers refuse bad chains before anything runs."""
    d = kvc.make_desc(100, 2, 128, torch.bfloat16, 2, 32)
    xp = kvc.Predictor(kvc.PRED_XLAYER_DPLR, 0, 0, 0, *([0x1000] * 12))
    preds = (kvc.Predictor * 2)(xp, xp)
    c = kvc.Codes(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000)
    codes = (kvc.Codes * 2)(c, c)
    P = lambda *a: (ctypes.c_void_p * len(a))(*a)
    x = P(0x1000, 0x2000)
    need = L.kvc_layers_workspace_bytes(kvc.OP_ENCODE, ctypes.byref(d), preds, 2)
    assert L.kvc_layers_workspace_bytes(kvc.OP_ATTEND, ctypes.byref(d), preds, 2) == 0
    assert L.kvc_layers_workspace_bytes(kvc.OP_ENCODE, ctypes.byref(d), preds, 0) == 0

    def enc(n=2, Kr=None, Vr=None, Ks=0x1000, ws=0x100000, wsn=None):
        Kr = Kr or P(0x3000, 0x5000)
        Vr = Vr or P(0x4000, 0x6000)
        return L.kvc_encode_layers(ctypes.byref(d), preds, n, x, x, Ks, 0x1000, codes, Kr, Vr, ws,
                                   need if wsn is None else wsn, None)

    assert enc(n=0) == 1
    assert enc(Ks=None) == 1                                   # layer 0's sources
    assert enc(Kr=P(0x3000, 0x3000)) == 1                      # layer 1 would overwrite its own source
    assert enc(Kr=P(0x1000, 0x5000)) == 1                      # layer 0 would overwrite the chain's source
    assert enc(Kr=P(0x3000, 0x5008)) == 3                      # misaligned
    if need:
        assert enc(wsn=need - 1) == 4
    tp = kvc.Predictor(kvc.PRED_TEMPORAL, 0, 0, 0, *([0x1000] * 12))
    assert L.kvc_decode_layers(ctypes.byref(kvc.make_desc(100, 2, 128, frame_tokens=10)), (kvc.Predictor * 1)(tp),
                               1, (kvc.Codes * 1)(c), 0x1000, 0x1000, P(0x3000), P(0x4000), None, 0, None) == 2


def test_multi_layer_binding_rejects_mismatched_lists():
    """The binding checks the per-layer lists before any call reaches the library."""
    d = kvc.make_desc(100, 2, 128, torch.bfloat16, 2, 32)
    p = kvc.Predictor(kvc.PRED_XLAYER_DPLR, 0, 0, 0)
    with pytest.raises(ValueError, match="K_rec has 1 entries for 2 layers"):
        kvc.kvc_encode_layers(d, [p, p], [None, None], [None, None], None, None, [None, None], [None], [None, None])
    with pytest.raises(ValueError, match="codes has 3 entries for 2 layers"):
        kvc.kvc_decode_layers(d, [p, p], [None, None, None], None, None, [None, None], [None, None])


def test_copy_helpers_reject_short_destinations():
    """A destination smaller than the copy is refused before any library call."""
    small, big = torch.empty(4, dtype=torch.uint8), torch.empty(8, dtype=torch.uint8)
    with pytest.raises(ValueError, match="destination holds 4 bytes, the copy 8"):
        kvc.kvc_copy_to_device(small, big)
    with pytest.raises(ValueError, match="destination holds 4 bytes, the copy 8"):
        kvc.kvc_copy_to_host(small, big)
