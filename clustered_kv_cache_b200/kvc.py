"""ctypes binding of libkvc.so (include/kvc.h).

Argument marshalling only: every function here turns torch tensors into device
pointers and forwards to the C entry point of the same name; all computation
happens in the library's CUDA kernels.  The library is loaded on first use and
a missing or unloadable library raises ``KvcError`` (there is no fallback).

A cross-layer chain, the anchor layer first and then layers 1 .. L-1 in one
launch each way::

    desc0 = make_desc(T, H, D, torch.bfloat16, 4, 32)          # INT4 anchor
    desc = make_desc(T, H, D, torch.bfloat16, 2, 32)           # INT2 residuals
    preds = [make_predictor(PRED_XLAYER_DPLR, w, rank=64) for w in weights]
    kvc_encode_layer(desc0, make_predictor(PRED_NONE), K[0], V[0], None, None, codes0, K0r, V0r)
    ws = alloc_layers_workspace(OP_ENCODE, desc, preds)
    kvc_encode_layers(desc, preds, K[1:], V[1:], K0r, V0r, codes, K_rec, V_rec, ws)
    kvc_decode_layers(desc, preds, codes, K0r, V0r, K_dec, V_dec,
                      alloc_layers_workspace(OP_DECODE, desc, preds))
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkvc.so")

KVC_F32, KVC_BF16, KVC_F16 = 0, 1, 2
PRED_NONE, PRED_XLAYER_DPLR, PRED_TEMPORAL, PRED_CLUSTER = 0, 1, 2, 3
OP_ENCODE, OP_DECODE, OP_ATTEND, OP_REFIT_K, OP_REFIT_V = 0, 1, 2, 3, 4

STATUS = {0: "KVC_OK", 1: "KVC_ERR_INVALID_ARGUMENT", 2: "KVC_ERR_UNSUPPORTED", 3: "KVC_ERR_MISALIGNED",
          4: "KVC_ERR_WORKSPACE_TOO_SMALL", 5: "KVC_ERR_CUDA", 6: "KVC_ERR_DEVICE_TIMEOUT"}

EXPORTED = ["kvc_codes_sizes", "kvc_codes_bytes", "kvc_workspace_bytes", "kvc_encode_layer", "kvc_decode_layer",
            "kvc_attend_compressed", "kvc_pack_codes", "kvc_unpack_codes", "kvc_get_device_error",
            "kvc_status_string", "kvc_last_cuda_error", "kvc_launch_counter", "kvc_testing_inject_stall",
            "kvc_attend_compressed_debiased", "kvc_refit_block_diag", "kvc_copy_to_device", "kvc_copy_to_host",
            "kvc_encode_layers", "kvc_decode_layers", "kvc_layers_workspace_bytes"]


class KvcError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}{(' (' + detail + ')') if detail else ''}")


class LayerDesc(ctypes.Structure):
    _fields_ = [("n_tokens", ctypes.c_int64), ("n_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("bits", ctypes.c_int32), ("group", ctypes.c_int32),
                ("param_dtype", ctypes.c_int32), ("frame_tokens", ctypes.c_int32), ("anchor_bits", ctypes.c_int32),
                ("residual_codec", ctypes.c_int32), ("q_heads", ctypes.c_int32)]


class Predictor(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("rank", ctypes.c_int32), ("n_clusters", ctypes.c_int32),
                ("code_dim", ctypes.c_int32)] + [(n, ctypes.c_void_p) for n in (
                    "k_block", "k_w", "k_u", "v_block", "v_w", "v_u", "k_centroids", "k_enc", "k_dec",
                    "v_centroids", "v_enc", "v_dec", "residual_codebook")]


class Codes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("k_codes", "k_params", "v_codes", "v_params", "k_assign", "v_assign")]


class CodesSize(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_size_t), ("params", ctypes.c_size_t), ("assign", ctypes.c_size_t)]


_LIB = None


def lib():
    """The loaded library; raises KvcError if it is missing or does not load."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise KvcError(-1, "load", f"{LIB_PATH} is missing; run clustered_kv_cache_b200.build")
    try:
        L = ctypes.CDLL(LIB_PATH)
    except OSError as e:  # pragma: no cover - environment dependent
        raise KvcError(-1, "load", str(e)) from e
    P, V, I64, I, SZ, F = (ctypes.POINTER, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t,
                           ctypes.c_float)
    D, PR, CO = P(LayerDesc), P(Predictor), P(Codes)
    sig = {
        "kvc_codes_sizes": (I, [D, PR, P(CodesSize)]),
        "kvc_codes_bytes": (SZ, [D, PR]),
        "kvc_workspace_bytes": (SZ, [I, D, PR, I64]),
        "kvc_encode_layer": (I, [D, PR, V, V, V, V, CO, V, V, V, SZ, V]),
        "kvc_decode_layer": (I, [D, PR, CO, V, V, V, V, V, SZ, V]),
        "kvc_attend_compressed": (I, [D, PR, V, I64, CO, V, V, V, V, I64, F, V, V, V, V, SZ, V]),
        "kvc_attend_compressed_debiased": (I, [D, PR, V, I64, CO, V, V, V, V, I64, F, V, V, V, V, SZ, V]),
        "kvc_refit_block_diag": (I, [D, PR, ctypes.c_int, V, V, V, F, V, V, SZ, V]),
        "kvc_copy_to_device": (I, [V, V, SZ, V]),
        "kvc_encode_layers": (I, [D, PR, I, P(V), P(V), V, V, CO, P(V), P(V), V, SZ, V]),
        "kvc_decode_layers": (I, [D, PR, I, CO, V, V, P(V), P(V), V, SZ, V]),
        "kvc_layers_workspace_bytes": (SZ, [I, D, PR, I]),
        "kvc_copy_to_host": (I, [V, V, SZ, V]),
        "kvc_pack_codes": (I, [V, I64, I, V, V]),
        "kvc_unpack_codes": (I, [V, I64, I, V, V]),
        "kvc_get_device_error": (I, [V]),
        "kvc_status_string": (ctypes.c_char_p, [I]),
        "kvc_last_cuda_error": (ctypes.c_char_p, []),
        "kvc_launch_counter": (ctypes.c_uint64, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = L
    return L


# ---------------------------------------------------------------- marshalling helpers

_DT = {torch.float32: KVC_F32, torch.bfloat16: KVC_BF16, torch.float16: KVC_F16}


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise KvcError(1, "argument", "tensor is not on a CUDA device")
    if not t.is_contiguous():
        raise KvcError(1, "argument", "tensor is not contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(status: int, where: str):
    if status != 0:
        detail = lib().kvc_last_cuda_error().decode() if status == 5 else ""
        raise KvcError(status, where, detail)


RESIDUAL_RTN, RESIDUAL_H64_EDEN2 = 0, 1


def make_desc(n_tokens: int, n_heads: int, head_dim: int, dtype=torch.bfloat16, bits: int = 2, group: int = 32,
              param_dtype=torch.float16, frame_tokens: int = 0, anchor_bits: int = 4,
              residual_codec: int = RESIDUAL_RTN, q_heads: int = 0) -> LayerDesc:
    return LayerDesc(n_tokens, n_heads, head_dim, _DT[dtype], bits, group, _DT[param_dtype], frame_tokens,
                     anchor_bits, residual_codec, q_heads)


def make_predictor(kind: int, weights: dict | None = None, rank: int = 0, n_clusters: int = 0,
                   code_dim: int = 0, residual_codebook: torch.Tensor | None = None) -> Predictor:
    """residual_codebook: the 16 H64 / EDEN-2 points, fp32 [16, 2] on the device."""
    p = Predictor(kind, rank, n_clusters, code_dim)
    weights = dict(weights or {})
    if residual_codebook is not None:
        weights["residual_codebook"] = residual_codebook
    for k, v in weights.items():
        if v is not None:
            setattr(p, k, _ptr(v))
    p._keep = weights  # keep the tensors alive with the struct
    return p


def codes_sizes(desc: LayerDesc, pred: Predictor) -> CodesSize:
    out = CodesSize()
    _check(lib().kvc_codes_sizes(ctypes.byref(desc), ctypes.byref(pred), ctypes.byref(out)), "kvc_codes_sizes")
    return out


def kvc_codes_bytes(desc: LayerDesc, pred: Predictor) -> int:
    return lib().kvc_codes_bytes(ctypes.byref(desc), ctypes.byref(pred))


def kvc_workspace_bytes(op: int, desc: LayerDesc, pred: Predictor, n_q: int = 0) -> int:
    return lib().kvc_workspace_bytes(op, ctypes.byref(desc), ctypes.byref(pred), n_q)


@dataclass
class CodeBuffers:
    """Device tensors holding one layer's compressed K and V."""

    k_codes: torch.Tensor
    k_params: torch.Tensor
    v_codes: torch.Tensor
    v_params: torch.Tensor
    k_assign: torch.Tensor | None = None
    v_assign: torch.Tensor | None = None

    def struct(self) -> Codes:
        return Codes(*(_ptr(t) for t in (self.k_codes, self.k_params, self.v_codes, self.v_params,
                                         self.k_assign, self.v_assign)))


def alloc_codes(desc: LayerDesc, pred: Predictor, device="cuda") -> CodeBuffers:
    s = codes_sizes(desc, pred)

    def buf(n):
        return torch.empty(max(int(n), 16), dtype=torch.uint8, device=device)

    assign = (buf(s.assign), buf(s.assign)) if s.assign else (None, None)
    return CodeBuffers(buf(s.codes), buf(s.params), buf(s.codes), buf(s.params), *assign)


def alloc_workspace(op: int, desc: LayerDesc, pred: Predictor, n_q: int = 0, device="cuda") -> torch.Tensor | None:
    n = kvc_workspace_bytes(op, desc, pred, n_q)
    return torch.empty(n, dtype=torch.uint8, device=device) if n else None


def _ws(ws):
    if ws is None:
        return None, 0
    return _ptr(ws), ws.numel() * ws.element_size()


# ---------------------------------------------------------------- entry points

def kvc_encode_layer(desc, pred, K, V, K_src, V_src, codes: CodeBuffers, K_rec=None, V_rec=None, ws=None,
                     stream=None):
    c = codes.struct()
    wp, wn = _ws(ws)
    _check(lib().kvc_encode_layer(ctypes.byref(desc), ctypes.byref(pred), _ptr(K), _ptr(V), _ptr(K_src),
                                  _ptr(V_src), ctypes.byref(c), _ptr(K_rec), _ptr(V_rec), wp, wn, _stream(stream)),
           "kvc_encode_layer")


def _preds(preds) -> ctypes.Array:
    return (Predictor * len(preds))(*preds)  # the structs' copies; the tensors stay with `preds`


def _codes(codes) -> ctypes.Array:
    return (Codes * len(codes))(*[c.struct() for c in codes])


def _ptrs(ts) -> ctypes.Array:
    return (ctypes.c_void_p * len(ts))(*[_ptr(t) for t in ts])


def kvc_layers_workspace_bytes(op: int, desc: LayerDesc, preds) -> int:
    return lib().kvc_layers_workspace_bytes(op, ctypes.byref(desc), _preds(preds), len(preds))


def alloc_layers_workspace(op: int, desc: LayerDesc, preds, device="cuda") -> torch.Tensor | None:
    n = kvc_layers_workspace_bytes(op, desc, preds)
    return torch.empty(n, dtype=torch.uint8, device=device) if n else None


def _same_length(n: int, **lists) -> None:
    for name, seq in lists.items():
        if len(seq) != n:
            raise ValueError(f"{name} has {len(seq)} entries for {n} layers")


def kvc_encode_layers(desc, preds, K, V, K_src, V_src, codes, K_rec, V_rec, ws=None, stream=None):
    """Layers i = 0 .. len(preds)-1 of a cross-layer chain in one call; layer i
    predicts from K_rec[i-1] / V_rec[i-1] (K_src / V_src for i = 0).  K, V, codes,
    K_rec, V_rec: lists of one entry per layer; ws from alloc_layers_workspace."""
    n = len(preds)
    _same_length(n, K=K, V=V, codes=codes, K_rec=K_rec, V_rec=V_rec)
    wp, wn = _ws(ws)
    _check(lib().kvc_encode_layers(ctypes.byref(desc), _preds(preds), n, _ptrs(K), _ptrs(V), _ptr(K_src),
                                   _ptr(V_src), _codes(codes), _ptrs(K_rec), _ptrs(V_rec), wp, wn, _stream(stream)),
           "kvc_encode_layers")


def kvc_decode_layers(desc, preds, codes, K_src, V_src, K_rec, V_rec, ws=None, stream=None):
    """The decode of kvc_encode_layers: layer i replays its prediction from
    K_rec[i-1] / V_rec[i-1] (K_src / V_src for i = 0) and adds its decoded
    residual; the reconstructions equal the encode's byte for byte."""
    n = len(preds)
    _same_length(n, codes=codes, K_rec=K_rec, V_rec=V_rec)
    wp, wn = _ws(ws)
    _check(lib().kvc_decode_layers(ctypes.byref(desc), _preds(preds), n, _codes(codes), _ptr(K_src), _ptr(V_src),
                                   _ptrs(K_rec), _ptrs(V_rec), wp, wn, _stream(stream)), "kvc_decode_layers")


def kvc_decode_layer(desc, pred, codes: CodeBuffers, K_src, V_src, K_rec, V_rec, ws=None, stream=None):
    c = codes.struct()
    wp, wn = _ws(ws)
    _check(lib().kvc_decode_layer(ctypes.byref(desc), ctypes.byref(pred), ctypes.byref(c), _ptr(K_src), _ptr(V_src),
                                  _ptr(K_rec), _ptr(V_rec), wp, wn, _stream(stream)), "kvc_decode_layer")


def kvc_attend_compressed(desc, pred, Q, codes: CodeBuffers, K_src, V_src, K_self, V_self, scale: float, O,
                          ws=None, stream=None, K_rec=None, V_rec=None):
    """K_rec / V_rec: optional outputs of the decoded history (K_rec_opt / V_rec_opt)."""
    c = codes.struct()
    wp, wn = _ws(ws)
    n_q = 0 if Q is None else Q.shape[0]
    n_self = 0 if K_self is None else K_self.shape[0]
    _check(lib().kvc_attend_compressed(ctypes.byref(desc), ctypes.byref(pred), _ptr(Q), n_q, ctypes.byref(c),
                                       _ptr(K_src), _ptr(V_src), _ptr(K_self), _ptr(V_self), n_self,
                                       ctypes.c_float(scale), _ptr(O), _ptr(K_rec), _ptr(V_rec), wp, wn,
                                       _stream(stream)),
           "kvc_attend_compressed")


def kvc_attend_compressed_debiased(desc, pred, Q, codes: CodeBuffers, K_src, V_src, K_self, V_self, scale: float,
                                   O, ws=None, stream=None, K_rec=None, V_rec=None):
    """kvc_attend_compressed with the Jensen-bias correction of the history keys."""
    c = codes.struct()
    wp, wn = _ws(ws)
    n_q = 0 if Q is None else Q.shape[0]
    n_self = 0 if K_self is None else K_self.shape[0]
    _check(lib().kvc_attend_compressed_debiased(ctypes.byref(desc), ctypes.byref(pred), _ptr(Q), n_q,
                                                ctypes.byref(c), _ptr(K_src), _ptr(V_src), _ptr(K_self),
                                                _ptr(V_self), n_self, ctypes.c_float(scale), _ptr(O), _ptr(K_rec),
                                                _ptr(V_rec), wp, wn, _stream(stream)),
           "kvc_attend_compressed_debiased")


def kvc_refit_block_diag(desc, pred, tensor: int, X0, X1, Y, ridge: float, block_out, ws=None, stream=None):
    """Video-adapted refit of the per-head blocks (tensor 0: K, 1: V)."""
    wp, wn = _ws(ws)
    _check(lib().kvc_refit_block_diag(ctypes.byref(desc), ctypes.byref(pred), int(tensor), _ptr(X0), _ptr(X1),
                                      _ptr(Y), ctypes.c_float(ridge), _ptr(block_out), wp, wn, _stream(stream)),
           "kvc_refit_block_diag")


def kvc_copy_to_device(dst: torch.Tensor, src: torch.Tensor, stream=None):
    """Copies a host tensor (pinned for asynchrony) into a device tensor of the same size."""
    n = src.numel() * src.element_size()
    if dst.numel() * dst.element_size() < n:
        raise ValueError(f"destination holds {dst.numel() * dst.element_size()} bytes, the copy {n}")
    _check(lib().kvc_copy_to_device(_ptr(dst), ctypes.c_void_p(src.data_ptr()), n, _stream(stream)),
           "kvc_copy_to_device")


def kvc_copy_to_host(dst: torch.Tensor, src: torch.Tensor, stream=None):
    """Copies a device tensor into a host tensor (pinned for asynchrony) of the same size."""
    n = src.numel() * src.element_size()
    if dst.numel() * dst.element_size() < n:
        raise ValueError(f"destination holds {dst.numel() * dst.element_size()} bytes, the copy {n}")
    _check(lib().kvc_copy_to_host(ctypes.c_void_p(dst.data_ptr()), _ptr(src), n, _stream(stream)),
           "kvc_copy_to_host")


def kvc_pack_codes(codes: torch.Tensor, bits: int, packed: torch.Tensor, stream=None):
    _check(lib().kvc_pack_codes(_ptr(codes), codes.numel(), bits, _ptr(packed), _stream(stream)), "kvc_pack_codes")


def kvc_unpack_codes(packed: torch.Tensor, n: int, bits: int, codes: torch.Tensor, stream=None):
    _check(lib().kvc_unpack_codes(_ptr(packed), n, bits, _ptr(codes), _stream(stream)), "kvc_unpack_codes")


def kvc_get_device_error(stream=None) -> int:
    return lib().kvc_get_device_error(_stream(stream))


def kvc_launch_counter() -> int:
    return int(lib().kvc_launch_counter())


def kvc_status_string(status: int) -> str:
    return lib().kvc_status_string(status).decode()


def kvc_encode_layer_cluster_static(desc, pred, K, V, codes: CodeBuffers, K_rec=None, V_rec=None, stream=None):
    """Clustered-codec encode that allocates nothing (its centre tables live in
    a static device array inside the library); for callers that cannot
    allocate device memory at encode time.  Same results as kvc_encode_layer."""
    fn = lib().kvc_encode_layer_cluster_static
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(LayerDesc), ctypes.POINTER(Predictor), ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.POINTER(Codes), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    c = codes.struct()
    _check(fn(ctypes.byref(desc), ctypes.byref(pred), _ptr(K), _ptr(V), ctypes.byref(c), _ptr(K_rec), _ptr(V_rec),
              _stream(stream)), "kvc_encode_layer_cluster_static")


def kvc_testing_inject_stall(what: int = 1):
    """Test hook (include/kvc_testing.h): the next tensor-core cross-layer codec
    launch leaves one pipeline stage unarmed, so a bounded device wait runs out
    and kvc_get_device_error() reports KVC_ERR_DEVICE_TIMEOUT."""
    fn = lib().kvc_testing_inject_stall
    fn.restype = None
    fn.argtypes = [ctypes.c_int]
    fn(int(what))
