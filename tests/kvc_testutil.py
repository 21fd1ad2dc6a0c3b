"""Helpers of the parity tests: moving codes between the GPU layout and the
oracle's unpacked form, and the tolerance checks.

Tolerances (one place for all tests):
  * packing / unpacking: bit-exact;
  * codes: >= 99.99 % of elements equal, any difference at most one level;
  * reconstructions: |gpu - oracle| <= 1e-3 (|x| + 1) wherever the codes agree,
    except where the exact value lies within fp32 accumulation error of a
    rounding midpoint of the state dtype (both roundings are then correct);
  * attention: relative L2 <= 1e-2 for bf16 outputs, <= 1e-4 for fp32.
"""

from __future__ import annotations

import numpy as np
import torch

from oracle import kvc_oracle as O

CODE_AGREE = 0.9999
ATT_TOL = {torch.bfloat16: 1e-2, torch.float32: 1e-4}


def to64(t) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def np_state(dtype) -> str:
    return {torch.bfloat16: "bf16", torch.float32: "f32"}[dtype]


def np_param(dtype) -> str:
    return {torch.float16: "f16", torch.float32: "f32"}[dtype]


def _params_dtype(param):
    return torch.float16 if param == "f16" else torch.float32


def params_from_gpu(buf: torch.Tensor, shape, param: str):
    """(scale, zero) pairs [..., 2] -> (s, z) float64 arrays of `shape`."""
    n = int(np.prod(shape))
    v = buf[: n * 2 * (2 if param == "f16" else 4)].view(_params_dtype(param)).reshape(*shape, 2)
    v = v.cpu().double().numpy()
    return v[..., 0], v[..., 1]


def params_to_gpu(s, z, param: str, device="cuda") -> torch.Tensor:
    pair = np.stack([s, z], axis=-1)
    t = torch.from_numpy(pair.astype(np.float16 if param == "f16" else np.float32))
    return t.reshape(-1).view(torch.uint8).to(device)


def codes_from_gpu(buf: torch.Tensor, shape, bits: int) -> np.ndarray:
    n = int(np.prod(shape))
    raw = buf[: n * bits // 8].cpu().numpy().reshape(*shape[:-1], shape[-1] * bits // 8)
    return O.unpack_codes(raw, bits, shape[-1])


def codes_to_gpu(q, bits: int, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(O.pack_codes(q, bits)).reshape(-1)).to(device)


def pad16(t: torch.Tensor) -> torch.Tensor:
    n = max(16, t.numel())
    out = torch.zeros(n, dtype=torch.uint8, device=t.device)
    out[: t.numel()] = t
    return out


def assert_codes_close(q_gpu, q_ref, what="codes", min_agree=CODE_AGREE):
    d = np.abs(q_gpu.astype(np.int64) - q_ref.astype(np.int64))
    agree = float((d == 0).mean()) if d.size else 1.0
    assert agree >= min_agree, f"{what}: agreement {agree:.6f} < {min_agree}"
    assert d.size == 0 or d.max() <= 1, f"{what}: a code differs by {d.max()} levels"
    return agree


def param_ulp(v, param: str) -> np.ndarray:
    """Spacing of the parameter dtype at v."""
    return np.spacing(np.abs(v).astype(np.float16 if param == "f16" else np.float32)).astype(np.float64)


PARAM_FLIP_BUDGET = 1e-2


def assert_params_close(s_gpu, z_gpu, s_ref, z_ref, param: str, what="params", levels: int = 3):
    """Stored (scale, zero) pairs.  They round the group's min and max of the
    residual, which the GPU forms in fp32 (about 1e-6 relative away from the
    oracle's fp64).  fp16 pairs: equal, or one fp16 rounding step apart, on at
    most 1 % of the groups (a shift of 1e-6 crosses an fp16 rounding boundary
    with probability about 2e-6 / 2^-11).  fp32 pairs: equal to 1e-5 relative.
    Returns the mask of groups whose pair differs."""
    ds = np.abs(s_gpu - s_ref)
    dz = np.abs(z_gpu - z_ref)
    if param == "f16":
        us = np.maximum(param_ulp(s_ref, param), param_ulp(s_gpu, param))
        uz = np.maximum(param_ulp(z_ref, param), param_ulp(z_gpu, param))
        assert np.all(ds <= us * 1.0001), f"{what}: a scale differs by more than one fp16 step"
        assert np.all(dz <= uz * 1.0001), f"{what}: a zero differs by more than one fp16 step"
        diff = (ds > 0) | (dz > 0)
        assert diff.mean() <= PARAM_FLIP_BUDGET, f"{what}: {diff.mean():.2e} of the groups differ"
        return diff
    span = np.abs(z_ref) + levels * np.abs(s_ref) + 1e-6
    assert np.all(ds <= 1e-5 * span), f"{what}: a scale differs by more than 1e-5 of the group's span"
    assert np.all(dz <= 1e-5 * span), f"{what}: a zero differs by more than 1e-5 of the group's span"
    return np.zeros(s_ref.shape, bool)


def assert_recon_close(rec_gpu, rec_ref, exact_ref, x, code_flip, state: str, what="recon"):
    """rec_gpu, rec_ref: values in the state dtype; exact_ref: the oracle's
    value before rounding to the state dtype; code_flip: elements whose code
    differs (excluded)."""
    tol = 1e-3 * (np.abs(x) + 1.0)
    bad = (np.abs(rec_gpu - rec_ref) > tol) & ~code_flip
    if np.any(bad) and state != "f64":
        # a mismatch is a rounding tie only if the exact value is at a midpoint
        # of the two neighbouring state values, within fp32 accumulation error
        mid = 0.5 * (rec_gpu + rec_ref)
        near = np.abs(exact_ref - mid) <= 2e-5 * (np.abs(exact_ref) + 1e-3)
        adjacent = O.round_to(mid, state) != mid  # mid is not itself representable
        bad &= ~(near & adjacent)
    n_bad = int(bad.sum())
    assert n_bad == 0, f"{what}: {n_bad} elements outside tolerance, worst {np.abs(rec_gpu - rec_ref)[bad].max()}"


def rel_l2(a, b) -> float:
    return O.rel_l2(a, b)


# ---------------------------------------------------------------- exact (unrounded) oracle values


def exact_none(c: "O.Coded", group: int):
    return O.dequantize_groups(c.q, c.s, c.z, group)


def exact_xlayer(d: "O.Desc", w: dict, ck, cv, K_src, V_src, K_hat):
    pk = O.xlayer_predict_k(K_src, w["k_block"], w["k_w"], w["k_u"])
    pv = O.xlayer_predict_v(K_hat, V_src, w["v_block"], w["v_w"], w["v_u"])
    return pk + O.dequantize_groups(ck.q, ck.s, ck.z, d.group), pv + O.dequantize_groups(cv.q, cv.s, cv.z, d.group)


def exact_temporal(d: "O.Desc", w: dict, ck, cv, K_hat, V_hat):
    T, H, D = K_hat.shape
    F = d.frame_tokens
    ek = np.zeros((T, H, D))
    ev = np.zeros((T, H, D))
    for f, a in enumerate(range(0, T, F)):
        b = min(T, a + F)
        n = b - a
        if f == 0:
            pk = np.zeros((n, H, D))
            pv = np.zeros((n, H, D))
        else:
            k2 = K_hat[a - 2 * F:a - 2 * F + n] if f >= 2 else np.zeros((n, H, D))
            pk = O._blockdiag(np.concatenate([K_hat[a - F:a - F + n], k2], -1), w["ak"])
            pv = O._blockdiag(np.concatenate([K_hat[a:b], V_hat[a - F:a - F + n]], -1), w["av"])
        ek[a:b] = pk + O.dequantize_groups(ck.q[a:b], ck.s[a:b], ck.z[a:b], d.group)
        ev[a:b] = pv + O.dequantize_groups(cv.q[a:b], cv.s[a:b], cv.z[a:b], d.group)
    return ek, ev
