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

# Observed agreement of every parity check in this process (written out by
# tests/conftest.py when KVC_PARITY_LOG names a file): the measured code
# agreement and the fraction of fp16 (scale, zero) groups that differ.
OBSERVED: list = []


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
    OBSERVED.append({"check": what, "code_agreement": agree, "elements": int(d.size)})
    if agree < min_agree:  # where the differences sit: spread thin (rounding) or bunched (one row / head)
        per_row = (d != 0).reshape(d.shape[0], -1).mean(axis=1)
        per_col = (d != 0).reshape(d.shape[0], d.shape[1], -1).mean(axis=(0, 2)) if d.ndim >= 3 else per_row[:0]
        raise AssertionError(f"{what}: agreement {agree:.6f} < {min_agree}; rows with a difference "
                             f"{int((per_row > 0).sum())} of {len(per_row)}, worst row {per_row.max():.3f}, "
                             f"worst second-axis index {int(per_col.argmax()) if per_col.size else -1} "
                             f"({per_col.max() if per_col.size else 0:.3f})")
    assert d.size == 0 or d.max() <= 1, f"{what}: a code differs by {d.max()} levels"
    return agree


def param_ulp(v, param: str) -> np.ndarray:
    """Spacing of the parameter dtype at v."""
    return np.spacing(np.abs(v).astype(np.float16 if param == "f16" else np.float32)).astype(np.float64)


# fp16 (scale, zero) pairs that may differ from the oracle's, as a fraction of
# the groups with identical inputs, plus three groups of slack for small
# samples.  Observed on a B200 over every parity check: at most 0.6 % of the
# groups in samples of 1000 or more (a residual moved by fp32 accumulation
# error crosses an fp16 rounding boundary), 1 group of 70 at worst in the
# small per-frame samples.
PARAM_FLIP_RATE = 2e-2
PARAM_FLIP_SLACK_GROUPS = 3


U32 = 2.0 ** -23  # fp32 rounding unit, allowing for truncating accumulation


def group_max(err, group):
    """Largest per-element bound inside each group of `group` channels."""
    return err.reshape(err.shape[:-1] + (err.shape[-1] // group, group)).max(axis=-1)


def assert_params_close(s_gpu, z_gpu, s_ref, z_ref, param: str, what="params", levels: int = 3, err=None,
                        group: int = 32, skip=None):
    """Stored (scale, zero) pairs round the group's min and max of the residual.
    The GPU forms the residual with fp32 accumulation; `err` [..., n] bounds,
    per element, how far its prediction can be from the exact one (0 when
    there is no prediction).  Each stored value may then differ from the
    oracle's by that bound plus one rounding step of the parameter dtype, and
    (fp16) at most PARAM_FLIP_RATE of the groups, plus PARAM_FLIP_SLACK_GROUPS
    groups, may differ at all (a residual moved by the accumulation error
    crosses an fp16 rounding boundary now and then).  `skip` marks groups whose inputs already
    differ (an earlier flipped code); they are not checked and do not count
    against the budget.  Returns the mask of groups whose pair differs."""
    ds = np.abs(s_gpu - s_ref)
    dz = np.abs(z_gpu - z_ref)
    e = np.zeros(s_ref.shape) if err is None else group_max(err, group)
    ok = np.ones(s_ref.shape, bool) if skip is None else ~skip
    us = np.maximum(param_ulp(s_ref, param), param_ulp(s_gpu, param)) + 2.0 * e / levels
    uz = np.maximum(param_ulp(z_ref, param), param_ulp(z_gpu, param)) + e
    if param == "f32":  # fp32 pairs are also rounded from fp32 min / max: allow a few rounding units
        span = np.abs(z_ref) + levels * np.abs(s_ref)
        us = us + 4 * U32 * span
        uz = uz + 4 * U32 * span
    assert np.all((ds <= us * 1.0001) | ~ok), f"{what}: a scale is outside its bound (worst {np.max((ds / us)[ok]):.2f})"
    assert np.all((dz <= uz * 1.0001) | ~ok), f"{what}: a zero is outside its bound (worst {np.max((dz / uz)[ok]):.2f})"
    diff = (ds > 0) | (dz > 0)
    n_ok = int(ok.sum())
    rate = float(diff[ok].mean()) if n_ok else 0.0  # among groups with the same inputs on both sides
    OBSERVED.append({"check": what, "param": param, "param_groups_differing": rate, "groups": n_ok})
    if param == "f16":
        budget = PARAM_FLIP_RATE + PARAM_FLIP_SLACK_GROUPS / max(n_ok, 1)
        assert rate <= budget, f"{what}: {rate:.2e} of the groups differ (budget {budget:.2e})"
        return diff
    return np.zeros(s_ref.shape, bool)


def assert_recon_close(rec_gpu, rec_ref, exact_ref, x, code_flip, state: str, what="recon", err=None, alt=None):
    """rec_gpu, rec_ref: values in the state dtype; exact_ref: the oracle's
    value before rounding to the state dtype; code_flip: elements whose stored
    code differs; err: per-element bound of the GPU's accumulation error;
    alt: for flipped elements, the exact value that the GPU's own stored code
    reconstructs (the oracle's prediction plus the GPU's dequantized code):
    the GPU's reconstruction must match it instead."""
    tol = 1e-3 * (np.abs(x) + 1.0)
    e_all = (0.0 if err is None else err) + 8 * U32 * (np.abs(exact_ref) + 1e-3)
    if alt is not None and np.any(code_flip):
        ulp = np.abs(O.round_to(alt, state) - alt) + np.spacing(np.abs(alt).astype(np.float32))
        badf = code_flip & (np.abs(rec_gpu - alt) > tol + e_all + ulp)
        assert not np.any(badf), f"{what}: {int(badf.sum())} flipped elements do not reconstruct their own code"
    bad = (np.abs(rec_gpu - rec_ref) > tol) & ~code_flip
    if np.any(bad) and state != "f64":
        # a mismatch is a rounding tie only if the exact value is at a midpoint
        # of the two neighbouring state values, within the accumulation error
        mid = 0.5 * (rec_gpu + rec_ref)
        near = np.abs(exact_ref - mid) <= e_all
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


def _temporal_preds(d: "O.Desc", w: dict, K_hat, V_hat, k_hist=None, v_hist=None, absolute=False):
    """Per-token predictions of the temporal maps from the given reconstructed
    frames (frame 0 predicted from k_hist / v_hist when given, else 0).  With
    `absolute`, the same on absolute values (for error bounds)."""
    T, H, D = K_hat.shape
    F = d.frame_tokens
    f_ = np.abs if absolute else (lambda x: x)
    hk = np.zeros((2 * F, H, D)) if k_hist is None else np.asarray(k_hist, np.float64).reshape(2 * F, H, D)
    hv = np.zeros((F, H, D)) if v_hist is None else np.asarray(v_hist, np.float64).reshape(F, H, D)
    Ka = f_(np.concatenate([hk, K_hat]))
    Va = f_(np.concatenate([hv, V_hat]))
    w = {k: f_(v) for k, v in w.items()}
    pk = np.zeros((T, H, D))
    pv = np.zeros((T, H, D))
    for f, a in enumerate(range(0, T, F)):
        if f == 0 and k_hist is None:
            continue
        b = min(T, a + F)
        n = b - a
        ko, vo = 2 * F + a, F + a
        pk[a:b] = O._blockdiag(np.concatenate([Ka[ko - F:ko - F + n], Ka[ko - 2 * F:ko - 2 * F + n]], -1), w["ak"])
        pv[a:b] = O._blockdiag(np.concatenate([Ka[ko:ko + n], Va[vo - F:vo - F + n]], -1), w["av"])
    return pk, pv


def exact_temporal(d: "O.Desc", w: dict, ck, cv, K_hat, V_hat, k_hist=None, v_hist=None):
    pk, pv = _temporal_preds(d, w, K_hat, V_hat, k_hist, v_hist)
    return (pk + O.dequantize_groups(ck.q, ck.s, ck.z, d.group),
            pv + O.dequantize_groups(cv.q, cv.s, cv.z, d.group))


# ---------------------------------------------------------------- a-priori accumulation bounds
#
# |fl(sum) - sum| <= n u sum|terms| for n terms accumulated in fp32 (u = 2^-23
# allows truncation).  The bound of a whole prediction is built by running the
# predictor on absolute values.


def err_xlayer(d: "O.Desc", w: dict, K_src, V_src, K_hat):
    aw = {k: np.abs(v) for k, v in w.items()}
    T, H, D = K_src.shape
    C = H * D
    r = w["k_w"].shape[0]
    blk_k = O._blockdiag(np.abs(K_src), aw["k_block"])
    blk_v = O._blockdiag(np.concatenate([np.abs(K_hat), np.abs(V_src)], -1), aw["v_block"])
    lat_k = O.xlayer_predict_k(np.abs(K_src), 0 * aw["k_block"], aw["k_w"], aw["k_u"])
    lat_v = O.xlayer_predict_v(np.abs(K_hat), np.abs(V_src), 0 * aw["v_block"], aw["v_w"], aw["v_u"])
    lat_gamma_k = (C + r) * U32 + 2.0 ** -16
    lat_gamma_v = (2 * C + r) * U32 + 2.0 ** -16
    return D * U32 * blk_k + lat_gamma_k * lat_k, 2 * D * U32 * blk_v + lat_gamma_v * lat_v


def err_temporal(d: "O.Desc", w: dict, K_hat, V_hat, k_hist=None, v_hist=None):
    """Bound of the temporal predictions (2D terms each), from the oracle's history."""
    D = K_hat.shape[-1]
    ak, av = _temporal_preds(d, w, K_hat, V_hat, k_hist, v_hist, absolute=True)
    return 2 * D * U32 * ak, 2 * D * U32 * av


def err_cluster(X_flat, cent, a, enc):
    """Bound of the coefficients enc (x - c_a) formed as enc x - enc c_a in fp32."""
    C = X_flat.shape[1]
    return C * U32 * (np.abs(X_flat) @ np.abs(enc).T + np.abs(cent[a]) @ np.abs(enc).T)
