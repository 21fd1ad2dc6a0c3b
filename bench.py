#!/usr/bin/env python
"""Benchmark of the predict-then-quantize-residual KV codec on one B200.

One step = closed-loop encode of every layer of a Wan-1.3B-shaped history
(30 layers x 32760 tokens x 12 heads x 128 channels, bf16; layer 0 INT4 anchor,
layers 1-29 block-DPLR prediction with rank-64 low-rank term and INT2 g32
residual with fp16 scale/zero) followed by the decode of every layer from the
codes.  Inputs (6 GB) are resident in HBM and larger than L2, so every step
streams from DRAM.  Metric: KV tokens encoded + decoded per second.

Also measured, in the same run (N = 1): the attention of a 4680-query chunk over
the compressed history of layer 15, one layer of the temporal codec (40 heads,
65536 tokens, INT4 g64), and one layer of the clustered codec with
mixed-dimensional attention (16 heads, 32768 tokens, 1560 queries).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 run under torch.distributed.run; every rank codes its own 32760-token
shard (weak scaling, no collective on the data path).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from clustered_kv_cache_b200 import kvc, synth  # noqa: E402

L_LAYERS, T_TOK, H, D, RANK = 30, 21 * 1560, 12, 128, 64
METRIC = "KV tokens/s encoded+decoded (GB/s vs HBM peak); compressed-attn TFLOP/s vs roofline"
UNIT = "KV tokens/s"


# DRAM bytes (read + write) per call, from the ncu captures summarised under
# profiles/ (codec_xlayer_wan_layer.md, codec_xlayer_fused_wan.md, attention_flash_wan.md,
# mixed_attention_cluster.md, cluster_codec_decode.md, temporal_codec_layer.md, codec_xlayer_eden2.md);
# set to None when a kernel changes after its capture.
TRAFFIC = {"encode_xlayer": 679453184 + 187834368, "decode_xlayer": 430907648 + 137585920,
           # per layer of the fused walk (a 4-layer launch's DRAM bytes / 4; scaled by the layer count)
           "encode_xlayer_fused": (2892781056 + 912364800) // 4, "decode_xlayer_fused": (2074051072 + 744571648) // 4,
           "attention_c2": 244925696 + 13229312, "attention_c4": 26439936 + 141056,
           "decode_c4": 9409024 + 214975232,
           "temporal_encode": 1424011008 + 351590400,
           "temporal_decode": 659118080 + 1286398464,
           "eden2_encode": None, "eden2_decode": 414407936 + 136523520}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p["bf16_tflops_sustained"], "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------- clocks during the timed region


class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.dev)], stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[4:8]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- the cross-layer workload


class XLayerBench:
    """Buffers and calls of the 30-layer encode + decode step."""

    def __init__(self, device, seed, layers=L_LAYERS):
        self.L = layers
        self.wl = synth.wan_xlayer(seed=seed, device=device, L=layers, T=T_TOK, H=H, D=D, rank=RANK)
        bf, hf = torch.bfloat16, torch.float16
        self.desc0 = kvc.make_desc(T_TOK, H, D, bf, 4, 32, hf)  # INT4 anchor
        self.desc = kvc.make_desc(T_TOK, H, D, bf, 2, 32, hf)
        self.pred0 = kvc.make_predictor(kvc.PRED_NONE)
        self.preds = [None] + [kvc.make_predictor(kvc.PRED_XLAYER_DPLR, self.wl.weights[l], rank=RANK)
                               for l in range(1, layers)]
        self.codes = [kvc.alloc_codes(self.desc0, self.pred0, device)] + \
                     [kvc.alloc_codes(self.desc, self.preds[l], device) for l in range(1, layers)]
        self.ws_enc = kvc.alloc_workspace(kvc.OP_ENCODE, self.desc, self.preds[1], device=device)
        self.ws_dec = kvc.alloc_workspace(kvc.OP_DECODE, self.desc, self.preds[1], device=device)
        if layers >= 2:  # the fused calls over layers 1 .. L-1 (one launch each way)
            self.ws_enc_all = kvc.alloc_layers_workspace(kvc.OP_ENCODE, self.desc, self.preds[1:], device=device)
            self.ws_dec_all = kvc.alloc_layers_workspace(kvc.OP_DECODE, self.desc, self.preds[1:], device=device)
        mk = lambda: torch.empty(T_TOK, H, D, dtype=bf, device=device)
        self.er = [(mk(), mk()), (mk(), mk())]  # encode-chain reconstructions (ping-pong)
        self.dr = [(mk(), mk()), (mk(), mk())]  # decode-chain reconstructions
        self.keep = None  # (K^_{l-1}, V^_{l-1}) for the attention row over layer l
        self.attn_layer = min(15, layers - 1)  # layer 15 of 30 (a smaller run: its last layer)

    def encode_chain(self, ev=None, keep_layer=None, before=None, after=None):
        """before(l) / after(l): hooks around the encode of layer l (the end-to-end
        step orders its copies against them)."""
        K, V = self.wl.K, self.wl.V
        Kr, Vr = self.er[0]
        if before:
            before(0)
        kvc.kvc_encode_layer(self.desc0, self.pred0, K[0], V[0], None, None, self.codes[0], Kr, Vr)
        if after:
            after(0)
        for l in range(1, self.L):
            Ks, Vs = self.er[(l - 1) % 2]
            Kr, Vr = self.er[l % 2]
            if before:
                before(l)
            if ev is not None:
                ev[l][0].record()
            kvc.kvc_encode_layer(self.desc, self.preds[l], K[l], V[l], Ks, Vs, self.codes[l], Kr, Vr, self.ws_enc)
            if ev is not None:
                ev[l][1].record()
            if after:
                after(l)
            if keep_layer is not None and l == keep_layer - 1:
                self.keep = (Kr.clone(), Vr.clone())

    def decode_chain(self, ev=None):
        Kr, Vr = self.dr[0]
        kvc.kvc_decode_layer(self.desc0, self.pred0, self.codes[0], None, None, Kr, Vr)
        for l in range(1, self.L):
            Ks, Vs = self.dr[(l - 1) % 2]
            Kr, Vr = self.dr[l % 2]
            if ev is not None:
                ev[l][0].record()
            kvc.kvc_decode_layer(self.desc, self.preds[l], self.codes[l], Ks, Vs, Kr, Vr, self.ws_dec)
            if ev is not None:
                ev[l][1].record()

    def encode_fused(self, ev=None):
        """The anchor layer, then layers 1 .. L-1 in one kvc_encode_layers launch
        (the same ping-pong reconstruction buffers as the per-layer chain)."""
        K, V = self.wl.K, self.wl.V
        Kr0, Vr0 = self.er[0]
        kvc.kvc_encode_layer(self.desc0, self.pred0, K[0], V[0], None, None, self.codes[0], Kr0, Vr0)
        if self.L < 2:
            return
        if ev is not None:
            ev[0].record()
        kvc.kvc_encode_layers(self.desc, self.preds[1:], K[1:], V[1:], Kr0, Vr0, self.codes[1:],
                              [self.er[l % 2][0] for l in range(1, self.L)],
                              [self.er[l % 2][1] for l in range(1, self.L)], self.ws_enc_all)
        if ev is not None:
            ev[1].record()

    def decode_fused(self, ev=None):
        Kr0, Vr0 = self.dr[0]
        kvc.kvc_decode_layer(self.desc0, self.pred0, self.codes[0], None, None, Kr0, Vr0)
        if self.L < 2:
            return
        if ev is not None:
            ev[0].record()
        kvc.kvc_decode_layers(self.desc, self.preds[1:], self.codes[1:], Kr0, Vr0,
                              [self.dr[l % 2][0] for l in range(1, self.L)],
                              [self.dr[l % 2][1] for l in range(1, self.L)], self.ws_dec_all)
        if ev is not None:
            ev[1].record()

    def step(self, ev_enc=None, ev_dec=None):
        self.encode_fused(ev_enc)
        self.decode_fused(ev_dec)

    # algorithmic traffic / work of one predicted layer
    def layer_bytes(self, encode: bool) -> int:
        C = H * D
        codes = kvc.kvc_codes_bytes(self.desc, self.preds[1])
        w = sum(t.numel() * t.element_size() for t in self.wl.weights[1].values())
        io = 2 * T_TOK * C * 2 * (3 if encode else 2)  # K,V in (encode) + sources in + recon out
        return io + codes + w

    @staticmethod
    def layer_flops() -> int:
        C = H * D
        return 2 * T_TOK * (H * D * D + C * RANK + RANK * C + H * 2 * D * D + 2 * C * RANK + RANK * C)


def time_events(pairs):
    return [s.elapsed_time(e) for s, e in pairs]


# ---------------------------------------------------------------- oracle timing (CPU)


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_xlayer_rate(wl, n_tok: int, layers: int, budget_s: float, threads: int = 1) -> dict:
    """Times the plain fp64 C++ oracle's closed-loop encode + decode of `n_tok`
    tokens through `layers` layers (tokens are independent, so this is an exact
    sample of the workload).  threads = 1: the single-threaded oracle; more:
    its thread driver over disjoint token runs.  Returns tokens/s (encoded +
    decoded)."""
    from oracle import kvc_oracle_c as O

    O.build()
    idx = torch.linspace(0, wl.K[0].shape[0] - 1, n_tok).long()
    t64 = lambda t: t[idx.to(t.device)].detach().cpu().double().numpy()
    K = [t64(k) for k in wl.K[:layers]]
    V = [t64(v) for v in wl.V[:layers]]
    W = [None] + [{k: v.detach().cpu().double().numpy() for k, v in wl.weights[l].items()} for l in range(1, layers)]
    d0 = O.Desc(n_tok, H, D, "bf16", 4, 32, "f16")
    d = O.Desc(n_tok, H, D, "bf16", 2, 32, "f16")
    t0 = time.perf_counter()
    done = 0
    ck, cv, Kh, Vh = O.encode_layer_none(d0, K[0], V[0], threads=threads)
    Kd, Vd = O.decode_layer_none(d0, ck, cv, threads=threads)
    done += 2
    for l in range(1, layers):
        ck, cv, Kh2, Vh2 = O.encode_layer_xlayer(d, W[l], K[l], V[l], Kh, Vh, threads=threads)
        Kd, Vd = O.decode_layer_xlayer(d, W[l], ck, cv, Kd, Vd, threads=threads)
        Kh, Vh = Kh2, Vh2
        done += 2
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": done * n_tok / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n_tok} of {T_TOK} tokens (evenly spaced) through {done // 2} of {L_LAYERS} layers, "
                      f"encode + decode, plain fp64 C++ oracle on {threads} thread(s); {dt:.1f} s"}


def cpu_baseline_line(wl, layers: int) -> dict:
    """The oracle on one host core (the baseline) and, beside it, its thread
    driver on every core of the box."""
    one = oracle_xlayer_rate(wl, 256, layers, 12.0, threads=1)
    n = O_threads()
    box = oracle_xlayer_rate(wl, 256 * n, layers, 12.0, threads=n)
    one["whole_box"] = {"value": box["value"], "unit": UNIT, "cores": n, "sample": box["sample"]}
    one["cpu_model"] = cpu_model()
    one["nproc"] = os.cpu_count()
    return one


def O_threads() -> int:
    from oracle import kvc_oracle_c as O

    return O.default_threads()


def run_reference(args, rank: int):
    """Reference arm: the fp64 oracle on the host cores, same metric and config."""
    if rank != 0:
        return
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    wl = synth.wan_xlayer(seed=synth.SEED_BASE + 1, device=dev, L=L_LAYERS, T=T_TOK if dev == "cuda" else 512,
                          H=H, D=D, rank=RANK)
    n = O_threads()
    for _ in range(args.warmup):
        oracle_xlayer_rate(wl, 4 * n, 2, 5.0, threads=n)
    vals, secs = [], []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        r = oracle_xlayer_rate(wl, 16 * n, L_LAYERS, 8.0, threads=n)
        secs.append(time.perf_counter() - t0)
        vals.append(r["value"])
    value = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * statistics.median(secs),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded Wan-1.3B-shaped trace, least-squares block-DPLR predictors)",
            "config": {"workload": "cross-layer codec, 30 layers x 32760 tokens x 12 heads x 128, INT2 g32 + INT4 "
                                   "anchor, rank 64; each step a bounded token sample", "global_batch": T_TOK,
                       "seq_len": T_TOK, "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": r["cores"], "kind": "oracle",
                             "sample": r["sample"], "cpu_model": cpu_model()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- extra rows (N = 1)


# ---------------------------------------------------------------- ranks (N > 1: weak scaling)


def shard_seed(rank: int) -> int:
    """Seed of a rank's own 32760-token shard (every rank codes different tokens)."""
    return synth.SEED_BASE + 1 + 1000 * rank


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's value: every multi-rank time is the max over ranks."""
    if world <= 1:
        return x
    t = torch.tensor([x], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_value(ms_step: float, world: int, layers: int) -> float:
    """Whole-job KV tokens/s: every rank's tokens, encoded and decoded through
    every layer, over the slowest rank's step time."""
    return 2 * T_TOK * layers * world / (ms_step * 1e-3)


def synced_ok():
    """Waits for the device and fails on a kernel-reported error (an expired
    wait, a bad launch): a timing of such a run is no measurement."""
    torch.cuda.synchronize()
    err = kvc.kvc_get_device_error()
    if err:
        raise RuntimeError(f"device error word 0x{err:x} after a timed row")


def row_attention(xb: XLayerBench, hbm, tf_burst, tf_sust, reps=3) -> dict:
    """4680 queries (3 latent frames) over layer 15's compressed history plus the
    chunk itself: one decode of the history (the codec kernel), then the flash
    attention kernel.  The decode is also timed alone, so that the attention
    kernel's own share and roofline are reported."""
    dev = xb.wl.K[0].device
    n_q = 3 * 1560
    Q = synth.queries(synth.SEED_BASE + 2, n_q, H, D, device=dev)
    Ks = synth.queries(synth.SEED_BASE + 12, n_q, H, D, device=dev)
    Vs = synth.queries(synth.SEED_BASE + 22, n_q, H, D, device=dev)
    O_ = torch.empty(n_q, H, D, dtype=torch.bfloat16, device=dev)
    l = xb.attn_layer
    ws = kvc.alloc_workspace(kvc.OP_ATTEND, xb.desc, xb.preds[l], n_q, device=dev)
    Kh, Vh = xb.keep
    call = lambda: kvc.kvc_attend_compressed(xb.desc, xb.preds[l], Q, xb.codes[l], Kh, Vh, Ks, Vs, D ** -0.5,
                                             O_, ws)
    call()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for s, e in ev:
        s.record()
        call()
        e.record()
    synced_ok()
    ms = statistics.median(time_events(ev))
    Kd, Vd = torch.empty_like(Kh), torch.empty_like(Vh)
    wsd = kvc.alloc_workspace(kvc.OP_DECODE, xb.desc, xb.preds[l], device=dev)
    dec = lambda: kvc.kvc_decode_layer(xb.desc, xb.preds[l], xb.codes[l], Kh, Vh, Kd, Vd, wsd)
    dec()
    torch.cuda.synchronize()
    evd = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for s, e in evd:
        s.record()
        dec()
        e.record()
    synced_ok()
    ms_dec = statistics.median(time_events(evd))
    attn_flops = 4 * n_q * (T_TOK + n_q) * H * D
    total = attn_flops + XLayerBench.layer_flops()
    tflops = total / (ms * 1e-3) / 1e12
    ms_attn = max(ms - ms_dec, 1e-6)
    tf_attn = attn_flops / (ms_attn * 1e-3) / 1e12
    return {"workload": "4680 queries x (32760 compressed + 4680 chunk) keys, 12 heads x 128, layer 15",
            "ms": ms, "value": tflops, "unit": "TFLOP/s (attention + one decode of the history)",
            "decode_ms": ms_dec, "attention_kernel_ms": ms_attn,
            "attention_kernel": {"achieved": tf_attn, "unit": "TFLOP/s", "frac": tf_attn / tf_burst,
                                 "traffic": TRAFFIC["attention_c2"]},
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": tf_burst, "unit": "TFLOP/s",
                         "frac": tflops / tf_burst, "traffic": TRAFFIC["attention_c2"] + TRAFFIC["decode_xlayer"],
                         "peak_kind": "burst bf16"}}


def row_attention_debiased(xb: XLayerBench, hbm, tf_burst, reps=3) -> dict:
    """The C2 attention with the Jensen-bias correction of the history keys
    (kvc_attend_compressed_debiased), same inputs and FLOP count."""
    dev = xb.wl.K[0].device
    n_q = 3 * 1560
    Q = synth.queries(synth.SEED_BASE + 2, n_q, H, D, device=dev)
    Ks = synth.queries(synth.SEED_BASE + 12, n_q, H, D, device=dev)
    Vs = synth.queries(synth.SEED_BASE + 22, n_q, H, D, device=dev)
    O_ = torch.empty(n_q, H, D, dtype=torch.bfloat16, device=dev)
    l = xb.attn_layer
    ws = kvc.alloc_workspace(kvc.OP_ATTEND, xb.desc, xb.preds[l], n_q, device=dev)
    Kh, Vh = xb.keep
    call = lambda: kvc.kvc_attend_compressed_debiased(xb.desc, xb.preds[l], Q, xb.codes[l], Kh, Vh, Ks, Vs,
                                                      D ** -0.5, O_, ws)
    call()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for s_, e_ in ev:
        s_.record()
        call()
        e_.record()
    synced_ok()
    ms = statistics.median(time_events(ev))
    total = 4 * n_q * (T_TOK + n_q) * H * D + XLayerBench.layer_flops()
    tflops = total / (ms * 1e-3) / 1e12
    return {"workload": "as c2_attention, with the Jensen-bias correction of the 32760 history keys",
            "ms": ms, "value": tflops, "unit": "TFLOP/s (attention + one decode of the history)",
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": tf_burst, "unit": "TFLOP/s",
                         "frac": tflops / tf_burst, "traffic": None, "peak_kind": "burst bf16"}}


def row_eden2(dev, hbm, reps=3) -> dict:
    """One predicted Wan-shaped layer (32760 tokens x 12 heads x 128, rank 64)
    coded with the H64 / EDEN-2 residual codec: encode and decode."""
    wl = synth.wan_xlayer(seed=synth.SEED_BASE + 1, device=dev, L=2, T=T_TOK, H=H, D=D, rank=RANK,
                          layers_needed=[1])
    cb = synth.eden2_codebook().to(dev)
    bf, hf = torch.bfloat16, torch.float16
    desc = kvc.make_desc(T_TOK, H, D, bf, 2, 64, hf, residual_codec=kvc.RESIDUAL_H64_EDEN2)
    pred = kvc.make_predictor(kvc.PRED_XLAYER_DPLR, wl.weights[1], rank=RANK, residual_codebook=cb)
    buf = kvc.alloc_codes(desc, pred, dev)
    Kr, Vr = torch.empty_like(wl.K[1]), torch.empty_like(wl.V[1])
    wse = kvc.alloc_workspace(kvc.OP_ENCODE, desc, pred, device=dev)
    wsd = kvc.alloc_workspace(kvc.OP_DECODE, desc, pred, device=dev)
    enc = lambda: kvc.kvc_encode_layer(desc, pred, wl.K[1], wl.V[1], wl.K[0], wl.V[0], buf, Kr, Vr, wse)
    dec = lambda: kvc.kvc_decode_layer(desc, pred, buf, wl.K[0], wl.V[0], Kr, Vr, wsd)
    out = {"workload": "cross-layer layer, 32760 tokens x 12 heads x 128, rank 64, H64 / EDEN-2 residuals "
                       "(4-bit index per pair, fp16 scale per 64 values)"}
    C = H * D
    w = sum(t.numel() * t.element_size() for t in wl.weights[1].values())
    for name, fn, nio in (("encode", enc, 3), ("decode", dec, 2)):
        fn()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for s_, e_ in ev:
            s_.record()
            fn()
            e_.record()
        synced_ok()
        ms = statistics.median(time_events(ev))
        byts = 2 * T_TOK * C * 2 * nio + kvc.kvc_codes_bytes(desc, pred) + w
        gbs = byts / (ms * 1e-3) / 1e9
        out[name] = {"ms": ms, "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                                            "frac": gbs / hbm, "traffic": TRAFFIC.get("eden2_" + name)}}
    return out


def row_temporal(dev, hbm, reps=3) -> dict:
    tw = synth.temporal_layer(seed=synth.SEED_BASE + 3, device=dev)
    T, Hh, Dd = tw.K.shape
    desc = kvc.make_desc(T, Hh, Dd, torch.bfloat16, 4, 64, torch.float16, tw.frame_tokens, 4)
    pred = kvc.make_predictor(kvc.PRED_TEMPORAL, {"k_block": tw.ak, "v_block": tw.av})
    buf = kvc.alloc_codes(desc, pred, dev)
    Kr, Vr = torch.empty_like(tw.K), torch.empty_like(tw.V)
    enc = lambda: kvc.kvc_encode_layer(desc, pred, tw.K, tw.V, None, None, buf, None, None)
    dec = lambda: kvc.kvc_decode_layer(desc, pred, buf, None, None, Kr, Vr)
    out = {}
    for name, fn in (("encode", enc), ("decode", dec)):
        fn()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for s, e in ev:
            s.record()
            fn()
            e.record()
        synced_ok()
        ms = statistics.median(time_events(ev))
        codes = kvc.kvc_codes_bytes(desc, pred)
        byts = 2 * T * Hh * Dd * 2 + codes + 2 * tw.ak.numel() * 2
        gbs = byts / (ms * 1e-3) / 1e9
        out[name] = {"ms": ms, "tokens_per_s": T / (ms * 1e-3),
                     "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                                  "traffic": TRAFFIC["temporal_" + name]}}
    out["workload"] = "temporal codec, one layer: 65536 tokens x 40 heads x 128, 1560-token frames, INT4 g64"
    return out


def row_cluster(dev, hbm, tf_burst, reps=3) -> dict:
    cw = synth.cluster_layer(seed=synth.SEED_BASE + 4, device=dev)
    T, Hh, Dd = cw.K.shape
    desc = kvc.make_desc(T, Hh, Dd, torch.bfloat16, 4, 32, torch.float16)
    w = dict(k_centroids=cw.k_centroids, k_enc=cw.k_enc, k_dec=cw.k_dec, v_centroids=cw.v_centroids,
             v_enc=cw.v_enc, v_dec=cw.v_dec)
    pred = kvc.make_predictor(kvc.PRED_CLUSTER, w, n_clusters=256, code_dim=128)
    buf = kvc.alloc_codes(desc, pred, dev)
    Kr, Vr = torch.empty_like(cw.K), torch.empty_like(cw.V)
    wse = kvc.alloc_workspace(kvc.OP_ENCODE, desc, pred, device=dev)
    wsd = kvc.alloc_workspace(kvc.OP_DECODE, desc, pred, device=dev)
    n_q = 1560
    Q = synth.queries(synth.SEED_BASE + 5, n_q, Hh, Dd, device=dev)
    O_ = torch.empty(n_q, Hh, Dd, dtype=torch.bfloat16, device=dev)
    wsa = kvc.alloc_workspace(kvc.OP_ATTEND, desc, pred, n_q, device=dev)
    calls = {"encode": lambda: kvc.kvc_encode_layer(desc, pred, cw.K, cw.V, None, None, buf, None, None, wse),
             "decode": lambda: kvc.kvc_decode_layer(desc, pred, buf, None, None, Kr, Vr, wsd),
             "attention": lambda: kvc.kvc_attend_compressed(desc, pred, Q, buf, None, None, None, None, Dd ** -0.5,
                                                            O_, wsa)}
    out = {"workload": "clustered codec, one layer: 32768 tokens x 16 heads x 128, 256 centres, 128 INT4 g32 "
                       "coefficients; mixed-dimensional attention of 1560 queries"}
    for name, fn in calls.items():
        fn()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for s, e in ev:
            s.record()
            fn()
            e.record()
        synced_ok()
        ms = statistics.median(time_events(ev))
        C = Hh * Dd
        if name == "attention":
            fl = 4 * n_q * T * Hh * 128
            tf = fl / (ms * 1e-3) / 1e12
            roof = {"bound": "tensor", "achieved": tf, "peak": tf_burst, "unit": "TFLOP/s", "frac": tf / tf_burst}
        elif name == "encode":
            # per token and tensor: distances to the 256 centres and the 128 coefficients
            # (the timed call asks for no reconstruction, so none is counted)
            fl = 2 * 2 * T * C * (256 + 128)
            tf = fl / (ms * 1e-3) / 1e12
            roof = {"bound": "tensor", "achieved": tf, "peak": tf_burst, "unit": "TFLOP/s", "frac": tf / tf_burst}
        else:
            byts = 2 * T * C * 2 + kvc.kvc_codes_bytes(desc, pred)
            gbs = byts / (ms * 1e-3) / 1e9
            roof = {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm}
        roof["traffic"] = {"attention": TRAFFIC["attention_c4"], "decode": TRAFFIC["decode_c4"]}.get(name)
        out[name] = {"ms": ms, "roofline": roof}
    return out


# ---------------------------------------------------------------- main


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-rows", action="store_true", help="skip the extra per-row measurements")
    ap.add_argument("--rows", default="c2,c2j,c3,c4,eden2",
                    help="which extra rows to measure (comma-separated)")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--layers", type=int, default=L_LAYERS,
                    help="layers of the cross-layer workload (the headline number uses all 30)")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the codec has no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    from clustered_kv_cache_b200 import build

    # one rank builds (if the in-tree library is stale); the others wait for it
    if rank == 0:
        build.build()
    if world > 1:
        torch.distributed.barrier()
    hbm, tf_burst, tf_sust, peak_kind = peaks()

    xb = XLayerBench(dev, shard_seed(rank), args.layers)
    L_RUN = args.layers
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        xb.step()
    torch.cuda.synchronize()
    assert kvc.kvc_get_device_error() == 0

    mk = lambda: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    ev_enc = [mk() for _ in range(args.steps)]  # around the fused call of layers 1 .. L-1
    ev_dec = [mk() for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    clocks = Clocks(vis.split(",")[local] if vis else local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    launches0 = kvc.kvc_launch_counter()
    t_start.record()
    for k in range(args.steps):
        xb.step(ev_enc[k], ev_dec[k])
    t_end.record()
    torch.cuda.synchronize()
    barrier()
    launches = kvc.kvc_launch_counter() - launches0
    clk = clocks.stop()
    assert kvc.kvc_get_device_error() == 0
    ms_total = max_over_ranks(t_start.elapsed_time(t_end), world, dev)
    ms_step = ms_total / args.steps
    value = job_value(ms_step, world, L_RUN)

    # the dominant launch: the fused call over the n_pred = L-1 predicted layers
    n_pred = max(L_RUN - 1, 1)
    enc_ms = statistics.mean(time_events(ev_enc)) if L_RUN >= 2 else float("nan")
    dec_ms = statistics.mean(time_events(ev_dec)) if L_RUN >= 2 else float("nan")
    enc_b, dec_b = n_pred * xb.layer_bytes(True), n_pred * xb.layer_bytes(False)
    enc_gbs, dec_gbs = enc_b / (enc_ms * 1e-3) / 1e9, dec_b / (dec_ms * 1e-3) / 1e9
    dom_enc = enc_ms >= dec_ms
    tkey = "encode_xlayer_fused" if dom_enc else "decode_xlayer_fused"
    roof = {"bound": "hbm", "achieved": enc_gbs if dom_enc else dec_gbs, "peak": hbm, "unit": "GB/s",
            "frac": (enc_gbs if dom_enc else dec_gbs) / hbm,
            "traffic": TRAFFIC[tkey] * n_pred if tkey in TRAFFIC else None,
            "kernel": f"kvc_encode_layers (cross-layer, {n_pred} layers in one launch)" if dom_enc else
                      f"kvc_decode_layers (cross-layer, {n_pred} layers in one launch)",
            "bytes_per_launch": enc_b if dom_enc else dec_b, "ms_per_launch": enc_ms if dom_enc else dec_ms,
            "peak_kind": peak_kind}
    flops = XLayerBench.layer_flops()
    detail = {"encode_layers": {"ms": enc_ms, "ms_per_layer": enc_ms / n_pred, "GB/s": enc_gbs,
                                "frac_hbm": enc_gbs / hbm, "bytes": enc_b,
                                "TFLOP/s": n_pred * flops / (enc_ms * 1e-3) / 1e12},
              "decode_layers": {"ms": dec_ms, "ms_per_layer": dec_ms / n_pred, "GB/s": dec_gbs,
                                "frac_hbm": dec_gbs / hbm, "bytes": dec_b,
                                "TFLOP/s": n_pred * flops / (dec_ms * 1e-3) / 1e12}}

    # end to end: inputs from pinned host memory, codes back to the host
    e2e = None
    if args.e2e_steps > 0:
        hK = [k.cpu().pin_memory() for k in xb.wl.K]
        hV = [v.cpu().pin_memory() for v in xb.wl.V]
        hcodes = [[torch.empty_like(t, device="cpu").pin_memory() for t in (c.k_codes, c.k_params, c.v_codes,
                                                                            c.v_params)] for c in xb.codes]
        bi = sum(t.numel() * t.element_size() for t in hK + hV)
        bo = sum(t.numel() * t.element_size() for c in hcodes for t in c)

        comp = torch.cuda.current_stream()
        h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(L_RUN)]    # layer l's inputs on the device
        ev_enc = [torch.cuda.Event() for _ in range(L_RUN)]   # layer l encoded (its inputs read, codes written)
        ev_out = [torch.cuda.Event() for _ in range(L_RUN)]   # layer l's codes on the host

        def e2e_step():
            # every byte moves through the library's C ABI: host inputs in, codes out.
            # Three streams, ordered per layer by events: the inputs of layer l+1
            # are copied in while layer l is encoded, and the codes of layer l are
            # copied out while the next layers run (copies in and out use the two
            # directions of the link at once).
            for l in range(L_RUN):
                h2d.wait_event(ev_enc[l])  # the previous step's encode of layer l has read its inputs
                kvc.kvc_copy_to_device(xb.wl.K[l], hK[l], h2d)
                kvc.kvc_copy_to_device(xb.wl.V[l], hV[l], h2d)
                ev_in[l].record(h2d)

            def before(l):
                comp.wait_event(ev_in[l])
                comp.wait_event(ev_out[l])  # the previous step's codes of layer l are out

            xb.encode_chain(before=before, after=lambda l: ev_enc[l].record(comp))
            for l, (c, hc) in enumerate(zip(xb.codes, hcodes)):
                d2h.wait_event(ev_enc[l])
                for src, dst in zip((c.k_codes, c.k_params, c.v_codes, c.v_params), hc):
                    kvc.kvc_copy_to_host(dst, src, d2h)
                ev_out[l].record(d2h)
            xb.decode_chain()
            comp.wait_stream(h2d)
            comp.wait_stream(d2h)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        h2d.wait_stream(comp)  # the timed copies start after the start event
        for _ in range(args.e2e_steps):
            e2e_step()
        e.record()
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(s.elapsed_time(e) / args.e2e_steps, world, dev)
        e2e = {"value": job_value(ms_e2e, world, L_RUN), "unit": UNIT, "h2d_bytes_per_step": bi,
               "d2h_bytes_per_step": bo, "ms_per_step": ms_e2e}
        del hK, hV, hcodes

    rows = None
    cpu = None
    if world == 1:
        want = set(args.rows.split(",")) if not args.no_rows else set()
        rows = {}
        if ("c2" in want or "c2j" in want) and L_RUN >= 2:
            xb.encode_chain(keep_layer=xb.attn_layer)
            torch.cuda.synchronize()
            if "c2" in want:
                rows["c2_attention"] = row_attention(xb, hbm, tf_burst, tf_sust)
            if "c2j" in want:
                rows["c2_attention_debiased"] = row_attention_debiased(xb, hbm, tf_burst)
            xb.keep = None
            torch.cuda.empty_cache()
        if "c3" in want:
            rows["c3_temporal"] = row_temporal(dev, hbm)
            torch.cuda.empty_cache()
        if "c4" in want:
            rows["c4_cluster"] = row_cluster(dev, hbm, tf_burst)
            torch.cuda.empty_cache()
        if "eden2" in want:
            rows["c1_eden2_layer"] = row_eden2(dev, hbm)
        rows = rows or None
        if not args.no_cpu:
            # about 25 s of host work: the single-threaded oracle, then its thread driver
            cpu = cpu_baseline_line(xb.wl, L_RUN)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded Wan-1.3B-shaped trace, inter-layer correlation 0.9; block-DPLR "
                        "predictors fitted by least squares on a separate 4096-token trace)",
                "config": {"workload": f"cross-layer codec: encode + decode of {L_RUN} layers x 32760 tokens x 12 "
                                       "heads x 128, bf16, INT2 g32 residual (INT4 anchor), block-DPLR rank 64",
                           "global_batch": T_TOK * world, "seq_len": T_TOK, "parallelism": f"dp{world}",
                           "l2": "inputs larger than L2 (6 GB per step streamed)"},
                "roofline": roof, "layers": detail, "clocks": clk, "gpu_launches": launches,
                "e2e": e2e, "cpu_baseline": cpu, "rows": rows}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
