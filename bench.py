#!/usr/bin/env python
"""Benchmark: TurboQuant_prod prefill encode of a KV-cache key batch plus decode scoring.

One step = the hot path over one batch:
  1. tq_quantize_prod of keys [1 batch, 32 heads, 32768 tokens, d=128] bf16
     (b = 3: 2-bit Lloyd-Max codes + 1-bit QJL, randomized Hadamard rotation, S bf16);
  2. tq_score of one bf16 decode query per head against that head's 32768 compressed keys.
Metric: quantize Mvec/s & score Gkeys/s (d=128, b=3); value = vectors that went through
the whole step per second over all ranks, in Mvec/s. Per-kernel rates and the HBM
roofline of the dominant kernel (the encoder) are reported beside it.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tq|reference]
For N > 1 launch with torchrun (one rank per GPU); each rank quantizes its own batch
(weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "quantize Mvec/s & score Gkeys/s (d=128, b=3); % of HBM roofline"
HEADS, TOKENS, D, BITS = 32, 32768, 128, 3
N_VEC = HEADS * TOKENS
# Algorithmic bytes per vector of the encoder: 256 B bf16 in; 32 B codes + 16 B QJL +
# 4 B norm + 4 B residual norm out.
ENC_BYTES_PER_VEC = 2 * D + (BITS - 1) * D // 8 + D // 8 + 8
# Per key of the scorer: 32 B codes + 16 B QJL + 8 B norms in, 4 B score out.
SCORE_BYTES_PER_KEY = (BITS - 1) * D // 8 + D // 8 + 8 + 4
WORKLOAD = "turboquant_prod b=3 RHT prefill encode of KV keys [1,32,32768,128] bf16 + one decode query per head scored"


def rank_seed(rank: int) -> int:
    """Each rank quantizes its own batch (weak scaling): a distinct data seed per rank."""
    return synth.SEED_DATA + 100 * rank


def max_over_ranks(values, dist, device):
    """Element-wise max of per-rank timings (the slowest rank sets the job's time)."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_rate(units_per_rank: int, world: int, ms: float) -> float:
    """Units processed by all ranks per second, in millions."""
    return units_per_rank * world / (ms / 1e3) / 1e6


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def tensor_peak():
    """Measured dense bf16 peak (burst: the kernels are timed alone)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"])
    return 1590.0


def stored_traffic(kernel_key: str):
    """Per-launch DRAM bytes of one kernel from the committed ncu figures (profiles/traffic.json),
    used only while the kernel's source file hashes to the captured source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        import hashlib
        with open(p) as f:
            entry = json.load(f).get(kernel_key)
        if not entry:
            return None
        src = os.path.join(ROOT, entry["source"])
        if hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != entry["source_sha"]:
            return None
        return float(entry["dram_bytes_per_launch"])
    except Exception:
        return None


def time_on_stream(torch, fn, stream, dev, reps: int, warmup: int) -> float:
    """Mean milliseconds of fn() over `reps` back-to-back calls, CUDA events on `stream`."""
    for _ in range(max(3, warmup)):
        fn()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    return e0.elapsed_time(e1) / reps


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                self.out = ""

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            f = [s.strip() for s in line.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[0]))
                mx = max(mx, float(f[1]))
            except ValueError:
                continue
            for nm, v in zip(names, f[3:7]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# Decode attention over a compressed cache (32 heads x 131072 tokens, d = 128): keys prod
# b=4 (48 B codes + 16 B QJL + 8 B norms), values mse b=4 (64 B codes + 4 B norm).
DEC_H, DEC_T = 32, 131072
DEC_BYTES_PER_TOKEN = (48 + 16 + 8) + (64 + 4)


def measure_decode(tq, torch, dev, stream, steps: int, warmup: int, peak: float):
    """Time tq_attend_decode on the decode-step workload (seeded synthetic cache, built on the GPU)."""
    d = D
    ks = tq.State(d, 4, tq.PROD, tq.ROT_DENSE, tq.F32, device=dev.index, gauss_pi=synth.gaussian_matrix(d, 0),
                  s=synth.gaussian_matrix(d, synth.SEED_S))
    vs = tq.State(d, 4, tq.MSE, tq.ROT_DENSE, tq.F32, device=dev.index, gauss_pi=synth.gaussian_matrix(d, 0))
    n = DEC_H * DEC_T
    kc, kz, kn, kr = ks.empty_planes(n, dev)
    vc, _, vn, _ = vs.empty_planes(n, dev)
    g = torch.Generator(device=dev)
    g.manual_seed(12345)
    for h in range(DEC_H):
        sl = slice(h * DEC_T, (h + 1) * DEC_T)
        k = torch.randn(DEC_T, d, generator=g, device=dev)
        v = torch.randn(DEC_T, d, generator=g, device=dev)
        k /= k.norm(dim=1, keepdim=True)
        v /= v.norm(dim=1, keepdim=True)
        tq.quantize_prod(ks, k, kc[sl], kz[sl], kn[sl], kr[sl], stream=stream)
        tq.quantize_mse(vs, v, vc[sl], vn[sl], stream=stream)
    q = torch.randn(DEC_H, d, generator=g, device=dev).to(torch.bfloat16)
    out = torch.empty((DEC_H, d), dtype=torch.float32, device=dev)
    ws = torch.empty(tq.attend_workspace(ks, vs, DEC_H, DEC_T), dtype=torch.uint8, device=dev)
    scale = 1.0 / d ** 0.5

    def run():
        tq.attend_decode(ks, vs, q, kc, kz, kn, kr, vc, vn, scale, out, ws, H=DEC_H, T=DEC_T, stream=stream)

    for _ in range(max(3, warmup)):
        run()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        run()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    gbs = DEC_BYTES_PER_TOKEN * n / (ms / 1e3) / 1e9
    ks.close()
    vs.close()
    return {"workload": "decode attention, 32 heads x 131072 tokens, d=128, K prod b=4, V mse b=4, one bf16 "
                        "query per head", "ms": ms, "gkeys_s": n / (ms / 1e3) / 1e9,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "algorithmic_bytes_per_launch": DEC_BYTES_PER_TOKEN * n},
            "gpu_launches_per_step": 3}


# Streaming decode step: 32 query heads sharing 8 KV heads (G = 4), a cache of 131,072 tokens
# per KV head (K prod b=4, V mse b=4, dense Pi); each step encodes one new K and V token per
# KV head into the cache and attends over every token (tq_attend_append_decode).
STR_H, STR_G, STR_T = 32, 4, 131072


def measure_streaming(tq, torch, dev, stream, steps: int, warmup: int, peak: float):
    """Time tq_attend_append_decode: the per-token append + decode step of a growing cache."""
    d = D
    hkv = STR_H // STR_G
    ks = tq.State(d, 4, tq.PROD, tq.ROT_DENSE, tq.F32, device=dev.index, gauss_pi=synth.gaussian_matrix(d, 0),
                  s=synth.gaussian_matrix(d, synth.SEED_S))
    vs = tq.State(d, 4, tq.MSE, tq.ROT_DENSE, tq.F32, device=dev.index, gauss_pi=synth.gaussian_matrix(d, 0))
    nstep = max(3, warmup) + steps
    t0 = STR_T - nstep   # the cache holds t0 tokens before the first step and STR_T after the last
    kc, kz, kn, kr = ks.empty_planes(hkv * STR_T, dev)
    vc, _, vn, _ = vs.empty_planes(hkv * STR_T, dev)
    g = torch.Generator(device=dev)
    g.manual_seed(54321)
    for h in range(hkv):
        sl = slice(h * STR_T, h * STR_T + t0)
        k = torch.randn(t0, d, generator=g, device=dev)
        v = torch.randn(t0, d, generator=g, device=dev)
        k /= k.norm(dim=1, keepdim=True)
        v /= v.norm(dim=1, keepdim=True)
        tq.quantize_prod(ks, k, kc[sl], kz[sl], kn[sl], kr[sl], stream=stream)
        tq.quantize_mse(vs, v, vc[sl], vn[sl], stream=stream)
    qs = torch.randn(nstep, STR_H, d, generator=g, device=dev).to(torch.bfloat16)
    knew = torch.randn(nstep, hkv, d, generator=g, device=dev).to(torch.bfloat16)
    vnew = torch.randn(nstep, hkv, d, generator=g, device=dev).to(torch.bfloat16)
    out = torch.empty((STR_H, d), dtype=torch.float32, device=dev)
    ws = torch.empty(tq.attend_workspace(ks, vs, STR_H, STR_T), dtype=torch.uint8, device=dev)
    scale = 1.0 / d ** 0.5

    def run(i):
        tq.attend_append_decode(ks, vs, qs[i], STR_G, knew[i], vnew[i], t0 + i, STR_T, kc, kz, kn, kr, vc, vn, scale,
                                out, ws, stream=stream)

    nw = max(3, warmup)
    for i in range(nw):
        run(i)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(nw, nstep):
        run(i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    tmean = t0 + nw + (steps + 1) / 2.0   # tokens attended per step, on average
    # the method must read every KV head's compressed cache once per step and write the new rows
    nbytes = hkv * tmean * DEC_BYTES_PER_TOKEN + hkv * (DEC_BYTES_PER_TOKEN + 2 * 2 * d) + STR_H * (2 + 4) * d
    gbs = nbytes / (ms / 1e3) / 1e9
    ks.close()
    vs.close()
    return {"workload": "streaming decode step: 32 query heads over 8 KV heads (GQA 4), 131,072-token cache, d=128, "
                        "K prod b=4, V mse b=4 (dense Pi); one new K/V token per KV head encoded into the cache, "
                        "then attention over every token", "ms": ms, "steps_per_s": 1e3 / ms,
            "head_tokens_gkeys_s": STR_H * tmean / (ms / 1e3) / 1e9,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "algorithmic_bytes_per_launch": nbytes},
            "gpu_launches_per_step": 3}


# Outlier-channel split of the same KV key batch: the 32 channels of largest mean square
# (over the first 32,768 keys) at prod b=3, the other 96 at prod b=2; each group rotated by
# its randomized Hadamard transform (orders 32 and 96 = 12 x 8), S stored bf16.
# Per vector: 256 B in; out 8 + 4 + 8 B (outer codes, QJL, norms) + 12 + 12 + 8 B (inner).
SPLIT_M, SPLIT_BO, SPLIT_BR = 32, 3, 2
SPLIT_BYTES_PER_VEC = 2 * D + (SPLIT_M * (SPLIT_BO - 1) // 8 + SPLIT_M // 8 + 8) + \
    ((D - SPLIT_M) * (SPLIT_BR - 1) // 8 + (D - SPLIT_M) // 8 + 8)


def measure_split(tq, torch, x, q, heads, dev, stream, steps: int, warmup: int, peak: float):
    """Time tq_split_quantize and tq_split_score on the prefill batch (x, q already on the device)."""
    nvec = x.shape[0]
    ms = torch.mean(x[:TOKENS].float() ** 2, dim=0)
    ch = np.sort(torch.argsort(ms, descending=True)[:SPLIT_M].cpu().numpy())
    so = tq.State(SPLIT_M, SPLIT_BO, tq.PROD, tq.ROT_RHT, tq.BF16, device=dev.index, seed_pi=20, seed_s=21)
    sr = tq.State(D - SPLIT_M, SPLIT_BR, tq.PROD, tq.ROT_RHT, tq.BF16, device=dev.index, seed_pi=22, seed_s=23)
    sp = tq.Split(so, sr, ch)
    po, pr = sp.empty_planes(nvec, dev)
    scores = torch.empty((heads, 1, TOKENS), dtype=torch.float32, device=dev)
    sws = torch.empty(max(1, tq.split_score_workspace(sp, tq.BF16, heads, 1)), dtype=torch.uint8, device=dev)

    def enc():
        tq.split_quantize(sp, x, po, pr, stream=stream)

    def sc():
        tq.split_score(sp, q, po, pr, scores, groups=heads, nq=1, n=TOKENS, stream=stream, workspace=sws)

    out = {}
    for name, fn in (("encode", enc), ("score", sc)):
        for _ in range(max(3, warmup)):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        out[name] = e0.elapsed_time(e1) / steps
    gbs = SPLIT_BYTES_PER_VEC * nvec / (out["encode"] / 1e3) / 1e9
    res = {"workload": f"outlier-channel split of the KV key batch: {SPLIT_M} channels at prod b={SPLIT_BO}, "
                       f"{D - SPLIT_M} at prod b={SPLIT_BR} (Hadamard Pi per group, S bf16), "
                       f"{SPLIT_M * SPLIT_BO + (D - SPLIT_M) * SPLIT_BR} bits per vector of codes",
           "effective_bits": (SPLIT_M * SPLIT_BO + (D - SPLIT_M) * SPLIT_BR) / D,
           "ms": out, "quantize_mvec_s": nvec / (out["encode"] / 1e3) / 1e6,
           "score_gkeys_s": nvec / (out["score"] / 1e3) / 1e9,
           "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                        "algorithmic_bytes_per_launch": SPLIT_BYTES_PER_VEC * nvec}}
    sp.close()
    so.close()
    sr.close()
    return res


# Prefix coding of b = 4 MSE codes (the V cache's width in the decode shape): 1,048,576 unit
# vectors, d = 128, RHT state; encode (lengths, scan, bit stream) and decode timed apart.
ENT_N = 1 << 20


def measure_entropy(tq, torch, dev, stream, steps: int, warmup: int):
    st = tq.State(D, 4, tq.MSE, tq.ROT_RHT, tq.F32, device=dev.index, signs=synth.rht_signs(D))
    g = torch.Generator(device=dev)
    g.manual_seed(777)
    x = torch.randn(ENT_N, D, generator=g, device=dev)
    x /= x.norm(dim=1, keepdim=True)
    codes, _, norms, _ = st.empty_planes(ENT_N, dev)
    tq.quantize_mse(st, x, codes, norms, stream=stream)
    offsets = torch.empty(ENT_N + 1, dtype=torch.int64, device=dev)
    sbuf = torch.empty(tq.entropy_max_bytes(st, ENT_N), dtype=torch.uint8, device=dev)
    ws = torch.empty(tq.entropy_workspace(st, ENT_N), dtype=torch.uint8, device=dev)
    back = torch.empty_like(codes)

    def enc():
        tq.entropy_encode(st, codes, offsets, sbuf, ws, cuda_stream=stream)

    def dec():
        tq.entropy_decode(st, sbuf, offsets, back, cuda_stream=stream)

    out = {}
    for name, fn in (("encode", enc), ("decode", dec)):
        for _ in range(max(2, min(warmup, 3))):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = max(2, min(steps, 10))
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        out[name] = e0.elapsed_time(e1) / reps
    total_bits = int(offsets[-1].item())
    _, _, mean = tq.entropy_table(st)
    ok = bool(torch.equal(back, codes))
    st.close()
    return {"workload": "prefix code of b=4 MSE codes: 1,048,576 unit vectors x 128 (Huffman of the Lemma-1 index "
                        "law, canonical)", "ms": out,
            "encode_mvec_s": ENT_N / (out["encode"] / 1e3) / 1e6, "decode_mvec_s": ENT_N / (out["decode"] / 1e3) / 1e6,
            "bits_per_coordinate": total_bits / (ENT_N * D), "law_mean_bits": mean,
            "saving_vs_fixed": 1 - total_bits / (ENT_N * D * 4), "round_trip_exact": ok}


# Embedding search (1,000,000 vectors, d = 1536, prod b = 2, dense Pi and S bf16, 1000 queries):
# algorithmic flops: encode 4 d^2 per vector (Pi x and S r); search 4 d per (query, key).
C5_N, C5_D, C5_NQ, C5_K = 1_000_000, 1536, 1000, 10


def measure_c5(tq, torch, dev, stream, steps: int, warmup: int, tflops_peak: float, n: int = None):
    """Time the tensor-core encode and the top-10 search on the embedding-search shape, with the
    dense Haar Pi and with the randomized Hadamard Pi (order 1536 = 12 x 128; S stays Gaussian).
    n: database size (default the full 1,000,000; a smaller n is for profiling captures)."""
    d = C5_D
    C5_N = globals()["C5_N"] if n is None else n
    g = torch.Generator(device=dev)
    g.manual_seed(4242)
    mu = torch.randn(256, d, generator=g, device=dev)
    mu /= mu.norm(dim=1, keepdim=True)
    lab = torch.randint(0, 256, (C5_N,), generator=g, device=dev)
    x = mu[lab] + 0.3 * torch.randn(C5_N, d, generator=g, device=dev) / d ** 0.5
    x = (x / x.norm(dim=1, keepdim=True)).to(torch.bfloat16)
    qlab = torch.randint(0, 256, (C5_NQ,), generator=g, device=dev)
    qv = mu[qlab] + 0.3 * torch.randn(C5_NQ, d, generator=g, device=dev) / d ** 0.5
    qv = (qv / qv.norm(dim=1, keepdim=True)).to(torch.bfloat16)
    idx = torch.empty((C5_NQ, C5_K), dtype=torch.int64, device=dev)
    vals = torch.empty((C5_NQ, C5_K), dtype=torch.float32, device=dev)
    res = {}
    for rot in (tq.ROT_DENSE, tq.ROT_RHT):
        if rot == tq.ROT_DENSE:
            st = tq.State(d, 2, tq.PROD, rot, tq.BF16, device=dev.index, gauss_pi=synth.gaussian_matrix(d, 0),
                          s=synth.gaussian_matrix(d, synth.SEED_S))
            enc_flops = 4.0 * d * d * C5_N          # Pi x and S r
        else:
            st = tq.State(d, 2, tq.PROD, rot, tq.BF16, device=dev.index, signs=synth.rht_signs(d),
                          s=synth.gaussian_matrix(d, synth.SEED_S))
            enc_flops = 2.0 * d * d * C5_N          # S r (the rotation is O(d log d) adds)
        codes, qjl, norms, rnorms = st.empty_planes(C5_N, dev)
        ws = torch.empty(tq.search_workspace(st, C5_NQ, C5_N, C5_K), dtype=torch.uint8, device=dev)
        ews = torch.empty(max(1, tq.quantize_workspace(st, C5_N, tq.BF16)), dtype=torch.uint8, device=dev)

        def enc():
            tq.quantize_prod(st, x, codes, qjl, norms, rnorms, stream=stream, workspace=ews)

        def srch():
            tq.search_topk(st, qv, codes, qjl, norms, rnorms, C5_K, idx, vals, ws, stream=stream)

        out = {}
        for name, fn, flops in (("encode", enc, enc_flops), ("search", srch, 4.0 * d * C5_NQ * C5_N)):
            for _ in range(max(2, min(warmup, 3))):
                fn()
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = max(2, min(steps, 20))   # a few hundred ms, so the clock record has samples
            with ClockSampler(dev.index) as clk:
                e0.record(stream)
                for _ in range(reps):
                    fn()
                e1.record(stream)
                torch.cuda.synchronize(dev)
            ms = e0.elapsed_time(e1) / reps
            tf = flops / (ms / 1e3) / 1e12
            out[name] = {"ms": ms, "reps": reps, "clocks": clk.summary(),
                         "roofline": {"bound": "tensor", "achieved": tf, "peak": tflops_peak, "unit": "TFLOP/s",
                                      "frac": tf / tflops_peak, "algorithmic_flops_per_launch": flops}}
        out["encode"]["mvec_s"] = C5_N / (out["encode"]["ms"] / 1e3) / 1e6
        st.close()
        res["dense" if rot == tq.ROT_DENSE else "rht"] = out
    res["dense"]["workload"] = (f"embedding search: {C5_N:,} x 1536 bf16 (Gaussian mixture, 256 centres), prod b=2, "
                                "dense Pi and S bf16 (tensor cores), 1000 queries, top-10")
    res["rht"]["workload"] = ("the same with Pi = H_1536 diag(eps) / sqrt(1536), H_1536 = H_12 (x) H_128 (CUDA cores), "
                              "S Gaussian bf16 (tensor cores)")
    return res


def host_threads():
    """(cores this process may run on, BLAS threads numpy uses)."""
    cores = len(os.sched_getaffinity(0))
    try:
        from threadpoolctl import threadpool_info
        blas = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        blas = cores
    return cores, blas


def oracle_sample(heads: int, seed: int, single_thread: bool = False):
    """The oracle (fp64 numpy) on `heads` heads of the workload; returns (vectors, seconds)."""
    from oracle import quantizer as OQ
    from oracle import rotation as OR
    eps = synth.rht_signs(D)
    S = OR.round_bf16(synth.gaussian_matrix(D, synth.SEED_S))
    Pi = OR.rht_matrix(eps)
    cb = OQ.make_codebook(D, BITS - 1)
    qv = synth.bf16_from_bits(synth.decode_queries(HEADS, D))
    data = [synth.bf16_from_bits(synth.kv_prefill_batch(HEADS, TOKENS, D, seed=seed, head_range=(h, h + 1))[0])
            for h in range(heads)]

    def work():
        t0 = time.perf_counter()
        for h in range(heads):
            codes, z, nu, rho, _, _ = OQ.encode_prod(data[h], Pi, S, cb)
            OQ.pack_bits(codes, BITS - 1)
            OQ.pack_bits(z, 1)
            xt = OQ.decode_prod(codes, z, nu, rho, Pi, S, cb)
            OQ.estimate(qv[h:h + 1], xt)
        return time.perf_counter() - t0

    if single_thread:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            return heads * TOKENS, work()
    return heads * TOKENS, work()


def oracle_c5_slice(nvec: int = 65536):
    """The oracle on a seeded slice of the embedding-search shape (d = 1536, prod b = 2, dense Pi
    and S bf16): encode + pack of `nvec` vectors, then the estimates of all 1000 queries against
    them and a top-10; the times extrapolate linearly to 10^6 vectors."""
    from oracle import attention as OA
    from oracle import quantizer as OQ
    from oracle import rotation as OR
    d = C5_D
    bits, _ = synth.mixture_vectors(nvec, d)
    qbits, _ = synth.mixture_vectors(C5_NQ, d, seed=synth.SEED_DATA + 9, centre_seed=synth.SEED_DATA)
    x, qv = synth.bf16_from_bits(bits), synth.bf16_from_bits(qbits)
    Pi = OR.round_bf16(OR.haar_from_gaussian(synth.gaussian_matrix(d, 0)))
    S = OR.round_bf16(synth.gaussian_matrix(d, synth.SEED_S))
    cb = OQ.make_codebook(d, 1)
    t0 = time.perf_counter()
    codes, z, nu, rho, _, _ = OQ.encode_prod(x, Pi, S, cb)
    OQ.pack_bits(codes, 1)
    OQ.pack_bits(z, 1)
    t1 = time.perf_counter()
    OA.topk(OQ.estimate(qv, OQ.decode_prod(codes, z, nu, rho, Pi, S, cb)), C5_K)
    t2 = time.perf_counter()
    scale = C5_N / nvec
    return {"sample": f"{nvec} of {C5_N} vectors x {d} (same recipe), all {C5_NQ} queries; times x {scale:.2f} "
                      f"to the full database (linear in the vectors)",
            "encode_s": t1 - t0, "search_s": t2 - t1, "encode_mvec_s": nvec / (t1 - t0) / 1e6,
            "search_s_extrapolated": (t2 - t1) * scale, "encode_s_extrapolated": (t1 - t0) * scale}


# Parity-size configuration: TurboQuant_mse b = 3, d = 128, 4096 unit vectors (fp32), dense
# Haar Pi; encode, decode, and 64 unit queries x 4096 estimates. It fits in L2, so only rates
# are reported.
C1_N, C1_NQ = 4096, 64


def measure_c1(tq, torch, dev, stream, steps: int, warmup: int):
    d = D
    st = tq.State(d, 3, tq.MSE, tq.ROT_DENSE, tq.F32, device=dev.index, gauss_pi=synth.gaussian_matrix(d, 0))
    x = torch.from_numpy(synth.unit_vectors(C1_N, d, seed=synth.SEED_DATA)).to(dev)
    q = torch.from_numpy(synth.unit_vectors(C1_NQ, d, seed=synth.SEED_DATA + 1)).to(dev)
    codes, _, norms, _ = st.empty_planes(C1_N, dev)
    xt = torch.empty_like(x)
    scores = torch.empty((1, C1_NQ, C1_N), dtype=torch.float32, device=dev)
    sws = torch.empty(max(1, tq.score_workspace(st, 1, C1_NQ)), dtype=torch.uint8, device=dev)
    reps = max(10, steps)
    ms = {
        "encode": time_on_stream(torch, lambda: tq.quantize_mse(st, x, codes, norms, stream=stream), stream, dev,
                                 reps, warmup),
        "decode": time_on_stream(torch, lambda: tq.dequant(st, codes, None, norms, None, xt, stream=stream), stream,
                                 dev, reps, warmup),
        "score": time_on_stream(torch, lambda: tq.score(st, q, codes, None, norms, None, scores, stream=stream,
                                                        workspace=sws), stream, dev, reps, warmup),
    }
    st.close()
    return {"workload": "turboquant_mse b=3, d=128, 4096 unit vectors fp32, dense Haar Pi: encode, decode, "
                        "64 queries x 4096 estimates (fits in L2: rates only, no roofline claim)",
            "ms": ms, "encode_mvec_s": C1_N / (ms["encode"] / 1e3) / 1e6,
            "decode_mvec_s": C1_N / (ms["decode"] / 1e3) / 1e6,
            "score_gpairs_s": C1_N * C1_NQ / (ms["score"] / 1e3) / 1e9}


# Distortion / bias sweep: 2^20 uniform unit vectors at d = 128 and 256, b = 1..4, MSE and
# prod (dense Haar Pi fp32, S fp32), 1024 unit queries; statistics reduced on the device.
C4_N, C4_NQ = 1 << 20, 1024


def measure_c4(tq, torch, dev, stream):
    import math
    rows = []
    for d in (128, 256):
        g = torch.Generator(device=dev)
        g.manual_seed(9000 + d)
        x = torch.randn(C4_N, d, generator=g, device=dev)
        x /= x.norm(dim=1, keepdim=True)
        q = torch.randn(C4_NQ, d, generator=g, device=dev)
        q /= q.norm(dim=1, keepdim=True)
        xt = torch.empty_like(x)
        sums = torch.zeros(6, dtype=torch.float64, device=dev)
        for mode in (tq.MSE, tq.PROD):
            for b in (1, 2, 3, 4):
                st = tq.State(d, b, mode, tq.ROT_DENSE, tq.F32, device=dev.index,
                              gauss_pi=synth.gaussian_matrix(d, 0), s=synth.gaussian_matrix(d, synth.SEED_S))
                codes, qjl, norms, rnorms = st.empty_planes(C4_N, dev)
                if mode == tq.MSE:
                    enc = lambda: tq.quantize_mse(st, x, codes, norms, stream=stream)  # noqa: E731
                else:
                    enc = lambda: tq.quantize_prod(st, x, codes, qjl, norms, rnorms, stream=stream)  # noqa: E731
                enc_ms = time_on_stream(torch, enc, stream, dev, 3, 1)
                dec = lambda: tq.dequant(st, codes, qjl, norms, rnorms, xt, stream=stream)  # noqa: E731
                dec_ms = time_on_stream(torch, dec, stream, dev, 3, 1)
                tq.ip_stats(x, xt, q, sums, device=dev.index, stream=stream)
                torch.cuda.synchronize(dev)
                s = sums.cpu().numpy()
                n_pairs = C4_N * C4_NQ
                mean_e = s[2] / n_pairs
                rows.append({"d": d, "b": b, "mode": "mse" if mode == tq.MSE else "prod",
                             "D_mse": s[0] / C4_N if mode == tq.MSE else None,
                             "D_mse_theory": st.dmse if mode == tq.MSE else None,
                             "lower_4^-b": 4.0 ** -b, "upper_sqrt3pi/2_4^-b": math.sqrt(3) * math.pi / 2 * 4.0 ** -b,
                             "D_prod": s[3] / n_pairs if mode == tq.PROD else None,
                             "slope": s[4] / s[5], "mean_ip_err": mean_e,
                             "sd_ip_err": math.sqrt(max(0.0, s[3] / n_pairs - mean_e ** 2)),
                             "encode_ms": enc_ms, "encode_mvec_s": C4_N / (enc_ms / 1e3) / 1e6,
                             "decode_ms": dec_ms, "decode_mvec_s": C4_N / (dec_ms / 1e3) / 1e6})
                st.close()
    return {"workload": "distortion / bias sweep: 2^20 uniform unit vectors, d=128 and 256, b=1..4, mse and prod, "
                        "dense Haar Pi, 1024 unit queries (statistics on the device)", "rows": rows}


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    heads = 4
    for _ in range(args.warmup):
        oracle_sample(heads, synth.SEED_DATA)
    times = []
    for _ in range(args.steps):
        _, dt = oracle_sample(heads, synth.SEED_DATA)
        times.append(dt)
    cores, blas = host_threads()
    tot = sum(times)
    value = heads * TOKENS * args.steps / tot / 1e6
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "Mvec/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample": f"{heads} of {HEADS} heads per step ({heads * TOKENS} vectors)"},
        "cpu_baseline": {"value": value, "unit": "Mvec/s", "cores": cores, "blas_threads": blas, "kind": "oracle",
                         "sample": f"{heads} heads x {TOKENS} tokens per step, fp64 numpy oracle"},
        "e2e": {"value": value, "unit": "Mvec/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--heads", type=int, default=HEADS, help="smaller batch for profiling runs")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode-attention measurement")
    ap.add_argument("--no-stream", action="store_true", help="skip the streaming append + decode measurement")
    ap.add_argument("--no-c5", action="store_true", help="skip the embedding-search measurement")
    ap.add_argument("--c5-keys", type=int, default=None, help="embedding database size (profiling runs)")
    ap.add_argument("--no-split", action="store_true", help="skip the outlier-channel split measurement")
    ap.add_argument("--no-entropy", action="store_true", help="skip the prefix-coding measurement")
    ap.add_argument("--no-c1", action="store_true", help="skip the parity-size configuration's rates")
    ap.add_argument("--no-c4", action="store_true", help="skip the distortion / bias sweep")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist
    import vector_quantization_tq_b200 as tq

    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    heads = args.heads
    nvec = heads * TOKENS

    # state: prod b=3, RHT signs (seed 0), S ~ N(0,1) stored bf16 (seed 1)
    st = tq.State(D, BITS, tq.PROD, tq.ROT_RHT, tq.BF16, device=local, signs=synth.rht_signs(D),
                  s=synth.gaussian_matrix(D, synth.SEED_S))
    # each rank its own batch (weak scaling)
    seed = rank_seed(rank)
    kbits = synth.kv_prefill_batch(HEADS, TOKENS, D, seed=seed, head_range=(0, heads)).reshape(nvec, D)
    qbits = synth.decode_queries(HEADS, D)[:heads]
    x = torch.from_numpy(kbits.view(np.int16)).to(dev).view(torch.bfloat16)
    q = torch.from_numpy(qbits.view(np.int16)).to(dev).view(torch.bfloat16)
    codes, qjl, norms, rnorms = st.empty_planes(nvec, dev)
    scores = torch.empty((heads, 1, TOKENS), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sws = torch.empty(max(1, tq.score_workspace(st, heads, 1)), dtype=torch.uint8, device=dev)
    assert tq.quantize_workspace(st, nvec, tq.BF16) == 0   # the d = 128 encoder is one pass

    def step():
        tq.quantize_prod(st, x, codes, qjl, norms, rnorms, stream=stream)
        tq.score(st, q, codes, qjl, norms, rnorms, scores, groups=heads, nq=1, n=TOKENS, stream=stream,
                 workspace=sws)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            tq.quantize_prod(st, x, codes, qjl, norms, rnorms, stream=stream)
            ev[i][1].record(stream)
            tq.score(st, q, codes, qjl, norms, rnorms, scores, groups=heads, nq=1, n=TOKENS, stream=stream,
                     workspace=sws)
            ev[i][2].record(stream)
        end.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    total_ms = start.elapsed_time(end)
    enc_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    sc_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    step_ms = total_ms / args.steps
    if world > 1:
        step_ms, enc_ms, sc_ms = max_over_ranks([step_ms, enc_ms, sc_ms], dist, dev)

    # end to end through the public API with host buffers (pinned), copies inside the timed region
    e2e = None
    if not args.no_e2e:
        hx = x.cpu().pin_memory()
        hq = q.cpu().pin_memory()
        hc = torch.empty(codes.shape, dtype=codes.dtype).pin_memory()
        hz = torch.empty(qjl.shape, dtype=qjl.dtype).pin_memory()
        hn = torch.empty(norms.shape, dtype=norms.dtype).pin_memory()
        hr = torch.empty(rnorms.shape, dtype=rnorms.dtype).pin_memory()
        hs = torch.empty(scores.shape, dtype=scores.dtype).pin_memory()
        dx = torch.empty_like(x)
        dq = torch.empty_like(q)
        # The batch goes through in groups of heads so that the copies overlap the kernels:
        # group g's inputs come in on `cin` while group g-1 is encoded and scored on `stream`
        # and group g-2's planes and scores go out on `cout` (the two copy directions run on
        # separate copy engines).
        cin, cout = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        hg = 4 if heads % 4 == 0 else 1
        groups_e2e = [(h0, h0 + hg) for h0 in range(0, heads, hg)]
        ev_in = [torch.cuda.Event() for _ in groups_e2e]
        ev_k = [torch.cuda.Event() for _ in groups_e2e]

        def e2e_step():
            cin.wait_stream(stream)    # the previous step's kernels are done with dx / dq
            for g, (h0, h1) in enumerate(groups_e2e):
                r0, r1 = h0 * TOKENS, h1 * TOKENS
                with torch.cuda.stream(cin):
                    dx[r0:r1].copy_(hx[r0:r1], non_blocking=True)
                    dq[h0:h1].copy_(hq[h0:h1], non_blocking=True)
                    ev_in[g].record(cin)
                stream.wait_event(ev_in[g])
                tq.quantize_prod(st, dx[r0:r1], codes[r0:r1], qjl[r0:r1], norms[r0:r1], rnorms[r0:r1],
                                 stream=stream)
                tq.score(st, dq[h0:h1], codes[r0:r1], qjl[r0:r1], norms[r0:r1], rnorms[r0:r1], scores[h0:h1],
                         groups=h1 - h0, nq=1, n=TOKENS, stream=stream, workspace=sws)
                ev_k[g].record(stream)
                cout.wait_event(ev_k[g])
                with torch.cuda.stream(cout):
                    hc[r0:r1].copy_(codes[r0:r1], non_blocking=True)
                    hz[r0:r1].copy_(qjl[r0:r1], non_blocking=True)
                    hn[r0:r1].copy_(norms[r0:r1], non_blocking=True)
                    hr[r0:r1].copy_(rnorms[r0:r1], non_blocking=True)
                    hs[h0:h1].copy_(scores[h0:h1], non_blocking=True)
            stream.wait_stream(cout)   # the step ends when its results are on the host

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        ne2e = max(3, args.steps // 2)
        for _ in range(ne2e):
            e2e_step()
        s1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = s0.elapsed_time(s1) / ne2e
        if world > 1:
            e2e_ms = max_over_ranks([e2e_ms], dist, dev)[0]
        h2d = hx.numel() * hx.element_size() + hq.numel() * hq.element_size()
        d2h = sum(t.numel() * t.element_size() for t in (hc, hz, hn, hr, hs))
        e2e = {"value": job_rate(nvec, world, e2e_ms), "unit": "Mvec/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cores, blas = host_threads()
        n_s, dt = oracle_sample(8, seed)
        n1, dt1 = oracle_sample(1, seed, single_thread=True)
        cpu = {"value": n_s / dt / 1e6, "unit": "Mvec/s", "cores": cores, "blas_threads": blas, "kind": "oracle",
               "sample": f"8 of 32 heads ({n_s} vectors) of the same batch: fp64 numpy encode + pack + decode + "
                         f"estimate, {dt:.2f} s wall, numpy/BLAS on {blas} threads",
               "single_thread": {"value": n1 / dt1 / 1e6, "unit": "Mvec/s", "cores": 1,
                                 "sample": f"1 head ({n1} vectors), BLAS limited to 1 thread, {dt1:.2f} s wall"}}
        if not args.no_c5:
            cpu["embedding_search_slice"] = oracle_c5_slice()

    peak, peak_kind = measured_peaks()
    decode = None
    if not args.no_decode:
        decode = measure_decode(tq, torch, dev, stream, args.steps, args.warmup, peak)
    streaming = None
    if not args.no_stream:
        streaming = measure_streaming(tq, torch, dev, stream, args.steps, args.warmup, peak)
    split = None
    if not args.no_split:
        split = measure_split(tq, torch, x, q, heads, dev, stream, args.steps, args.warmup, peak)
    ent = None
    if not args.no_entropy:
        ent = measure_entropy(tq, torch, dev, stream, args.steps, args.warmup)
    c5 = None
    if not args.no_c5:
        c5 = measure_c5(tq, torch, dev, stream, args.steps, args.warmup, tensor_peak(), n=args.c5_keys)
    c1 = None if args.no_c1 else measure_c1(tq, torch, dev, stream, args.steps, args.warmup)
    c4 = None if args.no_c4 else measure_c4(tq, torch, dev, stream)
    enc_gbs = ENC_BYTES_PER_VEC * nvec / (enc_ms / 1e3) / 1e9
    sc_gbs = SCORE_BYTES_PER_KEY * nvec / (sc_ms / 1e3) / 1e9
    traffic = stored_traffic("encode_prod_d128")
    line = {
        "metric": METRIC,
        "value": job_rate(nvec, world, step_ms),
        "unit": "Mvec/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(3, args.warmup),
        "ms_per_step": step_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "vectors_per_rank": nvec, "heads": heads, "tokens": TOKENS, "d": D,
                   "b": BITS, "mode": "prod", "rotation": "rht", "matrix_dtype": "bf16",
                   "l2": "inputs larger than L2 (256 MiB of bf16 keys per step per rank)",
                   "parallelism": f"dp{world} (independent batches)"},
        "quantize_mvec_s": nvec * world / (enc_ms / 1e3) / 1e6,
        "score_gkeys_s": nvec * world / (sc_ms / 1e3) / 1e9,
        "kernels_ms": {"encode": enc_ms, "score": sc_ms},
        "roofline": {"bound": "hbm", "achieved": enc_gbs, "peak": peak, "unit": "GB/s", "frac": enc_gbs / peak,
                     "traffic": traffic, "kernel": "encode (tq_quantize_prod)",
                     "algorithmic_bytes_per_launch": ENC_BYTES_PER_VEC * nvec, "peak_kind": peak_kind},
        "score_roofline": {"bound": "hbm", "achieved": sc_gbs, "peak": peak, "unit": "GB/s", "frac": sc_gbs / peak},
        "gpu_launches": 3 * args.steps,   # encoder; query tables + scorer
        "clocks": clk.summary(),
        "e2e": e2e,
        "decode_attention": decode,
        "streaming_step": streaming,
        "embedding_search": c5,
        "outlier_split": split,
        "prefix_code": ent,
        "parity_config": c1,
        "distortion_sweep": c4,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    st.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
