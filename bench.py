#!/usr/bin/env python
"""Benchmark of the GIFT whitened-FP8 gradient codec on B200.

Workload (one step): the Llama-600M-sized stand-in stack of 24 layers x
{qkv 1536->4608, o 1536->1536, up 1536->4096, down 4096->1536} bf16
gradients (528.5 M elements, 1.06 GB).  Selective deployment: o and down
are whitened at rank 32, qkv and up take the Euclidean per-block E4M3
codec.  A step runs the whole per-step hot path of the paper:
  * every K_REFRESH = 50 steps (section V.E, Algorithm 1), the factor
    refresh of all 48 whitened layers (A = X^T X / N on 8192 tokens each,
    subspace iteration, Rayleigh-Ritz) in one batched call; timed steps
    0, 50, 100, ... carry it, so the default 50 timed steps hold exactly one;
  * encode of all 96 gradients, then decode of all 96;
  * the one-step round-trip error of one whitened layer.
value = gradient bytes of the stack / step time (GB/s).

Multi-GPU (`--gpus N` under torchrun): replicas only -- the codec has no
exchange step, so every rank runs its own copy of the stack (weak scaling);
the timed region is bracketed by barriers and the reported time is the max
over ranks.

`--impl reference` times the CPU oracle (oracle/gift_oracle.py) on a
bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "whitened FP8 encode+decode GB/s of gradient and % of B200 HBM roofline"
UNIT = "GB/s"
WORKLOAD = ("llama600m-standin stack: 24 x {qkv 4608x1536, o 1536x1536, up 4096x1536, down 1536x4096} "
            "bf16 gradients; o/down whitened rank 32 (refresh N=8192), qkv/up Euclidean; E4M3 block 128")
REFRESH_N = 8192
RANK, OVERSAMPLE, ITERS = 32, 16, 4
K_REFRESH = 50
HBM_FALLBACK = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10 * K_REFRESH)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="gift", choices=["gift", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-nvfp4", action="store_true", help="skip the NVFP4 measurement on the 11008x4096 gradient")
    ap.add_argument("--no-layers", action="store_true", help="skip the single-layer codec measurements")
    ap.add_argument("--no-staleness", action="store_true", help="skip the factor-staleness sweep")
    ap.add_argument("--depth", type=int, default=24, help="layers in the stack (24 = the full stand-in)")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", HBM_FALLBACK), "measured"
    return HBM_FALLBACK, "fallback"


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            # the timed region starts once the sampler has written its first sample
            t_end = time.time() + 3.0
            while time.time() < t_end and os.path.getsize(self.path) == 0:
                time.sleep(0.01)
        except Exception:
            self.proc = None

    def stop(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": []}
        if self.proc is None:
            return out
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if sm:
            out = {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                   "samples": len(sm)}
        return out


# ---------------------------------------------------------------------------
# rank plumbing (replicas only: the one collective is the timing reduction)
# ---------------------------------------------------------------------------
def max_over_ranks(ms: float, device=None) -> float:
    """Max of a per-rank device time over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, bytes_per_rank: float, ms_per_step: float) -> float:
    """Whole-job throughput in GB/s: every rank processes its own replica (weak scaling)."""
    return world * bytes_per_rank / (ms_per_step * 1e-3) / 1e9


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def build_workload(torch, ops, synth, dev, depth, seed):
    """Device-resident stack: G, codes, scales, G_hat in single buffers; per whitened layer X and factors."""
    shapes = synth.stack_shapes(depth)
    n_el = sum(d_out * d_in for _, _, d_out, d_in, _ in shapes)
    G_all = torch.empty((n_el,), device=dev, dtype=torch.bfloat16)
    Gh_all = torch.empty((n_el,), device=dev, dtype=torch.bfloat16)
    C_all = torch.empty((n_el,), device=dev, dtype=torch.uint8)
    S_all = torch.empty((n_el // 128,), device=dev, dtype=torch.float32)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    Qs = {}
    for d in (1536, 4096):
        Qs[d] = torch.from_numpy(synth.haar_orthogonal(d, 3000 + d).astype(np.float32)).to(dev)
    layers, whitened = [], []
    off = 0
    for (l, name, d_out, d_in, wh) in shapes:
        n = d_out * d_in
        G = G_all[off:off + n].view(d_out, d_in)
        G.copy_(synth.device_gradient(d_out, d_in, 1.0, Qs[d_in], gen, torch.bfloat16))
        L = ops.LayerArgs(d_out=d_out, d_in=d_in, rank=RANK if wh else 0, dtype=torch.bfloat16, G=G,
                          G_hat=Gh_all[off:off + n].view(d_out, d_in), codes=C_all[off:off + n].view(d_out, d_in),
                          scales=S_all[off // 128:(off + n) // 128].view(d_out, d_in // 128))
        if wh:
            sigma = torch.arange(1, d_in + 1, device=dev, dtype=torch.float32) ** -1.0
            X = synth.device_activations(REFRESH_N, sigma, Qs[d_in], gen, torch.bfloat16)
            L.U = torch.empty((d_in, RANK), device=dev, dtype=torch.float32)
            L.lam = torch.empty((RANK,), device=dev, dtype=torch.float32)
            L.rho = torch.empty((1,), device=dev, dtype=torch.float32)
            ws = torch.empty((ops.refresh_workspace_size(REFRESH_N, d_in, RANK, OVERSAMPLE),), device=dev,
                             dtype=torch.uint8)
            st = torch.zeros((1,), device=dev, dtype=torch.int32)
            whitened.append(dict(layer=L, X=X, ws=ws, st=st, seed=7000 + len(whitened)))
        layers.append(L)
        off += n
    ews = torch.empty((max(ops.error_workspace_size(4096, 4096), 16),), device=dev, dtype=torch.uint8)
    err = torch.empty((3,), device=dev, dtype=torch.float64)
    wl = [L for L in layers if L.rank > 0]
    el = [L for L in layers if L.rank == 0]
    jobs = ops.make_refresh_jobs([(w["X"], w["layer"].U, w["layer"].lam, w["layer"].rho, w["ws"], w["st"],
                                   w["seed"], None) for w in whitened])
    W = dict(layers=layers, whitened=whitened, G_all=G_all, Gh_all=Gh_all, C_all=C_all, S_all=S_all,
                n_el=n_el, ews=ews, err=err, jobs=jobs,
                n_wh=sum(L.d_out * L.d_in for L in wl), n_eu=sum(L.d_out * L.d_in for L in el),
                packed_wh=ops.make_layers(wl), n_packed_wh=len(wl),
                packed_eu=ops.make_layers(el), n_packed_eu=len(el))
    W["sets"] = [dict(packed_wh=W["packed_wh"], packed_eu=W["packed_eu"],
                      err_pairs=[(w["layer"].G, w["layer"].G_hat) for w in whitened], G_all=G_all, Gh_all=Gh_all,
                      err=err)]
    return W


def nvfp4_measure(torch, ops, synth, dev, peak, reps=20):
    """NVFP4 codec on one 11008 x 4096 bf16 gradient (an MLP projection of the
    stand-in model's larger sibling), whitened with a rank-32 factor refreshed
    from 8192 tokens, and the Euclidean NVFP4 codec on the same tensor.
    Algorithmic bytes per element and direction: 2 + 0.5 + 1/16 = 2.5625."""
    d_out, d_in = 11008, 4096
    gen = torch.Generator(device=dev)
    gen.manual_seed(5005)
    Q = torch.from_numpy(synth.haar_orthogonal(d_in, 5003).astype(np.float32)).to(dev)
    G = synth.device_gradient(d_out, d_in, 1.0, Q, gen, torch.bfloat16)
    sigma = torch.arange(1, d_in + 1, device=dev, dtype=torch.float32) ** -1.0
    X = synth.device_activations(REFRESH_N, sigma, Q, gen, torch.bfloat16)
    U, lam, rho, _ = ops.factor_refresh(X, RANK, OVERSAMPLE, ITERS, seed=5004)
    del X
    codes = torch.empty((d_out, d_in // 2), device=dev, dtype=torch.uint8)
    sb = torch.empty((d_out, d_in // 16), device=dev, dtype=torch.uint8)
    ts = torch.empty((1,), device=dev, dtype=torch.float32)
    Gh = torch.empty_like(G)
    flush = torch.empty((256 << 20,), device=dev, dtype=torch.uint8)  # > L2 between timed calls
    err = torch.empty((3,), device=dev, dtype=torch.float64)
    ews = torch.empty((ops.error_workspace_size(d_out, d_in),), device=dev, dtype=torch.uint8)

    def timed(fn):
        ts_ms = []
        for i in range(reps + 3):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if i >= 3:
                ts_ms.append(a.elapsed_time(b))
        return float(np.median(ts_ms))

    out = {"workload": f"G {d_out}x{d_in} bf16, rank {RANK} factor from X {REFRESH_N}x{d_in}; "
                       "median of 20 calls, L2 flushed between calls",
           "bytes_per_element_each_way": 2.5625}
    n = d_out * d_in
    for name, args in (("whitened", (U, lam, rho)), ("euclid", (None, None, None))):
        enc = timed(lambda: ops.encode_nvfp4(G, *args, codes=codes, block_scales=sb, tensor_scale=ts))
        dec = timed(lambda: ops.decode_nvfp4(codes, sb, ts, *args, out=Gh))
        ops.roundtrip_error(G, Gh, out=err, ws=ews)
        gbs = 2 * n / ((enc + dec) * 1e-3) / 1e9
        out[name] = {"encode_ms": enc, "decode_ms": dec, "gradient_gbs": gbs,
                     "roofline_frac": 2 * 2.5625 * n / ((enc + dec) * 1e-3) / 1e9 / peak,
                     "roundtrip_rel_error": float(err[0].item())}
    return out


def layers_measure(torch, ops, synth, dev, peak, reps=20):
    """The whitened E4M3 codec called on one layer at a time (gift_encode then
    gift_decode, G_hat in G's dtype), for the single-layer shapes: 512 x 512
    fp32 (factor from 2048 fp32 tokens, G exponent 0.8), the 4096 x 1536 bf16
    MLP up-projection stand-in and the largest shape, 11008 x 4096 bf16 (both
    from 8192 bf16 tokens, exponent 1.0). One layer has d_out / 128 panels, so
    a single call fills at most that many of the 148 SMs.
    Algorithmic bytes per element each way: bytes(G) + 1 + 4/128."""
    flush = torch.empty((256 << 20,), device=dev, dtype=torch.uint8)  # > L2 between timed calls

    def timed(fn):
        ts_ms = []
        for i in range(reps + 3):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if i >= 3:
                ts_ms.append(a.elapsed_time(b))
        return float(np.median(ts_ms))

    out = {"workload": "one layer per call, rank-32 factor refreshed once (untimed); "
                       "median of 20 calls, L2 flushed between calls"}
    specs = (("512x512_f32", 512, 512, torch.float32, 2048, 0.8, 6001),
             ("4096x1536_bf16", 4096, 1536, torch.bfloat16, REFRESH_N, 1.0, 6002),
             ("11008x4096_bf16", 11008, 4096, torch.bfloat16, REFRESH_N, 1.0, 6003))
    for name, d_out, d_in, dt, n_tok, expo, seed in specs:
        gen = torch.Generator(device=dev)
        gen.manual_seed(seed)
        Q = torch.from_numpy(synth.haar_orthogonal(d_in, seed + 10).astype(np.float32)).to(dev)
        G = synth.device_gradient(d_out, d_in, expo, Q, gen, dt)
        sigma = torch.arange(1, d_in + 1, device=dev, dtype=torch.float32) ** -1.0
        X = synth.device_activations(n_tok, sigma, Q, gen, dt)
        U, lam, rho, _ = ops.factor_refresh(X, RANK, OVERSAMPLE, ITERS, seed=seed + 20)
        del X
        codes = torch.empty((d_out, d_in), device=dev, dtype=torch.uint8)
        scales = torch.empty((d_out, d_in // 128), device=dev, dtype=torch.float32)
        Gh = torch.empty_like(G)
        enc = timed(lambda: ops.encode(G, U, lam, rho, codes=codes, scales=scales))
        dec = timed(lambda: ops.decode(codes, scales, U, lam, rho, out=Gh))
        n = d_out * d_in
        gb = G.element_size()
        t = (enc + dec) * 1e-3
        out[name] = {"encode_ms": enc, "decode_ms": dec, "gradient_gbs": gb * n / t / 1e9,
                     "elements_per_s": n / t, "panels": (d_out + 127) // 128,
                     "roofline_frac": 2 * (gb + 1 + 4 / 128) * n / t / 1e9 / peak}
        del G, Gh, codes, scales
    del flush
    torch.cuda.empty_cache()
    return out


def staleness_measure(torch, dev):
    """The falsifier of the review page ("What would settle it"): the FP8
    round-trip error of GIFT, with its factor refreshed every K steps, against
    the Euclidean codec as a function of the steps since the last refresh, for
    K in {10, 25, 50, 100} (referee report, section V.E / Algorithm 1).  One
    1536 x 1536 bf16 layer (the stack's o-projection), 4096 tokens a step, 100
    steps of activations whose basis turns by exp(theta S) a step (slow and
    fast drift); errors in the Frobenius norm and in the coordinates whitened
    by the step's fresh factor.  Every refresh, codec and error step runs in
    the library (see geometry_aware_fp8_b200/staleness.py)."""
    from geometry_aware_fp8_b200 import staleness as stl
    T, Ks = 100, (10, 25, 50, 100)
    out = {"workload": "1536x1536 bf16 layer, X 4096x1536 bf16 per step, 100 steps, "
                       "Q_t = Q_0 exp(theta S)^t, G_t = Delta_t^T X_t / N; rank 32, E4M3 block 128",
           "K": list(Ks)}
    for theta in (0.002, 0.01):
        step = stl.drifting_device(T, 4096, 1536, 1536, theta, 8000, dtype=torch.bfloat16, device=dev)
        t0 = time.time()
        res = stl.sweep(step, T, Ks, seed=8100)
        summ = stl.summary(res, Ks)
        summ["seconds"] = time.time() - t0
        out[f"theta={theta}"] = summ
    return out


def refresh_all(ops, W):
    """Factor refresh of every whitened layer in one batched call."""
    ops.factor_refresh_many(W["jobs"], len(W["whitened"]), RANK, OVERSAMPLE, ITERS)


PHASES = ("refresh", "encode_euclid", "encode_whitened", "decode_euclid", "decode_whitened", "error")


def step(ops, W, k, ev=None, S=None):
    """Step k: on every K_REFRESH-th step the batched refresh of all whitened
    layers; then encode and decode all 96 gradients (each codec phase is one
    grouped launch) and the round-trip error of one whitened layer.
    If `ev` (len(PHASES)+1 events) is given, phase boundaries are recorded.
    S selects the G / G_hat buffer set (default: the workload's own)."""
    S = S or W["sets"][0]
    i = k % len(W["whitened"])
    rec = (lambda j: ev[j].record()) if ev else (lambda j: None)
    rec(0)
    if k % K_REFRESH == 0:
        refresh_all(ops, W)
    rec(1)
    ops.encode_many(S["packed_eu"], W["n_packed_eu"])
    rec(2)
    ops.encode_many(S["packed_wh"], W["n_packed_wh"])
    rec(3)
    ops.decode_many(S["packed_eu"], W["n_packed_eu"])
    rec(4)
    ops.decode_many(S["packed_wh"], W["n_packed_wh"])
    rec(5)
    G, Gh = S["err_pairs"][i]
    ops.roundtrip_error(G, Gh, out=S["err"], ws=W["ews"])
    rec(6)


def buffer_set(ops, W, G_all, Gh_all):
    import torch
    """Layer descriptors of the stack over other G / G_hat buffers (same offsets,
    shared codes, scales and factors)."""
    import copy
    layers, off = [], 0
    for L in W["layers"]:
        n = L.d_out * L.d_in
        M = copy.copy(L)
        M.G = G_all[off:off + n].view(L.d_out, L.d_in)
        M.G_hat = Gh_all[off:off + n].view(L.d_out, L.d_in)
        layers.append(M)
        off += n
    wl = [L for L in layers if L.rank > 0]
    el = [L for L in layers if L.rank == 0]
    return dict(packed_wh=ops.make_layers(wl), packed_eu=ops.make_layers(el),
                err_pairs=[(L.G, L.G_hat) for L in wl], G_all=G_all, Gh_all=Gh_all, err=torch.empty_like(W["err"]))


# DRAM traffic (read + write bytes per gradient element) of the whitened codec
# launches from one ncu capture of the depth-8 stack (16 whitened layers); the
# kernels' work grows in proportion to the elements, so the bench's launch is
# that figure x its elements.  Valid only for the kernel source it was taken
# on (sha256 of the file); otherwise the bench reports traffic as null.
TRAFFIC = {
    "encode_whitened": {"bytes_per_element": (201.796864e6 + 21.118976e6) / 69206016,
                        "profile": "profiles/whiten_encode_tc_stack8.md"},
    "decode_whitened": {"bytes_per_element": (96.061952e6 + 80.016384e6) / 69206016,
                        "profile": "profiles/whiten_decode_tc_stack8.md"},
}
TRAFFIC_SOURCE = ("geometry_aware_fp8_b200/csrc/codec_tc.cu",
                  "a125250a24fa765d34175b4edf167016c9cb2d44bef6f718aafcde2f7c51a943")


def traffic_for(phase, n_elements):
    import hashlib
    t = TRAFFIC.get(phase)
    path = os.path.join(ROOT, TRAFFIC_SOURCE[0])
    if t is None or not os.path.exists(path):
        return None
    with open(path, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != TRAFFIC_SOURCE[1]:
            return None
    return t["bytes_per_element"] * n_elements


def phase_bytes(W):
    """Algorithmic bytes of each codec launch: encode reads G (2 B/element) and
    writes codes (1 B) + scales (4/128 B); decode the reverse; plus U per layer."""
    enc = 2 + 1 + 4 / 128
    dec = 1 + 4 / 128 + 2
    u_bytes = sum(w["layer"].d_in * RANK * 4 for w in W["whitened"])
    return {"encode_euclid": W["n_eu"] * enc, "encode_whitened": W["n_wh"] * enc + u_bytes,
            "decode_euclid": W["n_eu"] * dec, "decode_whitened": W["n_wh"] * dec + u_bytes}


def count_launches(torch, ops, W, K):
    """libgift kernels launched inside a timed region of K steps, counted with
    the CUDA profiler on an untimed refresh step and an untimed codec step."""
    try:
        from torch.profiler import ProfilerActivity, profile

        def run(k):
            with profile(activities=[ProfilerActivity.CUDA]) as prof:
                step(ops, W, k)
                torch.cuda.synchronize()
            names = [e.name for e in prof.events() if e.device_type.name == "CUDA"]
            return [n for n in names if "gift" in n]

        with_refresh, plain = run(0), run(1)
        n_ref = (K + K_REFRESH - 1) // K_REFRESH
        total = n_ref * len(with_refresh) + (K - n_ref) * len(plain)
        return total, sorted(set(with_refresh))
    except Exception as e:  # pragma: no cover
        return None, [f"profiler unavailable: {e}"]


def cpu_baseline(sample_seconds=12.0):
    """The oracle as it stands on the host cores: bounded sample of the same workload."""
    from oracle import gift_oracle as O
    from geometry_aware_fp8_b200 import synth
    t_end = time.time() + sample_seconds
    nbytes, t_used, reps = 0, 0.0, 0
    Q = synth.haar_orthogonal(1536, 11)
    X = synth.to_storage(synth.activations(REFRESH_N, Q, synth.column_power(1536, 1.0), 12), "bf16")
    Go = synth.to_storage(synth.gradient(1536, Q, 1.0, 13), "bf16")
    Gq = synth.to_storage(synth.gradient(4608, Q, 1.0, 14), "bf16")
    while time.time() < t_end or reps == 0:
        t0 = time.perf_counter()
        A = O.input_factor(X)
        U, lam, rho, _ = O.factor_refresh(A, RANK, OVERSAMPLE, ITERS, seed=reps)
        c, s = O.encode_e4m3(Go, U, lam, rho)
        Gh = O.bf16_round(O.decode_e4m3(c, s, U, lam, rho))
        O.roundtrip_error(Go, Gh)
        c2, s2 = O.quantize_e4m3_blocks(Gq)
        O.bf16_round(O.dequantize_e4m3_blocks(c2, s2))
        t_used += time.perf_counter() - t0
        nbytes += 2 * (Go.size + Gq.size)
        reps += 1
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    return {"value": nbytes / t_used / 1e9, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": (f"{reps} x [o-projection 1536x1536 bf16: refresh from X 8192x1536 + whitened encode + "
                       f"decode + error; qkv 4608x1536 Euclidean encode + decode], {t_used:.1f} s"),
            "host_cpus": os.cpu_count()}


def run_gpu(args):
    import torch
    import torch.distributed as dist
    from geometry_aware_fp8_b200 import ops, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.warmup < 3:
        args.warmup = 3
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    W = build_workload(torch, ops, synth, dev, args.depth, seed=1234 + rank)
    refresh_all(ops, W)
    torch.cuda.synchronize()

    for k in range(args.warmup):
        step(ops, W, k)  # step 0 includes a batched refresh
    torch.cuda.synchronize()

    # ---- timed region: device resident inputs (1.06 GB of G > 126 MB L2) ----
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(PHASES) + 1)] for _ in range(K)]
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for k in range(K):
        step(ops, W, k, evs[k])
    t1.record()
    torch.cuda.synchronize()
    barrier()
    clock_info = clocks.stop()
    ms_total = t0.elapsed_time(t1)
    phase = np.array([[e[i].elapsed_time(e[i + 1]) for i in range(len(PHASES))] for e in evs])
    pm = {n: float(phase[:, i].mean()) for i, n in enumerate(PHASES)}
    ms_total = max_over_ranks(ms_total, dev)
    ms_step = ms_total / K
    g_bytes = W["n_el"] * 2
    value = job_value(world, g_bytes, ms_step)

    pb = phase_bytes(W)
    peak, peak_kind = measured_peaks()
    dom = max(pb, key=lambda n: pm[n])
    achieved = pb[dom] / (pm[dom] * 1e-3) / 1e9
    roofline = {"bound": "hbm", "kernel": f"{dom} (one grouped launch over its layers of the stack)",
                "achieved": achieved, "peak": peak, "peak_source": peak_kind, "unit": "GB/s",
                "frac": achieved / peak,
                "traffic": traffic_for(dom, W["n_wh"] if dom.endswith("whitened") else W["n_eu"]),
                "traffic_unit": "bytes per launch (DRAM read + write, ncu, scaled from the depth-8 capture)"}
    codec_ms = sum(pm[n] for n in pb)
    ref_steps = [k for k in range(K) if k % K_REFRESH == 0]
    codec = {"phase_ms": pm,
             "refresh_batched_ms": float(np.mean([phase[k, 0] for k in ref_steps])) if ref_steps else None,
             "refresh_layers": len(W["whitened"]),
             "phase_gbs": {n: pb[n] / (pm[n] * 1e-3) / 1e9 for n in pb},
             "phase_roofline_frac": {n: pb[n] / (pm[n] * 1e-3) / 1e9 / peak for n in pb},
             "codec_gradient_gbs": g_bytes / (codec_ms * 1e-3) / 1e9,
             "codec_roofline_frac": sum(pb.values()) / (codec_ms * 1e-3) / 1e9 / peak}

    launches, names = count_launches(torch, ops, W, K)
    nvfp4 = nvfp4_measure(torch, ops, synth, dev, peak) if not args.no_nvfp4 else None
    single = layers_measure(torch, ops, synth, dev, peak) if not args.no_layers else None
    stale = staleness_measure(torch, dev) if not args.no_staleness else None

    # ---- end to end through host buffers: the same schedule, with every
    # step's gradients copied in from pinned host memory, the activations of
    # all whitened layers copied in on refresh steps, and G_hat copied back ----
    e2e = None
    if not args.no_e2e:
        # Through host buffers: every step's gradients come in from pinned host
        # memory (and all activations on refresh steps), G_hat and the error go
        # back.  Copies in, compute and copies out run on three streams over two
        # device buffer sets, so step k+1's upload and step k-1's download
        # overlap step k (PCIe is full duplex); every byte still crosses inside
        # the timed region.
        G_host = torch.empty((W["n_el"],), dtype=torch.bfloat16, pin_memory=True)
        G_host.copy_(W["G_all"].cpu())
        Gh_host = torch.empty_like(G_host, pin_memory=True)
        X_host = [w["X"].cpu().pin_memory() for w in W["whitened"]]
        err_host = torch.empty((3,), dtype=torch.float64, pin_memory=True)
        x_bytes = sum(x.numel() * 2 for x in X_host)
        if len(W["sets"]) < 2:
            W["sets"].append(buffer_set(ops, W, torch.empty_like(W["G_all"]), torch.empty_like(W["Gh_all"])))
        comp = torch.cuda.current_stream()
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        E = torch.cuda.Event

        def run_e2e(ks):
            done = {}     # k -> event: step k's compute finished (its G buffer is free)
            out_done = {} # k -> event: step k's download finished (its G_hat buffer is free)
            last_ref = None
            for k in ks:
                S = W["sets"][k % 2]
                with torch.cuda.stream(s_in):
                    if k - 2 in done:
                        s_in.wait_event(done[k - 2])
                    S["G_all"].copy_(G_host, non_blocking=True)
                    if k % K_REFRESH == 0:
                        if last_ref is not None:
                            s_in.wait_event(last_ref)
                        for w, xh in zip(W["whitened"], X_host):
                            w["X"].copy_(xh, non_blocking=True)
                    ev_in = E()
                    ev_in.record(s_in)
                comp.wait_event(ev_in)
                if k - 2 in out_done:
                    comp.wait_event(out_done[k - 2])
                step(ops, W, k, S=S)
                ev_c = E()
                ev_c.record(comp)
                done[k] = ev_c
                if k % K_REFRESH == 0:
                    last_ref = ev_c
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_c)
                    Gh_host.copy_(S["Gh_all"], non_blocking=True)
                    err_host.copy_(S["err"], non_blocking=True)
                    ev_o = E()
                    ev_o.record(s_out)
                out_done[k] = ev_o
            return ev_o

        run_e2e(range(1, 3))
        torch.cuda.synchronize()
        barrier()
        a = E(enable_timing=True)
        b = E(enable_timing=True)
        a.record(comp)
        s_in.wait_event(a)
        last = run_e2e(range(K))
        comp.wait_event(last)
        b.record(comp)
        torch.cuda.synchronize()
        ms_e = max_over_ranks(a.elapsed_time(b), dev)
        n_ref = (K + K_REFRESH - 1) // K_REFRESH
        e2e = {"value": job_value(world, g_bytes, ms_e / K), "unit": UNIT,
               "h2d_bytes_per_step": int(g_bytes + n_ref * x_bytes / K), "d2h_bytes_per_step": int(g_bytes + 24),
               "ms_per_step": ms_e / K,
               "pipeline": "uploads, compute and downloads on three streams over two G / G_hat buffer sets"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline()

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
                "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f32", "data": "synthetic",
                "config": {"workload": WORKLOAD, "depth": args.depth, "gradient_elements": W["n_el"],
                           "gradient_bytes": g_bytes, "storage": "bf16 G / e4m3 codes / fp32 scales",
                           "l2": "inputs larger than L2 (1.06 GB of gradients streamed per step)",
                           "parallelism": f"replicas x{world}"},
                "roofline": roofline, "codec": codec, "layers": single, "staleness": stale, "nvfp4": nvfp4, "e2e": e2e, "cpu_baseline": cpu,
                "gpu_launches": launches, "kernels": names, "clocks": clock_info}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle on the host cores
# ---------------------------------------------------------------------------
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    warm = max(args.warmup, 0)
    for _ in range(min(warm, 2)):
        cpu_baseline(sample_seconds=0.0)
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        r = cpu_baseline(sample_seconds=0.0)
        vals.append(r["value"])
    wall = time.perf_counter() - t0
    v = float(statistics.mean(vals))
    cpu = dict(r, value=v)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": 0, "steps": args.steps,
            "warmup": warm, "ms_per_step": wall / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": cpu["sample"]},
            "cpu_baseline": cpu, "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_gpu(a)
