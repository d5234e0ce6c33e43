#!/usr/bin/env python
"""Benchmark of the GIFT whitened-FP8 gradient codec on B200.

Workload (one step): the Llama-600M-sized stand-in stack of 24 layers x
{qkv 1536->4608, o 1536->1536, up 1536->4096, down 4096->1536} bf16
gradients (528.5 M elements, 1.06 GB).  Selective deployment: o and down
are whitened at rank 32, qkv and up take the Euclidean per-block E4M3
codec.  A step is the whole per-step hot path of the paper:
  * encode of all 96 gradients, then decode of all 96 (each codec phase one
    grouped launch), and the one-step round-trip error of one whitened layer;
  * the factor refresh of all 48 whitened layers (A = X^T X / N on 8192
    tokens each, subspace iteration, Rayleigh-Ritz; one batched call), which
    Algorithm 1 (section V.E) runs once every K_REFRESH = 50 steps: a step
    carries 1/50 of it.
The codec steps and the refresh are timed in two regions, each bracketed
by a barrier and a device synchronisation and timed with CUDA events:
K codec steps, and R batched refreshes.  ms_per_step = codec step + refresh
/ 50, so the value does not depend on --steps.
value = gradient bytes of the stack / ms_per_step (GB/s).

Multi-GPU (`--gpus N` under torchrun): replicas only -- the codec has no
exchange step, so every rank runs its own copy of the stack (weak scaling);
the timed regions are bracketed by barriers and the reported times are the
max over ranks.

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
BF16_FALLBACK = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100, help="timed codec steps")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--refreshes", type=int, default=3, help="timed batched refreshes (each counts 1/50 of a step)")
    ap.add_argument("--impl", default="gift", choices=["gift", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-nvfp4", action="store_true", help="skip the NVFP4 measurement on the 11008x4096 gradient")
    ap.add_argument("--no-layers", action="store_true", help="skip the single-layer codec measurements")
    ap.add_argument("--no-staleness", action="store_true", help="skip the factor-staleness sweep")
    ap.add_argument("--no-config2", action="store_true", help="skip the config-2 batch of 24 layers")
    ap.add_argument("--no-config4", action="store_true", help="skip the config-4 refresh at scale")
    ap.add_argument("--no-variants", action="store_true", help="skip the dense-transform variants")
    ap.add_argument("--depth", type=int, default=24, help="layers in the stack (24 = the full stand-in)")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", HBM_FALLBACK), "measured"
    return HBM_FALLBACK, "fallback"


def measured_bf16_peak():
    """Dense bf16 TFLOP/s for a kernel timed alone (the burst figure)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f).get("bf16_tflops", BF16_FALLBACK))
    return BF16_FALLBACK


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
            L.U_split = torch.empty((2, d_in, 64), device=dev, dtype=torch.int16)
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
                       "median of 20 calls, L2 flushed between calls; graph_replay: the same two calls "
                       "captured in CUDA graphs and replayed (no host work per call)"}
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
        # the same calls captured once in CUDA graphs and replayed: kernel time
        # without the binding's host work
        side = torch.cuda.Stream()
        ge, gd = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(ge, stream=side):
            ops.encode(G, U, lam, rho, codes=codes, scales=scales)
        with torch.cuda.graph(gd, stream=side):
            ops.decode(codes, scales, U, lam, rho, out=Gh)
        enc_g, dec_g = timed(ge.replay), timed(gd.replay)
        n = d_out * d_in
        gb = G.element_size()
        t = (enc + dec) * 1e-3
        tg = (enc_g + dec_g) * 1e-3
        out[name] = {"encode_ms": enc, "decode_ms": dec, "gradient_gbs": gb * n / t / 1e9,
                     "elements_per_s": n / t, "panels": (d_out + 127) // 128,
                     "roofline_frac": 2 * (gb + 1 + 4 / 128) * n / t / 1e9 / peak,
                     "graph_replay": {"encode_ms": enc_g, "decode_ms": dec_g, "gradient_gbs": gb * n / tg / 1e9,
                                      "roofline_frac": 2 * (gb + 1 + 4 / 128) * n / tg / 1e9 / peak}}
        del G, Gh, codes, scales, ge, gd
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
    """Factor refresh of every whitened layer in one batched call, then the U
    split the tensor-core codec loads (gift_split_u_many: one launch for all
    layers of the grouped codec's array)."""
    ops.factor_refresh_many(W["jobs"], len(W["whitened"]), RANK, OVERSAMPLE, ITERS)
    ops.split_u_many(W["packed_wh"], W["n_packed_wh"])


PHASES = ("encode_euclid", "encode_whitened", "decode_euclid", "decode_whitened", "error")


def step(ops, W, k, ev=None, S=None):
    """Codec step k: encode and decode all 96 gradients (each codec phase is
    one grouped launch) and the round-trip error of one whitened layer.  The
    factor refresh, which Algorithm 1 runs every K_REFRESH steps, is timed
    on its own (refresh_all).  If `ev` (len(PHASES)+1 events) is given, phase
    boundaries are recorded.  S selects the G / G_hat buffer set (default:
    the workload's own)."""
    S = S or W["sets"][0]
    i = k % len(W["whitened"])
    rec = (lambda j: ev[j].record()) if ev else (lambda j: None)
    rec(0)
    ops.encode_many(S["packed_eu"], W["n_packed_eu"])
    rec(1)
    ops.encode_many(S["packed_wh"], W["n_packed_wh"])
    rec(2)
    ops.decode_many(S["packed_eu"], W["n_packed_eu"])
    rec(3)
    ops.decode_many(S["packed_wh"], W["n_packed_wh"])
    rec(4)
    G, Gh = S["err_pairs"][i]
    ops.roundtrip_error(G, Gh, out=S["err"], ws=W["ews"])
    rec(5)


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


# Memory traffic of the whitened codec launches from one ncu capture of the
# depth-8 stack (16 whitened layers; profiles/ names the command), per
# gradient element: DRAM read bytes, and the bytes the kernel wrote into L2
# (L2 write sectors from the SMs x 32 B).  Every written line reaches DRAM,
# but lines still dirty in L2 when a kernel ends are written back during
# later kernels, so the kernel's own DRAM write counter sees only part of
# them; the L2 write-in is the full write traffic (sector-granular: the
# encoder's 4-byte scale stores count as whole 32-byte sectors there, an upper
# bound that L2 merges before DRAM).  The kernels' work grows in
# proportion to the elements, so the bench's launch is that figure x its
# elements.  Valid only for the kernel source it was taken on (sha256 of the
# file); otherwise the bench reports traffic as null.
TRAFFIC = {
    "decode_whitened": {"read_per_element": 1.482048, "l2_write_per_element": 2.006570,
                        "dram_write_per_element": 1.148715, "profile": "profiles/whiten_decode_tc_stack8.md"},
    "encode_whitened": {"read_per_element": 2.949004, "l2_write_per_element": 1.250000,
                        "dram_write_per_element": 0.298965, "profile": "profiles/whiten_encode_tc_stack8.md"},
}
TRAFFIC_SOURCE = ("geometry_aware_fp8_b200/csrc/codec_tc.cu",
                  "4dd3db93aff24074a976fe973fc77adf86a1e11c3075d8f80168cac25f3a2a08")


def traffic_for(phase, n_elements, alg_read, alg_write):
    import hashlib
    t = TRAFFIC.get(phase)
    path = os.path.join(ROOT, TRAFFIC_SOURCE[0])
    if t is None or not os.path.exists(path):
        return None
    with open(path, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != TRAFFIC_SOURCE[1]:
            return None
    rd, wr = t["read_per_element"] * n_elements, t["l2_write_per_element"] * n_elements
    return {"bytes": rd + wr, "read_bytes": rd, "write_bytes": wr, "read_excess": rd / alg_read,
            "write_excess": wr / alg_write,
            "dram_write_during_kernel_bytes": t["dram_write_per_element"] * n_elements, "profile": t["profile"]}


def phase_bytes(W):
    """Algorithmic bytes of each codec launch, split into reads and writes:
    encode reads G (2 B/element) and writes codes (1 B) + scales (4/128 B);
    decode the reverse; a whitened launch also reads U once per layer."""
    u_bytes = sum(w["layer"].d_in * RANK * 4 for w in W["whitened"])
    n_wh, n_eu = W["n_wh"], W["n_eu"]
    rw = {"encode_euclid": (2 * n_eu, (1 + 4 / 128) * n_eu),
          "encode_whitened": (2 * n_wh + u_bytes, (1 + 4 / 128) * n_wh),
          "decode_euclid": ((1 + 4 / 128) * n_eu, 2 * n_eu),
          "decode_whitened": ((1 + 4 / 128) * n_wh + u_bytes, 2 * n_wh)}
    return {k: r + w for k, (r, w) in rw.items()}, rw


def profile_kernels(torch, fn):
    """Device time of each libgift kernel in one call of fn, from the CUDA
    profiler: {kernel name: (launches, total ms)}."""
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    out = {}
    for e in prof.events():
        if e.device_type.name == "CUDA" and "gift" in e.name:
            n, t = out.get(e.name, (0, 0.0))
            out[e.name] = (n + 1, t + e.device_time_total / 1e3)
    return out


def kernel_short_name(name):
    """'void gift::(anonymous namespace)::syrk_tc_kernel<...>(...)' -> 'syrk_tc_kernel'."""
    import re
    m = re.search(r"([A-Za-z_][A-Za-z0-9_]*)(<[^()]*>)?\(", name)
    return m.group(1) if m else name


def count_launches(torch, ops, W, K, n_refresh):
    """libgift kernels launched inside the two timed regions (K codec steps,
    n_refresh batched refreshes), counted with the CUDA profiler on one
    untimed codec step and one untimed refresh."""
    try:
        codec = profile_kernels(torch, lambda: step(ops, W, 1))
        ref = profile_kernels(torch, lambda: refresh_all(ops, W))
        per_step = sum(n for n, _ in codec.values())
        per_ref = sum(n for n, _ in ref.values())
        return K * per_step + n_refresh * per_ref, sorted(set(codec) | set(ref)), per_step, per_ref
    except Exception as e:  # pragma: no cover
        return None, [f"profiler unavailable: {e}"], None, None


def config2_batch_measure(torch, ops, synth, dev, peak, reps=20, batch=24):
    """Config 2 (the MLP up-projection stand-in, d_in 1536, d_out 4096, bf16,
    exponent 1.0) as a batch of `batch` distinct gradients of that layer, each
    with its own rank-32 factor refreshed from 8192 bf16 tokens (one batched
    refresh and its U splits, untimed), coded by one grouped whitened encode
    and one grouped decode.  The batch (302 MB of G) is larger than L2, and L2 is flushed
    between timed repetitions."""
    d_out, d_in = 4096, 1536
    gen = torch.Generator(device=dev)
    gen.manual_seed(2001)
    Q = torch.from_numpy(synth.haar_orthogonal(d_in, 2003).astype(np.float32)).to(dev)
    sigma = torch.arange(1, d_in + 1, device=dev, dtype=torch.float32) ** -1.0
    layers, items = [], []
    for b in range(batch):
        G = synth.device_gradient(d_out, d_in, 1.0, Q, gen, torch.bfloat16)
        L = ops.LayerArgs(d_out=d_out, d_in=d_in, rank=RANK, dtype=torch.bfloat16, G=G, G_hat=torch.empty_like(G),
                          codes=torch.empty((d_out, d_in), device=dev, dtype=torch.uint8),
                          scales=torch.empty((d_out, d_in // 128), device=dev, dtype=torch.float32),
                          U=torch.empty((d_in, RANK), device=dev), lam=torch.empty((RANK,), device=dev),
                          rho=torch.empty((1,), device=dev))
        X = synth.device_activations(REFRESH_N, sigma, Q, gen, torch.bfloat16)
        ws = torch.empty((ops.refresh_workspace_size(REFRESH_N, d_in, RANK, OVERSAMPLE),), device=dev,
                         dtype=torch.uint8)
        items.append((X, L.U, L.lam, L.rho, ws, torch.zeros((1,), device=dev, dtype=torch.int32), 2004 + b, None))
        layers.append(L)
    jobs = ops.make_refresh_jobs(items)
    ops.factor_refresh_many(jobs, batch, RANK, OVERSAMPLE, ITERS)
    for L in layers:
        L.U_split = ops.split_u(L.U)
    torch.cuda.synchronize()
    del items, jobs
    packed = ops.make_layers(layers)
    flush = torch.empty((256 << 20,), device=dev, dtype=torch.uint8)
    st = torch.zeros((1,), device=dev, dtype=torch.int32)
    te, td = [], []
    for i in range(reps + 3):
        flush.zero_()
        a, b, c = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        a.record()
        ops.encode_many(packed, batch, dev_status=st)
        b.record()
        ops.decode_many(packed, batch, dev_status=st)
        c.record()
        torch.cuda.synchronize()
        if i >= 3:
            te.append(a.elapsed_time(b))
            td.append(b.elapsed_time(c))
    n = batch * d_out * d_in
    u = batch * d_in * RANK * 4
    enc, dec = float(np.median(te)), float(np.median(td))
    e_b, d_b = n * (2 + 1 + 4 / 128) + u, n * (1 + 4 / 128 + 2) + u
    out = {"workload": f"{batch} distinct 4096x1536 bf16 gradients (config 2's layer), each with its own rank-32 "
                       f"factor from X {REFRESH_N}x1536 bf16; one grouped encode + one grouped decode; "
                       f"median of {reps}, L2 flushed between repetitions",
           "encode_ms": enc, "decode_ms": dec, "gradient_gbs": 2 * n / ((enc + dec) * 1e-3) / 1e9,
           "elements_per_s": n / ((enc + dec) * 1e-3),
           "encode_roofline_frac": e_b / (enc * 1e-3) / 1e9 / peak,
           "decode_roofline_frac": d_b / (dec * 1e-3) / 1e9 / peak,
           "roofline_frac": (e_b + d_b) / ((enc + dec) * 1e-3) / 1e9 / peak,
           "dev_status": int(st.item())}
    del layers, packed, flush
    torch.cuda.empty_cache()
    return out


def config4_refresh_measure(torch, ops, synth, dev, bf16_peak, reps=5):
    """Config 4, the factor refresh at scale: X 65536 x 4096 bf16 with
    eigenvalues i^-1.2 and five 100x spikes; A = X^T X / N and its top-32
    eigenpairs by 4 iterations of subspace iteration with oversample 16.
    Useful flops of the contraction: 2 N d (d + 1) / 2 (the symmetric half).
    Per-kernel device times come from the CUDA profiler on one more call."""
    N, d = 65536, 4096
    gen = torch.Generator(device=dev)
    gen.manual_seed(4001)
    Qd = torch.from_numpy(synth.haar_orthogonal(d, 4003).astype(np.float32)).to(dev)
    sig = torch.from_numpy(synth.spectrum_power(d, 1.2, 5, 100.0).astype(np.float32)).to(dev)
    X = synth.device_activations(N, sig, Qd, gen, torch.bfloat16)
    del Qd
    A = torch.empty((d, d), device=dev, dtype=torch.float32)
    U = torch.empty((d, RANK), device=dev)
    lam = torch.empty((RANK,), device=dev)
    rho = torch.empty((1,), device=dev)
    ws = torch.empty((ops.refresh_workspace_size(N, d, RANK, OVERSAMPLE, True),), device=dev, dtype=torch.uint8)
    st = torch.zeros((1,), device=dev, dtype=torch.int32)
    call = lambda: ops.factor_refresh(X, RANK, OVERSAMPLE, ITERS, 4004, A_out=A, ws=ws, dev_status=st,
                                      out=(U, lam, rho))
    ts = []
    for i in range(reps + 3):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        call()
        b.record()
        torch.cuda.synchronize()
        if i >= 3:
            ts.append(a.elapsed_time(b))
    ms = float(np.median(ts))
    flops = 2.0 * N * d * (d + 1) / 2
    kern = profile_kernels(torch, call)
    tot = sum(t for _, t in kern.values())
    syrk = sum(t for k, (_, t) in kern.items() if "syrk" in k)
    out = {"workload": "X 65536x4096 bf16, eigenvalues i^-1.2 with five 100x spikes; rank 32, oversample 16, "
                       f"4 iterations; median of {reps} calls",
           "ms": ms, "useful_flops": flops, "tflops": flops / (ms * 1e-3) / 1e12,
           "frac_of_bf16_peak": flops / (ms * 1e-3) / 1e12 / bf16_peak,
           "syrk_ms": syrk, "syrk_tflops": flops / (syrk * 1e-3) / 1e12 if syrk else None,
           "syrk_frac_of_bf16_peak": flops / (syrk * 1e-3) / 1e12 / bf16_peak if syrk else None,
           "syrk_share": syrk / tot if tot else None,
           "kernels_ms": {kernel_short_name(k): round(t, 4) for k, (_, t) in kern.items()},
           "lambda_1": float(lam[0].item()), "rho": float(rho.item()), "dev_status": int(st.item())}
    del X, A, ws
    torch.cuda.empty_cache()
    return out


def variants_measure(torch, ops, synth, dev, bf16_peak, reps=10):
    """The variants GIFT is simplified from, on the GPU (review page, "What
    carries the argument"; Fig. 2 caption; section IV.A, Eq. (14)): the E4M3
    round trip of one gradient under the Euclidean codec, the rank-32 codec,
    full-rank input whitening A^{-1/2} and the input-side Cholesky form
    L_A^{-T}, on draws with a linear layer's structure (d_in 512, d_out 256,
    N 4096, sigma_i = i^-1, G = Delta^T X / N with Delta's columns scaled by
    j^-1/2): relative Frobenius errors from gift_roundtrip_error.  Then the
    dense codec's speed at config 2's layer shape (4096 x 1536 bf16, median
    of `reps`, L2 flushed): it is a pair of GEMMs, so it is tensor bound;
    flops count the bf16 products the kernels issue (3 parts of M on encode,
    2 of M^{-1} on decode; the Cholesky form skips the zero blocks of its
    triangle)."""
    d_in, d_out, N = 512, 256, 4096
    Q = synth.haar_orthogonal(d_in, 41)
    X = synth.activations(N, Q, synth.column_power(d_in, 1.0), 42)
    rng = np.random.default_rng(43)
    Delta = rng.standard_normal((N, d_out)) * (np.arange(1, d_out + 1) ** -0.5)[None, :]
    G = torch.from_numpy(synth.to_storage(Delta.T @ X / N, "bf16")).to(dev).to(torch.bfloat16)
    Xd = torch.from_numpy(X.astype(np.float32)).to(dev)
    A = torch.empty((d_in, d_in), device=dev)
    U, lam, rho, _ = ops.factor_refresh(Xd, RANK, OVERSAMPLE, ITERS, 44, A_out=A)
    err = torch.empty((3,), device=dev, dtype=torch.float64)
    out = {"workload": "d_in 512, d_out 256, N 4096, sigma_i = i^-1, G = Delta^T X / N (bf16), Delta columns "
                       "scaled j^-1/2; E4M3 block 128; relative Frobenius round-trip error",
           "frobenius_error": {}}

    def rt(c, s_, dec):
        Gh = dec(c, s_)
        ops.roundtrip_error(G, Gh, out=err)
        return float(err[0].item())

    c, s_ = ops.encode(G)
    out["frobenius_error"]["euclid"] = rt(c, s_, lambda c, s_: ops.decode(c, s_, out_dtype=torch.bfloat16))
    c, s_ = ops.encode(G, U, lam, rho)
    out["frobenius_error"]["input_rank32"] = rt(c, s_, lambda c, s_: ops.decode(c, s_, U, lam, rho))
    facs = {}
    for name, kind in (("input_full", ops.DENSE_INVSQRT), ("input_cholesky", ops.DENSE_CHOLESKY)):
        M, Mi, Ms, Mis, st = ops.dense_factor(A, kind)
        up = kind == ops.DENSE_CHOLESKY
        c, s_ = ops.dense_encode(G, Ms, up)
        out["frobenius_error"][name] = rt(c, s_, lambda c, s_: ops.dense_decode(c, s_, Mis, up))
        out[f"{name}_factor_status"] = int(st.item())
    # speed at the config-2 layer shape, factor of A from 8192 tokens
    d_in, d_out = 1536, 4096
    gen = torch.Generator(device=dev)
    gen.manual_seed(2001)
    Qd = torch.from_numpy(synth.haar_orthogonal(d_in, 2003).astype(np.float32)).to(dev)
    G2 = synth.device_gradient(d_out, d_in, 1.0, Qd, gen, torch.bfloat16)
    sigma = torch.arange(1, d_in + 1, device=dev, dtype=torch.float32) ** -1.0
    X2 = synth.device_activations(REFRESH_N, sigma, Qd, gen, torch.bfloat16)
    A2 = torch.empty((d_in, d_in), device=dev)
    ops.factor_refresh(X2, RANK, OVERSAMPLE, ITERS, 2004, A_out=A2)
    del X2
    flush = torch.empty((256 << 20,), device=dev, dtype=torch.uint8)
    codes = torch.empty((d_out, d_in), device=dev, dtype=torch.uint8)
    scales = torch.empty((d_out, d_in // 128), device=dev, dtype=torch.float32)
    Gh = torch.empty_like(G2)

    def timed(fn):
        ts = []
        for i in range(reps + 3):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if i >= 3:
                ts.append(a.elapsed_time(b))
        return float(np.median(ts))

    for name, kind in (("input_full", ops.DENSE_INVSQRT), ("input_cholesky", ops.DENSE_CHOLESKY)):
        t_fac = timed(lambda: ops.dense_factor(A2, kind))
        M, Mi, Ms, Mis, st = ops.dense_factor(A2, kind)
        up = kind == ops.DENSE_CHOLESKY
        enc = timed(lambda: ops.dense_encode(G2, Ms, up, codes=codes, scales=scales))
        dec = timed(lambda: ops.dense_decode(codes, scales, Mis, up, out=Gh))
        nblk = d_in // 128
        frac_k = (nblk + 1) / (2 * nblk) if up else 1.0  # share of the K range a tile runs
        one = 2.0 * d_out * d_in * d_in * frac_k          # one product G M (or W_hat M^{-1})
        fe, fd = 3 * one, 2 * one                          # bf16 parts of M: 3 (encode), 2 (decode)
        out[f"{name}_4096x1536"] = {"factor_ms": t_fac, "encode_ms": enc, "decode_ms": dec,
                                    "encode_tflops": fe / (enc * 1e-3) / 1e12,
                                    "decode_tflops": fd / (dec * 1e-3) / 1e12,
                                    "encode_frac_of_bf16_peak": fe / (enc * 1e-3) / 1e12 / bf16_peak,
                                    "decode_frac_of_bf16_peak": fd / (dec * 1e-3) / 1e12 / bf16_peak,
                                    "factor_status": int(st.item())}
    del G2, A2, flush, codes, scales, Gh
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------
# CPU baseline: the oracle as it stands, on the host cores
# ---------------------------------------------------------------------------
def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def _oracle_layer(O, synth, d_out, d_in, whitened, seed, with_refresh=True):
    """One layer through the oracle: (gradient bytes, refresh s, codec s).
    Whitened: refresh from X 8192 x d_in bf16, encode, decode (G_hat rounded
    to bf16), error.  Euclidean: per-block E4M3 encode and decode."""
    Q = synth.haar_orthogonal(d_in, seed)
    G = synth.to_storage(synth.gradient(d_out, Q, 1.0, seed + 1), "bf16")
    t_ref = 0.0
    if whitened:
        X = synth.to_storage(synth.activations(REFRESH_N, Q, synth.column_power(d_in, 1.0), seed + 2), "bf16")
        t0 = time.perf_counter()
        U, lam, rho, _ = O.factor_refresh(O.input_factor(X), RANK, OVERSAMPLE, ITERS, seed=seed)
        t_ref = time.perf_counter() - t0
        t0 = time.perf_counter()
        c, s_ = O.encode_e4m3(G, U, lam, rho)
        Gh = O.bf16_round(O.decode_e4m3(c, s_, U, lam, rho))
        O.roundtrip_error(G, Gh)
    else:
        t0 = time.perf_counter()
        c, s_ = O.quantize_e4m3_blocks(G)
        O.bf16_round(O.dequantize_e4m3_blocks(c, s_))
    return 2 * G.size, t_ref, time.perf_counter() - t0


def cpu_stack_group(O, synth, seed=11):
    """One layer of each shape of the stack (qkv and up Euclidean, o and down
    whitened) through the oracle: (gradient bytes, refresh s, codec s)."""
    tot = [0, 0.0, 0.0]
    for j, (d_out, d_in, wh) in enumerate(((4608, 1536, False), (1536, 1536, True), (4096, 1536, False),
                                           (1536, 4096, True))):
        r = _oracle_layer(O, synth, d_out, d_in, wh, seed + 10 * j)
        for i in range(3):
            tot[i] += r[i]
    return tuple(tot)


def cpu_baseline():
    """The oracle (numpy fp64, unchanged) on the host cores, on bounded samples
    of the workloads: all cores (numpy's BLAS threads) and one thread.
    value: one layer of each stack shape, gradient GB/s with the refresh
    amortised over K_REFRESH steps as in the GPU figure."""
    from oracle import gift_oracle as O
    from geometry_aware_fp8_b200 import synth
    try:
        from threadpoolctl import threadpool_info, threadpool_limits
    except Exception:  # pragma: no cover
        threadpool_info = threadpool_limits = None
    cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1]) if threadpool_info else os.cpu_count()

    def amortised(b, t_ref, t_codec):
        return b / (t_codec + t_ref / K_REFRESH) / 1e9

    out = {"kind": "oracle", "unit": UNIT, "cores": cores, "host_cpus": os.cpu_count(), "cpu_model": cpu_model()}
    t_all = time.perf_counter()
    b, tr, tc = cpu_stack_group(O, synth)
    out["value"] = amortised(b, tr, tc)
    out["stack_layer_group"] = {"gradient_gbs": out["value"], "refresh_s": tr, "codec_s": tc, "threads": cores}
    b, tr, tc = _oracle_layer(O, synth, 512, 512, True, 1001)
    out["config1_512x512"] = {"gradient_gbs": amortised(b, tr, tc), "codec_gbs": b / tc / 1e9, "refresh_s": tr,
                              "codec_s": tc, "threads": cores}
    b, tr, tc = _oracle_layer(O, synth, 4096, 1536, True, 2001)
    out["config2_4096x1536"] = {"gradient_gbs": amortised(b, tr, tc), "codec_gbs": b / tc / 1e9, "refresh_s": tr,
                                "codec_s": tc, "threads": cores}
    # config 4, the refresh at scale (d = 4096): A from a sample of 16384 of the
    # 65536 tokens (its time scaled by 4 for the whole range), then the
    # subspace iteration and Rayleigh-Ritz on that d x d matrix
    N, d, n_s = 65536, 4096, 16384
    rng = np.random.default_rng(4001)
    Q = synth.haar_orthogonal(d, 4003)
    sig = synth.spectrum_power(d, 1.2, 5, 100.0)
    Xs = synth.to_storage((rng.standard_normal((n_s, d)) * sig[None, :]) @ Q, "bf16")
    t0 = time.perf_counter()
    A = O.input_factor(Xs)
    t_A = time.perf_counter() - t0
    del Xs
    t0 = time.perf_counter()
    O.factor_refresh(A, RANK, OVERSAMPLE, ITERS, seed=4004)
    t_eig = time.perf_counter() - t0
    out["config4_refresh"] = {"A_s_for_65536_tokens": t_A * N / n_s, "eig_s": t_eig,
                              "refresh_s": t_A * N / n_s + t_eig, "threads": cores,
                              "sample": f"A timed on {n_s} of the {N} tokens and scaled by {N // n_s}"}
    if threadpool_limits is not None:
        with threadpool_limits(limits=1):
            b, tr, tc = _oracle_layer(O, synth, 512, 512, True, 1001)
            out["config1_512x512_1thread"] = {"gradient_gbs": amortised(b, tr, tc), "codec_gbs": b / tc / 1e9,
                                              "refresh_s": tr, "codec_s": tc, "threads": 1}
            b, tr, tc = _oracle_layer(O, synth, 1536, 1536, True, 21)
            out["o_1536x1536_1thread"] = {"gradient_gbs": amortised(b, tr, tc), "codec_gbs": b / tc / 1e9,
                                          "refresh_s": tr, "codec_s": tc, "threads": 1}
    out["sample"] = ("one layer of each stack shape (qkv 4608x1536 and up 4096x1536 Euclidean; o 1536x1536 and "
                     "down 1536x4096 whitened, refresh from X 8192 x d_in, encode, decode, error) for value; "
                     "configs 1 and 2, the config-4 refresh, and configs 1 and o on one thread; "
                     f"{time.perf_counter() - t_all:.1f} s in all")
    return out


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
        step(ops, W, k)
    refresh_all(ops, W)
    torch.cuda.synchronize()

    K = args.steps
    R = max(1, args.refreshes)
    clocks = ClockSampler(local)
    # ---- timed region 1: K codec steps, device-resident inputs (1.06 GB of G > 126 MB L2) ----
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(PHASES) + 1)] for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for k in range(K):
        step(ops, W, k, evs[k])
    t1.record()
    torch.cuda.synchronize()
    barrier()
    # ---- timed region 2: R batched refreshes of the 48 whitened layers ----
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    r0.record()
    for _ in range(R):
        refresh_all(ops, W)
    r1.record()
    torch.cuda.synchronize()
    barrier()
    clock_info = clocks.stop()
    codec_ms = max_over_ranks(t0.elapsed_time(t1), dev) / K
    refresh_ms = max_over_ranks(r0.elapsed_time(r1), dev) / R
    ms_step = codec_ms + refresh_ms / K_REFRESH
    phase = np.array([[e[i].elapsed_time(e[i + 1]) for i in range(len(PHASES))] for e in evs])
    pm = {n: float(phase[:, i].mean()) for i, n in enumerate(PHASES)}
    g_bytes = W["n_el"] * 2
    value = job_value(world, g_bytes, ms_step)
    status = [int(w["st"].item()) for w in W["whitened"]]

    pb, rw = phase_bytes(W)
    peak, peak_kind = measured_peaks()
    dom = max(pb, key=lambda n: pm[n])
    achieved = pb[dom] / (pm[dom] * 1e-3) / 1e9
    n_dom = W["n_wh"] if dom.endswith("whitened") else W["n_eu"]
    roofline = {"bound": "hbm", "kernel": f"{dom} (one grouped launch over its layers of the stack)",
                "achieved": achieved, "peak": peak, "peak_source": peak_kind, "unit": "GB/s",
                "frac": achieved / peak,
                "traffic": None, "traffic_detail": traffic_for(dom, n_dom, *rw[dom]),
                "algorithmic_bytes": pb[dom], "algorithmic_read_bytes": rw[dom][0],
                "algorithmic_write_bytes": rw[dom][1]}
    if roofline["traffic_detail"]:
        roofline["traffic"] = roofline["traffic_detail"]["bytes"]
    codec_sum = sum(pm[n] for n in pb)
    codec = {"codec_step_ms": codec_ms, "refresh_batched_ms": refresh_ms, "refresh_layers": len(W["whitened"]),
             "refresh_amortised_ms": refresh_ms / K_REFRESH, "refreshes_timed": R,
             "phase_ms": pm,
             "phase_gbs": {n: pb[n] / (pm[n] * 1e-3) / 1e9 for n in pb},
             "phase_roofline_frac": {n: pb[n] / (pm[n] * 1e-3) / 1e9 / peak for n in pb},
             "codec_gradient_gbs": g_bytes / (codec_sum * 1e-3) / 1e9,
             "codec_roofline_frac": sum(pb.values()) / (codec_sum * 1e-3) / 1e9 / peak,
             "whitened_roofline_frac": (pb["encode_whitened"] + pb["decode_whitened"]) /
                                       ((pm["encode_whitened"] + pm["decode_whitened"]) * 1e-3) / 1e9 / peak,
             "refresh_dev_status": sorted(set(status))}

    launches, names, per_step, per_ref = count_launches(torch, ops, W, K, R)
    bf16_peak = measured_bf16_peak()
    c4 = config4_refresh_measure(torch, ops, synth, dev, bf16_peak) if not args.no_config4 else None
    c2 = config2_batch_measure(torch, ops, synth, dev, peak) if not args.no_config2 else None
    variants = variants_measure(torch, ops, synth, dev, bf16_peak) if not args.no_variants else None
    nvfp4 = nvfp4_measure(torch, ops, synth, dev, peak) if not args.no_nvfp4 else None
    single = layers_measure(torch, ops, synth, dev, peak) if not args.no_layers else None
    stale = staleness_measure(torch, dev) if not args.no_staleness else None

    # ---- end to end through host buffers: every codec step's gradients come
    # in from pinned host memory and G_hat and the error go back; the refresh
    # is timed with the activations of all whitened layers copied in first.
    # Copies in, compute and copies out run on three streams over two device
    # buffer sets, so step k+1's upload and step k-1's download overlap step k
    # (PCIe is full duplex); every byte still crosses inside a timed region.
    e2e = None
    if not args.no_e2e:
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
            done, out_done = {}, {}
            for k in ks:
                S = W["sets"][k % 2]
                with torch.cuda.stream(s_in):
                    if k - 2 in done:
                        s_in.wait_event(done[k - 2])
                    S["G_all"].copy_(G_host, non_blocking=True)
                    ev_in = E()
                    ev_in.record(s_in)
                comp.wait_event(ev_in)
                if k - 2 in out_done:
                    comp.wait_event(out_done[k - 2])
                step(ops, W, k, S=S)
                ev_c = E()
                ev_c.record(comp)
                done[k] = ev_c
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
        a, b = E(enable_timing=True), E(enable_timing=True)
        a.record(comp)
        s_in.wait_event(a)
        last = run_e2e(range(K))
        comp.wait_event(last)
        b.record(comp)
        torch.cuda.synchronize()
        barrier()
        ms_codec_e = max_over_ranks(a.elapsed_time(b), dev) / K
        a, b = E(enable_timing=True), E(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        a.record(comp)
        for w, xh in zip(W["whitened"], X_host):
            w["X"].copy_(xh, non_blocking=True)
        refresh_all(ops, W)
        b.record(comp)
        torch.cuda.synchronize()
        barrier()
        ms_ref_e = max_over_ranks(a.elapsed_time(b), dev)
        ms_e = ms_codec_e + ms_ref_e / K_REFRESH
        e2e = {"value": job_value(world, g_bytes, ms_e), "unit": UNIT,
               "h2d_bytes_per_step": int(g_bytes + x_bytes / K_REFRESH), "d2h_bytes_per_step": int(g_bytes + 24),
               "ms_per_step": ms_e, "codec_step_ms": ms_codec_e, "refresh_with_upload_ms": ms_ref_e,
               "pipeline": "uploads, compute and downloads on three streams over two G / G_hat buffer sets; "
                           "activations uploaded before each timed refresh, amortised over 50 steps"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline()

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
                "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f32", "data": "synthetic",
                "config": {"workload": WORKLOAD, "depth": args.depth, "gradient_elements": W["n_el"],
                           "gradient_bytes": g_bytes, "storage": "bf16 G / e4m3 codes / fp32 scales",
                           "step": "codec step + batched refresh / 50 (Algorithm 1's K = 50), timed separately",
                           "l2": "inputs larger than L2 (1.06 GB of gradients streamed per step)",
                           "parallelism": f"replicas x{world}"},
                "roofline": roofline, "codec": codec, "config2_batch": c2, "config4_refresh": c4, "variants": variants, "layers": single,
                "staleness": stale, "nvfp4": nvfp4, "e2e": e2e, "cpu_baseline": cpu,
                "gpu_launches": launches, "gpu_launches_per_codec_step": per_step,
                "gpu_launches_per_refresh": per_ref, "kernels": names, "clocks": clock_info}
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
    from oracle import gift_oracle as O
    from geometry_aware_fp8_b200 import synth
    warm = max(args.warmup, 0)
    for _ in range(min(warm, 1)):
        cpu_stack_group(O, synth)
    steps = max(1, min(args.steps, 20))
    byt, t_ref, t_codec = 0, 0.0, 0.0
    t0 = time.perf_counter()
    for k in range(steps):
        b, tr, tc = cpu_stack_group(O, synth, seed=11 + 100 * k)
        byt, t_ref, t_codec = byt + b, t_ref + tr, t_codec + tc
    wall = time.perf_counter() - t0
    v = byt / (t_codec + t_ref / K_REFRESH) / 1e9
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        cores = os.cpu_count()
    sample = (f"{steps} x one layer of each stack shape (qkv 4608x1536 and up 4096x1536 Euclidean; o 1536x1536 "
              f"and down 1536x4096 whitened with a refresh from X 8192 x d_in), refresh amortised over "
              f"{K_REFRESH} steps; {wall:.1f} s")
    cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample, "cpu_model": cpu_model(),
           "refresh_s_per_group": t_ref / steps, "codec_s_per_group": t_codec / steps}
    # n_gpus: the N this arm was launched for (it runs on rank 0's host cores)
    n_launch = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": n_launch, "steps": steps,
            "warmup": warm, "ms_per_step": (t_codec + t_ref / K_REFRESH) / steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": sample},
            "cpu_baseline": cpu, "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_gpu(a)
