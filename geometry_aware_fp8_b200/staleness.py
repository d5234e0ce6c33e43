"""Staleness of the input factor on the GPU.

GIFT review page, "What would settle it": measure the FP8 round-trip error of
GIFT against the Euclidean baseline as a function of the steps since the last
refresh of A; if just before a refresh the error reaches the Euclidean one,
the benefit depends on the refresh interval.  The referee report on section
V.E / Algorithm 1 asks for the intervals K in {10, 25, 50, 100}.

``sweep`` runs that measurement over a sequence of steps whose activations
drift (``synth.drifting_layer`` on the CPU, ``drifting_device`` here on the
device).  At every step t it refreshes the factor of A_t (the geometry the
gradient has at t), codes G_t with the Euclidean codec and, for each K, with
GIFT under the factor refreshed at step K floor(t / K); it records the
Frobenius round-trip error and the error in the coordinates whitened by the
fresh factor of step t.  Every refresh, codec and error step runs in the
library's kernels (gift_factor_refresh, gift_encode, gift_decode,
gift_roundtrip_error, gift_whitened_error); torch draws the synthetic inputs
and holds device memory.
"""
from __future__ import annotations

import numpy as np
import torch

from . import ops, synth


def sweep(step_inputs, T: int, Ks, rank: int = 32, oversample: int = 16, iters: int = 4, seed: int = 0):
    """step_inputs(t) -> (X_t, G_t) on the device.  Returns per-step errors as
    {"euclid": {"frob": [...], "white": [...]}, K: {"frob": [...], "white": [...]}}
    (Python floats; the factor of step t uses Rademacher seed (seed + t))."""
    fresh = []
    rec = {"euclid": []}
    for K in Ks:
        rec[K] = []
    ws_e = ws_w = None
    for t in range(T):
        X, G = step_inputs(t)
        U, lam, rho, _ = ops.factor_refresh(X, rank, oversample, iters, seed=seed + t)
        fresh.append((U, lam, rho))
        del X
        d_out, d_in = G.shape
        if ws_e is None:
            ws_e = torch.empty((ops.error_workspace_size(d_out, d_in),), device=G.device, dtype=torch.uint8)
            ws_w = torch.empty((ops.whitened_error_workspace_size(d_out, d_in),), device=G.device, dtype=torch.uint8)

        def errors(Gh):
            e = ops.roundtrip_error(G, Gh, ws=ws_e)
            w = ops.whitened_error(G, Gh, U, lam, rho, ws=ws_w)
            return torch.stack((e[0], w[0]))

        codes, scales = ops.encode(G)
        rec["euclid"].append(errors(ops.decode(codes, scales, out_dtype=G.dtype)))
        for K in Ks:
            f = fresh[K * (t // K)]
            codes, scales = ops.encode(G, *f)
            rec[K].append(errors(ops.decode(codes, scales, *f, out_dtype=G.dtype)))
    out = {}
    for key, vals in rec.items():
        v = torch.stack(vals).cpu().numpy()
        out[key] = {"frob": v[:, 0].tolist(), "white": v[:, 1].tolist()}
    return out


def drifting_device(T: int, N: int, d_in: int, d_out: int, theta: float, seed: int, dtype=torch.bfloat16,
                    device="cuda:0", a: float = 1.0):
    """step_inputs for ``sweep`` with the drift model of ``synth.drifting_layer``
    drawn on the device: Q_0 and the generator S come from the same seeded CPU
    draws, R = exp(theta S) is formed once on the device, and step t draws
    Z_t and Delta_t from a torch generator seeded with seed + 1000 + t."""
    Q0 = torch.from_numpy(synth.haar_orthogonal(d_in, seed).astype(np.float32)).to(device)
    S = torch.from_numpy(synth.drift_generator(d_in, seed + 1)).to(device)
    R = torch.linalg.matrix_exp(theta * S).to(torch.float32)
    sigma = torch.arange(1, d_in + 1, device=device, dtype=torch.float32) ** (-a)
    state = {"t": 0, "Q": Q0}

    def step(t):
        if t != state["t"]:
            raise ValueError("steps must be drawn in order")
        gen = torch.Generator(device=device)
        gen.manual_seed(seed + 1000 + t)
        Z = torch.randn((N, d_in), generator=gen, device=device, dtype=torch.float32)
        X = (Z * sigma[None, :]) @ state["Q"]
        D = torch.randn((N, d_out), generator=gen, device=device, dtype=torch.float32)
        G = (D.T @ X) / N
        state["Q"] = state["Q"] @ R
        state["t"] = t + 1
        return X.to(dtype), G.to(dtype)

    return step


def summary(res, Ks):
    """Mean errors by the factor's age (steps since its refresh) for each K,
    against the Euclidean codec over the same steps."""
    eu_f = float(np.mean(res["euclid"]["frob"]))
    eu_w = float(np.mean(res["euclid"]["white"]))
    out = {"euclid": {"frob": eu_f, "white": eu_w}}
    for K in Ks:
        f = np.asarray(res[K]["frob"])
        w = np.asarray(res[K]["white"])
        age = np.arange(len(f)) % K
        last = age == min(K - 1, len(f) - 1)
        out[f"K={K}"] = {"white_fresh": float(w[age == 0].mean()), "white_stalest": float(w[last].mean()),
                         "white_mean": float(w.mean()), "frob_fresh": float(f[age == 0].mean()),
                         "frob_stalest": float(f[last].mean()), "frob_mean": float(f.mean()),
                         "stalest_reaches_euclid_white": bool(w[last].mean() >= eu_w)}
    return out
