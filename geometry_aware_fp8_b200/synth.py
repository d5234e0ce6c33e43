"""Seeded synthetic inputs for the GIFT gradient codec.

This module only draws random matrices with the shapes and spectra of the
workloads; it holds none of the codec's arithmetic, so both the CUDA library
and the CPU oracle may consume what it produces.  The pages measure on real
Llama-300M/600M activations and gradients, which are not available; these
power-law stand-ins replace them.

Recipes (all fp64 draws from numpy's PCG64 ``default_rng(seed)`` on the CPU,
or torch's Philox generator on a CUDA device for the large stacks, then one
round-to-nearest-even cast to the storage dtype):

* Q: Haar-random orthogonal d x d (QR of a Gaussian matrix with the signs of
  diag(R) folded into Q).
* activations X (N x d_in) = Z diag(sigma) Q, Z iid N(0,1), so that the
  input factor A = X^T X / N has population eigenvalues sigma_i^2.
  ``column_power(a)``: sigma_i = i^-a.  ``spectrum_power(b, spikes, mult)``:
  sigma_i^2 = i^-b, multiplied by ``mult`` for i <= spikes.
* gradient G (d_out x d_in) = Z diag(j^-e) Q^T (the literal form of the
  layer configurations, whose anisotropy axes are not A's), or
  ``aligned=True`` for Z diag(j^-e) Q, whose principal axes coincide with
  the activations' principal axes.
* drifting layer (the staleness sweep): the activation basis rotates slowly,
  Q_t = Q_0 R^t with R = exp(theta S) and S = (B - B^T) / sqrt(2 d) for a
  Gaussian B (skew-symmetric, spectral norm about 2), X_t = Z_t diag(sigma)
  Q_t, and the gradient follows the activations as a linear layer's does,
  G_t = Delta_t^T X_t / N with Delta_t iid N(0,1) of shape N x d_out.
"""
from __future__ import annotations

import numpy as np

try:  # torch is only needed for bf16 casts and device-side stacks
    import torch
except Exception:  # pragma: no cover
    torch = None


def haar_orthogonal(d: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    Z = rng.standard_normal((d, d))
    Q, R = np.linalg.qr(Z)
    return Q * np.sign(np.diag(R))[None, :]


def column_power(d: int, a: float) -> np.ndarray:
    """sigma_i = i^-a, i = 1..d."""
    return np.arange(1, d + 1, dtype=np.float64) ** (-a)


def spectrum_power(d: int, b: float, spikes: int = 0, mult: float = 1.0) -> np.ndarray:
    """sigma_i = sqrt(i^-b), with the first `spikes` eigenvalues multiplied by `mult`."""
    ev = np.arange(1, d + 1, dtype=np.float64) ** (-b)
    ev[:spikes] *= mult
    return np.sqrt(ev)


def activations(N: int, Q: np.ndarray, sigma: np.ndarray, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    Z = rng.standard_normal((N, Q.shape[0]))
    return (Z * sigma[None, :]) @ Q


def gradient(d_out: int, Q: np.ndarray, exponent: float, seed: int,
             aligned: bool = False) -> np.ndarray:
    d_in = Q.shape[0]
    rng = np.random.default_rng(seed)
    Z = rng.standard_normal((d_out, d_in))
    D = column_power(d_in, exponent)
    # X = Z diag(sigma) Q puts A's principal axes on the rows of Q; the
    # literal recipe multiplies by Q^T (axes on Q's columns), the aligned
    # variant by Q (axes shared with A).
    return (Z * D[None, :]) @ (Q if aligned else Q.T)


def drift_generator(d: int, seed: int) -> np.ndarray:
    """S = (B - B^T) / sqrt(2 d), B iid N(0,1): the generator of the drift."""
    rng = np.random.default_rng(seed)
    B = rng.standard_normal((d, d))
    return (B - B.T) / np.sqrt(2.0 * d)


def drift_rotation(d: int, theta: float, seed: int) -> np.ndarray:
    """R = exp(theta S): the orthogonal one-step rotation of the activation basis."""
    from scipy.linalg import expm
    return expm(theta * drift_generator(d, seed))


def drifting_layer(T: int, N: int, d_in: int, d_out: int, theta: float, seed: int, a: float = 1.0):
    """T steps of (X_t, G_t) on the CPU (fp64): X_t = Z_t diag(i^-a) Q_0 R^t,
    G_t = Delta_t^T X_t / N.  Step t draws from default_rng(seed + 1000 + t)."""
    Q = haar_orthogonal(d_in, seed)
    R = drift_rotation(d_in, theta, seed + 1)
    sigma = column_power(d_in, a)
    out = []
    for t in range(T):
        rng = np.random.default_rng(seed + 1000 + t)
        X = (rng.standard_normal((N, d_in)) * sigma[None, :]) @ Q
        D = rng.standard_normal((N, d_out))
        out.append((X, D.T @ X / N))
        Q = Q @ R
    return out


def to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round to the storage dtype ('f32' or 'bf16'); returned as float32 values."""
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    if dtype == "f32":
        return x32
    if dtype == "bf16":
        t = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float32)
        return t.numpy()
    raise ValueError(dtype)


# --------------------------------------------------------------------------
# The five layer configurations (seeds: config k uses 1000k+1 for X,
# 1000k+2 for G, 1000k+3 for Q).
# --------------------------------------------------------------------------

def config1(aligned: bool = False):
    """One 512x512 fp32 layer, X: 2048 rows, sigma_i = i^-1, G exponent 0.8."""
    Q = haar_orthogonal(512, 1003)
    X = activations(2048, Q, column_power(512, 1.0), 1001)
    G = gradient(512, Q, 0.8, 1002, aligned=aligned)
    return to_storage(X, "f32"), to_storage(G, "f32")


def config2():
    """MLP up-projection stand-in: d_in 1536, d_out 4096, bf16, exponent 1.0, X: 8192 rows."""
    Q = haar_orthogonal(1536, 2003)
    X = activations(8192, Q, column_power(1536, 1.0), 2001)
    G = gradient(4096, Q, 1.0, 2002)
    return to_storage(X, "bf16"), to_storage(G, "bf16")


# Llama-600M-sized stand-in layer stack: (name, d_in, d_out, whitened)
STACK_LAYERS = (
    ("qkv", 1536, 4608, False),
    ("o", 1536, 1536, True),
    ("up", 1536, 4096, False),
    ("down", 4096, 1536, True),
)
STACK_DEPTH = 24


def stack_shapes(depth: int = STACK_DEPTH):
    """[(layer index, name, d_out, d_in, whitened)] in stack order."""
    out = []
    for l in range(depth):
        for name, d_in, d_out, wh in STACK_LAYERS:
            out.append((l, name, d_out, d_in, wh))
    return out


def device_gradient(d_out: int, d_in: int, exponent: float, Q_dev, gen, dtype):
    """G = Z diag(j^-e) Q^T drawn on the device (for the full-size stack)."""
    Z = torch.randn((d_out, d_in), generator=gen, device=Q_dev.device, dtype=torch.float32)
    D = torch.arange(1, d_in + 1, device=Q_dev.device, dtype=torch.float32) ** (-exponent)
    return ((Z * D[None, :]) @ Q_dev.T).to(dtype)


def device_activations(N: int, sigma_dev, Q_dev, gen, dtype, chunk: int = 8192):
    """X = Z diag(sigma) Q drawn on the device in row chunks."""
    d = Q_dev.shape[0]
    X = torch.empty((N, d), device=Q_dev.device, dtype=dtype)
    for r0 in range(0, N, chunk):
        r1 = min(N, r0 + chunk)
        Z = torch.randn((r1 - r0, d), generator=gen, device=Q_dev.device, dtype=torch.float32)
        X[r0:r1] = ((Z * sigma_dev[None, :]) @ Q_dev).to(dtype)
    return X
