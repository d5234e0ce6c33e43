"""Plain float64 CPU oracle for the GIFT gradient round trip.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, table or helper with the CUDA library under
``geometry_aware_fp8_b200/``; the two meet only through the seeded input
generators, which hold none of the method's arithmetic.

What it computes (sources):

* GIFT: Geometry-Informed Low-precision Gradient Communication for LLM
  Pretraining (arXiv 2607.07494), review page, "What carries the argument":
  the gradient of a linear layer is moved into coordinates given by the
  input-side K-FAC factor A = E[a a^T], kept at rank 32, quantised to FP8,
  sent, dequantised and mapped back; the optimizer never sees the change.
  Abstract: the same coordinate change serves FP8 and NVFP4.
* Same page, referee report on section V.B / Table II: the factor is kept
  at rank 32.  Section V.E / Algorithm 1: A is refreshed every K = 50 steps.
* The low-rank transform itself is not printed on the pages.  This library
  fixes it as M = rho^{-1/2} I + U diag((lambda+rho)^{-1/2} - rho^{-1/2}) U^T
  with (U, lambda) the top-r eigenpairs of A and rho the mean of A's other
  eigenvalues; the inverse uses exponent +1/2.  Written in projector form,
  M = rho^{-1/2}(I - U U^T) + U diag((lambda+rho)^{-1/2}) U^T, which is the
  same matrix for any U and also covers r = d_in (rho := 0).
* E4M3: "FP8 Formats for Deep Learning" (Micikevicius et al., reference [28]
  of the GIFT paper): 1 sign, 4 exponent bits with bias 7, 3 mantissa bits,
  no infinities, the all-ones pattern S.1111.111 is NaN, largest finite
  value 448, smallest subnormal 2^-9.
* E2M1 (the NVFP4 element, named in the GIFT abstract): 1 sign, 2 exponent
  bits with bias 1, 1 mantissa bit; magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}.

Where a floating-point value decides a code, the oracle takes that decision
in fp32, the precision the GPU kernels work in: W is formed in fp64, rounded
once to fp32, and the block maximum, the reciprocal scale and the scaled
value are fp32 operations with IEEE rounding.  Everything else is fp64.

Pins: every function here is checked in ``tests/test_oracle_*.py`` against
hand-derived format values, brute-force nearest-value search, library
routines (LAPACK eigh, ml_dtypes casts, matrix functions) and closed-form
invariants of the transform.  The fidelity claim of the pages (about 67 %
lower round-trip error than Euclidean FP8 on real Llama-600M gradients,
Tables I-II) is parity unpinned: those gradients are not available.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E2M1_MAX = 6.0
BLOCK_E4M3 = 128
BLOCK_NVFP4 = 16

_F32 = np.float32


# ---------------------------------------------------------------------------
# Scalar number formats (FP8 Formats for Deep Learning, E4M3 definition;
# E2M1 as used by NVFP4).  Vectorised over numpy arrays, exact in fp64.
# ---------------------------------------------------------------------------

def e4m3_decode(codes) -> np.ndarray:
    """Value of each E4M3 byte (NaN for S.1111.111)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = np.ldexp(1.0 + m / 8.0, e - 7)
    sub = np.ldexp(m / 8.0, -6)
    v = np.where(e == 0, sub, normal)
    v = np.where((e == 15) & (m == 7), np.nan, v)
    return sign * v


def e4m3_encode(y) -> np.ndarray:
    """Round-to-nearest-even with saturation to +-448; the sign of zero follows y.

    Values at or above 448 in magnitude clamp to 448 (S.1111.110): inside
    [448, 464) RNE already lands on 448, and from 464 up the neighbour above
    would be the NaN pattern, so saturation returns the largest finite value.
    """
    y = np.asarray(y, dtype=np.float64)
    neg = np.signbit(y)
    a = np.minimum(np.abs(y), E4M3_MAX)
    _, ex = np.frexp(a)                       # a = f * 2**ex, f in [0.5, 1)
    e = ex.astype(np.int64) - 1                # a in [2**e, 2**(e+1))
    normal = (a >= 2.0 ** -6)
    qe = np.where(normal, e, -6) - 3           # exponent of one mantissa step
    r = np.rint(np.ldexp(a, -qe))              # ties to even, exact in fp64
    # normal: r in [8, 16]; subnormal: r in [0, 8]
    E = np.where(normal, e + 7, 0)
    M = np.where(normal, r - 8, r)
    carry = M >= 8
    E = np.where(carry, E + 1, E)
    M = np.where(carry, M - 8, M)
    code = (E.astype(np.int64) << 3) | M.astype(np.int64)
    code = code | np.where(neg, 0x80, 0)
    return code.astype(np.uint8)


def e2m1_decode(codes) -> np.ndarray:
    """Value of each 4-bit E2M1 code (low nibble of the input)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = c & 0x1
    v = np.where(e == 0, 0.5 * m, np.ldexp(1.0 + 0.5 * m, e - 1))
    return sign * v


def e2m1_encode(y) -> np.ndarray:
    """Round-to-nearest-even with saturation to +-6; returns 4-bit codes."""
    y = np.asarray(y, dtype=np.float64)
    neg = np.signbit(y)
    a = np.minimum(np.abs(y), E2M1_MAX)
    _, ex = np.frexp(a)
    e = ex.astype(np.int64) - 1
    normal = a >= 1.0
    qe = np.where(normal, e, 0) - 1            # one mantissa step
    r = np.rint(np.ldexp(a, -qe))
    E = np.where(normal, e + 1, 0)
    M = np.where(normal, r - 2, r)             # normal r in [2, 4]; subnormal [0, 2]
    carry = M >= 2
    E = np.where(carry, E + 1, E)
    M = np.where(carry, M - 2, M)
    code = (E.astype(np.int64) << 1) | M.astype(np.int64)
    code = code | np.where(neg, 0x8, 0)
    return code.astype(np.uint8)


def bf16_round(x) -> np.ndarray:
    """fp64 -> fp32 (RNE) -> bf16 (RNE); returned as float32 holding bf16 values."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) >> 16 << 16
    out = (u & 0xFFFFFFFF).astype(np.uint32).view(np.float32)
    return np.where(np.isnan(f), f, out)


# ---------------------------------------------------------------------------
# Counter-based generator for the random start block of subspace iteration.
# SplitMix64 output function (Steele, Lea & Flood, "Fast splittable
# pseudorandom number generators", OOPSLA 2014), applied to a counter.
# ---------------------------------------------------------------------------

_MASK64 = (1 << 64) - 1


def splitmix64(x: int) -> int:
    z = (x + 0x9E3779B97F4A7C15) & _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def rademacher_start(d: int, m: int, seed: int) -> np.ndarray:
    """Omega[i, j] = +1 if the top bit of splitmix64(seed XOR (i*m + j)) is 0, else -1."""
    om = np.empty((d, m))
    for i in range(d):
        for j in range(m):
            h = splitmix64((seed ^ (i * m + j)) & _MASK64)
            om[i, j] = -1.0 if (h >> 63) else 1.0
    return om


# ---------------------------------------------------------------------------
# Factor refresh: A = X^T X / N, randomised subspace iteration, Rayleigh-Ritz,
# rho = mean of the eigenvalues left out.  (GIFT review page, "What carries
# the argument" and the section V.E / Algorithm 1 refresh of the input-side
# factor; rank 32 from section V.B / Table II.)
# ---------------------------------------------------------------------------

def input_factor(X) -> np.ndarray:
    """A = X^T X / N with X's stored values read exactly (N x d_in -> d_in x d_in)."""
    X = np.asarray(X, dtype=np.float64)
    return (X.T @ X) / X.shape[0]


def householder_q(Y) -> np.ndarray:
    """Thin Q of Y = QR by Householder reflections (columns of Q orthonormal)."""
    Y = np.array(Y, dtype=np.float64, copy=True)
    n, m = Y.shape
    vs = []
    for k in range(m):
        x = Y[k:, k]
        alpha = np.linalg.norm(x)
        v = x.copy()
        if alpha == 0.0:
            vs.append(None)
            continue
        v[0] += np.copysign(alpha, x[0]) if x[0] != 0 else alpha
        v /= np.linalg.norm(v)
        Y[k:, k:] -= 2.0 * np.outer(v, v @ Y[k:, k:])
        vs.append(v)
    Q = np.zeros((n, m))
    Q[:m, :m] = np.eye(m)
    for k in reversed(range(m)):
        v = vs[k]
        if v is None:
            continue
        Q[k:, :] -= 2.0 * np.outer(v, v @ Q[k:, :])
    return Q


def jacobi_eigh(B, sweeps: int = 60, tol: float = 1e-15):
    """Cyclic Jacobi eigen-solver for a small symmetric matrix.

    Returns (w, V) with eigenvalues w in descending order and V's columns the
    matching unit eigenvectors.  Rotation angles follow the classical
    Jacobi choice that zeroes B[p, q] (Golub & Van Loan, section 8.5).
    """
    B = np.array(B, dtype=np.float64, copy=True)
    n = B.shape[0]
    V = np.eye(n)
    for _ in range(sweeps):
        off = np.sqrt(np.sum(np.tril(B, -1) ** 2))
        if off <= tol * np.sqrt(np.sum(B * B)):
            break
        for p in range(n - 1):
            for q in range(p + 1, n):
                bpq = B[p, q]
                if bpq == 0.0:
                    continue
                with np.errstate(over="ignore"):
                    theta = (B[q, q] - B[p, p]) / (2.0 * bpq)
                if abs(theta) > 1e150:          # theta^2 would overflow: t ~ 1/(2 theta)
                    t = 0.5 / theta
                else:
                    t = np.copysign(1.0, theta) / (abs(theta) + np.sqrt(theta * theta + 1.0))
                c = 1.0 / np.sqrt(t * t + 1.0)
                s = t * c
                bp = B[p, :].copy()
                bq = B[q, :].copy()
                B[p, :] = c * bp - s * bq
                B[q, :] = s * bp + c * bq
                bp = B[:, p].copy()
                bq = B[:, q].copy()
                B[:, p] = c * bp - s * bq
                B[:, q] = s * bp + c * bq
                vp = V[:, p].copy()
                vq = V[:, q].copy()
                V[:, p] = c * vp - s * vq
                V[:, q] = s * vp + c * vq
    w = np.diag(B).copy()
    order = np.argsort(-w, kind="stable")
    return w[order], V[:, order]


def factor_refresh(A, rank: int = 32, oversample: int = 16, iters: int = 4,
                   seed: int = 0, rho_floor_rel: float = 2.0 ** -24):
    """Top-`rank` eigenpairs of A by randomised subspace iteration, and rho.

    Steps: Omega (d x (rank+oversample), Rademacher from the counter
    generator); Q = orth(Omega); `iters` times Q = orth(A Q); Rayleigh-Ritz
    B = Q^T A Q, eigenpairs of B by Jacobi, keep the top `rank`, U = Q V;
    rho = (tr A - sum(lambda)) / (d - rank), floored at rho_floor_rel *
    lambda_1.  With rank == d the subspace is the whole space and rho := 0.

    Returns (U [d x rank], lam [rank], rho, flags) where flags has bit 0 set
    when the rho floor was applied.
    """
    A = np.asarray(A, dtype=np.float64)
    d = A.shape[0]
    if rank == d:
        w, V = jacobi_eigh(A)
        return V, w, 0.0, 0
    m = min(rank + oversample, d)
    Q = householder_q(rademacher_start(d, m, seed))
    for _ in range(iters):
        Q = householder_q(A @ Q)
    B = Q.T @ (A @ Q)
    B = 0.5 * (B + B.T)
    w, V = jacobi_eigh(B)
    lam = w[:rank]
    U = Q @ V[:, :rank]
    rho = (np.trace(A) - np.sum(lam)) / (d - rank)
    flags = 0
    floor = rho_floor_rel * lam[0]
    if not rho > floor:
        rho = floor
        flags |= 1
    return U, lam, float(rho), flags


# ---------------------------------------------------------------------------
# Whitening transform and its inverse (projector form of the rank-r
# construction above).
# ---------------------------------------------------------------------------

def transform_matrix(U, lam, rho, inverse: bool = False) -> np.ndarray:
    """M (inverse=False) or M^{-1} (inverse=True) as an explicit d x d matrix.

    M^{+-1} = rho^{-+1/2} (I - U U^T) + U diag((lam + rho)^{-+1/2}) U^T.
    An empty U (rank 0) gives the identity: the Euclidean codec.
    """
    U = np.asarray(U, dtype=np.float64)
    d, r = U.shape
    if r == 0:
        return np.eye(d)
    p = 0.5 if inverse else -0.5
    lam = np.asarray(lam, dtype=np.float64)
    core = U @ np.diag((lam + rho) ** p) @ U.T
    if rho == 0.0:
        return core
    return rho ** p * (np.eye(d) - U @ U.T) + core


# ---------------------------------------------------------------------------
# Per-block E4M3 codec on the whitened gradient.
# ---------------------------------------------------------------------------

def quantize_e4m3_blocks(W, block: int = BLOCK_E4M3):
    """Per-row, per-`block` E4M3 quantisation of W (d_out x d_in).

    For each block: amax = max|W| (fp32); scale s = amax/448 (fp32);
    codes = E4M3_RNE_satfinite(W * fp32(448/amax)).  A block whose amax is 0,
    or so small that fp32(448/amax) overflows, is flushed: s = 0 and all
    codes 0x00.
    """
    W32 = np.asarray(W, dtype=np.float64).astype(_F32)
    d_out, d_in = W32.shape
    nb = d_in // block
    Wb = W32.reshape(d_out, nb, block)
    amax = np.max(np.abs(Wb), axis=2)                       # exact in fp32
    with np.errstate(divide="ignore", over="ignore"):
        inv = (_F32(E4M3_MAX) / np.where(amax > 0, amax, _F32(1))).astype(_F32)
    live = (amax > 0) & np.isfinite(inv)
    inv = np.where(live, inv, _F32(0)).astype(_F32)
    scales = np.where(live, amax / _F32(E4M3_MAX), _F32(0)).astype(_F32)
    y = (Wb * inv[:, :, None]).astype(_F32)
    codes = e4m3_encode(y)
    codes = np.where(live[:, :, None], codes, np.uint8(0)).astype(np.uint8)
    return codes.reshape(d_out, d_in), scales


def dequantize_e4m3_blocks(codes, scales, block: int = BLOCK_E4M3) -> np.ndarray:
    """W_hat = value(code) * s per block (fp64)."""
    codes = np.asarray(codes, dtype=np.uint8)
    d_out, d_in = codes.shape
    nb = d_in // block
    v = e4m3_decode(codes).reshape(d_out, nb, block)
    s = np.asarray(scales, dtype=np.float64).reshape(d_out, nb, 1)
    return (v * s).reshape(d_out, d_in)


def whiten(G, U, lam, rho) -> np.ndarray:
    """W = G M (fp64), M from transform_matrix."""
    return np.asarray(G, dtype=np.float64) @ transform_matrix(U, lam, rho)


def encode_e4m3(G, U, lam, rho, block: int = BLOCK_E4M3):
    """GIFT encode: whiten on the input side, then per-block E4M3.

    Pass an empty U (shape d_in x 0) for the Euclidean codec.
    Returns (codes uint8 [d_out, d_in], scales float32 [d_out, d_in/block]).
    """
    return quantize_e4m3_blocks(whiten(G, U, lam, rho), block)


def decode_e4m3(codes, scales, U, lam, rho, block: int = BLOCK_E4M3) -> np.ndarray:
    """GIFT decode: dequantise, then apply the inverse transform.  fp64 result."""
    W_hat = dequantize_e4m3_blocks(codes, scales, block)
    return W_hat @ transform_matrix(U, lam, rho, inverse=True)


# ---------------------------------------------------------------------------
# NVFP4 codec: E2M1 elements, E4M3 scale per 16 elements, fp32 tensor scale.
# ---------------------------------------------------------------------------

def quantize_nvfp4(W, block: int = BLOCK_NVFP4, S_t=None):
    """Two-level NVFP4 quantisation of W (d_out x d_in), decisions in fp32.

    S_t = amax(W) / (6*448); per block b: s_b = E4M3(amax_b / (6*S_t));
    element codes E2M1(W * fp32(1 / (value(s_b) * S_t))); a block whose
    scale code is zero, or whose reciprocal overflows fp32, gets scale code 0
    and all-zero element codes.
    Returns (codes packed two per byte, low nibble = even column;
    block scale codes uint8 [d_out, d_in/16]; tensor scale float32).
    S_t, if given, is the tensor scale of a larger tensor whose rows W are.
    """
    W32 = np.asarray(W, dtype=np.float64).astype(_F32)
    d_out, d_in = W32.shape
    nb = d_in // block
    if S_t is None:
        amax_t = _F32(np.max(np.abs(W32))) if W32.size else _F32(0)
        S_t = _F32(amax_t / _F32(6.0 * E4M3_MAX))
    else:  # rows of a larger tensor: its tensor scale is given
        S_t = _F32(S_t)
    Wb = W32.reshape(d_out, nb, block)
    amax_b = np.max(np.abs(Wb), axis=2).astype(_F32)
    denom = _F32(_F32(6.0) * S_t)
    if denom > 0:
        ratio = (amax_b / denom).astype(_F32)
    else:
        ratio = np.zeros_like(amax_b)
    sb = e4m3_encode(ratio)
    sbv = e4m3_decode(sb).astype(_F32)
    dq = (sbv * S_t).astype(_F32)
    with np.errstate(divide="ignore", over="ignore"):
        inv = (_F32(1.0) / np.where(dq > 0, dq, _F32(1))).astype(_F32)
    live = (dq > 0) & np.isfinite(inv)
    inv = np.where(live, inv, _F32(0)).astype(_F32)
    sb = np.where(live, sb, np.uint8(0)).astype(np.uint8)
    y = (Wb * inv[:, :, None]).astype(_F32)
    q = e2m1_encode(y)
    q = np.where(live[:, :, None], q, np.uint8(0)).reshape(d_out, d_in)
    packed = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)
    return packed, sb.astype(np.uint8), S_t


def dequantize_nvfp4(packed, sb, S_t, block: int = BLOCK_NVFP4) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    d_out = packed.shape[0]
    d_in = packed.shape[1] * 2
    q = np.empty((d_out, d_in), dtype=np.uint8)
    q[:, 0::2] = packed & 0xF
    q[:, 1::2] = packed >> 4
    v = e2m1_decode(q).reshape(d_out, d_in // block, block)
    s = e4m3_decode(sb).reshape(d_out, d_in // block, 1) * float(S_t)
    return (v * s).reshape(d_out, d_in)


def encode_nvfp4(G, U, lam, rho, block: int = BLOCK_NVFP4):
    return quantize_nvfp4(whiten(G, U, lam, rho), block)


def decode_nvfp4(packed, sb, S_t, U, lam, rho, block: int = BLOCK_NVFP4) -> np.ndarray:
    return dequantize_nvfp4(packed, sb, S_t, block) @ transform_matrix(U, lam, rho, inverse=True)


# ---------------------------------------------------------------------------
# Fidelity metrics (the one-step round-trip error of Tables I-II).
# ---------------------------------------------------------------------------

def roundtrip_error(G, G_hat) -> float:
    """||G_hat - G||_F / ||G||_F in fp64."""
    G = np.asarray(G, dtype=np.float64)
    D = np.asarray(G_hat, dtype=np.float64) - G
    return float(np.sqrt(np.sum(D * D)) / np.sqrt(np.sum(G * G)))


def whitened_error(G, G_hat, M) -> float:
    """||(G_hat - G) M||_F / ||G M||_F: the error measured in whitened coordinates."""
    G = np.asarray(G, dtype=np.float64)
    D = (np.asarray(G_hat, dtype=np.float64) - G) @ M
    W = G @ M
    return float(np.sqrt(np.sum(D * D)) / np.sqrt(np.sum(W * W)))


# ---------------------------------------------------------------------------
# Staleness of the factor (review page, "What would settle it": the round-trip
# error of GIFT against the Euclidean baseline as a function of the steps since
# the last refresh of A; referee report on section V.E / Algorithm 1: refresh
# intervals K in {10, 25, 50, 100}).
# ---------------------------------------------------------------------------

def staleness_sweep(steps, Ks, rank: int = 32, oversample: int = 16, iters: int = 4, seed: int = 0,
                    ghat_bf16: bool = False):
    """Per-step errors of the Euclidean codec and of GIFT with its factor
    refreshed every K steps, for a sequence steps = [(X_t, G_t), ...].

    The factor of step t is the refresh of A_t = X_t^T X_t / N with Rademacher
    seed (seed + t); GIFT under interval K codes G_t with the factor of step
    K floor(t / K).  Errors: the Frobenius round-trip error and the error in
    the coordinates whitened by the fresh factor of step t (the geometry the
    gradient has at that step).  G_hat is kept in fp64, or rounded to bf16 by
    round-to-nearest-even (ghat_bf16) as a codec whose G is bf16 returns it.
    Returns {"euclid": {"frob": [...], "white": [...]}, K: {"frob": [...],
    "white": [...]}, ...}."""
    fresh = []
    for t, (X, _) in enumerate(steps):
        U, lam, rho, _ = factor_refresh(input_factor(X), rank, oversample, iters, seed=seed + t)
        fresh.append((U, lam, rho))
    M_now = [transform_matrix(*f) for f in fresh]
    empty = np.zeros((steps[0][1].shape[1], 0))
    out_round = bf16_round if ghat_bf16 else (lambda x: x)
    out = {"euclid": {"frob": [], "white": []}}
    for t, (_, G) in enumerate(steps):
        c, s = encode_e4m3(G, empty, np.zeros(0), 1.0)
        Gh = out_round(decode_e4m3(c, s, empty, np.zeros(0), 1.0))
        out["euclid"]["frob"].append(roundtrip_error(G, Gh))
        out["euclid"]["white"].append(whitened_error(G, Gh, M_now[t]))
    for K in Ks:
        out[K] = {"frob": [], "white": []}
        for t, (_, G) in enumerate(steps):
            f = fresh[K * (t // K)]
            c, s = encode_e4m3(G, *f)
            Gh = out_round(decode_e4m3(c, s, *f))
            out[K]["frob"].append(roundtrip_error(G, Gh))
            out[K]["white"].append(whitened_error(G, Gh, M_now[t]))
    return out


# ---------------------------------------------------------------------------
# The variants GIFT is simplified from (review page, "What carries the
# argument": full two-sided K-FAC whitening, then the input side alone, then
# rank 32; section IV.A, Eq. (14) writes the input-side Cholesky form L_A^{-T},
# which the referee report's minor comment 3 reads as (L_A^{-1})^T).  Oracle
# only: the library codes the rank-r eigen transform.
# ---------------------------------------------------------------------------

def full_rank_transform(A, inverse: bool = False) -> np.ndarray:
    """A^{-1/2} (inverse: A^{1/2}) by LAPACK eigh: the rank-r construction at
    r = d_in, where the floor rho is empty (reading C3: rho := 0)."""
    lam, V = np.linalg.eigh(np.asarray(A, dtype=np.float64))
    p = 0.5 if inverse else -0.5
    return (V * lam ** p) @ V.T


def cholesky_transform(A, inverse: bool = False) -> np.ndarray:
    """L^{-T} with A = L L^T (Eq. 14's L_A^{-T}); inverse: L^T.  W = G L^{-T}
    has input-side covariance L^{-1} A L^{-T} = I."""
    L = np.linalg.cholesky(np.asarray(A, dtype=np.float64))
    if inverse:
        return L.T
    return np.linalg.inv(L).T


def encode_dense(G, M, block: int = BLOCK_E4M3):
    """Per-block E4M3 of W = G M for a dense d_in x d_in transform M (the
    full-rank or Cholesky variant): (codes, scales) as encode_e4m3."""
    return quantize_e4m3_blocks(np.asarray(G, dtype=np.float64) @ np.asarray(M, dtype=np.float64), block)


def decode_dense(codes, scales, M_inv, block: int = BLOCK_E4M3) -> np.ndarray:
    """G_hat = W_hat M^{-1} for a dense transform (fp64)."""
    return dequantize_e4m3_blocks(codes, scales, block) @ np.asarray(M_inv, dtype=np.float64)


def two_sided_encode_decode(G, A, B, block: int = BLOCK_E4M3):
    """Full two-sided Cholesky whitening: W = L_B^{-1} G L_A^{-T}, per-block
    E4M3, G_hat = L_B W_hat L_A^T (B = E[delta delta^T], the output-side
    factor, d_out x d_out)."""
    LB = np.linalg.cholesky(np.asarray(B, dtype=np.float64))
    W = np.linalg.solve(LB, np.asarray(G, dtype=np.float64)) @ cholesky_transform(A)
    c, s = quantize_e4m3_blocks(W, block)
    return LB @ dequantize_e4m3_blocks(c, s, block) @ cholesky_transform(A, inverse=True)


def transform_comparison(G, X, Delta, rank: int = 32, oversample: int = 16, iters: int = 4, seed: int = 0):
    """Round-trip errors of the E4M3 codec under each coordinate choice, for a
    layer with activations X (N x d_in), output-side errors Delta (N x d_out)
    and gradient G (d_out x d_in): Euclidean, input-side rank-r (the codec's
    transform), input-side full rank (A^{-1/2}), input-side Cholesky (L_A^{-T})
    and two-sided Cholesky.  Each reports the Frobenius error and the error in
    the coordinates whitened by the input-side A^{-1/2} (a Table I/II-style
    comparison on synthetic data)."""
    A = input_factor(X)
    B = input_factor(Delta)
    M_ref = full_rank_transform(A)
    U, lam, rho, _ = factor_refresh(A, rank, oversample, iters, seed=seed)
    out = {}

    def record(name, Gh):
        out[name] = {"frob": roundtrip_error(G, Gh), "white": whitened_error(G, Gh, M_ref)}

    c, s = quantize_e4m3_blocks(G)
    record("euclid", dequantize_e4m3_blocks(c, s))
    c, s = encode_e4m3(G, U, lam, rho)
    record(f"input_rank{rank}", decode_e4m3(c, s, U, lam, rho))
    for name, fn in (("input_full", full_rank_transform), ("input_cholesky", cholesky_transform)):
        c, s = quantize_e4m3_blocks(np.asarray(G, dtype=np.float64) @ fn(A))
        record(name, dequantize_e4m3_blocks(c, s) @ fn(A, inverse=True))
    record("two_sided_cholesky", two_sided_encode_decode(G, A, B))
    return out
