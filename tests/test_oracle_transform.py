"""Pins for the oracle's transform and codecs (CPU only).

The transform is checked against an independent matrix-function route
(LAPACK eigh of the rank-r-plus-floor factor, raised to -1/2), the exact
inverse, sign invariance, the full-rank isotropy identity, and scaling
laws that are exact in binary floating point.  The codec is checked on
hand-built blocks whose codes are known, on the zero block, against the
per-element E4M3 error bound, and through its NVFP4 counterpart.
"""
import numpy as np
import pytest

from oracle import gift_oracle as O
from geometry_aware_fp8_b200 import synth


def _random_factor(d, r, seed):
    rng = np.random.default_rng(seed)
    U = np.linalg.qr(rng.standard_normal((d, r)))[0]
    lam = np.sort(rng.uniform(0.5, 20.0, r))[::-1]
    rho = 0.07
    return U, lam, rho


def test_transform_is_inverse_sqrt_of_lowrank_plus_floor():
    d, r = 96, 32
    U, lam, rho = _random_factor(d, r, 1)
    Ahat = U @ np.diag(lam) @ U.T + rho * np.eye(d)
    w, V = np.linalg.eigh(Ahat)
    ref = V @ np.diag(w ** -0.5) @ V.T
    M = O.transform_matrix(U, lam, rho)
    assert np.allclose(M, ref, atol=1e-12)
    Minv = O.transform_matrix(U, lam, rho, inverse=True)
    assert np.allclose(Minv, V @ np.diag(w ** 0.5) @ V.T, atol=1e-12)
    assert np.allclose(M @ Minv, np.eye(d), atol=1e-12)


def test_transform_roundtrip_without_quantisation():
    d, r = 128, 32
    U, lam, rho = _random_factor(d, r, 2)
    G = np.random.default_rng(3).standard_normal((40, d))
    W = O.whiten(G, U, lam, rho)
    back = W @ O.transform_matrix(U, lam, rho, inverse=True)
    assert np.max(np.abs(back - G)) / np.max(np.abs(G)) < 1e-12


def test_transform_sign_invariance():
    d, r = 64, 32
    U, lam, rho = _random_factor(d, r, 4)
    flip = np.where(np.arange(r) % 3 == 0, -1.0, 1.0)
    assert np.allclose(O.transform_matrix(U, lam, rho),
                       O.transform_matrix(U * flip, lam, rho), atol=1e-14)


def test_rank_zero_is_euclidean():
    G = np.random.default_rng(5).standard_normal((8, 256)).astype(np.float32)
    U0 = np.zeros((256, 0))
    c1, s1 = O.encode_e4m3(G, U0, np.zeros(0), 1.0)
    c2, s2 = O.quantize_e4m3_blocks(G)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)
    back = O.decode_e4m3(c1, s1, U0, np.zeros(0), 1.0)
    assert np.array_equal(back, O.dequantize_e4m3_blocks(c1, s1))


def test_whitened_activations_are_isotropic_at_full_rank():
    # r = d: M = A^{-1/2}, so the whitened activations have identity second moment
    Q = synth.haar_orthogonal(32, 11)
    X = synth.activations(500, Q, synth.column_power(32, 1.0), 12)
    A = O.input_factor(X)
    U, lam, rho, _ = O.factor_refresh(A, 32)
    Xw = X @ O.transform_matrix(U, lam, rho)
    assert np.allclose(Xw.T @ Xw / X.shape[0], np.eye(32), atol=1e-9)


def test_scaling_activations_by_two_halves_scales_exactly():
    # X -> 2X: A -> 4A, lam -> 4 lam, rho -> 4 rho, M -> M/2, so W halves:
    # identical codes, scales halved exactly.
    Q = synth.haar_orthogonal(256, 21)
    X = synth.activations(600, Q, synth.column_power(256, 1.0), 22)
    G = synth.gradient(16, Q, 1.0, 23).astype(np.float32)
    A = O.input_factor(X)
    U, lam, rho, _ = O.factor_refresh(A, 32, 16, 4, seed=5)
    c1, s1 = O.encode_e4m3(G, U, lam, rho)
    c2, s2 = O.encode_e4m3(G, U, 4 * lam, 4 * rho)
    assert np.array_equal(c1, c2)
    assert np.array_equal(s2, (s1 / 2).astype(np.float32))


def test_rows_are_independent():
    d = 256
    U, lam, rho = _random_factor(d, 32, 6)
    G = np.random.default_rng(7).standard_normal((20, d)).astype(np.float32)
    c, s = O.encode_e4m3(G, U, lam, rho)
    c2, s2 = O.encode_e4m3(G[5:9], U, lam, rho)
    assert np.array_equal(c[5:9], c2) and np.array_equal(s[5:9], s2)


def test_quantize_hand_built_block():
    # block with amax 448*2^-3 = 56: the scale is exactly 1/8 and
    # W*448/amax = 8 W; pick W = v/8 for representable v so codes are exact.
    vals = O.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    rng = np.random.default_rng(0)
    pick = rng.choice(vals, 127)
    v = np.concatenate([[448.0], pick])
    W = (v / 8.0)[None, :]
    codes, scales = O.quantize_e4m3_blocks(W)
    assert scales[0, 0] == np.float32(56.0 / 448.0)
    assert np.array_equal(O.e4m3_decode(codes[0]), v)
    assert np.array_equal(O.dequantize_e4m3_blocks(codes, scales)[0], W[0])


def test_zero_block_and_signed_zero_codes():
    W = np.zeros((2, 256))
    W[1, 128:] = -1e-30
    W[1, 130] = 1.0
    codes, scales = O.quantize_e4m3_blocks(W)
    assert np.all(codes[0] == 0) and np.all(scales[0] == 0)
    assert np.all(codes[1, :128] == 0) and scales[1, 0] == 0
    assert codes[1, 130] == 0x7E
    assert codes[1, 129] == 0x80  # tiny negative value -> signed zero
    assert np.all(O.dequantize_e4m3_blocks(codes, scales)[0] == 0)


def test_e4m3_block_error_bound():
    # |W_hat - W| <= half a mantissa step of E4M3 at |W|, in units of s
    W = np.random.default_rng(9).standard_normal((64, 512)) * np.exp(
        np.random.default_rng(10).uniform(-6, 6, (64, 1)))
    codes, scales = O.quantize_e4m3_blocks(W)
    Wh = O.dequantize_e4m3_blocks(codes, scales)
    W32 = W.astype(np.float32).astype(np.float64)
    s = np.repeat(scales.astype(np.float64), 128, axis=1)
    y = np.abs(W32) / s
    step = np.where(y >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(y, 2.0 ** -6))) - 3), 2.0 ** -9)
    assert np.all(np.abs(Wh - W32) <= (0.5 * step * (1 + 1e-6) + 1e-7 * y) * s)


def test_nvfp4_hand_built_and_bounds():
    # a 16-block scaled so that S_t = 1/448/6*6 ... exact values
    W = np.array([[6.0, -3.0, 1.5, 0.5, 0.0, 2.0, -4.0, 1.0, 0.75, 5.0, -6.0, 3.5, 0.25, 1.25, 1.75, 2.5]])
    packed, sb, St = O.quantize_nvfp4(W)
    assert St == np.float32(6.0 / (6 * 448))
    # amax_b / (6 S_t) = 448 -> scale code 0x7E, value 448, so dq = 448 * S_t = 1
    assert sb[0, 0] == 0x7E
    q = np.empty(16, dtype=np.uint8)
    q[0::2] = packed[0] & 0xF
    q[1::2] = packed[0] >> 4
    want = O.e2m1_encode(W[0])
    assert np.array_equal(q, want)
    back = O.dequantize_nvfp4(packed, sb, St)
    assert np.array_equal(back[0], O.e2m1_decode(want) * 448 * np.float64(St))


def test_nvfp4_zero_tensor():
    packed, sb, St = O.quantize_nvfp4(np.zeros((3, 32)))
    assert St == 0 and np.all(packed == 0) and np.all(sb == 0)


def test_fidelity_report_whitened_norm():
    """Mechanism check (not a pin of the pages' 67 % figure, which used real
    gradients): on gradients built as Delta^T X / N, whitening spreads the
    FP8 error evenly over the directions of A, so the error measured in the
    whitened norm is lower than Euclidean FP8's."""
    d = 256
    Q = synth.haar_orthogonal(d, 31)
    X = synth.activations(4096, Q, synth.column_power(d, 1.0), 32)
    rng = np.random.default_rng(33)
    Delta = rng.standard_normal((4096, 64))
    G = (Delta.T @ X / 4096).astype(np.float32)
    A = O.input_factor(X)
    U, lam, rho, _ = O.factor_refresh(A, 32, 16, 4, seed=1)
    M = O.transform_matrix(U, lam, rho)
    c, s = O.encode_e4m3(G, U, lam, rho)
    Gh = O.decode_e4m3(c, s, U, lam, rho)
    ce, se = O.quantize_e4m3_blocks(G)
    Ge = O.dequantize_e4m3_blocks(ce, se)
    gift_w = O.whitened_error(G, Gh, M)
    eucl_w = O.whitened_error(G, Ge, M)
    assert gift_w < eucl_w


def test_block_too_small_for_the_fp32_reciprocal_is_flushed():
    # 448/amax overflows fp32 for amax below ~1.3e-36: such a block is flushed
    W = np.zeros((1, 256))
    W[0, 5] = -2.5e-38          # 448/2.5e-38 = 1.8e40 > FLT_MAX
    W[0, 130] = 1e-30           # 448/1e-30 = 4.5e32 is representable
    codes, scales = O.quantize_e4m3_blocks(W)
    assert scales[0, 0] == 0 and np.all(codes[0, :128] == 0)
    assert scales[0, 1] == np.float32(1e-30) / np.float32(448) and codes[0, 130] == 0x7E


def test_nvfp4_hand_derived_blocks_between_and_on_scale_ties():
    """Six blocks whose scale ratios amax_b / (6 S_t) fall between E4M3 values
    or exactly on ties (tests/golden/nvfp4_hand_blocks.txt): the block scale
    codes, the element codes and the dequantised values of the oracle must be
    the hand-derived ones."""
    from _golden import nvfp4_hand_blocks
    W, st, sb_want, q_want, _ = nvfp4_hand_blocks()
    packed, sb, St = O.quantize_nvfp4(W)
    assert St == np.float32(st)
    assert np.array_equal(sb[0], sb_want), (sb[0], sb_want)
    q = np.empty(96, dtype=np.uint8)
    q[0::2] = packed[0] & 0xF
    q[1::2] = packed[0] >> 4
    assert np.array_equal(q, q_want), np.nonzero(q != q_want)
    back = O.dequantize_nvfp4(packed, sb, St)[0]
    want = O.e2m1_decode(q_want) * np.repeat(O.e4m3_decode(sb_want), 16) * st
    assert np.array_equal(back, want)
    # the scale of the 8.25 block is 8 (not 9), of the 8.5 tie 8, of the 15.5 tie 16
    assert list(O.e4m3_decode(sb_want[1:5])) == [8.0, 8.0, 16.0, 12.0]
