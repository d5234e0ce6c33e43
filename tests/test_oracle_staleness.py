"""CPU pins of the staleness sweep (review page, "What would settle it";
referee report on section V.E / Algorithm 1: refresh intervals K): the drift
model's rotation and the sweep's bookkeeping of which factor codes which step.
The codec and refresh functions it calls are pinned elsewhere; the error in
whitened coordinates is pinned here by closed forms."""
import numpy as np
import pytest

from oracle import gift_oracle as O
from geometry_aware_fp8_b200 import synth


def test_drift_rotation_is_orthogonal_and_exp_of_the_generator():
    S = synth.drift_generator(64, 5)
    assert np.allclose(S, -S.T)
    R = synth.drift_rotation(64, 0.1, 5)
    assert np.allclose(R.T @ R, np.eye(64), atol=1e-12)
    assert np.allclose(synth.drift_rotation(64, 0.0, 5), np.eye(64))
    # exp(2 theta S) = exp(theta S)^2, and to first order R = I + theta S
    assert np.allclose(synth.drift_rotation(64, 0.2, 5), R @ R, atol=1e-12)
    assert np.allclose(synth.drift_rotation(64, 1e-6, 5), np.eye(64) + 1e-6 * S, atol=1e-11)


def test_drifting_layer_gradient_follows_the_activations():
    steps = synth.drifting_layer(3, 256, 128, 32, 0.05, 11)
    for X, G in steps:
        # G = Delta^T X / N lies in the row space of X
        P = np.linalg.pinv(X) @ X
        assert np.allclose(G @ P, G, atol=1e-10)
    # the principal axis of A_t moves from step to step
    v = [np.linalg.eigh(X.T @ X)[1][:, -1] for X, _ in steps]
    assert abs(v[0] @ v[2]) < 0.9999


def _same_x_steps(T, seed):
    base = synth.drifting_layer(1, 512, 256, 128, 0.0, seed)[0][0]
    rng = np.random.default_rng(seed + 5)
    return [(base, rng.standard_normal((512, 128)).T @ base / 512) for _ in range(T)]


def test_sweep_uses_the_factor_of_the_last_refresh():
    T = 6
    steps = _same_x_steps(T, 21)
    res = O.staleness_sweep(steps, [1, 2, 4], seed=0)
    fresh = O.staleness_sweep(steps, [1], seed=0)
    # each refresh draws its own Rademacher start (seed + step), so the errors
    # of each K are checked against the factor of that K's last refresh
    for K in (1, 2, 4):
        for t in range(T):
            U, lam, rho, _ = O.factor_refresh(O.input_factor(steps[K * (t // K)][0]), 32, 16, 4, seed=K * (t // K))
            c, s = O.encode_e4m3(steps[t][1], U, lam, rho)
            e = O.roundtrip_error(steps[t][1], O.decode_e4m3(c, s, U, lam, rho))
            assert res[K]["frob"][t] == e
    assert res[1] == fresh[1]
    # the Euclidean errors do not depend on K and are the rank-0 codec's
    for t, (_, G) in enumerate(steps):
        c, s = O.quantize_e4m3_blocks(G)
        assert res["euclid"]["frob"][t] == O.roundtrip_error(G, O.dequantize_e4m3_blocks(c, s))


def test_whitened_error_is_measured_with_the_fresh_factor():
    steps = synth.drifting_layer(4, 512, 256, 128, 0.05, 31)
    res = O.staleness_sweep(steps, [4], seed=2)
    U3, l3, r3, _ = O.factor_refresh(O.input_factor(steps[3][0]), 32, 16, 4, seed=5)
    U0, l0, r0, _ = O.factor_refresh(O.input_factor(steps[0][0]), 32, 16, 4, seed=2)
    c, s = O.encode_e4m3(steps[3][1], U0, l0, r0)
    Gh = O.decode_e4m3(c, s, U0, l0, r0)
    assert res[4]["white"][3] == O.whitened_error(steps[3][1], Gh, O.transform_matrix(U3, l3, r3))
    # with the drift the stale factor loses to the fresh one in whitened coordinates
    assert res[4]["white"][3] > res[4]["white"][0]


def test_bf16_output_rounds_g_hat_before_the_errors():
    steps = synth.drifting_layer(2, 512, 256, 128, 0.05, 41)
    res = O.staleness_sweep(steps, [2], seed=4, ghat_bf16=True)
    _, G = steps[1]
    c, s = O.quantize_e4m3_blocks(G)
    assert res["euclid"]["frob"][1] == O.roundtrip_error(G, O.bf16_round(O.dequantize_e4m3_blocks(c, s)))


def test_whitened_error_closed_forms():
    d = 256
    rng = np.random.default_rng(3)
    G = rng.standard_normal((4, d))
    # an error proportional to G is the same fraction in any coordinates
    U = np.linalg.qr(rng.standard_normal((d, 32)))[0]
    lam = np.sort(rng.uniform(1, 10, 32))[::-1]
    M = O.transform_matrix(U, lam, 0.01)
    assert O.whitened_error(G, 1.03 * G, M) == pytest.approx(0.03, rel=1e-12)
    # M = I is the Frobenius round-trip error
    Gh = G + 0.01 * rng.standard_normal(G.shape)
    assert O.whitened_error(G, Gh, np.eye(d)) == pytest.approx(O.roundtrip_error(G, Gh), rel=1e-12)
    # one row along e_1 (inside span U = {e_1}) and an error delta e_2 (outside it):
    # ||(G_hat - G) M|| = delta rho^{-1/2}, ||G M|| = (lambda + rho)^{-1/2}
    E = np.eye(d)
    lam1, rho, delta = 4.0, 0.25, 1e-3
    M1 = O.transform_matrix(E[:, :1], np.array([lam1]), rho)
    got = O.whitened_error(E[:1], E[:1] + delta * E[1:2], M1)
    assert got == pytest.approx(delta * np.sqrt((lam1 + rho) / rho), rel=1e-12)
