"""GPU parity of the staleness measurement against the CPU oracle, through
the C ABI: the error in whitened coordinates (gift_whitened_error) and the
whole sweep on a small drifting layer (review page, "What would settle it")."""
import numpy as np
import pytest
import torch

from oracle import gift_oracle as O
from geometry_aware_fp8_b200 import ops, staleness, synth

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _factor(d_in, seed):
    Q = synth.haar_orthogonal(d_in, seed)
    X = synth.activations(2 * d_in, Q, synth.column_power(d_in, 1.0), seed + 1)
    U, lam, rho, _ = O.factor_refresh(O.input_factor(X), 32, 16, 4, seed=seed)
    return Q, U.astype(np.float32), lam.astype(np.float32), np.float32(rho)


@pytest.mark.parametrize("dtype,d_out,d_in", [("bf16", 300, 512), ("f32", 129, 256), ("bf16", 3, 1536)])
def test_whitened_error_matches_oracle(dtype, d_out, d_in):
    Q, U, lam, rho = _factor(d_in, 60 + d_in)
    G = synth.to_storage(synth.gradient(d_out, Q, 1.0, 61), dtype)
    rng = np.random.default_rng(62)
    Gh = synth.to_storage(G * (1 + 0.05 * rng.standard_normal(G.shape)), dtype)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    Gd, Ghd = torch.from_numpy(G).to(DEV).to(tdt), torch.from_numpy(Gh).to(DEV).to(tdt)
    Ud, ld, rd = torch.from_numpy(U).to(DEV), torch.from_numpy(lam).to(DEV), torch.tensor([rho], device=DEV)
    got = ops.whitened_error(Gd, Ghd, Ud, ld, rd).cpu().numpy()
    # the oracle's projector form with the same fp32 factor (U orthonormal to fp32 rounding)
    M = O.transform_matrix(U.astype(np.float64), lam.astype(np.float64), float(rho))
    want = O.whitened_error(G, Gh, M)
    assert got[0] == pytest.approx(want, rel=1e-4)
    D = (Gh.astype(np.float64) - G) @ M
    assert got[1] == pytest.approx(np.sum(D * D), rel=2e-4)
    # deterministic: a second call gives the same bits
    again = ops.whitened_error(Gd, Ghd, Ud, ld, rd).cpu().numpy()
    assert np.array_equal(got, again)
    # rank 0: M = I, the plain round-trip error
    plain = ops.whitened_error(Gd, Ghd).cpu().numpy()
    assert plain[0] == pytest.approx(O.roundtrip_error(G, Gh), rel=1e-5)


def test_staleness_sweep_matches_oracle():
    T, Ks = 8, [4, 8]
    steps = synth.drifting_layer(T, 1024, 256, 128, 0.05, 7)
    steps = [(synth.to_storage(X, "bf16"), synth.to_storage(G, "bf16")) for X, G in steps]
    want = O.staleness_sweep(steps, Ks, seed=3, ghat_bf16=True)  # the codec returns G_hat in G's dtype
    dev = [(torch.from_numpy(X).to(DEV).to(torch.bfloat16), torch.from_numpy(G).to(DEV).to(torch.bfloat16))
           for X, G in steps]
    got = staleness.sweep(lambda t: dev[t], T, Ks, seed=3)
    for key in ["euclid"] + Ks:
        for m in ("frob", "white"):
            assert np.allclose(got[key][m], want[key][m], rtol=2e-2), (key, m, got[key][m], want[key][m])
    # the stale factor loses to the fresh one as the activations drift
    assert got[8]["white"][7] > 2 * got[8]["white"][0]


def test_device_drift_draws_the_same_model():
    """The device generator follows synth.drifting_layer's recipe: its rotation
    R and basis Q_0 are those of the CPU draws, so A_t's spectrum is i^-2 in a
    basis that turns by R each step."""
    step = staleness.drifting_device(3, 4096, 256, 64, 0.05, 17, dtype=torch.float32, device=DEV)
    R = synth.drift_rotation(256, 0.05, 18)
    Q = synth.haar_orthogonal(256, 17)
    for t in range(3):
        X, G = step(t)
        A = (X.double().T @ X.double() / 4096).cpu().numpy()
        C = Q @ A @ Q.T  # diag(i^-2) up to sampling noise
        diag = np.diag(C)
        assert np.allclose(diag[:8], np.arange(1, 9) ** -2.0, rtol=0.15)
        assert np.abs(C - np.diag(diag)).max() < 0.1 * diag[0]
        Q = Q @ R
