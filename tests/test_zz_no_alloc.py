"""The allocation-free factor refresh against the regular one (GPU).

gift_factor_refresh_noalloc serves callers that cannot give the library a
workspace (their device memory belongs to another allocator, or they may
not call cudaMalloc in that step).  It must return what gift_factor_refresh
returns, within the refresh tolerances: top-32 eigenvalues within 1e-4
relative, rho within the fp32-accumulation bound of its numerator, A within
1e-5 of max|A|, and the transform within 1e-2 in relative Frobenius norm.
Two calls in a row check that the shared scratch array is reused cleanly,
and every call must leave its device status word at zero.  One case is also
compared with the CPU oracle directly, under the same criteria.
This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from oracle import gift_oracle as O
from geometry_aware_fp8_b200 import ops, synth

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _rho_tol(rho, trace, N, d, r):
    return max(1e-4 * rho, 2.0 ** -24 * np.sqrt(N) * trace / (d - r))


def _compare(ref, got, A_ref, A_got, N):
    U0, l0, r0, _ = [t.cpu().numpy().astype(np.float64) for t in ref]
    U1, l1, r1, s1 = [t.cpu().numpy().astype(np.float64) for t in got]
    assert int(s1[0]) == 0, f"device status {int(s1[0]):#x}"
    A0 = A_ref.cpu().numpy().astype(np.float64)
    A1 = A_got.cpu().numpy().astype(np.float64)
    d, r = U0.shape
    assert np.max(np.abs(A1 - A0)) <= 1e-5 * np.max(np.abs(A0))
    assert np.allclose(l1, l0, rtol=1e-4, atol=0)
    assert abs(r1[0] - r0[0]) <= _rho_tol(r0[0], np.trace(A0), N, d, r)
    M0 = O.transform_matrix(U0, l0, r0[0])
    M1 = O.transform_matrix(U1, l1, r1[0])
    assert np.linalg.norm(M1 - M0) / np.linalg.norm(M0) < 1e-2


@pytest.mark.parametrize("N,d,dtype,rank,over", [(8192, 1536, "bf16", 32, 16), (4096, 4096, "bf16", 32, 16),
                                                 (2048, 512, "f32", 32, 16), (4096, 4096, "bf16", 48, 16)])
def test_noalloc_refresh_matches_regular_refresh_twice(N, d, dtype, rank, over):
    Q = synth.haar_orthogonal(d, 77 + d)
    X = synth.to_storage(synth.activations(N, Q, synth.column_power(d, 1.0), 78), dtype)
    Xd = torch.from_numpy(X).to(DEV)
    if dtype == "bf16":
        Xd = Xd.to(torch.bfloat16)
    A_ref = torch.empty((d, d), device=DEV, dtype=torch.float32)
    ref = ops.factor_refresh(Xd, rank, over, 4, 9, A_out=A_ref)
    first = None
    for call in range(2):
        A_got = torch.empty((d, d), device=DEV, dtype=torch.float32)
        got = ops.factor_refresh_noalloc(Xd, A_got, rank, over, 4, 9)
        torch.cuda.synchronize()
        _compare(ref, got, A_ref, A_got, N)
        if first is None:
            first = [t.clone() for t in got[:3]]
        else:
            for a, b in zip(first, got[:3]):
                assert torch.equal(a, b)


def test_noalloc_refresh_matches_oracle():
    """One case against the CPU oracle directly (config 1's shape: X 2048 x
    512 fp32, sigma_i = i^-1): A, the top-32 eigenvalues, rho, the floor bit,
    U's orthonormality, the Ritz property and the transform, under the
    criteria of the regular refresh's parity tests."""
    d, N = 512, 2048
    Q = synth.haar_orthogonal(d, 1003)
    X = synth.activations(N, Q, synth.column_power(d, 1.0), 1001).astype(np.float32)
    Xd = torch.from_numpy(X).to(DEV)
    A_got = torch.empty((d, d), device=DEV, dtype=torch.float32)
    U, lam, rho, st = ops.factor_refresh_noalloc(Xd, A_got, 32, 16, 4, 1004)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    A = O.input_factor(X)
    Uo, lo, ro, fo = O.factor_refresh(A, 32, 16, 4, seed=1004)
    Ag = A_got.cpu().numpy().astype(np.float64)
    Ug, lg, rg = U.cpu().numpy().astype(np.float64), lam.cpu().numpy().astype(np.float64), float(rho.item())
    assert np.max(np.abs(Ag - A)) <= 1e-5 * np.max(np.abs(A))
    assert np.allclose(lg, lo, rtol=1e-4, atol=0)
    assert abs(rg - ro) <= _rho_tol(ro, np.trace(A), N, d, 32), (rg, ro)
    assert fo == 0
    assert np.max(np.abs(Ug.T @ Ug - np.eye(32))) < 1e-5
    assert np.max(np.abs(Ug.T @ A @ Ug - np.diag(lg))) < 1e-4 * lg[0]
    Mg, Mo = O.transform_matrix(Ug, lg, rg), O.transform_matrix(Uo, lo, ro)
    assert np.linalg.norm(Mg - Mo) / np.linalg.norm(Mo) < 1e-2


def test_noalloc_refresh_rejects_what_it_cannot_hold():
    X = torch.zeros((256, 4224), device=DEV, dtype=torch.bfloat16)
    A = torch.empty((4224, 4224), device=DEV, dtype=torch.float32)
    with pytest.raises(ops.GiftError) as e:
        ops.factor_refresh_noalloc(X, A, 32, 16, 4, 0)
    assert e.value.status == 2  # GIFT_ERR_SHAPE: d_in above 4096
    X = torch.zeros((256, 512), device=DEV, dtype=torch.bfloat16)
    A = torch.empty((512, 512), device=DEV, dtype=torch.float32)
    with pytest.raises(ops.GiftError) as e:
        ops.factor_refresh_noalloc(X, A, 48, 17, 4, 0)
    assert e.value.status == 2  # rank + oversample above 64
    L = ops.lib()
    st = L.gift_factor_refresh_noalloc(X.data_ptr(), 1, 256, 512, 32, 16, 4, 0, A.data_ptr(), A.data_ptr(),
                                       A.data_ptr(), None, None, None)
    assert st == 1  # GIFT_ERR_INVALID_ARG: A_out is required
