"""GPU parity of the factor refresh against the CPU oracle, through the C ABI.

Criteria: A entries within 1e-5 of max|A| (fp32 accumulation of exact bf16/fp32
products); the top-32 Ritz values within 1e-4 relative (same algorithm, same
SplitMix64 start block); U orthonormal to 1e-5; rho within 1e-4 relative or
within the fp32-accumulation bound of its numerator: rho = (tr A - sum
lambda)/(d - r) is a small difference of two sums of size tr A, and A's
diagonal carries the rounding of an fp32 sum over N tokens, about
2^-24 sqrt(N) relative, so |d rho| <= 2^-24 sqrt(N) tr(A) / (d - r);
the Ritz property U^T A U = diag(lambda) on the oracle's fp64 A.  The
transform M is compared in relative Frobenius norm within 1e-2: after four
iterations the Ritz vectors next to the rank cut (lambda_32 vs lambda_33)
rotate by about |dB| / (theta_32 - theta_33), which for fp32 arithmetic and
the i^-2 spectra here is ~1e-3 of M's norm.
"""
import numpy as np
import pytest
import torch

from oracle import gift_oracle as O
from geometry_aware_fp8_b200 import ops, synth

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _refresh_both(X, rank=32, over=16, iters=4, seed=7, dtype="f32"):
    Xs = synth.to_storage(X, dtype)
    Xd = torch.from_numpy(Xs).to(DEV)
    if dtype == "bf16":
        Xd = Xd.to(torch.bfloat16)
    d = X.shape[1]
    A_out = torch.empty((d, d), device=DEV, dtype=torch.float32)
    U, lam, rho, st = ops.factor_refresh(Xd, rank, over, iters, seed, A_out=A_out)
    torch.cuda.synchronize()
    A = O.input_factor(Xs)
    Uo, lo, ro, fo = O.factor_refresh(A, rank, over, iters, seed=seed)
    return (A_out.cpu().numpy().astype(np.float64), U.cpu().numpy().astype(np.float64),
            lam.cpu().numpy().astype(np.float64), float(rho.item()), int(st.item())), (A, Uo, lo, ro, fo)


def rho_tol(rho, trace, N, d, r):
    return max(1e-4 * rho, 2.0 ** -24 * np.sqrt(N) * trace / (d - r))


def _check(gpu, orc, N, m_tol=1e-2):
    Ag, Ug, lg, rg, sg = gpu
    A, Uo, lo, ro, fo = orc
    assert np.max(np.abs(Ag - A)) <= 1e-5 * np.max(np.abs(A))
    assert np.allclose(lg, lo, rtol=1e-4, atol=0)
    assert abs(rg - ro) <= rho_tol(ro, np.trace(A), N, A.shape[0], Ug.shape[1]), (rg, ro)
    assert (sg & ops.DEV_RHO_FLOORED) == (fo & 1)
    r = Ug.shape[1]
    assert np.max(np.abs(Ug.T @ Ug - np.eye(r))) < 1e-5
    R = Ug.T @ A @ Ug
    assert np.max(np.abs(R - np.diag(lg))) < 1e-4 * lg[0]
    Mg = O.transform_matrix(Ug, lg, rg)
    Mo = O.transform_matrix(Uo, lo, ro)
    assert np.linalg.norm(Mg - Mo) / np.linalg.norm(Mo) < m_tol


def test_refresh_config1_fp32():
    """One 512-wide layer: X 2048 x 512 fp32, sigma_i = i^-1."""
    Q = synth.haar_orthogonal(512, 1003)
    X = synth.activations(2048, Q, synth.column_power(512, 1.0), 1001)
    g, o = _refresh_both(X, dtype="f32", seed=1004)
    _check(g, o, 2048)


def test_refresh_bf16_spiked_spectrum():
    """bf16 X with the config-4 spectrum shape (i^-1.2, five spikes of 100x), scaled down."""
    d = 1024
    Q = synth.haar_orthogonal(d, 11)
    X = synth.activations(4096, Q, synth.spectrum_power(d, 1.2, 5, 100.0), 12)
    g, o = _refresh_both(X, dtype="bf16", seed=13)
    _check(g, o, 4096)


@pytest.mark.parametrize("rank,over,iters", [(8, 8, 2), (32, 0, 3), (16, 17, 1)])
def test_refresh_rank_and_oversample_variants(rank, over, iters):
    d = 256
    Q = synth.haar_orthogonal(d, 21)
    X = synth.activations(1024, Q, synth.spectrum_power(d, 2.0), 22)
    g, o = _refresh_both(X, rank, over, iters, seed=23)
    _check(g, o, 1024, m_tol=5e-2)


def test_refresh_rank_deficient_input_sets_status():
    """N = 20 tokens < rank + oversample: A has rank 20, the sampled subspace
    loses columns (status bit), the nonzero Ritz values still match."""
    d = 128
    Q = synth.haar_orthogonal(d, 31)
    X = synth.activations(20, Q, synth.column_power(d, 0.5), 32)
    g, o = _refresh_both(X, 32, 16, 2, seed=33)
    Ag, Ug, lg, rg, sg = g
    A, Uo, lo, ro, fo = o
    assert sg & ops.DEV_RANK_DEFICIENT
    assert sg & ops.DEV_RHO_FLOORED and fo & 1
    assert np.allclose(lg[:20], lo[:20], rtol=1e-4)
    assert np.all(np.isfinite(Ug)) and np.isfinite(rg) and rg > 0


def test_refresh_is_deterministic():
    d = 512
    Q = synth.haar_orthogonal(d, 41)
    X = torch.from_numpy(synth.activations(2048, Q, synth.column_power(d, 1.0), 42).astype(np.float32)).to(DEV)
    a = ops.factor_refresh(X, 32, 16, 4, 5)
    b = ops.factor_refresh(X, 32, 16, 4, 5)
    for x, y in zip(a[:3], b[:3]):
        assert torch.equal(x, y)


def test_refresh_config2_bf16_split_k():
    """MLP up-projection stand-in: X 8192 x 1536 bf16 (sigma_i = i^-1); the
    tensor-core syrk splits the token range four ways here."""
    Q = synth.haar_orthogonal(1536, 2003)
    X = synth.activations(8192, Q, synth.column_power(1536, 1.0), 2001)
    g, o = _refresh_both(X, dtype="bf16", seed=2004)
    _check(g, o, 8192)


@pytest.fixture(scope="module")
def config4():
    """Factor refresh at scale: X 65536 x 4096 bf16, eigenvalues i^-1.2 with
    five 100x spikes, 4 iterations, oversample 16, on the GPU."""
    N, d = 65536, 4096
    gen = torch.Generator(device=DEV)
    gen.manual_seed(4001)
    Qd = torch.from_numpy(synth.haar_orthogonal(d, 4003).astype(np.float32)).to(DEV)
    sig = torch.from_numpy(synth.spectrum_power(d, 1.2, 5, 100.0).astype(np.float32)).to(DEV)
    X = synth.device_activations(N, sig, Qd, gen, torch.bfloat16)
    A_out = torch.empty((d, d), device=DEV, dtype=torch.float32)
    U, lam, rho, st = ops.factor_refresh(X, 32, 16, 4, 4004, A_out=A_out)
    torch.cuda.synchronize()
    Xh = X.float().cpu().numpy()
    del X
    out = dict(N=N, d=d, Xh=Xh, A=A_out.cpu().numpy(), U=U.cpu().numpy().astype(np.float64),
               lam=lam.cpu().numpy().astype(np.float64), rho=float(rho.item()), st=int(st.item()))
    del A_out
    torch.cuda.empty_cache()
    yield out


def test_refresh_config4_full_size_properties(config4):
    """Config 4 checked through what holds at any size: sampled entries of A
    (exact fp64 dot products of bf16 columns), the Rayleigh-Ritz property
    (XU)^T (XU) / N = diag(lambda) in fp64, and rho against the trace
    identity on the GPU's own U."""
    N, d, Xh, Ah = config4["N"], config4["d"], config4["Xh"], config4["A"]
    assert config4["st"] == 0
    rng = np.random.default_rng(0)
    idx = rng.integers(0, d, size=(200, 2))
    idx[:20, 1] = idx[:20, 0]                       # include diagonal entries
    want = np.array([np.dot(Xh[:, i].astype(np.float64), Xh[:, j].astype(np.float64)) / N for i, j in idx])
    got = Ah[idx[:, 0], idx[:, 1]]
    scale = np.sqrt(Ah[idx[:, 0], idx[:, 0]].astype(np.float64) * Ah[idx[:, 1], idx[:, 1]])
    assert np.max(np.abs(got - want) / scale) < 1e-5
    assert np.array_equal(Ah, Ah.T)
    Ug, lg = config4["U"], config4["lam"]
    XU = np.zeros((32, 32))
    fro = 0.0
    for r0 in range(0, N, 8192):
        blk = Xh[r0:r0 + 8192].astype(np.float64)
        P = blk @ Ug
        XU += P.T @ P
        fro += np.sum(blk * blk)
    R = XU / N
    assert np.allclose(np.diag(R), lg, rtol=1e-4)
    assert np.max(np.abs(R - np.diag(np.diag(R)))) < 1e-4 * lg[0]
    rho = config4["rho"]
    rho_ref = (fro / N - np.trace(R)) / (d - 32)
    rel = abs(rho - rho_ref) / rho_ref
    print(f"config4 rho {rho:.6e} vs trace identity {rho_ref:.6e} (rel {rel:.2e}); lambda_1 {lg[0]:.4f}")
    assert abs(rho - rho_ref) <= rho_tol(rho_ref, fro / N, N, d, 32)


def test_refresh_config4_matches_oracle(config4):
    """Config 4 against the oracle at full size: the oracle forms A = X^T X / N
    in fp64 from the same 65536 x 4096 bf16 activations and runs its own
    subspace iteration (Householder QR, Jacobi) from the same SplitMix64 start
    block.  Criteria as for every refresh: A within 1e-5 of max|A|, the top-32
    eigenvalues within 1e-4 relative, rho within its fp32-accumulation bound,
    the floor bit equal, U orthonormal, U^T A U = diag(lambda), and the
    transform M within 1e-2 in relative Frobenius norm."""
    N = config4["N"]
    A = O.input_factor(config4["Xh"])
    Uo, lo, ro, fo = O.factor_refresh(A, 32, 16, 4, seed=4004)
    gpu = (config4["A"].astype(np.float64), config4["U"], config4["lam"], config4["rho"], config4["st"])
    lam_rel = np.max(np.abs(config4["lam"] - lo) / lo)
    print(f"config4 vs oracle: max lambda rel err {lam_rel:.2e}, rho {config4['rho']:.6e} vs {ro:.6e} "
          f"(rel {abs(config4['rho'] - ro) / ro:.2e}); oracle lambda_1 {lo[0]:.4f}, lambda_32 {lo[31]:.6f}")
    _check(gpu, (A, Uo, lo, ro, fo), N)


def test_refresh_many_matches_single_refreshes_bitwise():
    """The batched refresh runs the same arithmetic per layer, side by side:
    each layer's result must equal its single refresh bit for bit (mixed
    widths and dtypes in one batch)."""
    specs = [(2048, 512, "f32", 3), (4096, 1536, "bf16", 4), (1024, 256, "bf16", 5), (8192, 1536, "bf16", 6)]
    items, singles = [], []
    for N, d, dtype, seed in specs:
        Q = synth.haar_orthogonal(d, 100 + seed)
        X = synth.to_storage(synth.activations(N, Q, synth.column_power(d, 1.0), 200 + seed), dtype)
        Xd = torch.from_numpy(X).to(DEV)
        if dtype == "bf16":
            Xd = Xd.to(torch.bfloat16)
        singles.append(ops.factor_refresh(Xd, 32, 16, 4, seed))
        U = torch.empty((d, 32), device=DEV)
        lam = torch.empty((32,), device=DEV)
        rho = torch.empty((1,), device=DEV)
        ws = torch.empty((ops.refresh_workspace_size(N, d, 32, 16),), device=DEV, dtype=torch.uint8)
        st = torch.zeros((1,), device=DEV, dtype=torch.int32)
        items.append((Xd, U, lam, rho, ws, st, seed, None))
    jobs = ops.make_refresh_jobs(items)
    ops.factor_refresh_many(jobs, len(items), 32, 16, 4)
    torch.cuda.synchronize()
    for (Xd, U, lam, rho, ws, st, seed, _), single in zip(items, singles):
        assert torch.equal(U, single[0]) and torch.equal(lam, single[1]) and torch.equal(rho, single[2])
        assert int(st.item()) == int(single[3].item())
