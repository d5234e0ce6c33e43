"""Parity at the benchmark's full size, in the launch configuration bench.py
times: the 24-layer stack (528.5 M gradient elements) built by the bench's own
workload builder, one batched refresh of the 48 whitened layers, then one step
of grouped encodes and decodes.  The oracle cannot redo the whole stack in
seconds, so it checks what it can compute piece by piece:

  * codec rows: every row of G is coded independently given the factor, so
    sampled rows (first, middle and last panel) of sampled whitened and
    Euclidean layers are encoded and decoded by the oracle with the GPU's own
    fp32 factor and compared under the criteria of _cmp.py;
  * refresh: for sampled whitened layers, the Rayleigh-Ritz property
    (X U)^T (X U) / N = diag(lambda) in fp64 on the layer's activations, and
    rho against the trace identity;
  * NVFP4 on the 11008 x 4096 gradient of the bench: the oracle forms W
    through the rank-32 factor for the whole tensor (cheap), so the tensor
    scale is checked exactly as defined, and sampled rows are coded with it.
"""
import numpy as np
import pytest
import torch

import bench
from oracle import gift_oracle as O
from geometry_aware_fp8_b200 import ops, synth

from _cmp import check_codes, check_nvfp4, check_rows, check_scales

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _rows(d_out):
    return np.r_[0:8, d_out // 2:d_out // 2 + 8, d_out - 8:d_out]


@pytest.fixture(scope="module")
def stack():
    W = bench.build_workload(torch, ops, synth, DEV, 24, seed=1234)
    bench.refresh_all(ops, W)
    bench.step(ops, W, 1)
    torch.cuda.synchronize()
    yield W
    del W
    torch.cuda.empty_cache()


@pytest.mark.parametrize("which", [0, 1, 46, 47])
def test_stack_whitened_rows_match_oracle(stack, which):
    L = stack["whitened"][which]["layer"]
    rows = _rows(L.d_out)
    U = L.U.cpu().numpy().astype(np.float64)
    lam = L.lam.cpu().numpy().astype(np.float64)
    rho = float(L.rho.item())
    G = L.G[rows].float().cpu().numpy().astype(np.float64)
    c_o, s_o = O.encode_e4m3(G, U, lam, rho)
    codes = L.codes[rows].cpu().numpy()
    check_codes(codes, c_o)
    check_scales(L.scales[rows].cpu().numpy(), s_o)
    want = O.decode_e4m3(codes, L.scales[rows].cpu().numpy(), U, lam, rho)
    check_rows(L.G_hat[rows].float().cpu().numpy(), want, bf16=True)


@pytest.mark.parametrize("which", [0, 1, 46, 47])
def test_stack_euclidean_rows_match_oracle(stack, which):
    L = [x for x in stack["layers"] if x.rank == 0][which]
    rows = _rows(L.d_out)
    G = L.G[rows].float().cpu().numpy().astype(np.float64)
    c_o, s_o = O.quantize_e4m3_blocks(G)
    assert np.array_equal(L.codes[rows].cpu().numpy(), c_o)
    assert np.array_equal(L.scales[rows].cpu().numpy(), s_o)
    want = O.dequantize_e4m3_blocks(c_o, s_o)
    check_rows(L.G_hat[rows].float().cpu().numpy(), want, rtol=1e-7, bf16=True)


@pytest.mark.parametrize("which", [0, 47])
def test_stack_refresh_rayleigh_ritz_and_rho(stack, which):
    w = stack["whitened"][which]
    L = w["layer"]
    X = w["X"].float().cpu().numpy().astype(np.float64)
    N, d = X.shape
    U = L.U.cpu().numpy().astype(np.float64)
    lam = L.lam.cpu().numpy().astype(np.float64)
    P = X @ U
    R = P.T @ P / N
    assert int(w["st"].item()) == 0
    assert np.allclose(np.diag(R), lam, rtol=1e-4)
    assert np.max(np.abs(R - np.diag(np.diag(R)))) < 1e-4 * lam[0]
    tr = np.sum(X * X) / N
    rho_ref = (tr - np.trace(R)) / (d - 32)
    tol = max(1e-4 * rho_ref, 2.0 ** -24 * np.sqrt(N) * tr / (d - 32))
    assert abs(float(L.rho.item()) - rho_ref) <= tol, (float(L.rho.item()), rho_ref)


def test_stack_nvfp4_full_tensor_scale_and_rows():
    d_out, d_in = 11008, 4096
    gen = torch.Generator(device=DEV)
    gen.manual_seed(5005)
    Q = torch.from_numpy(synth.haar_orthogonal(d_in, 5003).astype(np.float32)).to(DEV)
    G = synth.device_gradient(d_out, d_in, 1.0, Q, gen, torch.bfloat16)
    sigma = torch.arange(1, d_in + 1, device=DEV, dtype=torch.float32) ** -1.0
    X = synth.device_activations(bench.REFRESH_N, sigma, Q, gen, torch.bfloat16)
    U, lam, rho, _ = ops.factor_refresh(X, 32, 16, 4, seed=5004)
    del X
    codes, sb, ts = ops.encode_nvfp4(G, U, lam, rho)
    torch.cuda.synchronize()
    U64 = U.cpu().numpy().astype(np.float64)
    lam64 = lam.cpu().numpy().astype(np.float64)
    r = float(rho.item())
    G64 = G.float().cpu().numpy().astype(np.float64)
    # W = G M for the whole tensor, through the oracle's transform
    W32 = O.whiten(G64, U64, lam64, r).astype(np.float32)
    S_t = np.float32(np.max(np.abs(W32)) / np.float32(6.0 * 448.0))
    rows = _rows(d_out)
    want_c, want_s, _ = O.quantize_nvfp4(W32[rows], S_t=S_t)
    check_nvfp4((codes[rows].cpu().numpy(), sb[rows].cpu().numpy(), ts.cpu().numpy()), (want_c, want_s, S_t))
