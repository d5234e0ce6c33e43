"""GPU parity of the E4M3 codec against the CPU oracle, through the C ABI.

Sizes span several 128-row panels with a ragged tail and several scale
blocks; the oracle gets the same fp32 factors (U, lambda, rho) as the GPU.
"""
import numpy as np
import pytest
import torch

from oracle import gift_oracle as O
from geometry_aware_fp8_b200 import ops, synth

from _cmp import check_codes, check_rows, check_scales

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _factor(d_in, seed, N=None, rank=32):
    """Oracle factor of synthetic activations, rounded to the fp32 the GPU consumes."""
    Q = synth.haar_orthogonal(d_in, seed)
    X = synth.activations(N or 2 * d_in, Q, synth.column_power(d_in, 1.0), seed + 1)
    A = O.input_factor(X)
    U, lam, rho, _ = O.factor_refresh(A, rank, 16, 4, seed=seed)
    U32, lam32, rho32 = U.astype(np.float32), lam.astype(np.float32), np.float32(rho)
    return Q, U32, lam32, rho32


def _to_dev(*arrs):
    return [torch.from_numpy(np.ascontiguousarray(a)).to(DEV) for a in arrs]


def _g(d_out, Q, seed, dtype):
    G = synth.to_storage(synth.gradient(d_out, Q, 1.0, seed), dtype)
    t = torch.from_numpy(G).to(DEV)
    return G, (t.to(torch.bfloat16) if dtype == "bf16" else t)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d_out,d_in", [(1, 128), (3, 256), (129, 512), (300, 1536)])
def test_euclidean_roundtrip(dtype, d_out, d_in):
    Q = synth.haar_orthogonal(d_in, 5)
    G, Gd = _g(d_out, Q, 6, dtype)
    codes, scales = ops.encode(Gd)
    c_o, s_o = O.quantize_e4m3_blocks(G)
    assert np.array_equal(codes.cpu().numpy(), c_o)
    assert np.array_equal(scales.cpu().numpy(), s_o)
    out = ops.decode(codes, scales, out_dtype=Gd.dtype)
    want = O.dequantize_e4m3_blocks(c_o, s_o)
    check_rows(out.float().cpu().numpy(), want, rtol=1e-6, bf16=(dtype == "bf16"))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d_out,d_in,rank", [(300, 1536, 32), (129, 512, 32), (64, 256, 7), (2, 128, 32)])
def test_whitened_encode_matches_oracle(dtype, d_out, d_in, rank):
    Q, U, lam, rho = _factor(d_in, 40 + d_in, rank=rank)
    G, Gd = _g(d_out, Q, 41, dtype)
    Ud, lamd, rhod = _to_dev(U, lam, np.array([rho], dtype=np.float32))
    codes, scales = ops.encode(Gd, Ud, lamd, rhod)
    c_o, s_o = O.encode_e4m3(G, U.astype(np.float64), lam.astype(np.float64), float(rho))
    check_codes(codes.cpu().numpy(), c_o)
    check_scales(scales.cpu().numpy(), s_o)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d_out,d_in,rank", [(300, 1536, 32), (129, 512, 32), (64, 256, 7)])
def test_whitened_decode_matches_oracle(dtype, d_out, d_in, rank):
    Q, U, lam, rho = _factor(d_in, 50 + d_in, rank=rank)
    G, _ = _g(d_out, Q, 51, dtype)
    U64, lam64 = U.astype(np.float64), lam.astype(np.float64)
    c_o, s_o = O.encode_e4m3(G, U64, lam64, float(rho))
    want = O.decode_e4m3(c_o, s_o, U64, lam64, float(rho))
    Ud, lamd, rhod, cd, sd = _to_dev(U, lam, np.array([rho], dtype=np.float32), c_o, s_o)
    out = ops.decode(cd, sd, Ud, lamd, rhod, out_dtype=torch.bfloat16 if dtype == "bf16" else torch.float32)
    check_rows(out.float().cpu().numpy(), want, bf16=(dtype == "bf16"))


def test_whitened_roundtrip_error_matches_oracle():
    d_out, d_in = 256, 1536
    Q, U, lam, rho = _factor(d_in, 60)
    G, Gd = _g(d_out, Q, 61, "bf16")
    Ud, lamd, rhod = _to_dev(U, lam, np.array([rho], dtype=np.float32))
    codes, scales = ops.encode(Gd, Ud, lamd, rhod)
    Gh = ops.decode(codes, scales, Ud, lamd, rhod, out_dtype=torch.bfloat16)
    err = ops.roundtrip_error(Gd, Gh).cpu().numpy()
    # the metric kernel itself, against fp64 on the same two tensors
    want = O.roundtrip_error(Gd.float().cpu().numpy(), Gh.float().cpu().numpy())
    assert err[0] == pytest.approx(want, rel=1e-12)
    # and the end-to-end round trip against the oracle's own round trip
    U64, lam64 = U.astype(np.float64), lam.astype(np.float64)
    c_o, s_o = O.encode_e4m3(G, U64, lam64, float(rho))
    e_o = O.roundtrip_error(G, O.bf16_round(O.decode_e4m3(c_o, s_o, U64, lam64, float(rho))))
    assert err[0] == pytest.approx(e_o, rel=1e-2)


def test_zero_rows_and_saturation():
    d_in = 256
    Q, U, lam, rho = _factor(d_in, 70)
    G = np.zeros((5, d_in), dtype=np.float32)
    G[1, :] = 1e30                       # huge, finite
    G[2, 3] = -2.5e-38                   # tiny single value
    G[3, 128:] = np.linspace(-1, 1, 128)
    Gd = torch.from_numpy(G).to(DEV)
    codes, scales = ops.encode(Gd)
    c_o, s_o = O.quantize_e4m3_blocks(G)
    assert np.array_equal(codes.cpu().numpy(), c_o) and np.array_equal(scales.cpu().numpy(), s_o)
    Ud, lamd, rhod = _to_dev(U, lam, np.array([rho], dtype=np.float32))
    G2 = G.copy()
    G2[1, :] = 3.0
    codes, scales = ops.encode(torch.from_numpy(G2).to(DEV), Ud, lamd, rhod)
    c_o, s_o = O.encode_e4m3(G2, U.astype(np.float64), lam.astype(np.float64), float(rho))
    check_codes(codes.cpu().numpy(), c_o)
    assert np.all(codes.cpu().numpy()[0] == 0) and np.all(scales.cpu().numpy()[0] == 0)


def test_empty_gradient_is_a_no_op():
    G = torch.empty((0, 256), device=DEV, dtype=torch.bfloat16)
    codes, scales = ops.encode(G)
    assert codes.shape == (0, 256)
    out = ops.decode(codes, scales, out_dtype=torch.bfloat16)
    assert out.shape == (0, 256)
