"""GPU parity of the dense input-side transforms (full-rank A^{-1/2} and the
Cholesky form L_A^{-T} of Eq. 14) and of the E4M3 codec under them, against
the CPU oracle, through the C ABI.

Criteria:
  * factor: M and M^{-1} (fp32 results of fp64 arithmetic on the same fp32 A)
    within 1e-5 of the oracle's in relative Frobenius norm; the sum of M's
    three bf16 parts within 2^-24 of M per element, of M^{-1}'s two parts
    within 2^-16 (relative to the largest entry);
  * codec, given the same fp32 M: codes and scales within the bound that the
    fp32 evaluation of W = G M allows (_cmp.check_codes_within_bound: the
    entries of a whitening transform are large next to W, whose sum cancels,
    so the rank-32 codec's 99.9 % exact-code criterion does not transfer),
    at least 99 % of codes exact; G_hat within 1e-3 of the row maximum with
    the decoder fed the oracle's codes (the criterion of _cmp.check_rows);
  * round trip on the GPU's own factor: the relative Frobenius error within
    1 % of the oracle's.
"""
import numpy as np
import pytest
import torch

from oracle import gift_oracle as O
from geometry_aware_fp8_b200 import ops, synth

from _cmp import check_codes_within_bound, check_rows

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
KINDS = {"cholesky": ops.DENSE_CHOLESKY, "invsqrt": ops.DENSE_INVSQRT}


def _oracle_M(A64, kind, inverse=False):
    if kind == "cholesky":
        return O.cholesky_transform(A64, inverse=inverse)
    return O.full_rank_transform(A64, inverse=inverse)


def _layer(d_in, d_out, N, seed):
    """Activations with sigma_i = i^-1 and a gradient of a linear layer's
    structure, G = Delta^T X / N (the draws of the Table I/II-style study)."""
    Q = synth.haar_orthogonal(d_in, seed)
    X = synth.activations(N, Q, synth.column_power(d_in, 1.0), seed + 1)
    rng = np.random.default_rng(seed + 2)
    Delta = rng.standard_normal((N, d_out)) * (np.arange(1, d_out + 1) ** -0.5)[None, :]
    G = synth.to_storage(Delta.T @ X / N, "bf16")
    A32 = O.input_factor(X).astype(np.float32)
    return A32, G


def _rel(a, b):
    return np.linalg.norm(np.asarray(a, dtype=np.float64) - b) / np.linalg.norm(b)


@pytest.mark.parametrize("kind", ["cholesky", "invsqrt"])
@pytest.mark.parametrize("d", [512, 1536])
def test_dense_factor_matches_oracle(kind, d):
    A32, _ = _layer(d, 8, 4 * d, 500 + d)
    A64 = A32.astype(np.float64)
    M, Mi, Ms, Mis, st = ops.dense_factor(torch.from_numpy(A32).to(DEV), KINDS[kind])
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    Mo, Mio = _oracle_M(A64, kind), _oracle_M(A64, kind, inverse=True)
    e, ei = _rel(M.cpu().numpy(), Mo), _rel(Mi.cpu().numpy(), Mio)
    print(f"{kind} d={d}: M rel err {e:.2e}, M_inv rel err {ei:.2e}")
    assert e <= 1e-5 and ei <= 1e-5
    for full, parts, tol in ((M, Ms, 2.0 ** -24), (Mi, Mis, 2.0 ** -16)):
        pv = parts.view(torch.bfloat16).float().cpu().numpy().astype(np.float64)
        back = pv.sum(axis=0)
        f = full.cpu().numpy().astype(np.float64)
        assert np.max(np.abs(back - f)) <= tol * np.max(np.abs(f))


@pytest.mark.parametrize("kind", ["cholesky", "invsqrt"])
@pytest.mark.parametrize("d_in,d_out", [(512, 300), (1536, 1024), (256, 129)])
def test_dense_codec_matches_oracle_given_the_same_transform(kind, d_in, d_out):
    A32, G = _layer(d_in, d_out, 4 * d_in, 600 + d_in)
    A64 = A32.astype(np.float64)
    M32 = np.ascontiguousarray(_oracle_M(A64, kind), dtype=np.float32)
    Mi32 = np.ascontiguousarray(_oracle_M(A64, kind, inverse=True), dtype=np.float32)
    Ms = ops.dense_split(torch.from_numpy(M32).to(DEV), 3)
    Mis = ops.dense_split(torch.from_numpy(Mi32).to(DEV), 2)
    Gd = torch.from_numpy(G).to(DEV).to(torch.bfloat16)
    upper = kind == "cholesky"
    st = torch.zeros((1,), device=DEV, dtype=torch.int32)
    codes, scales = ops.dense_encode(Gd, Ms, upper, dev_status=st)
    G64, M64 = G.astype(np.float64), M32.astype(np.float64)
    c_o, s_o = O.encode_dense(G64, M64)
    W = G64 @ M64
    E = (d_in + 1) * 2.0 ** -24 * (np.abs(G64) @ np.abs(M64))
    rate = check_codes_within_bound(codes.cpu().numpy(), scales.cpu().numpy(), W, E, want_codes=c_o)
    if upper:  # the full K loop over the zero blocks meets the same bound
        c2, s2 = ops.dense_encode(Gd, Ms, False)
        check_codes_within_bound(c2.cpu().numpy(), s2.cpu().numpy(), W, E, want_codes=c_o)
    want = O.decode_dense(c_o, s_o, Mi32.astype(np.float64))
    cd, sd = torch.from_numpy(c_o).to(DEV), torch.from_numpy(s_o).to(DEV)
    for dt in (torch.bfloat16, torch.float32):
        out = ops.dense_decode(cd, sd, Mis, upper, out_dtype=dt, dev_status=st)
        check_rows(out.float().cpu().numpy(), want, bf16=dt == torch.bfloat16)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    print(f"{kind} {d_out}x{d_in}: code match {rate:.6f}")


@pytest.mark.parametrize("kind", ["cholesky", "invsqrt"])
def test_dense_round_trip_error_on_the_gpu_factor_matches_oracle(kind):
    """The whole variant on the GPU (factor from A, encode, decode) against the
    oracle's same variant: the Table I/II-style Frobenius errors agree."""
    d_in, d_out = 512, 256
    A32, G = _layer(d_in, d_out, 4096, 44)
    A64 = A32.astype(np.float64)
    M, Mi, Ms, Mis, st = ops.dense_factor(torch.from_numpy(A32).to(DEV), KINDS[kind])
    Gd = torch.from_numpy(G).to(DEV).to(torch.bfloat16)
    upper = kind == "cholesky"
    codes, scales = ops.dense_encode(Gd, Ms, upper)
    Gh = ops.dense_decode(codes, scales, Mis, upper, out_dtype=torch.float32)
    err = ops.roundtrip_error(Gd.float(), Gh)
    torch.cuda.synchronize()
    G64 = G.astype(np.float64)
    c_o, s_o = O.encode_dense(G64, _oracle_M(A64, kind))
    e_o = O.roundtrip_error(G64, O.decode_dense(c_o, s_o, _oracle_M(A64, kind, inverse=True)))
    e_g = float(err[0].item())
    print(f"{kind}: round-trip error GPU {e_g:.5f}, oracle {e_o:.5f}")
    assert abs(e_g - e_o) <= 1e-2 * e_o


def test_dense_entry_points_reject_bad_arguments():
    L = ops.lib()
    a = torch.zeros((256, 256), device=DEV)
    assert L.gift_dense_factor(a.data_ptr(), 256, 3, a.data_ptr(), a.data_ptr(), a.data_ptr(), a.data_ptr(),
                               a.data_ptr(), 1 << 30, None, None) == 1
    assert L.gift_dense_factor(a.data_ptr(), 200, 1, a.data_ptr(), a.data_ptr(), a.data_ptr(), a.data_ptr(),
                               a.data_ptr(), 1 << 30, None, None) == 2
    assert L.gift_dense_factor(a.data_ptr(), 256, 1, a.data_ptr(), a.data_ptr(), a.data_ptr(), a.data_ptr(),
                               a.data_ptr(), 16, None, None) == 4
    assert L.gift_dense_encode(a.data_ptr(), 4, 200, a.data_ptr(), 0, a.data_ptr(), a.data_ptr(), None, None) == 2
    assert L.gift_dense_encode(a.data_ptr(), 0, 256, None, 0, None, None, None, None) == 0
