"""Device status reporting of the codec and the refresh (GPU, through the C ABI).

Failure detection is exercised without faulting the GPU:
  * a bounded wait that gives up: gift_codec_stall_test makes every CTA of
    the tensor-core encoder or decoder wait a few polls on a barrier that
    nothing arrives at, before any work; the call must complete, report
    GIFT_DEV_TIMEOUT in the caller's status word, leave the outputs alone,
    and the context must stay usable (the next regular call matches the
    oracle);
  * non-finite inputs: an infinity or NaN in X, G or a block scale must set
    GIFT_DEV_NONFINITE, blocks without one must still match the oracle, and
    clean inputs must leave the status word at zero.
"""
import numpy as np
import pytest
import torch

from oracle import gift_oracle as O
from geometry_aware_fp8_b200 import ops, synth

from _cmp import check_codes, check_scales
from test_gpu_codec import _factor, _g, _to_dev

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _status():
    return torch.zeros((1,), device=DEV, dtype=torch.int32)


def _layer(d_out=300, d_in=1536, seed=90):
    Q, U, lam, rho = _factor(d_in, seed)
    G, Gd = _g(d_out, Q, seed + 1, "bf16")
    Ud, lamd, rhod = _to_dev(U, lam, np.array([rho], dtype=np.float32))
    return G, Gd, (U, lam, rho), (Ud, lamd, rhod)


@pytest.mark.parametrize("encode", [True, False])
def test_codec_wait_that_runs_out_reports_timeout_and_context_stays_usable(encode):
    G, Gd, (U, lam, rho), (Ud, lamd, rhod) = _layer()
    d_out, d_in = G.shape
    codes = torch.full((d_out, d_in), 0xAB, device=DEV, dtype=torch.uint8)
    scales = torch.full((d_out, d_in // 128), 7.0, device=DEV, dtype=torch.float32)
    Gh = torch.full((d_out, d_in), 3.0, device=DEV, dtype=torch.bfloat16)
    L = ops.LayerArgs(d_out=d_out, d_in=d_in, rank=32, dtype=torch.bfloat16, G=Gd, G_hat=Gh, codes=codes,
                      scales=scales, U=Ud, lam=lamd, rho=rhod)
    st = _status()
    ops.codec_stall_test(L, encode, 2000, st)
    torch.cuda.synchronize()
    assert int(st.item()) & ops.DEV_TIMEOUT
    # nothing was written
    assert bool((codes == 0xAB).all()) and bool((scales == 7.0).all()) and bool((Gh == 3.0).all())
    # the context is still usable: a regular call afterwards matches the oracle
    st2 = _status()
    U64, lam64 = U.astype(np.float64), lam.astype(np.float64)
    c_o, s_o = O.encode_e4m3(G, U64, lam64, float(rho))
    if encode:
        ops.encode(Gd, Ud, lamd, rhod, codes=codes, scales=scales, dev_status=st2)
        torch.cuda.synchronize()
        check_codes(codes.cpu().numpy(), c_o)
        check_scales(scales.cpu().numpy(), s_o)
    else:
        cd, sd = _to_dev(c_o, s_o)
        ops.decode(cd, sd, Ud, lamd, rhod, out=Gh, dev_status=st2)
        torch.cuda.synchronize()
        want = O.decode_e4m3(c_o, s_o, U64, lam64, float(rho))
        got = Gh.float().cpu().numpy()
        assert np.max(np.abs(got - want)) <= 1e-2 * np.max(np.abs(want))
    assert int(st2.item()) == 0


def test_refresh_of_activations_with_an_infinity_reports_nonfinite():
    d = 256
    Q = synth.haar_orthogonal(d, 91)
    X = synth.activations(1024, Q, synth.column_power(d, 1.0), 92).astype(np.float32)
    clean = ops.factor_refresh(torch.from_numpy(X).to(DEV), 32, 16, 4, 3)[3]
    X[17, 5] = np.inf
    st = ops.factor_refresh(torch.from_numpy(X).to(DEV), 32, 16, 4, 3)[3]
    torch.cuda.synchronize()
    assert int(clean.item()) == 0
    assert int(st.item()) & ops.DEV_NONFINITE


@pytest.mark.parametrize("rank", [0, 32])
@pytest.mark.parametrize("bad", [np.inf, np.nan])
def test_encode_of_a_non_finite_gradient_reports_nonfinite(rank, bad):
    G, Gd, (U, lam, rho), (Ud, lamd, rhod) = _layer(d_out=260, d_in=512, seed=93)
    args = (Ud, lamd, rhod) if rank else (None, None, None)
    st = _status()
    ops.encode(Gd, *args, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    Gb = G.copy()
    Gb[7, 300] = bad
    st = _status()
    codes, scales = ops.encode(torch.from_numpy(Gb).to(DEV).to(torch.bfloat16), *args, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & ops.DEV_NONFINITE
    # the other rows are coded as before (a row depends only on its own gradient)
    keep = np.r_[0:7, 8:260]
    U64, lam64 = (U.astype(np.float64), lam.astype(np.float64)) if rank else (np.zeros((512, 0)), np.zeros(0))
    c_o, s_o = O.encode_e4m3(G[keep], U64, lam64, float(rho) if rank else 1.0)
    check_codes(codes.cpu().numpy()[keep], c_o)
    check_scales(scales.cpu().numpy()[keep], s_o)


@pytest.mark.parametrize("rank", [0, 32])
def test_decode_of_a_non_finite_scale_reports_nonfinite(rank):
    G, Gd, (U, lam, rho), (Ud, lamd, rhod) = _layer(d_out=200, d_in=512, seed=95)
    args = (Ud, lamd, rhod) if rank else (None, None, None)
    codes, scales = ops.encode(Gd, *args)
    st = _status()
    ops.decode(codes, scales, *args, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    scales[3, 1] = float("inf")
    st = _status()
    ops.decode(codes, scales, *args, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & ops.DEV_NONFINITE


def test_grouped_calls_report_into_one_status_word():
    G, Gd, (U, lam, rho), (Ud, lamd, rhod) = _layer(d_out=256, d_in=1536, seed=97)
    Gb = Gd.clone()
    Gb[5, 9] = float("inf")
    mk = lambda g, r: ops.LayerArgs(d_out=256, d_in=1536, rank=r, dtype=torch.bfloat16, G=g,
                                    G_hat=torch.empty_like(g), codes=torch.empty((256, 1536), device=DEV,
                                                                                 dtype=torch.uint8),
                                    scales=torch.empty((256, 12), device=DEV), U=Ud if r else None,
                                    lam=lamd if r else None, rho=rhod if r else None)
    layers = [mk(Gd, 32), mk(Gd, 0)]
    st = _status()
    ops.encode_many(ops.make_layers(layers), 2, dev_status=st)
    ops.decode_many(ops.make_layers(layers), 2, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for r in (32, 0):
        st = _status()
        ops.encode_many(ops.make_layers([mk(Gd, 32 - r), mk(Gb, r)]), 2, dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) & ops.DEV_NONFINITE
