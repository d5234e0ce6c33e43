"""Config 1 end to end at its full size, through the C ABI: one 512 x 512 fp32
layer, factor refreshed on the GPU from X 2048 x 512 fp32 (sigma_i = i^-1),
then encode and decode of the fp32 gradient (exponent 0.8).  fp32 G takes the
CUDA-core codec.  Every element is checked: codes and scales against the
oracle fed the GPU's own fp32 factor, G_hat against the oracle's decode of the
GPU's codes, and the round-trip error against the oracle's own end-to-end
round trip (its fp64 factor): within 1 %."""
import numpy as np
import pytest
import torch

from oracle import gift_oracle as O
from geometry_aware_fp8_b200 import ops, synth

from _cmp import check_codes, check_rows, check_scales

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.mark.parametrize("aligned", [False, True])
def test_config1_round_trip_matches_oracle(aligned):
    X, G = synth.config1(aligned=aligned)
    Xd, Gd = torch.from_numpy(X).to(DEV), torch.from_numpy(G).to(DEV)
    U, lam, rho, st = ops.factor_refresh(Xd, 32, 16, 4, seed=1004)
    codes, scales = ops.encode(Gd, U, lam, rho)
    Gh = ops.decode(codes, scales, U, lam, rho, out_dtype=torch.float32)
    err = ops.roundtrip_error(Gd, Gh)
    torch.cuda.synchronize()
    assert int(st.item()) & ops.DEV_RHO_FLOORED == 0
    U64 = U.cpu().numpy().astype(np.float64)
    l64 = lam.cpu().numpy().astype(np.float64)
    r = float(rho.item())
    c_o, s_o = O.encode_e4m3(G, U64, l64, r)
    c_g, s_g = codes.cpu().numpy(), scales.cpu().numpy()
    check_codes(c_g, c_o)
    check_scales(s_g, s_o)
    check_rows(Gh.cpu().numpy(), O.decode_e4m3(c_g, s_g, U64, l64, r))
    # the oracle's own round trip, factor and all
    Uo, lo, ro, _ = O.factor_refresh(O.input_factor(X), 32, 16, 4, seed=1004)
    c, s = O.encode_e4m3(G, Uo, lo, ro)
    e_o = O.roundtrip_error(G, O.decode_e4m3(c, s, Uo, lo, ro))
    assert float(err[0].item()) == pytest.approx(e_o, rel=1e-2)
