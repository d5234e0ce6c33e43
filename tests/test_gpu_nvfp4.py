"""GPU parity of the NVFP4 codec (E2M1 codes, E4M3 scales per 16, fp32 tensor
scale) against the CPU oracle, through the C ABI.  Criteria in _cmp.py."""
import numpy as np
import pytest
import torch

from oracle import gift_oracle as O
from geometry_aware_fp8_b200 import ops, synth

from _cmp import check_nvfp4, check_rows
from test_gpu_codec import _factor, _g, _to_dev

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d_out,d_in", [(1, 16), (3, 48), (129, 528), (300, 1536)])
def test_nvfp4_euclidean_bit_exact(dtype, d_out, d_in):
    Q = synth.haar_orthogonal(d_in, 7)
    G, Gd = _g(d_out, Q, 8, dtype)
    codes, sb, st = ops.encode_nvfp4(Gd)
    want = O.quantize_nvfp4(G)
    check_nvfp4((codes.cpu().numpy(), sb.cpu().numpy(), st.cpu().numpy()), want, exact=True)
    out = ops.decode_nvfp4(codes, sb, st, out_dtype=Gd.dtype)
    ref = O.dequantize_nvfp4(*want)
    check_rows(out.float().cpu().numpy(), ref, rtol=1e-7, bf16=(dtype == "bf16"))


def test_nvfp4_zero_tensor_and_empty():
    Gd = torch.zeros((5, 64), device=DEV, dtype=torch.bfloat16)
    codes, sb, st = ops.encode_nvfp4(Gd)
    assert float(st.item()) == 0.0
    assert not codes.any().item() and not sb.any().item()
    out = ops.decode_nvfp4(codes, sb, st)
    assert not out.float().abs().sum().item()
    E = torch.empty((0, 128), device=DEV, dtype=torch.bfloat16)
    c, s, t = ops.encode_nvfp4(E)
    assert c.shape == (0, 64) and s.shape == (0, 8)


def test_nvfp4_saturating_block_and_tiny_values():
    # one huge element per row next to tiny ones: per-16 scales keep the small blocks
    G = np.zeros((4, 64), dtype=np.float32)
    G[:, 0] = 1e4
    G[:, 17:32] = 1e-3 * np.arange(1, 16)
    G[1, 40:56] = -2.5e-2
    Gd = torch.from_numpy(G).to(DEV)
    codes, sb, st = ops.encode_nvfp4(Gd)
    check_nvfp4((codes.cpu().numpy(), sb.cpu().numpy(), st.cpu().numpy()), O.quantize_nvfp4(G), exact=True)


@pytest.mark.parametrize("d_out,d_in", [(300, 1536), (129, 512), (2, 128)])
def test_nvfp4_whitened_encode_matches_oracle(d_out, d_in):
    Q, U, lam, rho = _factor(d_in, 60 + d_in)
    G, Gd = _g(d_out, Q, 61, "bf16")
    Ud, lamd, rhod = _to_dev(U, lam, np.array([rho], dtype=np.float32))
    codes, sb, st = ops.encode_nvfp4(Gd, Ud, lamd, rhod)
    want = O.encode_nvfp4(G, U.astype(np.float64), lam.astype(np.float64), float(rho))
    check_nvfp4((codes.cpu().numpy(), sb.cpu().numpy(), st.cpu().numpy()), want)


@pytest.mark.parametrize("d_out,d_in", [(300, 1536), (129, 512)])
def test_nvfp4_whitened_decode_matches_oracle(d_out, d_in):
    Q, U, lam, rho = _factor(d_in, 70 + d_in)
    G, _ = _g(d_out, Q, 71, "bf16")
    U64, lam64 = U.astype(np.float64), lam.astype(np.float64)
    c_o, s_o, t_o = O.encode_nvfp4(G, U64, lam64, float(rho))
    want = O.decode_nvfp4(c_o, s_o, t_o, U64, lam64, float(rho))
    Ud, lamd, rhod, cd, sd, td = _to_dev(U, lam, np.array([rho], dtype=np.float32), c_o, s_o,
                                         np.array([t_o], dtype=np.float32))
    out = ops.decode_nvfp4(cd, sd, td, Ud, lamd, rhod, out_dtype=torch.bfloat16)
    check_rows(out.float().cpu().numpy(), want, bf16=True)


@pytest.mark.parametrize("rank", [0, 32])
def test_nvfp4_roundtrip_error_matches_oracle(rank):
    """The whole round trip on the GPU (encode then decode) has the oracle's
    relative error, whitened and Euclidean."""
    d_out, d_in = 256, 1536
    Q, U, lam, rho = _factor(d_in, 80)
    G, Gd = _g(d_out, Q, 81, "bf16")
    G64 = G.astype(np.float64)
    if rank:
        Ud, lamd, rhod = _to_dev(U, lam, np.array([rho], dtype=np.float32))
        U64, lam64 = U.astype(np.float64), lam.astype(np.float64)
        want = O.decode_nvfp4(*O.encode_nvfp4(G64, U64, lam64, float(rho)), U64, lam64, float(rho))
        got = ops.decode_nvfp4(*ops.encode_nvfp4(Gd, Ud, lamd, rhod), Ud, lamd, rhod, out_dtype=torch.bfloat16).float()
    else:
        want = O.dequantize_nvfp4(*O.quantize_nvfp4(G64))
        got = ops.decode_nvfp4(*ops.encode_nvfp4(Gd), out_dtype=torch.float32)
    e_o = O.roundtrip_error(G64, want)
    e_g = O.roundtrip_error(G64, got.cpu().numpy())
    assert abs(e_g - e_o) <= 1e-3 * e_o, (e_g, e_o)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_nvfp4_euclidean_hand_derived_blocks(dtype):
    """The hand-derived row of tests/golden/nvfp4_hand_blocks.txt (block scale
    ratios between E4M3 values and on ties) through the GPU's Euclidean NVFP4
    codec: tensor scale, block scale codes and element codes must be the
    hand-derived ones (every value of the row except one in the flushed
    block is exact in bf16, and that block stays flushed)."""
    from _golden import nvfp4_hand_blocks
    W, st, sb_want, q_want, _ = nvfp4_hand_blocks()
    Gd = torch.from_numpy(np.repeat(W, 3, axis=0).astype(np.float32)).to(DEV).to(dtype)
    codes, sb, ts = ops.encode_nvfp4(Gd)
    torch.cuda.synchronize()
    assert float(ts.item()) == st
    from _cmp import unpack_nibbles
    for r in range(3):
        assert np.array_equal(sb[r].cpu().numpy(), sb_want)
        assert np.array_equal(unpack_nibbles(codes[r:r + 1].cpu().numpy())[0], q_want)
    out = ops.decode_nvfp4(codes, sb, ts, out_dtype=torch.float32)[0].cpu().numpy().astype(np.float64)
    want = O.e2m1_decode(q_want) * np.repeat(O.e4m3_decode(sb_want), 16) * st
    assert np.array_equal(out, want)
