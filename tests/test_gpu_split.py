"""The tensor-core whitened codec with a panel split across a thread-block
cluster (2 or 4 CTAs share each 128-row panel's chunks and add their partial
projections in cluster-rank order), against the CPU oracle.

A launch takes a cluster split when every cluster can own one panel and
the shorter chunk range outweighs the cluster's fixed cost (about 6 chunk
steps for 2 CTAs, 15 for 4): single layers such as the 4096 x 1536
up-projection stand-in (32 panels, 12 chunks: 2 CTAs) or a 4096 x 4096
layer (32 chunks: 4 CTAs).  Launches of many panels, like the grouped stack
or the 11008 x 4096 projection (86 panels), keep one CTA per panel.  The
planned split is read back through gift_codec_split, so each case states
which path it covers, including chunk counts that do not divide evenly
(9 chunks over 2 CTAs, 21 over 4).
"""
import numpy as np
import pytest
import torch

import bench
from oracle import gift_oracle as O
from geometry_aware_fp8_b200 import ops, synth

from _cmp import check_codes, check_rows, check_scales

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _factor(d_in, seed, rank=32):
    Q = synth.haar_orthogonal(d_in, seed)
    X = synth.activations(2 * d_in, Q, synth.column_power(d_in, 1.0), seed + 1)
    U, lam, rho, _ = O.factor_refresh(O.input_factor(X), rank, 16, 4, seed=seed)
    return Q, U.astype(np.float32), lam.astype(np.float32), np.float32(rho)


def _split(d_out, d_in, encode=True, rank=32, dtype=torch.bfloat16):
    L = ops.LayerArgs(d_out=d_out, d_in=d_in, rank=rank, dtype=dtype, G=None, G_hat=None, codes=None,
                      scales=None, U=None, lam=None, rho=None)
    return ops.codec_split(ops.make_layers([L]), 1, encode)


@pytest.mark.parametrize("d_out,d_in,want", [(300, 1152, 2), (300, 2688, 4), (130, 4096, 4), (260, 1536, 2),
                                             (4096, 1536, 2), (2048, 1536, 2), (4096, 4096, 4), (11008, 4096, 1),
                                             (128, 128, 1), (300, 256, 1), (130, 768, 1)])
def test_planned_split(d_out, d_in, want):
    assert _split(d_out, d_in, True) == want
    assert _split(d_out, d_in, False) == want


def test_planned_split_of_the_grouped_stack_is_one():
    W = [ops.LayerArgs(d_out=o, d_in=i, rank=32 if wh else 0, dtype=torch.bfloat16, G=None, G_hat=None,
                       codes=None, scales=None, U=None, lam=None, rho=None)
         for _, _, o, i, wh in synth.stack_shapes(24) if wh]
    assert ops.codec_split(ops.make_layers(W), len(W), True) == 1
    assert ops.codec_split(ops.make_layers(W), len(W), False) == 1
    # rank-0 and fp32 layers do not take the tensor-core path
    assert _split(256, 256, rank=0) == 0
    assert _split(256, 256, dtype=torch.float32) == 0


@pytest.mark.parametrize("d_out,d_in", [(300, 1152), (300, 2688), (130, 4096), (260, 1536)])
def test_split_codec_matches_oracle(d_out, d_in):
    Q, U, lam, rho = _factor(d_in, 80 + d_in)
    G = synth.to_storage(synth.gradient(d_out, Q, 1.0, 81 + d_in), "bf16")
    Gd = torch.from_numpy(G).to(DEV).to(torch.bfloat16)
    Ud, lamd = torch.from_numpy(U).to(DEV), torch.from_numpy(lam).to(DEV)
    rhod = torch.tensor([rho], device=DEV)
    codes, scales = ops.encode(Gd, Ud, lamd, rhod)
    U64, lam64 = U.astype(np.float64), lam.astype(np.float64)
    c_o, s_o = O.encode_e4m3(G, U64, lam64, float(rho))
    check_codes(codes.cpu().numpy(), c_o)
    check_scales(scales.cpu().numpy(), s_o)
    # decode the oracle's codes, so a code flip cannot spread into G_hat
    out = ops.decode(torch.from_numpy(c_o).to(DEV), torch.from_numpy(s_o).to(DEV), Ud, lamd, rhod)
    check_rows(out.float().cpu().numpy(), O.decode_e4m3(c_o, s_o, U64, lam64, float(rho)), bf16=True)


@pytest.mark.parametrize("d_out,d_in,seed,split", [(4096, 1536, 9100, 2), (4096, 4096, 9300, 4),
                                                   (11008, 4096, 9200, 1)])
def test_single_layer_full_size_rows_match_oracle(d_out, d_in, seed, split):
    """Full-size single layers (rank-32 factor refreshed on the GPU from 8192
    bf16 tokens): sampled rows of the codes, scales and G_hat against the oracle
    fed the GPU's fp32 factor."""
    assert _split(d_out, d_in) == split
    gen = torch.Generator(device=DEV)
    gen.manual_seed(seed)
    Q = torch.from_numpy(synth.haar_orthogonal(d_in, seed + 1).astype(np.float32)).to(DEV)
    G = synth.device_gradient(d_out, d_in, 1.0, Q, gen, torch.bfloat16)
    sigma = torch.arange(1, d_in + 1, device=DEV, dtype=torch.float32) ** -1.0
    X = synth.device_activations(bench.REFRESH_N, sigma, Q, gen, torch.bfloat16)
    U, lam, rho, st = ops.factor_refresh(X, 32, 16, 4, seed=seed + 2)
    del X
    codes, scales = ops.encode(G, U, lam, rho)
    Gh = ops.decode(codes, scales, U, lam, rho)
    torch.cuda.synchronize()
    rows = np.r_[0:8, d_out // 2:d_out // 2 + 8, d_out - 8:d_out]
    U64 = U.cpu().numpy().astype(np.float64)
    lam64 = lam.cpu().numpy().astype(np.float64)
    r = float(rho.item())
    c_o, s_o = O.encode_e4m3(G[rows].float().cpu().numpy().astype(np.float64), U64, lam64, r)
    c_g = codes[rows].cpu().numpy()
    s_g = scales[rows].cpu().numpy()
    check_codes(c_g, c_o)
    check_scales(s_g, s_o)
    check_rows(Gh[rows].float().cpu().numpy(), O.decode_e4m3(c_g, s_g, U64, lam64, r), bf16=True)
