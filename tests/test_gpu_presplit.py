"""The tensor-core codec with a pre-split U (gift_split_u + gift_layer.U_split),
through the C ABI on the GPU.

The split is an implementation format, so it is checked against its
definition (round-to-nearest-even bf16 and f16 parts, computed here with plain
PyTorch casts), and the codec with it must give bit-identical codes, scales
and G_hat to the same grouped call without it (whose parity with the oracle
the other codec tests establish); one layer is also compared with the oracle
directly.  Layers span ragged panels, both codec launch shapes (many panels,
and few panels, where CTAs share a panel in a cluster) and a Euclidean layer
in the same group.
"""
import numpy as np
import pytest
import torch

from oracle import gift_oracle as O
from geometry_aware_fp8_b200 import ops

from _cmp import check_codes, check_rows, check_scales
from test_gpu_codec import _factor, _g, _to_dev

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def test_split_u_matches_its_definition():
    _, U, _, _ = _factor(512, 71)
    Ud = torch.from_numpy(U).to(DEV)
    S = ops.split_u(Ud)
    torch.cuda.synchronize()
    bh = Ud.to(torch.bfloat16)
    bl = (Ud - bh.float()).to(torch.bfloat16)
    fh = Ud.to(torch.float16)
    fl = ((Ud - fh.float()) * 2048.0).to(torch.float16)
    want0 = torch.cat([bh.view(torch.int16), bl.view(torch.int16)], dim=1)
    want1 = torch.cat([fh.view(torch.int16), fl.view(torch.int16)], dim=1)
    assert torch.equal(S[0], want0)
    assert torch.equal(S[1], want1)


def _layers(shapes, seed):
    out = []
    for i, (d_out, d_in, rank) in enumerate(shapes):
        if rank:
            Q, U, lam, rho = _factor(d_in, seed + 10 * i)
            G, Gd = _g(d_out, Q, seed + 10 * i + 1, "bf16")
            Ud, lamd, rhod = _to_dev(U, lam, np.array([rho], dtype=np.float32))
            fac = (U, lam, rho)
        else:
            from geometry_aware_fp8_b200 import synth
            G, Gd = _g(d_out, synth.haar_orthogonal(d_in, seed + 10 * i), seed + 10 * i + 1, "bf16")
            Ud = lamd = rhod = None
            fac = None
        out.append((G, Gd, Ud, lamd, rhod, fac))
    return out


def _args(d_out, d_in, rank, Gd, Ud, lamd, rhod, presplit):
    return ops.LayerArgs(d_out=d_out, d_in=d_in, rank=rank, dtype=torch.bfloat16, G=Gd,
                         G_hat=torch.empty_like(Gd),
                         codes=torch.empty((d_out, d_in), device=DEV, dtype=torch.uint8),
                         scales=torch.empty((d_out, d_in // 128), device=DEV, dtype=torch.float32),
                         U=Ud, lam=lamd, rho=rhod,
                         U_split=ops.split_u(Ud) if (presplit and rank) else None)


def test_split_u_many_matches_split_u_per_layer():
    """gift_split_u_many writes, in one launch, each U_split layer's
    gift_split_u result; layers without a U_split or with rank 0 are left
    alone."""
    layers, want = [], []
    rng = np.random.default_rng(80)
    for i, (d_out, d_in) in enumerate([(256, 512), (300, 1536), (128, 128), (256, 4096), (256, 640)]):
        # any fp32 matrix will do for the split; columns of unit norm, as U's are
        Ud = torch.from_numpy((rng.standard_normal((d_in, 32)) / np.sqrt(d_in)).astype(np.float32)).to(DEV)
        keep = i != 2  # layer 2 carries no U_split
        sp = torch.full((2, d_in, 64), 0x5A5A, device=DEV, dtype=torch.int16) if keep else None
        layers.append(ops.LayerArgs(d_out=d_out, d_in=d_in, rank=32, dtype=torch.bfloat16, U=Ud, U_split=sp))
        want.append(ops.split_u(Ud) if keep else None)
    eu_split = torch.full((2, 256, 64), 0x1234, device=DEV, dtype=torch.int16)
    layers.append(ops.LayerArgs(d_out=64, d_in=256, rank=0, dtype=torch.bfloat16, U_split=eu_split))
    ops.split_u_many(ops.make_layers(layers), len(layers))
    torch.cuda.synchronize()
    for L, w in zip(layers, want):
        if w is not None:
            assert torch.equal(L.U_split, w)
    assert bool((eu_split == 0x1234).all())


def test_split_u_many_over_more_layers_than_one_launch_takes():
    """520 layers (one launch takes at most 512): every split is that of
    gift_split_u for its layer."""
    rng = np.random.default_rng(81)
    n = 520
    U = torch.from_numpy((rng.standard_normal((n, 128, 32)) / np.sqrt(128)).astype(np.float32)).to(DEV)
    S = torch.zeros((n, 2, 128, 64), device=DEV, dtype=torch.int16)
    layers = [ops.LayerArgs(d_out=128, d_in=128, rank=32, dtype=torch.bfloat16, U=U[i], U_split=S[i]) for i in range(n)]
    ops.split_u_many(ops.make_layers(layers), n)
    torch.cuda.synchronize()
    for i in (0, 1, 511, 512, 519):
        assert torch.equal(S[i], ops.split_u(U[i]))
    assert int((S == 0).all(dim=(1, 2, 3)).sum().item()) == 0  # every layer was written


def test_split_u_many_rejects_bad_arguments():
    L = ops.lib()
    assert L.gift_split_u_many(None, 0, None) == 0
    assert L.gift_split_u_many(None, 1, None) == 1
    U = torch.zeros((512, 32), device=DEV)
    sp = torch.zeros((2 * 512 * 64 + 8,), device=DEV, dtype=torch.int16)
    bad = ops.LayerArgs(d_out=128, d_in=512, rank=32, dtype=torch.bfloat16, U=U, lam=torch.zeros((32,), device=DEV),
                        rho=torch.ones((1,), device=DEV), U_split=sp[1:])  # 2-byte offset: misaligned
    assert L.gift_split_u_many(ops.make_layers([bad]), 1, None) == 3
    assert int(sp[1:].abs().sum().item()) == 0  # nothing was launched


@pytest.mark.parametrize("shapes", [
    [(300, 1536, 32), (129, 512, 32), (1536, 4096, 32), (200, 1536, 0)],  # many panels: one CTA each
    [(4096, 1536, 32)],                                                   # few panels: a cluster per panel
])
def test_grouped_codec_with_presplit_u_is_bit_identical(shapes):
    data = _layers(shapes, 300)
    runs = {}
    for presplit in (False, True):
        args = [_args(d_out, d_in, rank, Gd, Ud, lamd, rhod, presplit)
                for (d_out, d_in, rank), (_, Gd, Ud, lamd, rhod, _) in zip(shapes, data)]
        packed = ops.make_layers(args)
        st = torch.zeros((1,), device=DEV, dtype=torch.int32)
        ops.encode_many(packed, len(args), dev_status=st)
        ops.decode_many(packed, len(args), dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        runs[presplit] = args
    for a, b in zip(runs[False], runs[True]):
        assert torch.equal(a.codes, b.codes)
        assert torch.equal(a.scales, b.scales)
        assert torch.equal(a.G_hat.view(torch.int16), b.G_hat.view(torch.int16))
    # and one whitened layer against the oracle directly, both directions
    (d_out, d_in, rank), (G, _, _, _, _, (U, lam, rho)) = shapes[0], data[0]
    U64, lam64 = U.astype(np.float64), lam.astype(np.float64)
    c_o, s_o = O.encode_e4m3(G.astype(np.float64), U64, lam64, float(rho))
    codes = runs[True][0].codes.cpu().numpy()
    scales = runs[True][0].scales.cpu().numpy()
    check_codes(codes, c_o)
    check_scales(scales, s_o)
    want = O.decode_e4m3(codes, scales, U64, lam64, float(rho))
    check_rows(runs[True][0].G_hat.float().cpu().numpy(), want, bf16=True)
