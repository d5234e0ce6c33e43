"""GPU decode-and-sum (gift_decode_sum) against the oracle: the sum, scaled by
alpha, of the oracle's decodes of several code sets, under the G_hat criteria
of _cmp.py (1e-3 of the row maximum, plus one bf16 rounding for bf16 output).
"""
import numpy as np
import pytest
import torch

from oracle import gift_oracle as O
from geometry_aware_fp8_b200 import ops, synth

from _cmp import check_rows
from test_gpu_codec import _factor, _to_dev

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.mark.parametrize("rank", [0, 32])
@pytest.mark.parametrize("parts,alpha", [(1, 1.0), (3, 1.0 / 3), (8, 0.125)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_decode_sum_matches_oracle(rank, parts, alpha, out_dtype):
    d_out, d_in = 130, 512
    Q, U, lam, rho = _factor(d_in, 300)
    U64, lam64 = U.astype(np.float64), lam.astype(np.float64)
    Ue = U64 if rank else np.zeros((d_in, 0))
    le = lam64 if rank else np.zeros(0)
    re = float(rho) if rank else 1.0
    cs, ss, want = [], [], 0.0
    for r in range(parts):
        G = synth.to_storage(synth.gradient(d_out, Q, 1.0, 310 + r), "bf16")
        c, s = O.encode_e4m3(G, Ue, le, re)
        cs.append(c)
        ss.append(s)
        want = want + O.decode_e4m3(c, s, Ue, le, re)
    want = alpha * want
    dev_args = _to_dev(U, lam, np.array([rho], dtype=np.float32)) if rank else (None, None, None)
    st = torch.zeros((1,), device=DEV, dtype=torch.int32)
    out = ops.decode_sum(_to_dev(*cs), _to_dev(*ss), *dev_args, alpha=alpha, out_dtype=out_dtype, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    check_rows(out.float().cpu().numpy(), want, bf16=out_dtype == torch.bfloat16)
