"""Data-parallel use of the codec (review page, referee report on section II.A,
Eq. (1): each rank r holds its own gradient g^(r); abstract: GIFT leaves the
communication collective unchanged).

coded_allreduce replaces the all-reduce of one layer's gradient: every rank
codes its gradient with the shared factor, the codes and block scales of all
ranks are all-gathered (NCCL over NVLink on a GPU node), and every rank
decodes the sum, alpha sum_r T^{-1}(W_hat_r) = alpha T^{-1}(sum_r W_hat_r)
(gift_decode_sum: the inverse transform is linear, so it is applied once).
The collective moves 1 + 4/128 bytes per element and rank instead of the
gradient's 2 or 4.  The gathered tensors are ordinary local buffers: no
kernel reads another GPU's memory.

`encode` and `decode_sum` default to the library's calls; they are
parameters so that the collective plumbing can run on CPU ranks with other
callables (the gloo tests do that).
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence

import torch
import torch.distributed as dist

from . import ops


def coded_allreduce(G: torch.Tensor, U=None, lam=None, rho=None, mean: bool = True, group=None,
                    encode: Optional[Callable] = None, decode_sum: Optional[Callable] = None,
                    out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """alpha * sum over ranks of the decoded gradients (alpha = 1/world for the
    mean, 1 for the sum), identical on every rank of `group`."""
    world = dist.get_world_size(group)
    alpha = 1.0 / world if mean else 1.0
    if encode is None:
        encode = lambda g: ops.encode(g, U, lam, rho)
    if decode_sum is None:
        decode_sum = lambda cs, ss, a: ops.decode_sum(cs, ss, U, lam, rho, alpha=a, out_dtype=G.dtype, out=out)
    codes, scales = encode(G)
    cs = [torch.empty_like(codes) for _ in range(world)]
    ss = [torch.empty_like(scales) for _ in range(world)]
    dist.all_gather(cs, codes, group=group)
    dist.all_gather(ss, scales, group=group)
    return decode_sum(cs, ss, alpha)
