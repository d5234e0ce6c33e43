"""Data-parallel plumbing of the codec on two CPU ranks (gloo).

geometry_aware_fp8_b200.dp.coded_allreduce codes each rank's gradient, all-
gathers the codes and block scales, and decodes their sum.  The kernels need
a GPU, so here the encode and decode-sum steps are the oracle's (numpy on the
CPU); what is tested is the collective: every rank must end with the mean of
every rank's decoded gradient, in the same order, bit for bit the same on
both ranks, and equal to the sum computed by one process from all ranks'
inputs.  The GPU decode-and-sum kernel is checked against the oracle in
tests/test_gpu_dp.py.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import gift_oracle as O
from geometry_aware_fp8_b200 import dp, synth

D_IN, D_OUT = 256, 40


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _factor():
    Q = synth.haar_orthogonal(D_IN, 71)
    X = synth.activations(1024, Q, synth.column_power(D_IN, 1.0), 72)
    U, lam, rho, _ = O.factor_refresh(O.input_factor(X), 32, 16, 4, seed=73)
    return Q, U, lam, rho


def _grad(rank, Q):
    return synth.to_storage(synth.gradient(D_OUT, Q, 1.0, 80 + rank), "f32")


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        Q, U, lam, rho = _factor()
        G = torch.from_numpy(_grad(rank, Q))

        def enc(g):
            c, s = O.encode_e4m3(g.numpy().astype(np.float64), U, lam, rho)
            return torch.from_numpy(c), torch.from_numpy(s)

        def dsum(cs, ss, alpha):
            tot = sum(O.dequantize_e4m3_blocks(c.numpy(), s.numpy()) for c, s in zip(cs, ss))
            return torch.from_numpy(alpha * (tot @ O.transform_matrix(U, lam, rho, inverse=True)))

        out = dp.coded_allreduce(G, mean=True, encode=enc, decode_sum=dsum)
        q.put((rank, out.numpy()))
    finally:
        dist.destroy_process_group()


def test_coded_allreduce_on_two_gloo_ranks_gives_the_mean_of_decoded_gradients():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert np.array_equal(res[0], res[1])
    Q, U, lam, rho = _factor()
    want = sum(O.decode_e4m3(*O.encode_e4m3(_grad(r, Q).astype(np.float64), U, lam, rho), U, lam, rho)
               for r in range(world)) / world
    # sum_r T^{-1}(W_hat_r) and T^{-1}(sum_r W_hat_r) differ only by fp64 rounding
    assert np.linalg.norm(res[0] - want) <= 1e-12 * np.linalg.norm(want)
    # the mean of the decoded gradients is close to the mean gradient itself
    G_mean = sum(_grad(r, Q).astype(np.float64) for r in range(world)) / world
    assert O.roundtrip_error(G_mean, res[0]) < 0.3
