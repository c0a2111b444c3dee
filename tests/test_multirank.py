"""The N > 1 path on the CPU with world_size-2 gloo process groups.

The layer solve itself runs on one GPU.  Under torchrun the benchmark gives each rank its
own independent layer (weak scaling, no collective on the data path) and reduces only the
timing (max over ranks).  The data-parallel form of the Hessian (each rank sums 2 x^T x over
its own calibration tokens, one all-reduce of H: gptq.allreduce_hessian) is checked here too,
with the oracle standing in for the device context.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from oracle import gptq_oracle as O
from post_weight_quantization_16_b200 import gptq as G
from post_weight_quantization_16_b200 import synth


class _OracleContext:
    """The host-side face of a context (get_hessian / set_hessian) over the oracle's Hessian."""

    def __init__(self, n):
        self.H = torch.zeros((n, n), dtype=torch.float64)
        self.n_tok = 0

    def accumulate_hessian(self, X):
        self.H += torch.from_numpy(O.hessian(X))
        self.n_tok += X.shape[0]

    def get_hessian(self):
        return self.H.clone(), self.n_tok

    def set_hessian(self, H, n_tok):
        self.H = H.clone()
        self.n_tok = n_tok


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, lr = bench.dist_env()
        layer0, _ = synth.WORKLOADS["tiny_256x512"]
        layer = bench.rank_layer(layer0, r)
        # timing reduction: the job time is the slowest rank's
        t = bench.max_over_ranks(1.0 + r, w)
        # token-split Hessian through the binding's exchange step (gptq.allreduce_hessian), the
        # oracle standing in for the device context: each rank accumulates its own share
        X = synth.bf16_bits_to_f32(synth.make_x_bf16(layer0)).astype(np.float64)
        shard = np.array_split(X, w)[r]
        ctx = _OracleContext(X.shape[1])
        ctx.accumulate_hessian(shard)
        total = G.allreduce_hessian(ctx)
        bench.barrier(w)
        q.put((r, w, lr, layer.x_seed, layer.w_seed, t, ctx.H.numpy(), total, ctx.n_tok))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=180) for _ in range(world)])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, l0, xs0, ws0, t0, H0, tot0, nt0), (r1, w1, l1, xs1, ws1, t1, H1, tot1, nt1) = res
    assert (r0, r1) == (0, 1) and w0 == w1 == 2 and (l0, l1) == (0, 1)
    # independent layers: rank 0 keeps the workload's own seeds, rank 1 gets other ones
    layer0, _ = synth.WORKLOADS["tiny_256x512"]
    assert (xs0, ws0) == (layer0.x_seed, layer0.w_seed)
    assert xs1 != xs0 and ws1 != ws0
    # max over ranks
    assert t0 == t1 == 2.0
    # all ranks hold the Hessian of the whole calibration set
    Href = O.hessian(synth.bf16_bits_to_f32(synth.make_x_bf16(layer0)))
    assert np.allclose(H0, Href, rtol=1e-12, atol=0) and np.array_equal(H0, H1)
    n_tok = layer0.n_tok
    assert tot0 == tot1 == nt0 == nt1 == n_tok


def test_single_rank_helpers_without_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    layer0, _ = synth.WORKLOADS["tiny_256x512"]
    assert bench.rank_layer(layer0, 0) is layer0
