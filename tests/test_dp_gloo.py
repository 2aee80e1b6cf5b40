"""Data-parallel exchange of the LoRA gradients on two CPU ranks (gloo).

The flat-buffer layout must be identical on every rank and the in-place
all-reduce must leave every rank with the mean of the ranks' gradients in
every view (or the sum, for the variant that leaves the 1/world to the
optimiser step); an AdamW step with grad_scale = 1/world after the sum must
leave every rank with the parameters of one step on the mean gradient.  CPU
only: the same code path runs over NCCL on GPUs.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from layer_streamed_qlora_b200 import dp
from oracle.optim import adamw_step

SHAPES = [(16, 4096), (6144, 16), (16, 4096), (4096, 16), (32, 4096), (28672, 16), (16, 14336), (4096, 16),
          (3, 5)]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        flat, views = dp.flat_views(SHAPES, "cpu")
        g = torch.Generator().manual_seed(100 + rank)
        vals = []
        for v in views:
            v.copy_(torch.randn(v.shape, generator=g))
            vals.append(v.clone())
        summed = flat.clone()
        dp.allreduce_mean_(flat)
        world_seen = dp.allreduce_sum_(summed)
        # the training step's exchange: a sum, then the optimiser step with
        # grad_scale = 1/world on parameters that start equal on every rank
        theta0 = np.linspace(-0.05, 0.05, summed.numel())
        z = np.zeros(summed.numel())
        theta1, _, _ = adamw_step(theta0, summed.numpy().astype(np.float64), z, z, 1, 5e-4,
                                  grad_scale=1.0 / world_seen)
        # numpy copies: plain pickles (tensors would travel as shared-memory handles)
        q.put((rank, [v.numpy().copy() for v in views], [v.numpy() for v in vals], dp.flat_layout(SHAPES),
               flat.numpy().copy(), summed.numpy().copy(), world_seen, theta1))
    finally:
        dist.destroy_process_group()


def test_flat_layout_alignment():
    offs, n = dp.flat_layout(SHAPES)
    assert all(o % dp.ALIGN == 0 for o in offs) and dp.ALIGN % 128 == 0
    assert n >= sum(a * b for a, b in SHAPES)
    # fp32 views (gradients, AdamW state) on 512-byte and bf16 views (the
    # factors the GEMMs read) on 256-byte boundaries, at the same offsets
    flat, views = dp.flat_views(SHAPES, "cpu")
    flat16, views16 = dp.flat_views(SHAPES, "cpu", torch.bfloat16)
    assert flat16.numel() == flat.numel()
    for v, w, sh in zip(views, views16, SHAPES):
        assert tuple(v.shape) == sh and v.is_contiguous() and (v.data_ptr() - flat.data_ptr()) % 512 == 0
        assert tuple(w.shape) == sh and w.is_contiguous() and (w.data_ptr() - flat16.data_ptr()) % 256 == 0
        assert (w.data_ptr() - flat16.data_ptr()) // 2 == (v.data_ptr() - flat.data_ptr()) // 4


def test_allreduce_sum_single_process_is_noop():
    flat, _ = dp.flat_views([(4, 4)], "cpu")
    flat.fill_(3.0)
    assert dp.allreduce_sum_(flat) == 1
    assert torch.all(flat == 3.0)


def test_allreduce_mean_single_process_is_noop():
    flat, _ = dp.flat_views([(4, 4)], "cpu")
    flat.fill_(3.0)
    dp.allreduce_mean_(flat)
    assert torch.all(flat == 3.0)


@pytest.mark.timeout(120)
def test_two_rank_gradient_average():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, after, before, layout, gap, summed, world_seen, theta1 = q.get(timeout=100)
        res[rank] = (after, before, layout, gap, summed, world_seen, theta1)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert res[0][2] == res[1][2]  # same layout on every rank
    for i in range(len(SHAPES)):
        mean = (res[0][1][i] + res[1][1][i]) / 2
        for r in range(world):
            torch.testing.assert_close(torch.from_numpy(res[r][0][i]), torch.from_numpy(mean), rtol=1e-6, atol=1e-6)
    # the sum variant leaves the 1/world to the caller and reports world
    offs, n = dp.flat_layout(SHAPES)
    for r in range(world):
        assert res[r][5] == world
        torch.testing.assert_close(torch.from_numpy(res[r][4]), torch.from_numpy(res[r][3]) * world, rtol=1e-6,
                                   atol=1e-6)
    # after the optimiser step every rank holds the same parameters: those of
    # one AdamW step on the mean gradient
    assert np.array_equal(res[0][6], res[1][6])
    mean_flat = (res[0][4] / world).astype(np.float64)
    z = np.zeros(mean_flat.size)
    ref, _, _ = adamw_step(np.linspace(-0.05, 0.05, mean_flat.size), mean_flat, z, z, 1, 5e-4)
    np.testing.assert_allclose(res[0][6], ref, rtol=1e-12, atol=1e-15)
    # the alignment padding between views stays zero
    for r in range(world):
        pad = torch.ones(n, dtype=torch.bool)
        for o, (a, b) in zip(offs, SHAPES):
            pad[o:o + a * b] = False
        assert torch.all(torch.from_numpy(res[r][3])[pad] == 0)
