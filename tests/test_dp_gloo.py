"""The data-parallel path of bench.py on two CPU ranks (gloo).

The layer is data parallel: every rank holds the same NF4 weights and its own
tokens, and the only exchange is the sum of the adapter gradients dA, dB over
ranks.  bench.py keeps every projection's dA and dB as views of one flat fp32
buffer (the kernels write into the views, one in-place all-reduce sums them)
and reports the slowest rank's time.  These tests run those helpers on two
gloo ranks: the views alias the buffer at 16-byte aligned offsets, every rank
ends with the sum of both ranks' gradients in every view, and the time
reduction returns the maximum.
"""
from __future__ import annotations

import importlib.util
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHAPES = (("q", 64, 128), ("gate", 192, 128), ("down", 128, 192))
R = 8


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _grads_of(rank):
    g = torch.Generator().manual_seed(1000 + rank)
    return [(torch.randn(R, K, generator=g), torch.randn(N, R, generator=g)) for _, N, K in SHAPES]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench = _bench()
        flat, views = bench.grad_buffer(SHAPES, R, "cpu")
        for (dA, dB), (a, b) in zip(views, _grads_of(rank)):
            dA.copy_(a)          # what the backward kernels write
            dB.copy_(b)
        bench.allreduce_sum(flat, world)
        want = [(sum(_grads_of(k)[i][0] for k in range(world)), sum(_grads_of(k)[i][1] for k in range(world)))
                for i in range(len(SHAPES))]
        ok = all(torch.allclose(dA, a, rtol=0, atol=1e-6) and torch.allclose(dB, b, rtol=0, atol=1e-6)
                 for (dA, dB), (a, b) in zip(views, want))
        slowest = bench.max_over_ranks(1.5 + rank, world, "cpu")
        out[rank] = (ok, slowest)
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_grad_buffer_views_alias_one_aligned_buffer():
    bench = _bench()
    flat, views = bench.grad_buffer(SHAPES, R, "cpu")
    assert flat.numel() == sum(R * K + N * R for _, N, K in SHAPES)
    base = flat.data_ptr()
    for (dA, dB), (_, N, K) in zip(views, SHAPES):
        assert dA.shape == (R, K) and dB.shape == (N, R)
        assert dA.is_contiguous() and dB.is_contiguous()
        assert (dA.data_ptr() - base) % 16 == 0 and (dB.data_ptr() - base) % 16 == 0
    views[1][0].fill_(3.0)             # a write through a view lands in the flat buffer
    assert float(flat.sum()) == 3.0 * R * SHAPES[1][2]


def test_single_rank_reductions_are_identity():
    bench = _bench()
    flat, _ = bench.grad_buffer(SHAPES, R, "cpu")
    flat.copy_(torch.arange(flat.numel(), dtype=torch.float32))
    before = flat.clone()
    bench.allreduce_sum(flat, 1)
    assert torch.equal(flat, before)
    assert bench.max_over_ranks(2.5, 1, "cpu") == 2.5


@pytest.mark.timeout(180)
def test_two_gloo_ranks_sum_gradients_and_take_slowest_time():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    for rank in range(world):
        ok, slowest = res[rank]
        assert ok, f"rank {rank}: gradients are not the sum over ranks"
        assert slowest == 2.5
