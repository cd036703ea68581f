"""Multi-rank host logic of bench.py on CPU: two gloo ranks, replicas only.

Each rank times its own replica; the reported time is the slowest rank's and
the throughput counts the cells of every rank. The reference arm runs on
rank 0 alone and the other ranks leave without work.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    local_ms = [120.0, 180.0][rank]
    got = bench.max_over_ranks(local_ms, dist, "cpu")
    val = bench.pair_cells_per_s(world, 10, 2, 768, got)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, got, val))


def test_two_rank_max_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [180.0, 180.0]
    expect = 2 * 10 * 2 * 768 * 768 / 0.18
    assert all(abs(r[2] - expect) < 1e-6 * expect for r in res)


def test_single_rank_passthrough():
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.pair_cells_per_s(1, 4, 2, 100, 1000.0) == 4 * 2 * 100 * 100


def test_reference_arm_other_ranks_do_no_work(capsys):
    class A:
        workload, steps, warmup, reference_budget = 3, 1, 3, 1.0
    bench.run_reference(A(), rank=1, world=2)
    assert capsys.readouterr().out == ""


def test_flop_and_byte_accounting():
    N = 768
    assert bench.flops_per_cell(N) * N * N == 2 * N ** 3 * 128 + 2 * N * N * (4 * 128 * 128 + 128 * 128 + 128 * 128)
    alg = bench.kernel_algorithmic(N)
    assert alg["contract_tc_kernel"][0] == 2 * N ** 3 * 128
    assert alg["prologue_tc_kernel"][0] == N * N * 770 + 131072
    assert alg["epilogue_tc_kernel"][0] == N * N * 768 + 65536


def test_backward_and_attention_accounting():
    """The secondary figures' work counts, restated from the shapes the steps run."""
    N, c = 768, 128
    gemm = lambda m, n, k: 2 * m * n * k
    cells = N * N
    per_call = (gemm(cells, 4 * c, c) + 2 * N ** 3 * c          # recomputed projections a, b and x
                + gemm(cells, 5 * c, c) + gemm(cells, c, c)      # P and Y
                + gemm(cells, c, c)                              # dL/dxh
                + 2 * 2 * N ** 3 * c                             # contraction adjoint dA, dB
                + gemm(6 * c, c, cells)                          # weight gradients (K = cells)
                + gemm(cells, c, 5 * c))                         # dL/dzh
    assert bench.backward_flops_per_cell(N) * cells == per_call
    # minimum bytes per cell, bf16 = 2 B, fp32 = 4 B, stats 8 B
    steps = [256 + 256 + 8, 256 + 256 + 8,             # LayerNorms
             256 + 5 * 256, 256 + 256,                 # P (bf16 out), Y
             256 + 256 + 256 + 256 + 256,              # gate adjoint: P_g, Y, dout in; dy, dP_g out
             256 + 512,                                # dL/dxh (fp32 out)
             512 + 256 + 8 + 256,                      # LN_out adjoint
             2 * (256 + 256 + 256),                    # contraction adjoint
             512 + 1024 + 2 + 1024,                    # input-gate adjoint
             1280 + 256 + 256 + 256,                   # weight-gradient partials
             1280 + 512,                               # dL/dzh
             512 + 256 + 8 + 256]                      # LN_in adjoint
    assert bench.BACKWARD_BYTES_PER_CELL == sum(steps)
    B, n, H = bench.ATTN_SHAPE["batch"], bench.ATTN_SHAPE["n_atoms"], bench.ATTN_SHAPE["heads"]
    assert (B, n, H, bench.ATTN_SHAPE["head_dim"]) == (8, 768 * 24, 4, 32)
