"""The multi-GPU split's host logic on CPU ranks (gloo), against the oracle.

pair_representation_b200.sharded cuts the layer into row blocks (prologue,
epilogue) and channel blocks (contraction) with two point-to-point exchanges.
Here each rank runs it with stand-in stages computed by the float64 oracle on
CPU tensors, over gloo, and checks its output rows against the oracle's whole
layer: a wrong block, a channel sent to the wrong owner, rows received at the
wrong offset or a missing self copy all change the result. World sizes 2 and 3
(ragged row and channel blocks), both directions.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from pair_representation_b200.sharded import ShardPlan, split

N = 37


class OracleStages:
    """The three per-rank stages, computed by the oracle on float64 CPU tensors in
    the library's layouts (a, b, x channel-major [channels][rows][ld])."""

    def __init__(self, case, eps=1e-5):
        self.case, self.eps = case, eps

    def _square(self, z_rows, extra=None):
        import oracle  # noqa: F401
        n = self.case["z"].shape[0]
        z = np.zeros((n, n, 128), dtype=np.float32)
        z[:z_rows.shape[0]] = z_rows.numpy()
        sq = {k: v for k, v in self.case.items() if k not in ("z", "mask", "m")}
        sq["z"] = z
        if extra is not None:
            m = np.zeros((n, n), dtype=np.float32)
            m[:extra.shape[0]] = extra.numpy()
            sq["mask"] = m
        return sq

    def prologue_rows(self, z_rows, mask_rows, rows, a, b):
        import torch

        import oracle
        pa, pb = oracle.project(self._square(z_rows, mask_rows), eps=self.eps)
        for src, dst in ((pa, a), (pb, b)):
            dst.zero_()
            dst[:, :, :N] = torch.from_numpy(src[:rows].transpose(2, 0, 1).copy())

    def contract_channels(self, direction, channels, a, b, x):
        import torch

        import oracle
        am = a[:, :, :N].numpy().transpose(1, 2, 0)
        bm = b[:, :, :N].numpy().transpose(1, 2, 0)
        xm = oracle.contract(am, bm, "incoming" if direction else "outgoing")
        x.zero_()
        x[:, :, :N] = torch.from_numpy(xm.transpose(2, 0, 1).copy())

    def epilogue_rows(self, z_rows, x_rows, rows, out_rows):
        import torch

        import oracle
        sq = self._square(z_rows)
        xs = np.zeros((N, N, 128))
        xs[:rows] = x_rows[:, :, :N].numpy().transpose(1, 2, 0)
        out_rows.copy_(torch.from_numpy(oracle.finish(sq, xs, eps=self.eps)[:rows]))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, direction, q):
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    import pair_inputs as pi
    from pair_representation_b200.sharded import ShardedTriangleMultiplication

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        case = pi.random_case(N, 900 + world, affine=True, mask="random")
        plan = ShardPlan(N, world)
        r0, r1 = plan.rows(rank)
        layer = ShardedTriangleMultiplication(plan, rank, direction, OracleStages(case), "cpu", torch.float64, dist)
        z_rows = torch.from_numpy(case["z"][r0:r1].astype(np.float64))
        m_rows = torch.from_numpy(case["mask"][r0:r1].astype(np.float64))
        out = layer(z_rows, m_rows).numpy()
        ref = oracle.trimul(case, "incoming" if direction else "outgoing")[r0:r1]
        err = float(np.abs(out - ref).max() / np.abs(ref).max())
        dist.barrier()
        q.put((rank, err, None))
    except Exception as e:  # noqa: BLE001 - reported to the parent
        q.put((rank, None, repr(e)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("direction", [0, 1])
def test_sharded_layer_matches_oracle(world, direction):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, direction, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, exc in res:
        assert exc is None, (rank, exc)
        assert err <= 1e-12, (rank, err)


def test_plan_blocks_cover_everything_once():
    for n, world in ((37, 3), (768, 8), (3605, 8), (5, 5), (128, 128)):
        plan = ShardPlan(n, world)
        rows = [plan.rows(r) for r in range(world)]
        chans = [plan.channels(r) for r in range(world)]
        assert rows[0][0] == 0 and rows[-1][1] == n
        assert chans[0][0] == 0 and chans[-1][1] == 128
        for (a0, a1), (b0, b1) in zip(rows, rows[1:]):
            assert a1 == b0 and a1 > a0
        assert max(b - a for a, b in rows) - min(b - a for a, b in rows) <= 1
        assert all(plan.owner_of_channel(c) == next(r for r, (a, b) in enumerate(chans) if a <= c < b)
                   for c in range(128))
    assert split(10, 3, 0) == (0, 4) and split(10, 3, 2) == (7, 10)
    with pytest.raises(ValueError):
        ShardPlan(4, 5)
