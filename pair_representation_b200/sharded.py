"""The triangle multiplicative update split over several GPUs (one process per GPU).

The pages' own subject is running this layer on many GPUs ("Scaling
biomolecular modeling with context parallelism in NVIDIA BioNeMo", sections
"2-D tiling of the pair representation" and "Context-parallel implementation
of triangle multiplication"), where the pair representation is tiled over a
2-D device grid and ring exchanges overlap with compute. On one B200 node,
where NVSwitch gives every GPU full bandwidth to every other, the plainest
split that the layer's structure allows is used instead:

  * rows: residue rows are cut into P contiguous blocks R_0 .. R_{P-1}; each
    rank holds z, the mask and the output for its block. The prologue and the
    epilogue are per cell, so a row block is just a grid of |R_r| x N cells.
  * channels: the 128 hidden channels are cut into P contiguous blocks C_r;
    the contraction of a channel needs all N rows of a_c and b_c and touches
    no other channel.
  * per call: prologue on R_r (all channels) -> exchange so that rank q holds
    a_c, b_c for c in C_q over all rows -> contraction of C_q -> exchange so
    that rank q holds x_c for every c over its rows R_q -> epilogue on R_q.

Both exchanges are point-to-point sends of contiguous rows: the rows R_r of
channel c (|R_r| x ld elements) go from rank r to the owner of c, and back for
x. They run as one batch of NCCL sends/receives per exchange
(torch.distributed.batch_isend_irecv); the rank's own share is a local copy.
Per rank and call the exchanges move 3 (P - 1) / P^2 of the bf16 a, b and x
arrays (N^2 x 128 x 2 bytes each).

The kernels are the library's (trimul_prologue_rows, trimul_contract_channels,
trimul_epilogue_rows); this module holds the host logic: the split, the
buffers and the exchanges. ``stages`` may be replaced (tests run the host
logic on CPU ranks with stand-in stages); the default is the CUDA library.
"""
from __future__ import annotations

from dataclasses import dataclass

C = 128


def split(n: int, parts: int, k: int):
    """[start, stop) of block k when n items are cut into `parts` contiguous blocks
    whose sizes differ by at most one (the first n % parts blocks are larger)."""
    base, extra = divmod(n, parts)
    start = k * base + min(k, extra)
    return start, start + base + (1 if k < extra else 0)


@dataclass(frozen=True)
class ShardPlan:
    """The row and channel blocks of a P-way split of an N-residue layer."""

    N: int
    world: int

    def __post_init__(self):
        if self.world < 1 or self.world > C or self.world > self.N:
            raise ValueError("need 1 <= world <= min(N, 128)")

    @property
    def ld(self) -> int:
        """Row pitch of the bf16 a, b, x blocks: N rounded up to 64 (the library's rule)."""
        return (self.N + 63) // 64 * 64

    def rows(self, r: int):
        return split(self.N, self.world, r)

    def channels(self, r: int):
        return split(C, self.world, r)

    def nrows(self, r: int) -> int:
        a, b = self.rows(r)
        return b - a

    def nchannels(self, r: int) -> int:
        a, b = self.channels(r)
        return b - a

    def owner_of_channel(self, c: int) -> int:
        for r in range(self.world):
            a, b = self.channels(r)
            if a <= c < b:
                return r
        raise ValueError(c)


class CudaStages:
    """The per-rank stages on the CUDA library (bf16), enqueued on torch's current
    stream, where the exchanges' NCCL calls are ordered too."""

    def __init__(self, tm, params):
        self.tm, self.p = tm, params

    def prologue_rows(self, z_rows, mask_rows, rows, a, b):
        self.tm.trimul_prologue_rows(z_rows, mask_rows, self.p, rows, a, b)

    def contract_channels(self, direction, channels, a, b, x):
        self.tm.trimul_contract_channels(self.p, direction, channels, a, b, x)

    def epilogue_rows(self, z_rows, x_rows, rows, out_rows):
        self.tm.trimul_epilogue_rows(z_rows, x_rows, self.p, rows, out_rows)


def exchange_rows_to_channels(plan: ShardPlan, rank: int, loc, ch, dist, group=None):
    """loc [128][|R_rank|][ld] (all channels, this rank's rows) -> ch [|C_rank|][N][ld]
    (this rank's channels, all rows). Rows R_r of channel c travel from rank r to
    the owner of c."""
    r0, r1 = plan.rows(rank)
    c0, c1 = plan.channels(rank)
    ops = []
    for q in range(plan.world):
        q0, q1 = plan.channels(q)
        s0, s1 = plan.rows(q)
        if q == rank:
            ch[:, r0:r1].copy_(loc[c0:c1])
            continue
        for c in range(q0, q1):
            ops.append(dist.P2POp(dist.isend, loc[c], q, group))
        for c in range(c0, c1):
            ops.append(dist.P2POp(dist.irecv, ch[c - c0, s0:s1], q, group))
    _run(ops, dist)


def exchange_channels_to_rows(plan: ShardPlan, rank: int, ch, loc, dist, group=None):
    """ch [|C_rank|][N][ld] (this rank's channels, all rows) -> loc [128][|R_rank|][ld]
    (all channels, this rank's rows): the inverse of exchange_rows_to_channels."""
    r0, r1 = plan.rows(rank)
    c0, c1 = plan.channels(rank)
    ops = []
    for q in range(plan.world):
        q0, q1 = plan.channels(q)
        s0, s1 = plan.rows(q)
        if q == rank:
            loc[c0:c1].copy_(ch[:, r0:r1])
            continue
        for c in range(c0, c1):
            ops.append(dist.P2POp(dist.isend, ch[c - c0, s0:s1], q, group))
        for c in range(q0, q1):
            ops.append(dist.P2POp(dist.irecv, loc[c], q, group))
    _run(ops, dist)


def _run(ops, dist):
    if ops:
        for w in dist.batch_isend_irecv(ops):
            w.wait()


class ShardedTriangleMultiplication:
    """One rank's part of a layer split over `plan.world` ranks.

    ``layer(z_rows, mask_rows)`` takes this rank's block of residue rows of z
    ([|R_rank|][N][128]) and of the mask ([|R_rank|][N] or None) and returns the
    same rows of the layer's output. Every rank must call it with the same
    direction and N; the exchanges are collective.
    """

    def __init__(self, plan: ShardPlan, rank: int, direction: int, stages, device, dtype, dist, group=None):
        import torch
        self.plan, self.rank, self.direction = plan, rank, direction
        self.stages, self.dist, self.group = stages, dist, group
        n, ld = plan.N, plan.ld
        nr, nc = plan.nrows(rank), plan.nchannels(rank)
        z = dict(device=device, dtype=dtype)
        # Every row a kernel writes is a contiguous [ld] slice, so the exchanges send
        # whole rows; the columns past N are padding.
        self.a_loc = torch.zeros((C, nr, ld), **z)
        self.b_loc = torch.zeros((C, nr, ld), **z)
        self.a_ch = torch.zeros((nc, n, ld), **z)
        self.b_ch = torch.zeros((nc, n, ld), **z)
        self.x_ch = torch.zeros((nc, n, ld), **z)
        self.x_loc = torch.zeros((C, nr, ld), **z)

    def __call__(self, z_rows, mask_rows=None, out_rows=None):
        import torch
        plan, rank, st = self.plan, self.rank, self.stages
        nr, nc = plan.nrows(rank), plan.nchannels(rank)
        if out_rows is None:
            out_rows = torch.empty_like(z_rows)
        st.prologue_rows(z_rows, mask_rows, nr, self.a_loc, self.b_loc)
        exchange_rows_to_channels(plan, rank, self.a_loc, self.a_ch, self.dist, self.group)
        exchange_rows_to_channels(plan, rank, self.b_loc, self.b_ch, self.dist, self.group)
        st.contract_channels(self.direction, nc, self.a_ch, self.b_ch, self.x_ch)
        exchange_channels_to_rows(plan, rank, self.x_ch, self.x_loc, self.dist, self.group)
        st.epilogue_rows(z_rows, self.x_loc, nr, out_rows)
        return out_rows
