"""Expert parallelism: the layer's experts split over ranks, one process per GPU.

Rank r holds experts [r E/N, (r+1) E/N) of the E experts (N ranks).  A
forward on a rank's own tokens is:

    route          routing over all E experts (moe_route)
    dispatch       the token rows in expert order (moe_dispatch); the rows for
                   rank r's experts form one segment, because the scatter orders
                   rows by expert (inblix article "Perplexity's Lily engine
                   beats MLX by 35% on M5 Max, no PyTorch needed", paragraph 3:
                   scatter into expert-contiguous order with a block map)
    exchange       per-(destination, expert) counts, then the row segments
                   (all-to-all: segment r to rank r)
    experts        the grouped GEMMs over the received rows for this rank's
                   experts (moe_experts_forward), tiled by a block map built
                   here from the received counts
    exchange back  the expert outputs, the same segments in reverse
    combine        the routing-weighted sum per token (moe_combine)

The received rows are laid out by source rank, and inside each source by local
expert; the block map tiles each (expert, source) segment, experts first, so
one expert's tiles run next to each other and share its weights in L2.  The
results equal those of moe_forward's batched kernels bit for bit: every row
meets the same GEMM arithmetic, only the tiling of rows differs.  (For batches
of at most 8 tokens moe_forward runs its small-batch kernel instead, which
rounds differently.)

The exchanges are torch.distributed all-to-alls (NCCL between GPUs).  The
compute runs in a backend: ``LibraryBackend`` (the CUDA library) is the only
one here; tests pass their own.  There is no CPU fallback.
"""
from __future__ import annotations

import numpy as np
import torch

from . import Plan


def expert_range(E: int, world: int, rank: int) -> tuple[int, int]:
    """The contiguous experts [lo, hi) that `rank` holds."""
    if world <= 0 or E % world != 0:
        raise ValueError("E = %d experts do not split evenly over %d ranks" % (E, world))
    n = E // world
    return rank * n, (rank + 1) * n


def split_counts(counts, world: int) -> np.ndarray:
    """Per-expert row counts [E] -> [world, E / world]: row r holds the counts of
    rank r's experts, in the order the dispatched rows list them."""
    c = np.asarray(counts, dtype=np.int64)
    if c.ndim != 1 or c.shape[0] % world != 0:
        raise ValueError("counts must be [E] with E a multiple of world")
    return c.reshape(world, c.shape[0] // world)


def build_block_map(recv_counts, block_t: int) -> tuple[np.ndarray, int]:
    """Block map of the received rows.

    recv_counts[s, e]: rows that source rank s sent for local expert e.  The
    rows from source s start at the sum of the rows of sources before it, and
    inside them expert e's rows follow those of experts before e.  Returns
    (int32 [nb, 3] entries (expert, first row, rows), total rows): for each
    expert, for each source, its segment in tiles of at most block_t rows.
    """
    rc = np.asarray(recv_counts, dtype=np.int64)
    if rc.ndim != 2 or (rc < 0).any():
        raise ValueError("recv_counts must be a non-negative [world, experts] table")
    world, n_exp = rc.shape
    src_base = np.concatenate([[0], np.cumsum(rc.sum(axis=1))])
    exp_off = np.concatenate([np.zeros((world, 1), np.int64), np.cumsum(rc, axis=1)], axis=1)
    entries = []
    for e in range(n_exp):
        for s in range(world):
            first = int(src_base[s] + exp_off[s, e])
            n = int(rc[s, e])
            for t0 in range(0, n, block_t):
                entries.append((e, first + t0, min(block_t, n - t0)))
    bm = np.asarray(entries, dtype=np.int32).reshape(-1, 3)
    return bm, int(src_base[-1])


class ExpertParallelMoE:
    """One rank of an expert-parallel MoE layer.

    backend: the compute (``LibraryBackend``); group: the torch.distributed
    process group of the ranks (None only with world == 1: the exchanges are
    then skipped, the rows staying where they are).
    """

    def __init__(self, backend, E: int, world: int = 1, rank: int = 0, group=None, block_t: int = 256):
        self.be = backend
        self.E, self.world, self.rank, self.group = E, world, rank, group
        self.lo, self.hi = expert_range(E, world, rank)
        self.block_t = block_t
        if group is None and world > 1:
            raise ValueError("more than one rank needs a process group")
        self._dist = None
        if group is not None:
            import torch.distributed as dist
            self._dist = dist
            self._comm_dev = (torch.device("cuda", torch.cuda.current_device())
                              if dist.get_backend(group) == "nccl" else torch.device("cpu"))

    def _exchange_counts(self, send: np.ndarray) -> np.ndarray:
        if self._dist is None:
            return send.copy()
        t = torch.from_numpy(np.ascontiguousarray(send, dtype=np.int64)).reshape(-1).to(self._comm_dev)
        out = torch.empty_like(t)
        self._dist.all_to_all_single(out, t, group=self.group)
        return out.cpu().numpy().reshape(send.shape)

    def _exchange_rows(self, rows: torch.Tensor, send_rows, recv_rows) -> torch.Tensor:
        if self._dist is None:
            return rows
        out = self.be.empty_rows(int(sum(recv_rows)), like=rows)
        self._dist.all_to_all_single(out, rows.contiguous(), [int(v) for v in recv_rows],
                                     [int(v) for v in send_rows], group=self.group)
        return out

    def forward(self, x):
        """The layer on this rank's tokens x [T, d]; returns y [T, d]."""
        be = self.be
        r = be.route(x)
        xs = be.dispatch(x, r)
        send = split_counts(be.counts(r), self.world)     # [destination, its experts]
        recv = self._exchange_counts(send)                 # [source, my experts]
        send_rows, recv_rows = send.sum(axis=1), recv.sum(axis=1)
        xs_recv = self._exchange_rows(xs, send_rows, recv_rows)
        bm, n_rows = build_block_map(recv, self.block_t)
        o_recv = be.experts(xs_recv, n_rows, bm)
        o_back = self._exchange_rows(o_recv, recv_rows, send_rows)
        return be.combine(o_back, r, x)


class LibraryBackend:
    """The CUDA library as the compute of one rank.

    Routing, dispatch and combine use a plan over all E experts; the GEMMs use
    a plan over this rank's experts with their prepacked weights.  A rank can
    receive every rank's rows, so that plan takes up to world * T_max * k rows.
    The experts of a rank must number a multiple of 8 (a plan's shape rule).
    gate/up/down: the logical int4 weights of ALL experts (numpy, as
    ``MoeLayer`` takes them); only this rank's slice is uploaded.
    """

    def __init__(self, T_max, d, E, k, f, group, gate, up, down, w_r, b_r=None, world=1, rank=0,
                 device="cuda"):
        from .layer import _dev
        self.device = torch.device(device)
        self.T_max, self.d, self.E, self.k, self.f, self.group = T_max, d, E, k, f, group
        lo, hi = expert_range(E, world, rank)
        self.plan = Plan(T_max, d, E, k, f, group)
        self.plan_e = Plan(world * T_max * k, d, hi - lo, 1, f, group)
        logical = [tuple(_dev(np.ascontiguousarray(getattr(p, n)[lo:hi]), self.device)
                         for n in ("q", "scale", "bias")) for p in (gate, up, down)]
        self.packed = torch.empty(self.plan_e.info.packed_weight_bytes, dtype=torch.uint8,
                                  device=self.device)
        self.plan_e.prepack_weights(*logical, self.packed)
        self.w_r = _dev(np.asarray(w_r, np.float32), self.device)
        self.b_r = None if b_r is None else _dev(np.asarray(b_r, np.float32), self.device)
        self.ws = torch.empty(self.plan.info.workspace_bytes, dtype=torch.uint8, device=self.device)
        self.ws_e = torch.empty(self.plan_e.info.workspace_bytes, dtype=torch.uint8, device=self.device)
        self._nb = torch.zeros(4, dtype=torch.int32, device=self.device)
        torch.cuda.synchronize(self.device)

    def empty_rows(self, n, like):
        return torch.empty((n, self.d), dtype=like.dtype, device=self.device)

    def route(self, x):
        T = x.shape[0]
        i32 = dict(dtype=torch.int32, device=self.device)
        r = {
            "topk_idx": torch.empty((max(T, 1), self.k), **i32),
            "topk_w": torch.empty((max(T, 1), self.k), dtype=torch.float32, device=self.device),
            "counts": torch.empty(self.E, **i32),
            "offsets": torch.empty(self.E + 1, **i32),
            "sorted_assign": torch.empty(max(T * self.k, 1), **i32),
            "pos": torch.empty(max(T * self.k, 1), **i32),
            "block_offsets": torch.empty(self.E + 1, **i32),
            "block_map": torch.empty((self.plan.info.max_blocks, 3), **i32),
            "num_blocks": torch.empty(4, **i32),
        }
        self.plan.route(T, x, self.w_r, self.b_r, r, self.ws)
        return r

    def dispatch(self, x, r):
        T = x.shape[0]
        xs = torch.empty((max(T * self.k, 1), self.d), dtype=torch.bfloat16, device=self.device)
        self.plan.dispatch(T, x, r["sorted_assign"], xs, self.ws)
        return xs[:T * self.k]

    def counts(self, r):
        return r["counts"].cpu().numpy()

    def experts(self, xs_recv, n_rows, bm):
        o = torch.empty((max(n_rows, 1), self.d), dtype=torch.bfloat16, device=self.device)
        if n_rows > 0:
            bm_dev = torch.from_numpy(np.ascontiguousarray(bm, dtype=np.int32)).to(self.device)
            self._nb[0] = bm.shape[0]
            self.plan_e.experts_forward(n_rows, xs_recv, bm_dev, self._nb, self.packed, o, self.ws_e)
        return o[:n_rows]

    def combine(self, o_back, r, x):
        T = x.shape[0]
        y = torch.empty((max(T, 1), self.d), dtype=torch.bfloat16, device=self.device)
        self.plan.combine(T, o_back, r["pos"], r["topk_w"], y, self.ws)
        return y[:T]

    def read_status(self):
        """(code, detail) of the routing/combine workspace and of the GEMM workspace."""
        return self.plan.read_status(self.ws), self.plan_e.read_status(self.ws_e)
