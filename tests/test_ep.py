"""Expert parallelism (int4_expert_grouped_b200/ep.py) on CPU.

The count split and the block map of the received rows against hand-worked
tables; then the whole expert-parallel forward as two (and four) gloo ranks,
with an oracle-backed stand-in for the CUDA compute, against the oracle's
single-process layer: every token's output must match it to rounding, which
fails if a row reaches the wrong rank, the wrong local expert or the wrong
slot on the way back.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def ep(built_library):
    from int4_expert_grouped_b200 import ep as m
    return m


def test_expert_range(ep):
    assert ep.expert_range(128, 8, 0) == (0, 16)
    assert ep.expert_range(128, 8, 7) == (112, 128)
    assert ep.expert_range(16, 1, 0) == (0, 16)
    with pytest.raises(ValueError):
        ep.expert_range(12, 8, 0)


def test_split_counts(ep):
    c = np.array([3, 0, 5, 1, 2, 2], np.int32)
    assert ep.split_counts(c, 2).tolist() == [[3, 0, 5], [1, 2, 2]]
    assert ep.split_counts(c, 3).tolist() == [[3, 0], [5, 1], [2, 2]]
    with pytest.raises(ValueError):
        ep.split_counts(c, 4)


def test_block_map_of_received_rows(ep):
    # two sources, two local experts.  Source 0 sent (300 rows of expert 0,
    # 1 of expert 1), source 1 sent (5, 0): received rows are
    #   [0, 300) src 0 / e0, [300, 301) src 0 / e1, [301, 306) src 1 / e0.
    # Tiles of 128 rows, expert-major, then by source:
    bm, n = ep.build_block_map([[300, 1], [5, 0]], 128)
    assert n == 306
    assert bm.tolist() == [[0, 0, 128], [0, 128, 128], [0, 256, 44], [0, 301, 5], [1, 300, 1]]
    # every received row is covered once
    cover = np.zeros(n, int)
    for e, r0, rows in bm:
        cover[r0:r0 + rows] += 1
    assert (cover == 1).all()


def test_block_map_empty_and_single_source(ep):
    bm, n = ep.build_block_map([[0, 0, 0]], 256)
    assert n == 0 and bm.shape == (0, 3)
    bm, n = ep.build_block_map([[256, 257]], 256)
    assert n == 513
    assert bm.tolist() == [[0, 0, 256], [1, 256, 256], [1, 512, 1]]
    with pytest.raises(ValueError):
        ep.build_block_map([[1, -1]], 256)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(T, E, k, bias_to_first_rank=False):
    import moe_inputs as mi
    inp = mi.make_inputs(mi.Shape(T, 256, E, k, 128, 32), seed=11)
    if bias_to_first_rank:
        # every token prefers the experts of rank 0: the other ranks receive
        # no rows at all
        b = np.full(E, -50.0, np.float32)
        b[: E // 2] = 0.0
        inp.b_r = b
    return inp


def _rank(rank, world, port, T, E, k, bias_to_first_rank, out):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, HERE)
    from ep_stand_in import OracleBackend

    from int4_expert_grouped_b200 import ep
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        inp = _inputs(T, E, k, bias_to_first_rank)
        lo, hi = ep.expert_range(E, world, rank)
        per = T // world
        x = torch.from_numpy(inp.x[rank * per:(rank + 1) * per].astype(np.int32))
        layer = ep.ExpertParallelMoE(OracleBackend(inp, lo, hi), E, world, rank, group=dist.group.WORLD)
        y = layer.forward(x)
        out[rank] = y.numpy().copy()
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,T,E,k,skew", [(2, 64, 16, 4, False), (4, 64, 16, 3, False),
                                              (2, 48, 16, 4, True)])
def test_expert_parallel_forward_gloo(ep, world, T, E, k, skew):
    import oracle
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, T, E, k, skew, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    y = np.concatenate([out[r] for r in range(world)])
    ref = oracle.forward(_inputs(T, E, k, skew))["y"]
    assert y.shape == ref.shape
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-15)


def test_expert_parallel_forward_one_rank(ep):
    """world = 1 needs no process group: the exchanges are local."""
    import torch

    import oracle
    sys.path.insert(0, HERE)
    from ep_stand_in import OracleBackend
    inp = _inputs(40, 16, 4)
    layer = ep.ExpertParallelMoE(OracleBackend(inp, 0, 16), 16)
    y = layer.forward(torch.from_numpy(inp.x.astype(np.int32))).numpy()
    np.testing.assert_allclose(y, oracle.forward(inp)["y"], rtol=1e-12, atol=1e-15)


def _rank_leaves(rank, world, port, mode, out):
    """Rank 1 leaves before the exchange (exits, or stalls without joining it);
    rank 0's forward must end in an error from the process group (the closed
    connection, or its 5 s timeout), not wait for ever."""
    import datetime
    import time

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, HERE)
    from ep_stand_in import OracleBackend

    from int4_expert_grouped_b200 import ep
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        out[rank] = "left"
        if mode == "stall":
            time.sleep(10)  # alive, but never joins the exchange
        os._exit(0)  # gone without a word: no barrier, no destroy
    inp = _inputs(32, 16, 4)
    x = torch.from_numpy(inp.x[:16].astype(np.int32))
    layer = ep.ExpertParallelMoE(OracleBackend(inp, 0, 8), 16, world, rank, group=dist.group.WORLD)
    t0 = time.time()
    try:
        layer.forward(x)
        out[rank] = "no error"
    except RuntimeError as e:
        out[rank] = "error after %.1f s: %s" % (time.time() - t0, str(e).splitlines()[0][:80])
    os._exit(0)


@pytest.mark.parametrize("mode", ["exit", "stall"])
def test_expert_parallel_rank_that_leaves_ends_in_error(ep, mode):
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_leaves, args=(r, 2, port, mode, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[1] == "left"
    assert out[0].startswith("error after"), out[0]
    assert float(out[0].split()[2]) < 15.0, out[0]
