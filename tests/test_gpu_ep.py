"""Expert-parallel building blocks on one B200, through the C ABI.

moe_dispatch, moe_experts_forward and moe_combine, chained by ep.py, must give
moe_forward's output bit for bit (the same GEMM arithmetic per row), also
through a one-rank NCCL group and with a block map cut into irregular tiles
in shuffled order; a block map out of range is refused on the device with
MOE_ERR_DEVICE_BOUNDS and leaves the output untouched.  Expert parallelism
over several GPUs is not run here (one GPU per run): its exchanges are
covered by the gloo tests in test_ep.py.
"""
import socket

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle

pytestmark = pytest.mark.gpu

Y_ATOL_REL = 2e-2     # |y - ref| <= 2e-2 * (1 + |ref|), as the layer tests


@pytest.fixture(scope="module")
def moe(built_library):
    assert torch.cuda.is_available(), "the gpu tests need a GPU"
    import int4_expert_grouped_b200 as m
    from int4_expert_grouped_b200 import ep
    from int4_expert_grouped_b200.layer import MoeLayer, bf16_tensor
    m.MoeLayer, m.bf16_tensor, m.ep = MoeLayer, bf16_tensor, ep
    return m


_cache = {}


def setup(moe, name):
    if name not in _cache:
        inp = mi.workload(name)
        s = inp.shape
        layer = moe.MoeLayer.from_inputs(inp)
        x = moe.bf16_tensor(inp.x, "cuda")
        bufs = layer.route_buffers(s.T)
        y = layer.forward(x, route_out=bufs)
        torch.cuda.synchronize()
        assert layer.read_status() == (0, 0)
        _cache[name] = (inp, layer, x, bufs, y.clone())
    return _cache[name]


def backend(moe, inp):
    s = inp.shape
    return moe.ep.LibraryBackend(s.T, s.d, s.E, s.k, s.f, s.group, inp.gate, inp.up, inp.down,
                                 inp.w_r, inp.b_r)


def check_oracle(y, inp):
    ref = oracle.forward(inp)["y"]
    got = y.float().cpu().numpy().astype(np.float64)
    assert (np.abs(got - ref) <= Y_ATOL_REL * (1.0 + np.abs(ref))).all()


@pytest.mark.parametrize("name", ["tiny", "prefill_t512"])
def test_expert_parallel_one_rank_equals_forward(moe, name):
    inp, layer, x, bufs, y_ref = setup(moe, name)
    be = backend(moe, inp)
    y = moe.ep.ExpertParallelMoE(be, inp.shape.E).forward(x)
    torch.cuda.synchronize()
    assert be.read_status() == ((0, 0), (0, 0))
    assert torch.equal(y, y_ref[:inp.shape.T])
    check_oracle(y, inp)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_expert_parallel_through_nccl_one_rank(moe):
    import datetime

    import torch.distributed as dist
    inp, layer, x, bufs, y_ref = setup(moe, "prefill_t512")
    be = backend(moe, inp)
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % _free_port(), rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        y = moe.ep.ExpertParallelMoE(be, inp.shape.E, 1, 0, group=dist.group.WORLD).forward(x)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert be.read_status() == ((0, 0), (0, 0))
    assert torch.equal(y, y_ref[:inp.shape.T])


def test_experts_forward_irregular_tiles(moe):
    """Rows cut into tiles of 1..256 rows, listed in shuffled order."""
    inp, layer, x, bufs, y_ref = setup(moe, "prefill_t512")
    s = inp.shape
    Tk = s.T * s.k
    plan, ws = layer.plan, layer.ws
    xs = torch.empty((Tk, s.d), dtype=torch.bfloat16, device="cuda")
    plan.dispatch(s.T, x, bufs["sorted_assign"], xs, ws)
    counts = bufs["counts"].cpu().numpy()
    offsets = bufs["offsets"].cpu().numpy()
    rng = np.random.default_rng(5)
    entries = []
    for e in range(s.E):
        r, end = int(offsets[e]), int(offsets[e] + counts[e])
        while r < end:
            n = int(min(end - r, rng.integers(1, 257)))
            entries.append((e, r, n))
            r += n
    bm = np.asarray(entries, np.int32)[rng.permutation(len(entries))]
    bm_dev = torch.from_numpy(bm).cuda()
    nb = torch.tensor([len(bm), 0, 0, 0], dtype=torch.int32, device="cuda")
    o = torch.empty((Tk, s.d), dtype=torch.bfloat16, device="cuda")
    plan.experts_forward(Tk, xs, bm_dev, nb, layer.packed, o, ws)
    y = torch.empty((s.T, s.d), dtype=torch.bfloat16, device="cuda")
    plan.combine(s.T, o, bufs["pos"], bufs["topk_w"], y, ws)
    torch.cuda.synchronize()
    assert layer.read_status() == (0, 0)
    assert torch.equal(y, y_ref[:s.T])


@pytest.mark.parametrize("bad", ["row_past_end", "expert_out_of_range", "too_many_entries"])
def test_experts_forward_refuses_bad_block_map(moe, bad):
    inp, layer, x, bufs, y_ref = setup(moe, "tiny")
    s = inp.shape
    rows = 64
    xs = torch.zeros((rows, s.d), dtype=torch.bfloat16, device="cuda")
    bm = np.array([[0, 0, 32], [1, 32, 32]], np.int32)
    n = 2
    if bad == "row_past_end":
        bm[1] = (1, 40, 32)
    elif bad == "expert_out_of_range":
        bm[0, 0] = s.E
    else:
        n = 3
    o = torch.full((rows, s.d), 7.0, dtype=torch.bfloat16, device="cuda")
    nb = torch.tensor([n, 0, 0, 0], dtype=torch.int32, device="cuda")
    layer.plan.experts_forward(rows, xs, torch.from_numpy(bm).cuda(), nb, layer.packed, o, layer.ws)
    torch.cuda.synchronize()
    assert layer.read_status() == (7, 400)
    assert bool((o == 7.0).all())
