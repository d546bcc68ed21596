"""CUDA path (through the C ABI) against the CPU oracle, element by element.

Integer outputs (top-k indices, counts, offsets, scatter order, inverse
positions, block map) must match bit for bit; routing weights within 1e-6
relative; the layer output within |y - ref| <= 2e-2 * (1 + |ref|) with the
relative RMS error also reported and bounded.  Small workloads are checked in
full; the 8K-token and the 32K-token Zipf prefill layers have every token's
output checked (the oracle computes them one token at a time).
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle

pytestmark = pytest.mark.gpu

Y_ATOL_REL = 2e-2     # |y - ref| <= 2e-2 * (1 + |ref|)
Y_REL_RMS = 1.5e-2    # ||y - ref|| / ||ref||
W_REL = 1e-6          # routing weights


@pytest.fixture(scope="module")
def moe(built_library):
    assert torch.cuda.is_available(), "the gpu tests need a GPU"
    import int4_expert_grouped_b200 as m
    from int4_expert_grouped_b200.layer import MoeLayer, bf16_tensor
    m.MoeLayer, m.bf16_tensor = MoeLayer, bf16_tensor
    return m


def oracle_route(inp, T=None, block_t=256):
    x = inp.x if T is None else inp.x[:T]
    logits = oracle.router_logits(x, inp.w_r, inp.b_r)
    idx = oracle.topk(logits, inp.shape.k)
    w = oracle.topk_weights(logits, idx)
    counts, offsets = oracle.counts_offsets(idx, inp.shape.E)
    sa, pos = oracle.scatter(idx, offsets)
    bo, bm, nb = oracle.block_map(counts, offsets, block_t)
    return dict(topk_idx=idx, topk_w=w, counts=counts, offsets=offsets, sorted_assign=sa,
                pos=pos, block_offsets=bo, block_map=bm, num_blocks=nb)


def check_route(got, ref, T, k):
    g = {n: t.cpu().numpy() for n, t in got.items()}
    assert np.array_equal(g["topk_idx"][:T], ref["topk_idx"]), "topk_idx"
    rel = np.abs(g["topk_w"][:T].astype(np.float64) - ref["topk_w"]) / np.abs(ref["topk_w"])
    assert rel.max() <= W_REL, ("topk_w", rel.max())
    assert np.array_equal(g["counts"], ref["counts"]), "counts"
    assert np.array_equal(g["offsets"], ref["offsets"]), "offsets"
    assert np.array_equal(g["sorted_assign"][:T * k], ref["sorted_assign"]), "sorted_assign"
    assert np.array_equal(g["pos"][:T * k], ref["pos"]), "pos"
    assert np.array_equal(g["block_offsets"], ref["block_offsets"]), "block_offsets"
    nb = int(g["num_blocks"][0])
    assert nb == ref["num_blocks"], "num_blocks"
    assert np.array_equal(g["block_map"][:nb], ref["block_map"]), "block_map"


def check_y(y_gpu: torch.Tensor, ref: np.ndarray, what=""):
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(y)), what
    err = np.abs(y - ref)
    bound = Y_ATOL_REL * (1.0 + np.abs(ref))
    worst = float((err / bound).max())
    rel_rms = float(np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-30))
    print("%s: max err/bound %.4f, rel-RMS %.3e, max |err| %.3e" % (what, worst, rel_rms, err.max()))
    assert worst <= 1.0, (what, worst)
    assert rel_rms <= Y_REL_RMS, (what, rel_rms)
    return rel_rms


_cache = {}


def workload(name):
    if name not in _cache:
        _cache[name] = mi.workload(name)
    return _cache[name]


@pytest.mark.parametrize("name", ["tiny", "decode_t1", "decode_t4", "prefill_t512"])
def test_layer_full(moe, name):
    inp = workload(name)
    s = inp.shape
    layer = moe.MoeLayer.from_inputs(inp)
    x = moe.bf16_tensor(inp.x, "cuda")
    bufs = layer.route_buffers(s.T)
    y = layer.forward(x, route_out=bufs)
    torch.cuda.synchronize()
    assert layer.read_status() == (0, 0)
    ref = oracle.forward(inp)
    rref = oracle_route(inp)
    check_route(bufs, rref, s.T, s.k)
    check_y(y[:s.T], ref["y"], name)


def test_layer_t8192_every_token(moe):
    # the 8192-token prefill layer: routing in full and the output of every
    # token against the oracle (about 9 s of CPU on 16 cores)
    inp = workload("prefill_t8192")
    s = inp.shape
    layer = moe.MoeLayer.from_inputs(inp)
    x = moe.bf16_tensor(inp.x, "cuda")
    bufs = layer.route_buffers(s.T)
    y = layer.forward(x, route_out=bufs)
    torch.cuda.synchronize()
    assert layer.read_status() == (0, 0)
    rref = oracle_route(inp)
    check_route(bufs, rref, s.T, s.k)
    toks = np.arange(s.T)
    yref, idx, _ = oracle.token_outputs(inp, toks)
    assert np.array_equal(idx, rref["topk_idx"])
    check_y(y[:s.T], yref, "prefill_t8192, every token")


def block_entry_tokens(rref, k):
    """Tokens of the first and the last row of every block-map entry."""
    bm = rref["block_map"]
    sa = rref["sorted_assign"]
    first = sa[bm[:, 1]] // k
    last = sa[bm[:, 1] + bm[:, 2] - 1] // k
    return np.unique(np.concatenate([first, last]))


def test_layer_t32768_zipf_every_token(moe):
    # the Zipf-skewed 32768-token layer: routing in full and the output of
    # every token (the first and last rows of every block-map entry, and every
    # row of the most and of the least loaded non-empty expert, among them)
    inp = workload("prefill_t32768_zipf")
    s = inp.shape
    layer = moe.MoeLayer.from_inputs(inp)
    x = moe.bf16_tensor(inp.x, "cuda")
    bufs = layer.route_buffers(s.T)
    y = layer.forward(x, route_out=bufs)
    torch.cuda.synchronize()
    assert layer.read_status() == (0, 0)
    rref = oracle_route(inp)
    check_route(bufs, rref, s.T, s.k)
    counts, offsets, sa = rref["counts"], rref["offsets"], rref["sorted_assign"]
    nonempty = np.flatnonzero(counts)
    hot = int(nonempty[np.argmax(counts[nonempty])])
    cold = int(nonempty[np.argmin(counts[nonempty])])
    expert_tokens = lambda e: sa[offsets[e]:offsets[e + 1]] // s.k
    toks = np.arange(s.T)
    covered = np.unique(np.concatenate([block_entry_tokens(rref, s.k), expert_tokens(hot),
                                        expert_tokens(cold)]))
    assert covered.size > 0 and covered.max() < s.T
    print("checking all %d tokens (%d block-map entries; expert %d has %d rows, expert %d has %d)"
          % (s.T, rref["num_blocks"], hot, counts[hot], cold, counts[cold]))
    yref, idx, _ = oracle.token_outputs(inp, toks)
    assert np.array_equal(idx, rref["topk_idx"])
    check_y(y[:s.T], yref, "prefill_t32768_zipf, every token")


def test_route_entry_point_matches_forward(moe):
    inp = workload("prefill_t512")
    s = inp.shape
    layer = moe.MoeLayer.from_inputs(inp)
    x = moe.bf16_tensor(inp.x, "cuda")
    a = layer.route(x)
    b = layer.route_buffers(s.T)
    layer.forward(x, route_out=b)
    torch.cuda.synchronize()
    for n in a:
        if n == "block_map":
            nb = int(a["num_blocks"][0])
            assert torch.equal(a[n][:nb], b[n][:nb])
        elif n == "num_blocks":
            assert int(a[n][0]) == int(b[n][0])
        else:
            assert torch.equal(a[n], b[n]), n


def test_repeat_calls_and_host_path(moe):
    inp = workload("tiny")
    s = inp.shape
    layer = moe.MoeLayer.from_inputs(inp)
    x = moe.bf16_tensor(inp.x, "cuda")
    y1 = layer.forward(x).clone()
    y2 = layer.forward(x).clone()
    xh = torch.from_numpy(inp.x.view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = torch.empty((s.T, s.d), dtype=torch.bfloat16).pin_memory()
    layer.forward_host(xh, yh)
    ref = oracle.forward(inp)["y"]
    check_y(y1, ref, "first call")
    check_y(y2, ref, "second call")
    check_y(yh, ref, "host buffers")
    # no floating-point atomics anywhere: repeated calls agree bit for bit
    assert torch.equal(y1, y2)


def test_empty_batch(moe):
    inp = workload("tiny")
    layer = moe.MoeLayer.from_inputs(inp)
    x = torch.empty((0, inp.shape.d), dtype=torch.bfloat16, device="cuda")
    bufs = layer.route_buffers(0)
    layer.forward(x, route_out=bufs)
    torch.cuda.synchronize()
    assert int(bufs["num_blocks"][0]) == 0
    assert torch.count_nonzero(bufs["counts"]).item() == 0
    assert torch.count_nonzero(bufs["offsets"]).item() == 0


@pytest.mark.parametrize("T", [1, 3, 31, 77, 129, 255, 257])
def test_ragged_token_counts(moe, T):
    shape = mi.Shape(T=300, d=256, E=8, k=2, f=128, group=32)
    inp = mi.make_inputs(shape, 40 + T)
    layer = moe.MoeLayer.from_inputs(inp)
    x = moe.bf16_tensor(inp.x[:T], "cuda")
    bufs = layer.route_buffers(T)
    y = layer.forward(x, route_out=bufs)
    torch.cuda.synchronize()
    sub = mi.Inputs(mi.Shape(T, 256, 8, 2, 128, 32), inp.seed, inp.x[:T], inp.w_r, inp.b_r,
                    inp.gate, inp.up, inp.down)
    ref = oracle.forward(sub)
    check_route(bufs, oracle_route(sub), T, 2)
    check_y(y[:T], ref["y"], "T=%d" % T)


def test_all_tokens_same_experts(moe):
    # a zero router with a decreasing bias sends every token to experts 0..k-1:
    # each of those experts gets T rows (several full blocks and a ragged one)
    shape = mi.Shape(T=300, d=256, E=8, k=2, f=128, group=32)
    inp = mi.make_inputs(shape, 7)
    inp.w_r = np.zeros_like(inp.w_r)
    inp.b_r = -np.arange(8, dtype=np.float32)
    layer = moe.MoeLayer.from_inputs(inp)
    x = moe.bf16_tensor(inp.x, "cuda")
    bufs = layer.route_buffers(300)
    y = layer.forward(x, route_out=bufs)
    torch.cuda.synchronize()
    rref = oracle_route(inp)
    assert list(rref["counts"]) == [300, 300, 0, 0, 0, 0, 0, 0]
    check_route(bufs, rref, 300, 2)
    check_y(y[:300], oracle.forward(inp)["y"], "concentrated")


def test_streaming_form_large_blocks(moe):
    # Fewer than 64 rows per expert on average (T*k = 600 < 64*E) takes the
    # GEMMs' streaming form, whose units are halves of a block's rows; a bias
    # that puts expert 0 first for every token gives it 300 rows (a full
    # 256-row block, both halves in use, and a 44-row block whose second half
    # is empty), while the other experts get a few rows each.
    shape = mi.Shape(T=300, d=256, E=64, k=2, f=128, group=32)
    assert shape.T * shape.k < 64 * shape.E
    inp = mi.make_inputs(shape, 8)
    inp.b_r = np.zeros(64, dtype=np.float32)
    inp.b_r[0] = 50.0
    layer = moe.MoeLayer.from_inputs(inp)
    x = moe.bf16_tensor(inp.x, "cuda")
    bufs = layer.route_buffers(300)
    y = layer.forward(x, route_out=bufs)
    torch.cuda.synchronize()
    assert layer.read_status() == (0, 0)
    rref = oracle_route(inp)
    assert rref["counts"][0] == 300
    check_route(bufs, rref, 300, 2)
    check_y(y[:300], oracle.forward(inp)["y"], "streaming form, large blocks")


def test_every_expert_selected(moe):
    shape = mi.Shape(T=64, d=256, E=8, k=8, f=128, group=64)
    inp = mi.make_inputs(shape, 17)
    layer = moe.MoeLayer.from_inputs(inp)
    x = moe.bf16_tensor(inp.x, "cuda")
    bufs = layer.route_buffers(64)
    y = layer.forward(x, route_out=bufs)
    torch.cuda.synchronize()
    check_route(bufs, oracle_route(inp), 64, 8)
    check_y(y[:64], oracle.forward(inp)["y"], "k=E")


def test_tied_logits(moe):
    # a zero router without bias ties every logit: ids 0..k-1 in id order,
    # equal weights
    shape = mi.Shape(T=40, d=256, E=16, k=4, f=128, group=32)
    inp = mi.make_inputs(shape, 5)
    inp.w_r = np.zeros_like(inp.w_r)
    layer = moe.MoeLayer.from_inputs(inp)
    bufs = layer.route(moe.bf16_tensor(inp.x, "cuda"))
    torch.cuda.synchronize()
    idx = bufs["topk_idx"][:40].cpu().numpy()
    assert (idx == np.arange(4)).all()
    assert torch.all(bufs["topk_w"][:40] == 0.25)
    check_route(bufs, oracle_route(inp), 40, 4)


# ---------------------------------------------------------------------------
# The small-batch (decode) kernels: T <= 8 on shapes they take.  They share the
# routing definition and the packed weights with the batched path, so the
# same oracle checks apply; these cases add group 32, blocks of several rows,
# ties, and the largest decode batch of the 2048-wide layer.
# ---------------------------------------------------------------------------
def run_layer(moe, inp, T):
    layer = moe.MoeLayer.from_inputs(inp)
    x = moe.bf16_tensor(inp.x[:T], "cuda")
    bufs = layer.route_buffers(T)
    y = layer.forward(x, route_out=bufs)
    torch.cuda.synchronize()
    assert layer.read_status() == (0, 0)
    return layer, bufs, y


@pytest.mark.parametrize("T", [1, 2, 3, 5, 8])
def test_decode_path_small_batches(moe, T):
    inp = mi.make_inputs(mi.Shape(T, 256, 32, 4, 128, 32), 60 + T)
    layer, bufs, y = run_layer(moe, inp, T)
    assert layer.plan.forward_path(T) == 1
    check_route(bufs, oracle_route(inp), T, 4)
    check_y(y[:T], oracle.forward(inp)["y"], "decode T=%d" % T)


def test_decode_path_tied_logits(moe):
    # zero router: every token ties all logits, so all 8 tokens take experts
    # 0..3 with weight 1/4 and each of those experts gets one block of 8 rows
    inp = mi.make_inputs(mi.Shape(8, 256, 32, 4, 128, 32), 9)
    inp.w_r = np.zeros_like(inp.w_r)
    layer, bufs, y = run_layer(moe, inp, 8)
    assert layer.plan.forward_path(8) == 1
    assert (bufs["topk_idx"][:8].cpu().numpy() == np.arange(4)).all()
    assert torch.all(bufs["topk_w"][:8] == 0.25)
    rref = oracle_route(inp)
    assert list(rref["counts"][:4]) == [8, 8, 8, 8]
    check_route(bufs, rref, 8, 4)
    check_y(y[:8], oracle.forward(inp)["y"], "decode ties")


@pytest.mark.parametrize("T", [2, 8])
def test_decode_path_wide_layer(moe, T):
    inp = mi.make_inputs(mi.Shape(T, 2048, 128, 8, 768, 64), 70 + T)
    layer, bufs, y = run_layer(moe, inp, T)
    assert layer.plan.forward_path(T) == 1
    check_route(bufs, oracle_route(inp), T, 8)
    check_y(y[:T], oracle.forward(inp)["y"], "decode wide T=%d" % T)


def test_chained_calls_read_previous_output(moe):
    # The next call's x is the previous call's y, with no synchronisation in
    # between: a batched call then a small-batch call, then a small-batch call
    # on that output.  Kernels chained by programmatic dependent launch may
    # start early, so each must read x only after its predecessor completed.
    inp = workload("prefill_t512")
    s = inp.shape
    layer = moe.MoeLayer.from_inputs(inp)
    assert layer.plan.forward_path(512) == 0 and layer.plan.forward_path(1) == 1
    x = moe.bf16_tensor(inp.x, "cuda")
    y1 = layer.forward(x)
    b2 = layer.route_buffers(1)
    y2 = layer.forward(y1[:1], route_out=b2)
    b3 = layer.route_buffers(4)
    y3 = layer.forward(torch.cat([y2[:1]] * 4), route_out=b3)  # torch's copy sits in between
    y4 = layer.forward(y3[:2])
    torch.cuda.synchronize()
    assert layer.read_status() == (0, 0)
    check_y(y1[:512], oracle.forward(inp)["y"], "batched call")
    bits = lambda t: t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    for xin, yout, bufs in ((y1[:1], y2, b2), (torch.cat([y2[:1]] * 4), y3, b3), (y3[:2], y4, None)):
        T = xin.shape[0]
        sub = mi.Inputs(mi.Shape(T, s.d, s.E, s.k, s.f, s.group), inp.seed, bits(xin), inp.w_r,
                        inp.b_r, inp.gate, inp.up, inp.down)
        if bufs is not None:
            check_route(bufs, oracle_route(sub), T, s.k)
        check_y(yout[:T], oracle.forward(sub)["y"], "chained T=%d" % T)



# ---------------------------------------------------------------------------
# The int8 tensor-core router (batches of 1024 tokens and more): exact ties,
# near ties and all-tied rows, where the fixed-order recheck decides.  Routing
# only (moe_route), compared bit for bit with the oracle.
# ---------------------------------------------------------------------------
def route_only(moe, T, d, E, k, x_bits, w_r, b_r):
    plan = moe.Plan(T, d, E, k, 128, 64)
    assert plan.forward_path(T) == 2  # the int8 tensor-core router
    ws = torch.empty(plan.info.workspace_bytes, dtype=torch.uint8, device="cuda")
    i32 = dict(dtype=torch.int32, device="cuda")
    out = {"topk_idx": torch.empty((T, k), **i32),
           "topk_w": torch.empty((T, k), dtype=torch.float32, device="cuda"),
           "counts": torch.empty(E, **i32), "offsets": torch.empty(E + 1, **i32),
           "sorted_assign": torch.empty(T * k, **i32), "pos": torch.empty(T * k, **i32),
           "block_offsets": torch.empty(E + 1, **i32),
           "block_map": torch.empty((plan.info.max_blocks, 3), **i32),
           "num_blocks": torch.empty(4, **i32)}
    x = moe.bf16_tensor(x_bits, "cuda")
    wr = torch.from_numpy(np.ascontiguousarray(w_r, np.float32)).cuda()
    br = None if b_r is None else torch.from_numpy(np.ascontiguousarray(b_r, np.float32)).cuda()
    plan.route(T, x, wr, br, out, ws)
    torch.cuda.synchronize()
    assert plan.read_status(ws) == (0, 0)
    return out


def fast_case(moe, T, d, E, k, seed, kind):
    inp = mi.make_inputs(mi.Shape(T, d, E, k, 128, 64), seed, weights=False)
    assert T >= 1024  # the int8 tensor-core router takes batches of 1024 tokens and more
    w = inp.w_r.copy()
    b = None
    if kind == "duplicate_columns":      # experts 2j and 2j+1 tie exactly for every token
        w[:, 1::2] = w[:, 0::2]
    elif kind == "one_ulp_apart":        # experts 2j and 2j+1 differ in one entry's last bit
        w[:, 1::2] = w[:, 0::2]
        w[5, 1::2] = np.nextafter(w[5, 0::2], np.float32(np.inf))
    elif kind == "all_tied":             # every logit 0: every expert is a candidate
        w[:] = 0.0
    elif kind == "bias_only":            # every token on experts 0..k-1
        w[:] = 0.0
        b = -np.arange(E, dtype=np.float32)
    out = route_only(moe, T, d, E, k, inp.x, w, b)
    sub = mi.Inputs(inp.shape, seed, inp.x, w, b, None, None, None)
    check_route(out, oracle_route(sub), T, k)
    return out


@pytest.mark.parametrize("kind", ["duplicate_columns", "one_ulp_apart", "all_tied", "bias_only"])
def test_fast_router_ties(moe, kind):
    out = fast_case(moe, 1500, 256, 16, 4, 90, kind)
    idx = out["topk_idx"].cpu().numpy()
    if kind in ("all_tied", "bias_only"):
        assert (idx == np.arange(4)).all()


def test_fast_router_near_ties_wide(moe):
    # the 2048-wide, 128-expert router with pairs of experts one ulp apart
    fast_case(moe, 1024, 2048, 128, 8, 91, "one_ulp_apart")


def test_device_timeout_is_reported_and_workspace_recovers(moe):
    # The test hook withholds one weight stage of the gate/up GEMM and cuts its
    # wait limit to 5 ms: the consumers' bounded waits run out, the kernel
    # records MOE_ERR_DEVICE_TIMEOUT with the role that gave up, drains its
    # copies, frees its TMEM and returns.  A normal call on the same workspace
    # afterwards is correct.
    inp = workload("tiny")
    s = inp.shape
    bad = moe.MoeLayer.from_inputs(inp, flags=moe.SHAPE_TEST_TIMEOUT)
    assert bad.plan.forward_path(s.T) == 0
    x = moe.bf16_tensor(inp.x, "cuda")
    bad.forward(x)
    torch.cuda.synchronize()
    code, detail = bad.read_status()
    assert code == 6, (code, detail)            # MOE_ERR_DEVICE_TIMEOUT
    assert 101 <= detail <= 106, detail         # a gate/up GEMM role
    good = moe.MoeLayer.from_inputs(inp)
    good.ws = bad.ws                            # same shape: same workspace layout
    y = good.forward(x)
    torch.cuda.synchronize()
    assert good.read_status() == (0, 0)
    check_y(y[:s.T], oracle.forward(inp)["y"], "after a timeout")

