"""The C-ABI library loads, exports every symbol include/moe.h declares, and
rejects bad arguments before launching anything (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def moe(built_library):
    import int4_expert_grouped_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)


def test_every_declared_symbol_is_exported(moe):
    names = declared_functions()
    assert len(names) == 16
    for n in names:
        assert hasattr(moe.lib(), n), n
    assert set(names) == set(moe.EXPORTED)


def test_abi_version_matches_header(moe):
    v = int(re.search(r"#define MOE_ABI_VERSION (\d+)", open(HEADER).read()).group(1))
    assert moe.abi_version() == v


def test_status_strings(moe):
    for code in range(8):
        assert moe.lib().moe_status_str(code)


SHAPES = [(64, 256, 8, 2, 128, 32), (8192, 2048, 128, 8, 768, 64), (1, 2048, 128, 8, 768, 64),
          (32768, 2048, 128, 8, 768, 64)]


@pytest.mark.parametrize("shape", SHAPES)
def test_plan_sizes(moe, shape):
    T, d, E, k, f, G = shape
    p = moe.Plan(*shape)
    info = p.info
    assert info.block_t == 256
    assert info.max_blocks == -(-T * k // 256) + min(E, T * k)
    logical = 3 * E * f * d // 2 + 3 * E * f * (d // G) * 4
    assert logical <= info.packed_weight_bytes <= logical + 256
    need = T * k * f * 2 + T * d * 4  # h and the fp32 combine accumulator at least
    assert info.workspace_bytes >= need
    assert info.host_workspace_bytes >= info.workspace_bytes + 2 * T * d * 2


@pytest.mark.parametrize("shape,code", [
    ((64, 255, 8, 2, 128, 32), 2),     # d not a multiple of 256
    ((64, 256, 8, 2, 100, 32), 2),     # f not a multiple of 128
    ((64, 256, 8, 2, 128, 16), 2),     # group 16
    ((64, 256, 7, 2, 128, 32), 2),     # E not a multiple of 8
    ((64, 256, 512, 2, 128, 32), 2),   # E > 256
    ((64, 256, 8, 9, 128, 32), 1),     # k > E
    ((0, 256, 8, 2, 128, 32), 1),      # T_max = 0
    ((64, 256, 8, 0, 128, 32), 1),     # k = 0
])
def test_plan_rejects_shapes(moe, shape, code):
    with pytest.raises(moe.MoeError) as ei:
        moe.Plan(*shape)
    assert ei.value.code == code


def _call_forward(moe, plan, T, x, wr, br, packed, y, ws, ws_bytes):
    return moe.lib().moe_forward(plan.handle, T, x, wr, br, packed, y, None, ws, ws_bytes, None)


def test_forward_argument_checks(moe):
    p = moe.Plan(64, 256, 8, 2, 128, 32)
    W = p.info.workspace_bytes
    good = dict(x=0x10000, wr=0x20000, br=None, packed=0x30000, y=0x40000, ws=0x50000)

    def call(T=64, ws_bytes=W, **over):
        a = dict(good, **over)
        return _call_forward(moe, p, T, a["x"], a["wr"], a["br"], a["packed"], a["y"], a["ws"],
                             ws_bytes)

    assert moe.lib().moe_forward(None, 64, 1, 1, None, 1, 1, None, 1, W, None) == 1
    assert call(T=65) == 1                      # T > T_max
    assert call(T=-1) == 1
    assert call(x=None) == 1
    assert call(y=None) == 1
    assert call(wr=None) == 1
    assert call(packed=None) == 1
    assert call(ws=None) == 1
    assert call(x=0x10008) == 3                 # misaligned
    assert call(br=0x60004) == 3
    assert call(ws=0x50001) == 3
    assert call(ws_bytes=W - 1) == 4            # workspace too small


def test_route_argument_checks(moe):
    p = moe.Plan(64, 256, 8, 2, 128, 32)
    W = p.info.workspace_bytes
    ro = moe.RouteOut(*([0x1000 * (i + 1) for i in range(9)]))
    lib = moe.lib()
    assert lib.moe_route(p.handle, 64, 0x10000, 0x20000, None, ctypes.byref(ro), 0x50000, W - 1, None) == 4
    bad = moe.RouteOut(*([0x1000 * (i + 1) for i in range(8)] + [None]))
    assert lib.moe_route(p.handle, 64, 0x10000, 0x20000, None, ctypes.byref(bad), 0x50000, W, None) == 1
    mis = moe.RouteOut(*([0x1000 * (i + 1) for i in range(8)] + [0x9004]))
    assert lib.moe_route(p.handle, 64, 0x10000, 0x20000, None, ctypes.byref(mis), 0x50000, W, None) == 3
    assert lib.moe_route(p.handle, 65, 0x10000, 0x20000, None, ctypes.byref(ro), 0x50000, W, None) == 1


def test_prepack_and_host_checks(moe):
    p = moe.Plan(64, 256, 8, 2, 128, 32)
    lib = moe.lib()
    proj = moe.Projection(0x1000, 0x2000, 0x3000)
    w = moe.ExpertWeights(proj, proj, moe.Projection(0x1000, None, 0x3000))
    assert lib.moe_prepack_weights(p.handle, ctypes.byref(w), 0x8000, None) == 1
    w = moe.ExpertWeights(proj, proj, moe.Projection(0x1001, 0x2000, 0x3000))
    assert lib.moe_prepack_weights(p.handle, ctypes.byref(w), 0x8000, None) == 3
    H = p.info.host_workspace_bytes
    assert lib.moe_forward_host(p.handle, 64, 0x1000, 0x2000, None, 0x3000, 0x4000, 0x5000, H - 1, None) == 4
    assert lib.moe_forward_host(p.handle, 64, None, 0x2000, None, 0x3000, 0x4000, 0x5000, H, None) == 1


def test_expert_parallel_entry_checks(moe):
    """moe_dispatch, moe_experts_forward and moe_combine reject bad arguments
    before launching anything."""
    p = moe.Plan(64, 256, 8, 2, 128, 32)
    W = p.info.workspace_bytes
    lib = moe.lib()
    # moe_dispatch(plan, T, x, sorted_assign, xs, ws, ws_bytes, stream)
    assert lib.moe_dispatch(None, 64, 0x1000, 0x2000, 0x3000, 0x5000, W, None) == 1
    assert lib.moe_dispatch(p.handle, 65, 0x1000, 0x2000, 0x3000, 0x5000, W, None) == 1
    assert lib.moe_dispatch(p.handle, 64, None, 0x2000, 0x3000, 0x5000, W, None) == 1
    assert lib.moe_dispatch(p.handle, 64, 0x1000, 0x2004, 0x3000, 0x5000, W, None) == 3
    assert lib.moe_dispatch(p.handle, 64, 0x1000, 0x2000, 0x3000, 0x5000, W - 1, None) == 4
    # moe_experts_forward(plan, rows, xs, block_map, num_blocks, max_blocks,
    #                     packed_w, o, ws, ws_bytes, stream); rows <= T_max * k
    ef = lib.moe_experts_forward
    assert ef(p.handle, 129, 0x1000, 0x2000, 0x3000, 4, 0x4000, 0x6000, 0x5000, W, None) == 1
    assert ef(p.handle, -1, 0x1000, 0x2000, 0x3000, 4, 0x4000, 0x6000, 0x5000, W, None) == 1
    assert ef(p.handle, 128, 0x1000, 0x2000, 0x3000, -1, 0x4000, 0x6000, 0x5000, W, None) == 1
    assert ef(p.handle, 128, 0x1000, None, 0x3000, 4, 0x4000, 0x6000, 0x5000, W, None) == 1
    assert ef(p.handle, 128, 0x1000, 0x2000, None, 4, 0x4000, 0x6000, 0x5000, W, None) == 1
    assert ef(p.handle, 128, 0x1000, 0x2000, 0x3000, 4, None, 0x6000, 0x5000, W, None) == 1
    assert ef(p.handle, 128, 0x1000, 0x2000, 0x3008, 4, 0x4000, 0x6000, 0x5000, W, None) == 3
    assert ef(p.handle, 128, 0x1000, 0x2000, 0x3000, 4, 0x4000, 0x6002, 0x5000, W, None) == 3
    assert ef(p.handle, 128, 0x1000, 0x2000, 0x3000, 4, 0x4000, 0x6000, 0x5000, W - 1, None) == 4
    # moe_combine(plan, T, o, pos, topk_w, y, ws, ws_bytes, stream)
    assert lib.moe_combine(p.handle, 64, 0x1000, None, 0x3000, 0x4000, 0x5000, W, None) == 1
    assert lib.moe_combine(p.handle, 64, 0x1000, 0x2000, 0x3000, 0x4004, 0x5000, W, None) == 3
    assert lib.moe_combine(p.handle, 64, 0x1000, 0x2000, 0x3000, 0x4000, 0x5000, W - 1, None) == 4
    assert lib.moe_combine(p.handle, -1, 0x1000, 0x2000, 0x3000, 0x4000, 0x5000, W, None) == 1


def test_forward_path_choice(moe):
    # host-only query: small batches of a supported shape take the decode kernel
    p = moe.Plan(8192, 2048, 128, 8, 768, 64)
    assert [p.forward_path(T) for T in (0, 1, 4, 8, 9, 1023, 1024, 8192)] == [0, 1, 1, 1, 0, 0, 2, 2]
    assert p.forward_path(-1) == -1 and p.forward_path(8193) == -1
    tiny = moe.Plan(64, 256, 8, 2, 128, 32)
    assert tiny.forward_path(3) == 1 and tiny.forward_path(9) == 0
    g32 = moe.Plan(64, 256, 32, 2, 128, 32)
    assert g32.forward_path(3) == 1 and g32.forward_path(9) == 0
    # d = 4096: the x rows of 8 tokens no longer fit beside the weight ring
    wide = moe.Plan(64, 4096, 128, 8, 768, 64)
    assert wide.forward_path(4) == 1 and wide.forward_path(8) == 0
    # f = 1024 at T = 8: 8 h rows and their sums still fit
    assert moe.Plan(64, 2048, 128, 8, 1024, 64).forward_path(8) == 1
    # f = 4096: more than 16 feature tiles per expert
    assert moe.Plan(64, 2048, 128, 8, 4096, 64).forward_path(1) == 0
    # E = 256: two routing items per CTA on 148 SMs, still one kernel
    assert moe.Plan(64, 2048, 256, 8, 768, 64).forward_path(1) == 1
    # at most 64 assignments per call: k = 16 takes batches of up to 4 tokens
    k16 = moe.Plan(64, 2048, 128, 16, 768, 64)
    assert k16.forward_path(4) == 1 and k16.forward_path(5) == 0
