"""moe_route_noalloc against moe_route.

moe_route_noalloc serves callers that cannot allocate device memory (for
example code running under a stream capture that forbids allocation, or a
runtime that owns all device memory): it keeps its routing scratch in a fixed
array inside the library instead of a caller workspace.  Its outputs must be
those of moe_route on the same inputs.  Two calls run back to back, the
second with fewer tokens, so scratch left over from the first call would
show up as a mismatch.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import moe_inputs as mi

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env(built_library):
    assert torch.cuda.is_available(), "the gpu tests need a GPU"
    import int4_expert_grouped_b200 as m
    from int4_expert_grouped_b200.layer import MoeLayer, bf16_tensor
    return m, MoeLayer, bf16_tensor


def _same_routing(a, b, T, k):
    A = {n: t.cpu().numpy() for n, t in a.items()}
    B = {n: t.cpu().numpy() for n, t in b.items()}
    for n in ("topk_idx",):
        assert np.array_equal(A[n][:T], B[n][:T]), n
    rel = np.abs(A["topk_w"][:T].astype(np.float64) - B["topk_w"][:T]) / np.abs(B["topk_w"][:T])
    assert rel.max() <= 1e-6, rel.max()
    for n in ("counts", "offsets", "block_offsets"):
        assert np.array_equal(A[n], B[n]), n
    for n in ("sorted_assign", "pos"):
        assert np.array_equal(A[n][:T * k], B[n][:T * k]), n
    nb = int(B["num_blocks"][0])
    assert int(A["num_blocks"][0]) == nb
    assert np.array_equal(A["block_map"][:nb], B["block_map"][:nb])


def test_noalloc_route_matches_route_twice(env):
    m, MoeLayer, bf16 = env
    inp = mi.workload("prefill_t512")
    layer = MoeLayer.from_inputs(inp)
    x = bf16(inp.x, "cuda")
    for T in (512, 77):
        ref = layer.route(x[:T])
        got = layer.route_buffers(T)
        layer.plan.route_noalloc(T, x[:T], layer.w_r, layer.b_r, got)
        torch.cuda.synchronize()
        _same_routing(got, ref, T, inp.shape.k)


def test_noalloc_route_rejects_oversize(env):
    m, MoeLayer, bf16 = env
    plan = m.Plan(8192, 2048, 128, 8, 768, 64)
    ro = m.RouteOut(*([0x10000 * (i + 1) for i in range(9)]))
    import ctypes
    code = m.lib().moe_route_noalloc(plan.handle, 8192, 0x1000000, 0x2000000, None,
                                     ctypes.byref(ro), None)
    assert code == 4  # MOE_ERR_WORKSPACE_TOO_SMALL, nothing launched
