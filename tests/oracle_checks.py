"""Pins of the CPU oracle against facts that do not come from the oracle.

Each ``check_*`` function raises AssertionError on a mismatch.  They are run
by ``test_oracle_pins.py`` against the oracle as built, and by
``test_oracle_mutants.py`` against copies of the oracle with one planted
mistake each, to show that every planted mistake fails at least one pin.

What pins what (no pin re-types the oracle's own formula):
* router order: hand-derived fixtures (tests/golden/router_order.txt) and
  the rounding-error bound of the fp32 sum against the exactly rounded
  float64 sum (math.fsum of exact products);
* top-k: brute force by numpy's lexicographic sort, crafted ties, and the
  closed case W_r = 0 with a decreasing bias;
* routing weights: sum to one, the k = 2 logistic closed form, and
  scipy's softmax when every expert is selected;
* counts / offsets / scatter / block map: numpy bincount, numpy's stable
  argsort and the tiling invariants;
* dequantisation: hand-set bytes, and all 16 nibbles against s * (q - 8);
* expert MLP and combine: one expert with top-1 equals a dense SwiGLU MLP
  computed with torch in float64, the dense-mask formulation (every token
  through every expert, masked) computed with torch equals the scatter
  path, and plain Python loops on tiny shapes.
"""
from __future__ import annotations

import math
import os

import numpy as np
import scipy.special
import torch

import moe_inputs as mi

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
U32 = 2.0 ** -24  # unit roundoff of fp32


def _parse_value(tok: str) -> float:
    return float.fromhex(tok) if "0x" in tok else float(tok)


def _parse_pairs(toks, n):
    out = np.zeros(n, np.float64)
    for tok in toks:
        key, val = tok.split(":")
        v = _parse_value(val)
        if ".." in key:
            a, b = key.split("..")
            out[int(a):int(b) + 1] = v
        else:
            out[int(key)] = v
    return out


def load_router_cases():
    cases, cur = [], None
    with open(os.path.join(GOLDEN, "router_order.txt")) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            if parts[0] == "case":
                cur = {"name": parts[1], "bias": None}
            elif parts[0] == "x":
                cur["x"] = _parse_pairs(parts[1:], 64)
            elif parts[0] == "w":
                cur["w"] = _parse_pairs(parts[1:], 64)
            elif parts[0] == "bias":
                cur["bias"] = _parse_value(parts[1])
            elif parts[0] == "expect":
                cur["expect"] = _parse_value(parts[1])
            elif parts[0] == "other":
                cur["other"] = _parse_value(parts[1])
            elif parts[0] == "end":
                cases.append(cur)
    return cases


# ----------------------------------------------------------------------------
# router
# ----------------------------------------------------------------------------

def check_router_fixtures(orc):
    for c in load_router_cases():
        x = mi.f64_to_bf16_bits(c["x"]).reshape(1, 64)
        assert np.array_equal(mi.bf16_bits_to_f32(x).astype(np.float64).ravel(), c["x"]), c["name"]
        w = c["w"].astype(np.float32).reshape(64, 1)
        assert np.array_equal(w.astype(np.float64).ravel(), c["w"]), c["name"]
        b = None if c["bias"] is None else np.array([c["bias"]], np.float32)
        got = float(orc.router_logits(x, w, b)[0, 0])
        assert got == c["expect"], (c["name"], got.hex(), c["expect"].hex())
        assert got != c["other"], c["name"]


def check_router_error_bound(orc, seed=11):
    T, d, E = 24, 256, 16
    inp = mi.make_inputs(mi.Shape(T, d, E, 2, 32, 32), seed, weights=False)
    b = (np.arange(E, dtype=np.float32) - 8) / np.float32(16)
    got = orc.router_logits(inp.x, inp.w_r, b).astype(np.float64)
    xf = mi.bf16_bits_to_f32(inp.x).astype(np.float64)
    wf = inp.w_r.astype(np.float64)
    n = d // 32 + 5
    gamma = n * U32 / (1 - n * U32)
    for t in range(T):
        for e in range(E):
            prods = xf[t] * wf[:, e]  # exact: 8-bit times 24-bit significands
            exact = math.fsum(prods)
            bound = gamma * math.fsum(np.abs(prods)) + U32 * (abs(exact) + abs(float(b[e]))) * 2
            assert abs(got[t, e] - (exact + float(b[e]))) <= bound, (t, e)


# ----------------------------------------------------------------------------
# top-k and weights
# ----------------------------------------------------------------------------

def _brute_topk(logits, k):
    T, E = logits.shape
    out = np.empty((T, k), np.int32)
    ids = np.arange(E)
    for t in range(T):
        # primary key: logit descending; secondary: id ascending.
        # (+0.0 is used so that -0 and +0 compare equal)
        order = np.lexsort((ids, -(logits[t].astype(np.float64) + 0.0)))
        out[t] = order[:k]
    return out


def check_topk_bruteforce(orc, seed=5):
    rng = np.random.default_rng(seed)
    for E, k in ((8, 2), (16, 5), (128, 8), (6, 6)):
        logits = rng.standard_normal((40, E)).astype(np.float32)
        # plant exact ties, signed zeros and a constant row
        logits[0, :] = 0.0
        logits[1, ::2] = -0.0
        logits[2, :] = np.float32(1.5)
        logits[3, E // 2] = logits[3, 0]
        logits[4, :] = np.repeat(rng.standard_normal(E // 2 + 1).astype(np.float32), 2)[:E]
        got = orc.topk(logits, k)
        assert np.array_equal(got, _brute_topk(logits, k)), (E, k)


def check_topk_ties(orc):
    # all equal: lowest ids first, in id order
    l = np.zeros((1, 8), np.float32)
    assert orc.topk(l, 3).tolist() == [[0, 1, 2]]
    # rank order, not id order, for distinct values
    l = np.array([[0.1, 0.9, 0.5, 0.9, -1.0]], np.float32)
    assert orc.topk(l, 3).tolist() == [[1, 3, 2]]
    # a zero router with a decreasing (Zipf) bias selects experts 0..k-1
    E, k = 128, 8
    x = mi.make_x(3, 4, 64)
    got = orc.topk(orc.router_logits(x, np.zeros((64, E), np.float32), mi.zipf_router_bias(E)), k)
    assert (got == np.arange(k)).all()


def check_topk_weights(orc, seed=7):
    rng = np.random.default_rng(seed)
    logits = rng.standard_normal((64, 16)).astype(np.float32) * 3
    idx = orc.topk(logits, 4)
    w = orc.topk_weights(logits, idx)
    assert np.all(np.abs(w.sum(1) - 1.0) <= 4e-16)
    assert np.all(np.diff(w, axis=1) <= 0)  # rank order = weight order
    # k = 2: w0 = 1 / (1 + exp(l1 - l0))
    idx2 = orc.topk(logits, 2)
    w2 = orc.topk_weights(logits, idx2)
    l0 = logits[np.arange(64), idx2[:, 0]].astype(np.float64)
    l1 = logits[np.arange(64), idx2[:, 1]].astype(np.float64)
    assert np.allclose(w2[:, 0], 1.0 / (1.0 + np.exp(l1 - l0)), rtol=1e-14, atol=0)
    # every expert selected: the full softmax (scipy)
    idxE = orc.topk(logits, 16)
    wE = orc.topk_weights(logits, idxE)
    ref = scipy.special.softmax(logits.astype(np.float64), axis=1)
    assert np.allclose(wE, np.take_along_axis(ref, idxE, 1), rtol=1e-13, atol=0)


# ----------------------------------------------------------------------------
# counts, scatter, block map
# ----------------------------------------------------------------------------

def _random_routing(rng, T, E, k):
    return np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)


def check_scan_scatter(orc, seed=9):
    rng = np.random.default_rng(seed)
    for T, E, k in ((1, 8, 2), (64, 8, 2), (300, 128, 8), (17, 5, 5)):
        idx = _random_routing(rng, T, E, k)
        if T > 20:
            idx[: T // 3, 0] = 3  # skew one expert
            for t in range(T // 3):
                if 3 in idx[t, 1:]:
                    idx[t, 1:] = np.array([e for e in range(E) if e != 3][: k - 1])
        counts, offsets = orc.counts_offsets(idx, E)
        assert np.array_equal(counts, np.bincount(idx.ravel(), minlength=E))
        assert offsets[0] == 0 and offsets[-1] == T * k
        assert np.array_equal(np.diff(offsets), counts)
        sa, pos = orc.scatter(idx, offsets)
        assert np.array_equal(np.sort(sa), np.arange(T * k))
        assert np.array_equal(pos[sa], np.arange(T * k))
        assert np.array_equal(sa, np.argsort(idx.ravel(), kind="stable"))
        assert np.all(np.diff(idx.ravel()[sa]) >= 0)


def check_block_map(orc, seed=13):
    rng = np.random.default_rng(seed)
    for E, BT in ((8, 4), (128, 128), (5, 1), (7, 64)):
        counts = rng.integers(0, 300, E).astype(np.int32)
        counts[rng.integers(0, E)] = 0
        offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        bo, bm, nb = orc.block_map(counts, offsets, BT)
        assert nb == sum(-(-int(c) // BT) for c in counts)
        assert bo[-1] == nb and bo[0] == 0
        cover = np.zeros(int(offsets[-1]), np.int32)
        for b in range(nb):
            e, r0, rows = bm[b]
            assert 1 <= rows <= BT
            assert offsets[e] <= r0 and r0 + rows <= offsets[e + 1]
            assert bo[e] <= b < bo[e + 1]
            cover[r0:r0 + rows] += 1
        assert np.all(cover == 1)
        assert np.all(np.diff(bm[:, 1]) > 0) if nb > 1 else True


# Block maps worked out by hand: expert e with c_e rows gets ceil(c_e / BT)
# tiles in ascending expert order; tile i starts at offsets[e] + i * BT and
# holds min(BT, c_e - i * BT) rows, so only an expert's last tile is ragged
# and experts without rows get no tile.
BLOCK_MAP_CASES = [
    # (counts, BT, expected (expert, first row, rows) entries, block_offsets)
    ((300, 0, 256, 1), 128,
     [(0, 0, 128), (0, 128, 128), (0, 256, 44), (2, 300, 128), (2, 428, 128), (3, 556, 1)],
     (0, 3, 3, 5, 6)),
    ((513, 255, 0, 256), 256,
     [(0, 0, 256), (0, 256, 256), (0, 512, 1), (1, 513, 255), (3, 768, 256)],
     (0, 3, 4, 4, 5)),
    ((0, 0, 7), 4, [(2, 0, 4), (2, 4, 3)], (0, 0, 0, 2)),
]


def check_block_map_hand(orc):
    for counts, BT, entries, bo_ref in BLOCK_MAP_CASES:
        counts = np.array(counts, np.int32)
        offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        bo, bm, nb = orc.block_map(counts, offsets, BT)
        assert nb == len(entries), (counts, nb)
        assert [tuple(int(v) for v in row) for row in bm] == entries, (counts, bm)
        assert tuple(int(v) for v in bo) == bo_ref, (counts, bo)


# ----------------------------------------------------------------------------
# dequantisation
# ----------------------------------------------------------------------------

def check_dequant_hand(orc):
    one = lambda v: mi.f64_to_bf16_bits(np.array([v], np.float64))
    # byte 0xF0: low nibble (k = 0) is 0, high nibble (k = 1) is 15
    q = np.zeros((1, 16), np.uint8)
    q[0, 0] = 0xF0
    s = np.repeat(one(0.5), 1).reshape(1, 1)
    b = np.repeat(one(-4.0), 1).reshape(1, 1)
    w = orc.dequant(q, s, b, 32)
    assert w[0, 0] == -4.0 and w[0, 1] == 3.5
    assert np.all(w[0, 2:] == -4.0)
    # two groups of 32 along K with their own scale and bias
    q = np.full((2, 32), 0x21, np.uint8)  # even k -> 1, odd k -> 2
    s = mi.f64_to_bf16_bits(np.array([[0.25, 2.0], [1.0, 0.125]]))
    b = mi.f64_to_bf16_bits(np.array([[1.0, -3.0], [0.0, 0.5]]))
    w = orc.dequant(q, s, b, 32)
    assert np.all(w[0, 0:32:2] == 1.25) and np.all(w[0, 1:32:2] == 1.5)
    assert np.all(w[0, 32::2] == -1.0) and np.all(w[0, 33::2] == 1.0)
    assert np.all(w[1, 0:32:2] == 1.0) and np.all(w[1, 1:32:2] == 2.0)
    assert np.all(w[1, 32::2] == 0.625) and np.all(w[1, 33::2] == 0.75)


def check_dequant_all_nibbles(orc):
    # every nibble value q at every position, with bias = -8 * scale, is
    # exactly scale * (q - 8)
    for sv in (0.5, 1.0 / 3.0, 7.25e-4, 3.0):
        q = np.zeros((16, 32), np.uint8)
        for n in range(16):
            q[n, :] = n | (((n + 5) % 16) << 4)
        s = np.full((16, 2), mi.f64_to_bf16_bits(np.array([sv]))[0], np.uint16)
        sf = float(mi.bf16_bits_to_f32(s[0, 0]))
        b = mi.f64_to_bf16_bits(np.full((16, 2), -8.0 * sf))
        w = orc.dequant(q, s, b, 32)
        for n in range(16):
            assert np.all(w[n, 0::2] == sf * (n - 8))
            assert np.all(w[n, 1::2] == sf * (((n + 5) % 16) - 8))


# ----------------------------------------------------------------------------
# expert MLP and combine
# ----------------------------------------------------------------------------

def _torch_dequant(p: mi.Projection, G: int) -> torch.Tensor:
    """[E, N, K] float64, unpacked with torch bit ops (independent of the oracle)."""
    q = torch.from_numpy(p.q.astype(np.int64))
    lo, hi = q & 15, q >> 4
    nib = torch.stack([lo, hi], dim=-1).reshape(q.shape[0], q.shape[1], -1).to(torch.float64)
    s = torch.from_numpy(mi.bf16_bits_to_f32(p.scale).astype(np.float64))
    b = torch.from_numpy(mi.bf16_bits_to_f32(p.bias).astype(np.float64))
    return nib * s.repeat_interleave(G, dim=-1) + b.repeat_interleave(G, dim=-1)


def _torch_mlp(xf, Wg, Wu, Wd):
    return (torch.nn.functional.silu(xf @ Wg.T) * (xf @ Wu.T)) @ Wd.T


def check_single_expert_is_dense_mlp(orc):
    shape = mi.Shape(T=16, d=64, E=1, k=1, f=64, group=32)
    inp = mi.make_inputs(shape, 21)
    r = orc.forward(inp)
    assert np.all(r["topk_idx"] == 0) and np.all(r["topk_w"] == 1.0)
    xf = torch.from_numpy(mi.bf16_bits_to_f32(inp.x).astype(np.float64))
    Wg, Wu, Wd = (_torch_dequant(p, 32)[0] for p in (inp.gate, inp.up, inp.down))
    ref = _torch_mlp(xf, Wg, Wu, Wd).numpy()
    assert np.allclose(r["y"], ref, rtol=1e-11, atol=1e-14)


def check_dense_mask_form(orc):
    for shape, seed in ((mi.Shape(T=40, d=64, E=6, k=3, f=64, group=32), 23),
                        (mi.Shape(T=64, d=256, E=8, k=2, f=128, group=32), 0)):
        inp = mi.make_inputs(shape, seed)
        r = orc.forward(inp)
        xf = torch.from_numpy(mi.bf16_bits_to_f32(inp.x).astype(np.float64))
        Wg, Wu, Wd = (_torch_dequant(p, shape.group) for p in (inp.gate, inp.up, inp.down))
        M = torch.zeros(shape.T, shape.E, dtype=torch.float64)
        M.scatter_(1, torch.from_numpy(r["topk_idx"].astype(np.int64)), torch.from_numpy(r["topk_w"]))
        y = torch.zeros(shape.T, shape.d, dtype=torch.float64)
        for e in range(shape.E):
            y += M[:, e:e + 1] * _torch_mlp(xf, Wg[e], Wu[e], Wd[e])
        assert np.allclose(r["y"], y.numpy(), rtol=1e-11, atol=1e-14)


def check_tiny_bruteforce(orc):
    shape = mi.Shape(T=4, d=32, E=3, k=2, f=32, group=32)
    inp = mi.make_inputs(shape, 31)
    r = orc.forward(inp, want_h=True)
    T, d, E, k, f = shape.T, shape.d, shape.E, shape.k, shape.f
    x = mi.bf16_bits_to_f32(inp.x).astype(float).tolist()

    def weight(p, e, n, kk):
        byte = int(p.q[e, n, kk // 2])
        nib = (byte >> 4) if kk % 2 else (byte & 15)
        s = float(mi.bf16_bits_to_f32(p.scale[e, n, kk // 32]))
        b = float(mi.bf16_bits_to_f32(p.bias[e, n, kk // 32]))
        return nib * s + b

    for t in range(T):
        # exact logits, then the selection must agree unless a near tie
        exact = [math.fsum(x[t][i] * float(inp.w_r[i, e]) for i in range(d)) for e in range(E)]
        order = sorted(range(E), key=lambda e: (-exact[e], e))
        gaps = [exact[order[i]] - exact[order[i + 1]] for i in range(E - 1)]
        if min(gaps) > 1e-5:
            assert r["topk_idx"][t].tolist() == order[:k]
        y = [0.0] * d
        for j in range(k):
            e = int(r["topk_idx"][t, j])
            h = []
            for n in range(f):
                g = sum(weight(inp.gate, e, n, kk) * x[t][kk] for kk in range(d))
                u = sum(weight(inp.up, e, n, kk) * x[t][kk] for kk in range(d))
                h.append(g / (1 + math.exp(-g)) * u)
            for m in range(d):
                o = sum(weight(inp.down, e, m, n) * h[n] for n in range(f))
                y[m] += float(r["topk_w"][t, j]) * o
        assert np.allclose(r["y"][t], y, rtol=1e-11, atol=1e-14), t


def check_token_outputs_match_forward(orc):
    inp = mi.workload("tiny")
    r = orc.forward(inp)
    toks = np.array([0, 1, 31, 63])
    y, idx, w = orc.token_outputs(inp, toks)
    assert np.array_equal(idx, r["topk_idx"][toks])
    assert np.allclose(w, r["topk_w"][toks], rtol=1e-15, atol=0)
    assert np.allclose(y, r["y"][toks], rtol=1e-12, atol=1e-15)


ALL_CHECKS = [
    check_router_fixtures,
    check_router_error_bound,
    check_topk_bruteforce,
    check_topk_ties,
    check_topk_weights,
    check_scan_scatter,
    check_block_map,
    check_block_map_hand,
    check_dequant_hand,
    check_dequant_all_nibbles,
    check_single_expert_is_dense_mlp,
    check_dense_mask_form,
    check_tiny_bruteforce,
    check_token_outputs_match_forward,
]
