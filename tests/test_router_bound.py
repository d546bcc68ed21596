"""The error bound of the int8 tensor-core router, checked on the CPU.

The batched router for 1024 tokens and more computes approximate logits
l' = x' . w' + b from two int8 digits of every x and W_r entry (exactly, in
int32 on the tensor cores) and evaluates the router's fixed fp32 order only
for the experts whose interval [l' - delta, l' + delta] reaches the token's
k-th largest lower bound.  That is exact only if delta bounds the distance
between l' and the fixed-order logit.  Here the digits and delta are formed
the way the kernels form them (power-of-two scales, |x/s| < 128 and
|w/u| < 64, round to nearest, the remainders' maxima, sums and norms) and the
fixed-order logits come from the CPU oracle; the bound must hold for every
(token, expert) pair, on the layer workloads and on inputs made to stress it.
"""
import math

import numpy as np
import pytest

import moe_inputs as mi
import oracle

GAMMA_72 = 72 * 2.0 ** -24 / (1 - 72 * 2.0 ** -24)


def pow2_scale(m, span_log2):
    f, ex = np.frexp(np.asarray(m, np.float64))
    return np.where(np.asarray(m) > 0, np.ldexp(1.0, ex - span_log2), 1.0)


def digits_and_delta(x_bits, w_r, b_r):
    x = mi.bf16_bits_to_f32(x_bits).astype(np.float64)
    W = np.asarray(w_r, np.float32).astype(np.float64)
    d, E = W.shape
    s = pow2_scale(np.abs(x).max(1), 7)
    z = x / s[:, None]
    a = np.clip(np.rint(z), -127, 127)
    b = np.rint((z - a) * 128)
    assert np.abs(b).max() <= 64
    xq = s[:, None] * (a + b / 128)
    Et = np.abs(x - xq).max(1)
    At = np.abs(x).sum(1) + d * Et
    Nt = np.sqrt((x ** 2).sum(1))
    u = pow2_scale(np.abs(W).max(0), 6)
    zw = W / u[None, :]
    c = np.rint(zw)
    dd = np.rint((zw - c) * 128)
    assert np.abs(c).max() <= 64 and np.abs(dd).max() <= 64
    wq = u[None, :] * (c + dd / 128)
    Fe = np.abs(W - wq).max(0)
    Be = np.abs(W).sum(0)
    Wn = np.sqrt((W ** 2).sum(0))
    bias = np.zeros(E) if b_r is None else np.asarray(b_r, np.float32).astype(np.float64)
    # the exact x'.w' (the int8 products and int32 sums are exact) with the bias
    L = (xq @ wq + bias).astype(np.float32).astype(np.float64)
    delta = (Fe[None, :] * At[:, None] + Et[:, None] * Be[None, :]
             + GAMMA_72 * (Nt[:, None] * Wn[None, :] + np.abs(bias)[None, :]) + 2.0 ** -23 * np.abs(L))
    return L, delta


def check(x_bits, w_r, b_r, k):
    L, delta = digits_and_delta(x_bits, w_r, b_r)
    lc = oracle.router_logits(x_bits, w_r, b_r).astype(np.float64)
    ratio = np.abs(lc - L) / delta
    assert ratio.max() <= 1.0, ratio.max()
    # the candidates contain the fixed-order top-k
    lo, up = L - delta, L + delta
    theta = -np.sort(-lo, axis=1)[:, k - 1]
    cand = up >= theta[:, None]
    idx = oracle.topk(lc.astype(np.float32), k)
    assert np.all(np.take_along_axis(cand, idx.astype(np.int64), 1))
    return ratio.max(), cand.sum(1).mean()


@pytest.mark.parametrize("name", ["prefill_t512", "prefill_t8192", "prefill_t32768_zipf"])
def test_bound_on_layer_workloads(name):
    inp = mi.workload(name, weights=False)
    T = min(inp.shape.T, 1024)
    worst, mean_cand = check(inp.x[:T], inp.w_r, inp.b_r, inp.shape.k)
    print("%s: worst |error| / delta = %.3f, %.2f candidates per token" % (name, worst, mean_cand))
    assert mean_cand < 12  # a few experts beyond k: the exact step stays small


def test_bound_on_stressed_inputs():
    rng = np.random.default_rng(5)
    T, d, E, k = 256, 2048, 128, 8
    # x with a wide dynamic range (tiny entries lose digits) and outliers;
    # W_r with a few large entries per column and a spread of scales
    x = rng.standard_normal((T, d)) * np.exp2(rng.integers(-20, 3, (T, d)))
    x[:, 7] = 300.0
    x[5] = 0.0
    W = (rng.standard_normal((d, E)) * np.exp2(rng.integers(-12, 0, (d, E)))).astype(np.float32)
    W[3, :] = 4.0
    W[:, 9] = 0.0
    b = rng.standard_normal(E).astype(np.float32) * 10
    worst, _ = check(mi.f64_to_bf16_bits(x), W, b, k)
    print("stressed: worst |error| / delta = %.3f" % worst)
