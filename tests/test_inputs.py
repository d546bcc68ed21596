"""The seeded input generator against its published definitions."""
import numpy as np

import moe_inputs as mi


def test_splitmix64_published_outputs():
    # SplitMix64 from state 0: the first outputs of the reference generator
    g = 0x9E3779B97F4A7C15
    outs = [int(mi._mix(np.array([(i * g) % 2 ** 64], np.uint64))[0]) for i in (1, 2, 3)]
    assert outs == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_counter_based_streams():
    a = mi.raw_u64(5, 2, 0, 100)
    b = mi.raw_u64(5, 2, 40, 10)
    assert np.array_equal(a[40:50], b)
    assert not np.array_equal(mi.raw_u64(5, 3, 0, 10), a[:10])
    z = mi.normal(1, 8, 0, 11)
    assert np.array_equal(mi.normal(1, 8, 3, 5), z[3:8])


def test_bf16_round_to_nearest_even():
    f = mi.f64_to_bf16_bits
    assert f(np.array([1.0]))[0] == 0x3F80
    assert f(np.array([1.0 + 2 ** -8]))[0] == 0x3F80          # tie -> even
    assert f(np.array([1.0 + 3 * 2 ** -8]))[0] == 0x3F82      # tie -> even (up)
    assert f(np.array([1.0 + 2 ** -8 + 2 ** -40]))[0] == 0x3F81  # above the tie
    assert f(np.array([-2.5]))[0] == 0xC020
    v = np.random.default_rng(0).standard_normal(1000)
    back = mi.bf16_bits_to_f32(f(v)).astype(np.float64)
    assert np.all(np.abs(back - v) <= np.abs(v) * 2 ** -8)


def test_distributions_and_shapes():
    inp = mi.workload("tiny")
    s = inp.shape
    assert inp.x.shape == (s.T, s.d) and inp.w_r.shape == (s.d, s.E)
    assert inp.gate.q.shape == (s.E, s.f, s.d // 2)
    assert inp.down.q.shape == (s.E, s.d, s.f // 2)
    assert inp.gate.scale.shape == (s.E, s.f, s.d // s.group)
    x = mi.bf16_bits_to_f32(inp.x)
    assert abs(x.mean()) < 0.05 and abs(x.std() - 1) < 0.05
    assert abs(inp.w_r.std() * np.sqrt(s.d) - 1) < 0.05
    nib = np.concatenate([inp.gate.q & 15, inp.gate.q >> 4]).ravel()
    assert np.bincount(nib, minlength=16).min() > 0.9 * nib.size / 16
    sc = mi.bf16_bits_to_f32(inp.gate.scale) * 8 * np.sqrt(s.d)
    assert sc.min() >= 0.49 and sc.max() <= 1.51
    assert np.array_equal(mi.bf16_bits_to_f32(inp.gate.bias), -8 * mi.bf16_bits_to_f32(inp.gate.scale))


def test_decode_shapes_share_first_token():
    a = mi.workload("decode_t1", weights=False)
    b = mi.workload("decode_t4", weights=False)
    assert np.array_equal(a.x[0], b.x[0]) and np.array_equal(a.w_r, b.w_r)


def test_zipf_bias():
    b = mi.zipf_router_bias(128).astype(np.float64)
    assert np.all(np.diff(b) < 0)
    assert abs(np.exp(b).sum() - 1) < 1e-6
