"""Seeded synthetic inputs for the int4 expert-grouped MoE layer.

This module only draws random numbers and lays them out in the logical
formats the layer consumes.  It holds none of the layer's arithmetic (no
routing, no dequantisation, no matrix product), so both the CPU oracle and
the CUDA path can take their inputs from here without sharing any
computation.

Generator (counter based, so any element can be drawn on its own):

* SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): the i-th output of a stream with state ``s`` is
  ``mix(s + (i + 1) * 0x9E3779B97F4A7C15)`` with the published 64-bit
  finaliser ``mix``.
* Each tensor has its own stream, keyed by ``mix(mix(seed) + stream_id)``.
* uniform u = (h >> 11) * 2**-53 in [0, 1).
* normal pairs by Box-Muller in float64 from two uniforms (u1 from even
  counters, u2 from odd): r = sqrt(-2 ln(1 - u1)), z0 = r cos(2 pi u2),
  z1 = r sin(2 pi u2).
* bf16 values are rounded once, round-to-nearest-even, straight from
  float64; fp32 values by numpy's float64 -> float32 cast (also RNE).
* packed nibbles are the little-endian bytes of the stream's outputs, so
  every nibble is uniform on 0..15.

Workloads (sizes of the five layer configurations this library is built
for): ``tiny`` T=64, d=256, E=8, k=2, f=128, group 32; the decode and
prefill shapes share d=2048, E=128, k=8, f=768, group 64 and differ in T,
seed and the router bias (the 32K-token prefill adds a Zipf(s=1.1) bias so
expert load is skewed).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# stream ids, one per tensor
STREAM_WR = 1
STREAM_GATE_Q, STREAM_GATE_S = 2, 3
STREAM_UP_Q, STREAM_UP_S = 4, 5
STREAM_DOWN_Q, STREAM_DOWN_S = 6, 7
STREAM_X = 8


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _mix_scalar(z: int) -> int:
    return int(_mix(np.array([z & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64))[0])


def stream_key(seed: int, stream_id: int) -> int:
    return _mix_scalar((_mix_scalar(seed) + stream_id) & 0xFFFFFFFFFFFFFFFF)


def raw_u64(seed: int, stream_id: int, start: int, count: int) -> np.ndarray:
    """Outputs start .. start+count-1 of one SplitMix64 stream."""
    key = np.uint64(stream_key(seed, stream_id))
    i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(key + i * _GAMMA)


def uniform(seed: int, stream_id: int, start: int, count: int) -> np.ndarray:
    h = raw_u64(seed, stream_id, start, count)
    return (h >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal(seed: int, stream_id: int, start: int, count: int) -> np.ndarray:
    """Standard normals number start .. start+count-1 of a stream (float64)."""
    first_pair = start // 2
    last_pair = (start + count + 1) // 2
    npairs = last_pair - first_pair
    u = uniform(seed, stream_id, 2 * first_pair, 2 * npairs).reshape(npairs, 2)
    r = np.sqrt(-2.0 * np.log1p(-u[:, 0]))
    ang = 2.0 * math.pi * u[:, 1]
    z = np.empty((npairs, 2), dtype=np.float64)
    z[:, 0] = r * np.cos(ang)
    z[:, 1] = r * np.sin(ang)
    off = start - 2 * first_pair
    return z.reshape(-1)[off:off + count]


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round float64 to bf16 (RNE, one rounding); returns uint16 bit patterns.

    Finite inputs within bf16's normal range are assumed (true for every
    tensor drawn here)."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    bits = v.view(np.uint64)
    # bf16 keeps 7 of float64's 52 mantissa bits: drop 45 with RNE
    lsb = (bits >> np.uint64(45)) & np.uint64(1)
    with np.errstate(over="ignore"):
        rounded = (bits + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    f32 = rounded.view(np.float64).astype(np.float32)  # exact: 8-bit significand
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass(frozen=True)
class Shape:
    T: int
    d: int
    E: int
    k: int
    f: int
    group: int


@dataclasses.dataclass
class Projection:
    """One int4 projection in logical layout.

    q:     uint8 [E, N, K/2]; byte kk>>1 of row n holds weight kk in its low
           nibble when kk is even and in its high nibble when kk is odd.
    scale: uint16 bf16 bits [E, N, K/group]
    bias:  uint16 bf16 bits [E, N, K/group]
    """
    q: np.ndarray
    scale: np.ndarray
    bias: np.ndarray


@dataclasses.dataclass
class Inputs:
    shape: Shape
    seed: int
    x: np.ndarray          # uint16 bf16 bits [T, d]
    w_r: np.ndarray        # float32 [d, E]
    b_r: np.ndarray | None  # float32 [E] or None
    gate: Projection       # N = f, K = d
    up: Projection         # N = f, K = d
    down: Projection       # N = d, K = f


def _projection(seed: int, sq: int, ss: int, E: int, N: int, K: int, G: int) -> Projection:
    nbytes = E * N * (K // 2)
    h = raw_u64(seed, sq, 0, (nbytes + 7) // 8)
    q = h.view(np.uint8)[:nbytes].reshape(E, N, K // 2).copy()
    ng = E * N * (K // G)
    u = uniform(seed, ss, 0, ng)
    s = (0.5 + u) / (8.0 * math.sqrt(K))
    scale = f64_to_bf16_bits(s).reshape(E, N, K // G)
    # bias = -8 * scale: flipping the sign bit and adding 3 to the exponent
    # is exact for every scale drawn here (normal bf16 values near 1e-3)
    sf = bf16_bits_to_f32(scale).astype(np.float64)
    bias = f64_to_bf16_bits(-8.0 * sf).reshape(E, N, K // G)
    return Projection(q, scale, bias)


def zipf_router_bias(E: int, s: float = 1.1) -> np.ndarray:
    """log of Zipf(s) rank weights, rank r = e + 1, computed in float64."""
    H = math.fsum((r ** -s) for r in range(1, E + 1))
    return np.array([-s * math.log(e + 1) - math.log(H) for e in range(E)],
                    dtype=np.float64).astype(np.float32)


def make_x(seed: int, T: int, d: int) -> np.ndarray:
    return f64_to_bf16_bits(normal(seed, STREAM_X, 0, T * d)).reshape(T, d)


def make_inputs(shape: Shape, seed: int, zipf_bias: bool = False,
                weights: bool = True) -> Inputs:
    T, d, E, k, f, G = shape.T, shape.d, shape.E, shape.k, shape.f, shape.group
    w_r = (normal(seed, STREAM_WR, 0, d * E) / math.sqrt(d)).astype(np.float32).reshape(d, E)
    b_r = zipf_router_bias(E) if zipf_bias else None
    if weights:
        gate = _projection(seed, STREAM_GATE_Q, STREAM_GATE_S, E, f, d, G)
        up = _projection(seed, STREAM_UP_Q, STREAM_UP_S, E, f, d, G)
        down = _projection(seed, STREAM_DOWN_Q, STREAM_DOWN_S, E, d, f, G)
    else:
        gate = up = down = None
    x = make_x(seed, T, d)
    return Inputs(shape, seed, x, w_r, b_r, gate, up, down)


# The five layer configurations: name -> (shape, seed, zipf bias)
WORKLOADS = {
    "tiny": (Shape(64, 256, 8, 2, 128, 32), 0, False),
    "decode_t1": (Shape(1, 2048, 128, 8, 768, 64), 1, False),
    "decode_t4": (Shape(4, 2048, 128, 8, 768, 64), 1, False),
    "prefill_t512": (Shape(512, 2048, 128, 8, 768, 64), 2, False),
    "prefill_t8192": (Shape(8192, 2048, 128, 8, 768, 64), 3, False),
    "prefill_t32768_zipf": (Shape(32768, 2048, 128, 8, 768, 64), 4, True),
}


def workload(name: str, weights: bool = True) -> Inputs:
    shape, seed, zipf = WORKLOADS[name]
    return make_inputs(shape, seed, zipf, weights)
