"""CPU oracle for the int4 expert-grouped MoE layer.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The CUDA library never imports,
links or runs anything here, and nothing here imports the CUDA library.

The arithmetic lives in ``moe_oracle.c`` (plain C, fp32 router in one fixed
order, float64 everywhere else); this module compiles it with gcc and wraps
each function over numpy arrays.  Every function states the passage it
follows in the C source.  Parity of every function is pinned by the
``-m "not gpu"`` tests in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared"]

_lib = None


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so next to it (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "gate_q", "up_q", "down_q",
        "gate_s", "gate_b", "up_s", "up_b", "down_s", "down_b")]


_SIGNATURES = {
    "oracle_router_logits": "PIIPIPP",
    "oracle_topk": "PIIIP",
    "oracle_topk_weights": "PPIIIP",
    "oracle_counts_offsets": "PIIIPP",
    "oracle_scatter": "PPIIIPP",
    "oracle_block_map": "PPIIPP",
    "oracle_dequant": "PPPIIIP",
    "oracle_expert_rows": "PIIIIII" + 6 * "P",
    "oracle_combine": "PPPIIIP",
    "oracle_forward": "PIIIIII" + 13 * "P",
    "oracle_token_outputs": "PIIIIIPPPPIPPP",
}


def configure(cdll):
    """Set argument types on a loaded oracle library and return it."""
    kinds = {"P": ctypes.c_void_p, "I": ctypes.c_int64}
    for name, args in _SIGNATURES.items():
        fn = getattr(cdll, name)
        fn.argtypes = [kinds[a] for a in args]
        fn.restype = None
    cdll.oracle_block_map.restype = ctypes.c_int64
    cdll.oracle_abi_version.restype = ctypes.c_int
    return cdll


def lib():
    global _lib
    if _lib is None:
        _lib = configure(ctypes.CDLL(build()))
    return _lib


class using_library:
    """Context manager: route every wrapper in this module through another
    build of the oracle (the mutation tests use it)."""

    def __init__(self, cdll):
        self.cdll = cdll

    def __enter__(self):
        global _lib
        self.saved = _lib
        _lib = self.cdll
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def router_logits(x, w_r, b_r=None):
    """fp32 logits [T, E] in the fixed chain-and-butterfly order."""
    x = _c(x, np.uint16)
    w_r = _c(w_r, np.float32)
    T, d = x.shape
    E = w_r.shape[1]
    b = None if b_r is None else _c(b_r, np.float32)
    out = np.empty((T, E), np.float32)
    lib().oracle_router_logits(_p(x), T, d, _p(w_r), E, _p(b), _p(out))
    return out


def topk(logits, k):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    out = np.empty((T, k), np.int32)
    lib().oracle_topk(_p(logits), T, E, k, _p(out))
    return out


def topk_weights(logits, idx):
    logits = _c(logits, np.float32)
    idx = _c(idx, np.int32)
    T, E = logits.shape
    k = idx.shape[1]
    out = np.empty((T, k), np.float64)
    lib().oracle_topk_weights(_p(logits), _p(idx), T, E, k, _p(out))
    return out


def counts_offsets(idx, E):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    lib().oracle_counts_offsets(_p(idx), T, k, E, _p(counts), _p(offsets))
    return counts, offsets


def scatter(idx, offsets):
    idx = _c(idx, np.int32)
    offsets = _c(offsets, np.int32)
    T, k = idx.shape
    E = offsets.shape[0] - 1
    sa = np.empty(T * k, np.int32)
    pos = np.empty(T * k, np.int32)
    lib().oracle_scatter(_p(idx), _p(offsets), T, k, E, _p(sa), _p(pos))
    return sa, pos


def block_map(counts, offsets, block_t):
    counts = _c(counts, np.int32)
    offsets = _c(offsets, np.int32)
    E = counts.shape[0]
    cap = int(sum((int(c) + block_t - 1) // block_t for c in counts))
    bo = np.empty(E + 1, np.int32)
    bm = np.empty((max(cap, 1), 3), np.int32)
    nb = lib().oracle_block_map(_p(counts), _p(offsets), E, block_t, _p(bo), _p(bm))
    return bo, bm[:nb].copy(), int(nb)


def dequant(q, scale, bias, group):
    """One expert's projection [N, K] in float64 from nibbles and groups."""
    q = _c(q, np.uint8)
    scale = _c(scale, np.uint16)
    bias = _c(bias, np.uint16)
    N, K2 = q.shape
    K = 2 * K2
    out = np.empty((N, K), np.float64)
    lib().oracle_dequant(_p(q), _p(scale), _p(bias), N, K, group, _p(out))
    return out


def _weights_struct(inp):
    keep = [
        _c(inp.gate.q, np.uint8), _c(inp.up.q, np.uint8), _c(inp.down.q, np.uint8),
        _c(inp.gate.scale, np.uint16), _c(inp.gate.bias, np.uint16),
        _c(inp.up.scale, np.uint16), _c(inp.up.bias, np.uint16),
        _c(inp.down.scale, np.uint16), _c(inp.down.bias, np.uint16),
    ]
    w = _Weights(*[a.ctypes.data for a in keep])
    return w, keep


def forward(inp, want_h=False):
    """The whole layer through routing, scan, scatter, expert rows, combine.

    Returns a dict of every intermediate (float ones in float64)."""
    s = inp.shape
    T, d, E, k, f, G = s.T, s.d, s.E, s.k, s.f, s.group
    x = _c(inp.x, np.uint16)
    w_r = _c(inp.w_r, np.float32)
    b_r = None if inp.b_r is None else _c(inp.b_r, np.float32)
    w, keep = _weights_struct(inp)
    r = {
        "logits": np.empty((T, E), np.float32),
        "topk_idx": np.empty((T, k), np.int32),
        "topk_w": np.empty((T, k), np.float64),
        "counts": np.empty(E, np.int32),
        "offsets": np.empty(E + 1, np.int32),
        "sorted_assign": np.empty(T * k, np.int32),
        "pos": np.empty(T * k, np.int32),
        "h": np.empty((T * k, f), np.float64) if want_h else None,
        "o": np.empty((T * k, d), np.float64),
        "y": np.empty((T, d), np.float64),
    }
    lib().oracle_forward(
        _p(x), T, d, E, k, f, G, _p(w_r), _p(b_r), ctypes.byref(w),
        *[_p(r[n]) for n in ("logits", "topk_idx", "topk_w", "counts", "offsets",
                             "sorted_assign", "pos", "h", "o", "y")])
    del keep
    return r


def token_outputs(inp, tokens):
    """Layer output (float64 [n, d]) for the chosen tokens, one at a time,
    plus their routing (indices [n, k], weights [n, k])."""
    s = inp.shape
    d, E, k, f, G = s.d, s.E, s.k, s.f, s.group
    x = _c(inp.x, np.uint16)
    w_r = _c(inp.w_r, np.float32)
    b_r = None if inp.b_r is None else _c(inp.b_r, np.float32)
    toks = _c(tokens, np.int64)
    n = toks.shape[0]
    w, keep = _weights_struct(inp)
    y = np.empty((n, d), np.float64)
    idx = np.empty((n, k), np.int32)
    rw = np.empty((n, k), np.float64)
    lib().oracle_token_outputs(_p(x), d, E, k, f, G, _p(w_r), _p(b_r), ctypes.byref(w),
                               _p(toks), n, _p(y), _p(idx), _p(rw))
    del keep
    return y, idx, rw
