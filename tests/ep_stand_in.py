"""An oracle-backed stand-in for ep.LibraryBackend, so that the expert-parallel
host logic (count split, exchanges, block map of the received rows) runs as
gloo ranks on CPU.  Test infrastructure: every number comes from oracle/.

Tensors: token rows as int32 tensors holding bf16 bits (x, dispatched rows;
gloo exchanges no 16-bit types), expert outputs as float64 tensors.
"""
from __future__ import annotations

import types

import numpy as np
import torch

import oracle


def _proj_slice(p, e):
    return types.SimpleNamespace(q=p.q[e:e + 1], scale=p.scale[e:e + 1], bias=p.bias[e:e + 1])


class OracleBackend:
    def __init__(self, inp, lo: int, hi: int):
        self.inp = inp
        s = inp.shape
        self.d, self.E, self.k, self.f, self.group = s.d, s.E, s.k, s.f, s.group
        self.lo, self.hi = lo, hi

    def empty_rows(self, n, like):
        return torch.empty((n,) + tuple(like.shape[1:]), dtype=like.dtype)

    def route(self, x):
        xb = x.numpy().astype(np.uint16)
        logits = oracle.router_logits(xb, self.inp.w_r, self.inp.b_r)
        idx = oracle.topk(logits, self.k)
        w = oracle.topk_weights(logits, idx)
        counts, offsets = oracle.counts_offsets(idx, self.E)
        sa, pos = oracle.scatter(idx, offsets)
        return {"idx": idx, "w": w, "counts": counts, "sa": sa, "pos": pos}

    def dispatch(self, x, r):
        return x[torch.from_numpy(r["sa"].astype(np.int64) // self.k)].contiguous()

    def counts(self, r):
        return r["counts"]

    def expert_rows(self, e_global: int, rows_bits: np.ndarray) -> np.ndarray:
        """One expert on some rows: the oracle's layer with that expert alone
        and top-1 (weight exactly 1), whose per-row outputs are the expert's."""
        n = rows_bits.shape[0]
        one = types.SimpleNamespace(
            shape=types.SimpleNamespace(T=n, d=self.d, E=1, k=1, f=self.f, group=self.group),
            x=np.ascontiguousarray(rows_bits), w_r=np.zeros((self.d, 1), np.float32), b_r=None,
            gate=_proj_slice(self.inp.gate, e_global), up=_proj_slice(self.inp.up, e_global),
            down=_proj_slice(self.inp.down, e_global))
        return oracle.forward(one)["o"]

    def experts(self, xs_recv, n_rows, bm):
        o = np.full((n_rows, self.d), np.nan)
        rows = xs_recv.numpy().astype(np.uint16)
        for e, r0, n in bm:
            o[r0:r0 + n] = self.expert_rows(self.lo + int(e), rows[r0:r0 + n])
        return torch.from_numpy(o)

    def combine(self, o_back, r, x):
        o = o_back.numpy()
        T = x.shape[0]
        y = np.zeros((T, self.d))
        for j in range(self.k):
            y += r["w"][:, j:j + 1] * o[r["pos"].reshape(T, self.k)[:, j]]
        return torch.from_numpy(y)
