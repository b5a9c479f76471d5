"""Shared helpers for the GPU parity tests: fill a cache from the seeded
workload streams, run decode steps through the C ABI, and compare with the
fp64 oracle.  Inputs come only from ``duo_workloads``; expected values only
from ``oracle``."""
from __future__ import annotations

import numpy as np
import torch

import duo_workloads as W
from oracle import duo_oracle as O

MAX_ABS = 2e-3      # parity bar on fp32 outputs (bf16 inputs, fp32 accumulation)
REL_L2 = 1e-3


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    max_abs = float(np.abs(got - ref).max()) if got.size else 0.0
    den = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(got - ref) / den) if den > 0 else float(np.linalg.norm(got - ref))
    return max_abs, rel


def assert_close(got, ref, what=""):
    m, r = errors(got, ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert m <= MAX_ABS and r <= REL_L2, f"{what}: max-abs {m:.3e} (bar {MAX_ABS}), rel-L2 {r:.3e} (bar {REL_L2})"
    return m, r


class History:
    """CPU bf16 K/V/q streams of one workload, cached per (layer, b, head, kind)."""

    def __init__(self, w: W.Workload):
        self.w = w
        self._c = {}

    def kv(self, layer, b, g, kind, p1):
        key = (layer, b, g, kind)
        have = self._c.get(key)
        if have is None or have.shape[0] < p1:
            self._c[key] = W.tokens(self.w, layer, b, g, kind, 0, p1)
        return self._c[key][:p1]

    def k64(self, layer, b, g, p1):
        return self.kv(layer, b, g, W.TENSOR_K, p1).double().numpy()

    def v64(self, layer, b, g, p1):
        return self.kv(layer, b, g, W.TENSOR_V, p1).double().numpy()

    def drop(self):
        self._c.clear()


def fill(cache, hist: History, layer: int, lens0, dev, slab: int = 8192):
    """Bulk-append tokens 0 .. lens0[b]-1 of every (b, g) to one layer, in
    slabs of up to ``slab`` tokens with per-sequence counts."""
    w = hist.w
    lens0 = np.asarray(lens0, dtype=np.int64)
    top = int(lens0.max())
    for p0 in range(0, top, slab):
        n = min(slab, top - p0)
        k = torch.zeros(w.batch, w.n_kv, n, w.d, dtype=torch.bfloat16)
        v = torch.zeros_like(k)
        counts = np.clip(lens0 - p0, 0, n).astype(np.int32)
        for b in range(w.batch):
            c = int(counts[b])
            if c == 0:
                continue
            for g in range(w.n_kv):
                k[b, g, :c] = W.tokens(w, layer, b, g, W.TENSOR_K, p0, p0 + c)
                v[b, g, :c] = W.tokens(w, layer, b, g, W.TENSOR_V, p0, p0 + c)
        before = torch.from_numpy(np.minimum(lens0, p0).astype(np.int32)).to(dev)
        cache.append(layer, k.to(dev), v.to(dev), before, torch.from_numpy(counts).to(dev))


def new_token_inputs(w: W.Workload, layer: int, lens_before):
    """(q, k_new, v_new) CPU bf16 for the decode step that appends token lens_before[b]."""
    lens_before = np.asarray(lens_before, dtype=np.int64)
    k, v = W.new_kv(w, layer, lens_before, 1)
    q = W.decode_q(w, layer, lens_before + 1)
    return q, k, v


def oracle_decode(hist: History, layer: int, q, lens_after, mask, pairs=None):
    """fp64 reference for decode (oracle.decode_attention on the seeded
    history).  pairs: optional list of (b, h) to evaluate."""
    lens_after = np.asarray(lens_after, dtype=np.int64)

    def kh(b, g):
        return hist.kv(layer, b, g, W.TENSOR_K, int(lens_after[b])).float().numpy()

    def vh(b, g):
        return hist.kv(layer, b, g, W.TENSOR_V, int(lens_after[b])).float().numpy()
    w = hist.w
    return O.decode_attention(q.double().numpy(), kh, vh, lens_after, mask, w.sink, w.window, w.scale,
                              pairs=pairs)
