"""Seeded synthetic inputs for the mixed-head (retrieval/streaming) KV-cache path.

This module only draws random numbers and lays them out.  It holds none of
the attention or cache arithmetic: both the fp64 oracle (``oracle/``) and the
CUDA library's tests and benchmark take their inputs from here, and nothing
here imports either of them.

Every tensor is a deterministic function of (workload, layer, sequence, head,
tensor kind, token block): token ``p`` of head ``g`` of sequence ``b`` always has
the same K, V and q, whichever call asks for it and in whatever order.  Draws
are fp32 N(0, 1) from numpy's PCG64 seeded by a ``SeedSequence`` over that key,
rounded to bf16 (round-to-nearest-even) -- the cache element type the pages
assume (DuoAttention guide, section 1, KV-cache-size equation: "16-bit").

Workloads (shapes, head split, sink/window sizes, length mix) follow the
model shapes the pages name: Llama-2-7B-like MHA and Llama-3-8B-like GQA.
"""
from __future__ import annotations

import functools
import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np
import torch

BLOCK_TOKENS = 4096          # token granularity of the seeded K/V streams
Q_BLOCK_TOKENS = 64          # token granularity of the seeded q streams
TENSOR_K, TENSOR_V, TENSOR_Q = 0, 1, 2
_POOL = ThreadPoolExecutor(max_workers=8)


@dataclass(frozen=True)
class Workload:
    name: str
    index: int                 # position in the workload list; seed = 1234 + index
    layers: int
    batch: int
    hq: int                    # query heads
    n_kv: int                  # KV heads
    d: int                     # head dim
    sink: int                  # S
    window: int                # W
    retrieval_frac: float      # fraction of KV heads per layer that are retrieval
    steps: int = 0             # decode steps after the prefilled context
    t0: int = 0                # prefilled context (fixed length)
    t0_range: tuple | None = None   # (lo, hi) inclusive: ragged prefilled lengths
    fixed_retrieval: tuple | None = None   # explicit retrieval KV heads (all layers)
    rope: bool = False         # K/q rotated (rotate-half, theta=1e4) at their positions
    sink_boost: float = 1.0    # key rows 0..3 multiplied by this factor
    prompt: int = 0            # chunked prefill: prompt length
    chunk: int = 0             # chunked prefill: chunk length
    desc: str = ""

    @property
    def seed(self) -> int:
        return 1234 + self.index

    @property
    def group(self) -> int:
        return self.hq // self.n_kv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def n_retrieval(self) -> int:
        if self.fixed_retrieval is not None:
            return len(self.fixed_retrieval)
        return int(math.ceil(self.retrieval_frac * self.n_kv))


WORKLOADS = {
    "tiny": Workload(
        name="tiny", index=0, layers=1, batch=1, hq=4, n_kv=4, d=64, sink=16, window=64,
        retrieval_frac=0.5, steps=16, t0=512, fixed_retrieval=(0, 2), rope=True,
        desc="1 layer, MHA 4 heads, d=64, B=1, T0=512, 16 decode steps, heads {0,2} retrieval, S=16, W=64"),
    "mha32k": Workload(
        name="mha32k", index=1, layers=1, batch=1, hq=32, n_kv=32, d=128, sink=64, window=256,
        retrieval_frac=0.25, steps=64, t0=32768, sink_boost=4.0,
        desc="Llama-2-7B attention: MHA 32 heads, d=128, B=1, T=32768, 8 retrieval heads, S=64, W=256"),
    "gqa128k": Workload(
        name="gqa128k", index=2, layers=1, batch=8, hq=32, n_kv=8, d=128, sink=64, window=256,
        retrieval_frac=0.5, steps=32, t0_range=(16384, 131072),
        desc="Llama-3-8B attention: GQA 32q/8kv, d=128, B=8, T_b~U[16K,128K], 4 retrieval KV heads, S=64, W=256"),
    "mtok": Workload(
        name="mtok", index=3, layers=32, batch=1, hq=32, n_kv=8, d=128, sink=64, window=1024,
        retrieval_frac=0.25, steps=1, t0=1048576,
        desc="32 layers GQA 32q/8kv, d=128, B=1, T=1048576, 2 retrieval KV heads per layer, S=64, W=1024"),
    "prefill64k": Workload(
        name="prefill64k", index=4, layers=1, batch=1, hq=32, n_kv=8, d=128, sink=64, window=1024,
        retrieval_frac=0.5, prompt=65536, chunk=4096,
        desc="GQA 32q/8kv, d=128, B=1, 65536-token prompt in 4096-token chunks, 4 retrieval KV heads, S=64, W=1024"),
}


def scaled(w: Workload, **kw) -> Workload:
    """A copy of ``w`` with some fields replaced (smaller parity cases)."""
    d = {k: getattr(w, k) for k in w.__dataclass_fields__}
    d.update(kw)
    return Workload(**d)


# ---------------------------------------------------------------- head roles
def retrieval_mask(w: Workload, layer: int) -> np.ndarray:
    """uint8 [n_kv], 1 = retrieval KV head.  Seeded permutation; the first
    ceil(frac * n_kv) heads of it are retrieval (one draw per layer)."""
    m = np.zeros(w.n_kv, dtype=np.uint8)
    if w.fixed_retrieval is not None:
        m[list(w.fixed_retrieval)] = 1
        return m
    rng = np.random.default_rng(np.random.SeedSequence([w.seed, 7, layer]))
    perm = rng.permutation(w.n_kv)
    m[perm[: w.n_retrieval()]] = 1
    return m


def retrieval_masks(w: Workload) -> np.ndarray:
    return np.stack([retrieval_mask(w, l) for l in range(w.layers)])


# ---------------------------------------------------------------- lengths
def context_lengths(w: Workload) -> np.ndarray:
    """int64 [B]: tokens already cached before the first decode step."""
    if w.t0_range is not None:
        lo, hi = w.t0_range
        rng = np.random.default_rng(np.random.SeedSequence([w.seed, 11]))
        return rng.integers(lo, hi, size=w.batch, endpoint=True).astype(np.int64)
    return np.full(w.batch, w.t0, dtype=np.int64)


def capacity(w: Workload) -> int:
    """Retrieval-cache rows per (sequence, head) that the workload needs."""
    if w.prompt:
        return w.prompt
    return int(context_lengths(w).max()) + w.steps


# ---------------------------------------------------------------- token streams
def _block_tokens(kind: int) -> int:
    return Q_BLOCK_TOKENS if kind == TENSOR_Q else BLOCK_TOKENS


@functools.lru_cache(maxsize=192)
def _block(w: Workload, layer: int, b: int, head: int, kind: int, blk: int) -> np.ndarray:
    ss = np.random.SeedSequence([w.seed, layer, b, head, kind, blk])
    rng = np.random.default_rng(ss)
    x = rng.standard_normal((_block_tokens(kind), w.d), dtype=np.float32)
    x.setflags(write=False)
    return x


def _rope(x: np.ndarray, p0: int, d: int) -> np.ndarray:
    """Rotate-half rotary embedding, theta = 10000, positions p0 .. p0+n-1.
    Used only to shape the synthetic data; kernels never apply it."""
    half = d // 2
    n = x.shape[0]
    pos = np.arange(p0, p0 + n, dtype=np.float64)[:, None]
    inv = 10000.0 ** (-np.arange(half, dtype=np.float64) * 2.0 / d)
    ang = pos * inv[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1 = x[:, :half].astype(np.float64)
    x2 = x[:, half:].astype(np.float64)
    out = np.empty_like(x, dtype=np.float64)
    out[:, :half] = x1 * c - x2 * s
    out[:, half:] = x2 * c + x1 * s
    return out.astype(np.float32)


def tokens_f32(w: Workload, layer: int, b: int, head: int, kind: int, p0: int, p1: int) -> np.ndarray:
    """fp32 [p1-p0][d] draws for token positions p0..p1-1 (before bf16 rounding).
    The result may be a read-only view of a cached block."""
    if p1 <= p0:
        return np.zeros((0, w.d), dtype=np.float32)
    bt = _block_tokens(kind)
    b0, b1 = p0 // bt, (p1 - 1) // bt
    if b1 == b0:
        x = _block(w, layer, b, head, kind, b0)
    else:
        x = np.concatenate(list(_POOL.map(lambda k: _block(w, layer, b, head, kind, k),
                                          range(b0, b1 + 1))), axis=0)
    x = x[p0 - b0 * bt: p1 - b0 * bt]
    if w.rope and kind in (TENSOR_K, TENSOR_Q):
        x = _rope(x, p0, w.d)
    if w.sink_boost != 1.0 and kind == TENSOR_K and p0 < 4:
        x = x.copy()
        x[: 4 - p0] *= w.sink_boost
    return x


def tokens(w: Workload, layer: int, b: int, head: int, kind: int, p0: int, p1: int) -> torch.Tensor:
    """bf16 CPU tensor [p1-p0][d]: K (kind 0) or V (1) of KV head ``head``, or
    q (2) of query head ``head``, for token positions p0..p1-1 of sequence b."""
    x = tokens_f32(w, layer, b, head, kind, p0, p1)
    if not x.flags.writeable:
        x = x.copy()
    return torch.from_numpy(x).to(torch.bfloat16)


def decode_q(w: Workload, layer: int, lens_after: np.ndarray) -> torch.Tensor:
    """bf16 [B][Hq][d]: each sequence's query for its newest token (position len-1)."""
    out = torch.empty(w.batch, w.hq, w.d, dtype=torch.bfloat16)
    for b in range(w.batch):
        p = int(lens_after[b]) - 1
        for h in range(w.hq):
            out[b, h] = tokens(w, layer, b, h, TENSOR_Q, p, p + 1)[0]
    return out


def new_kv(w: Workload, layer: int, lens_before: np.ndarray, n_new: int):
    """bf16 k_new, v_new [B][n_kv][n_new][d]: tokens lens_before[b] .. +n_new-1."""
    k = torch.empty(w.batch, w.n_kv, n_new, w.d, dtype=torch.bfloat16)
    v = torch.empty_like(k)
    for b in range(w.batch):
        p = int(lens_before[b])
        for g in range(w.n_kv):
            k[b, g] = tokens(w, layer, b, g, TENSOR_K, p, p + n_new)
            v[b, g] = tokens(w, layer, b, g, TENSOR_V, p, p + n_new)
    return k, v


def chunk_q(w: Workload, layer: int, p0: int, c: int) -> torch.Tensor:
    """bf16 [B][Hq][c][d]: queries for positions p0 .. p0+c-1 (chunked prefill)."""
    out = torch.empty(w.batch, w.hq, c, w.d, dtype=torch.bfloat16)
    for b in range(w.batch):
        for h in range(w.hq):
            out[b, h] = tokens(w, layer, b, h, TENSOR_Q, p0, p0 + c)
    return out

