"""fp64 CPU oracle for mixed-head (retrieval / streaming) KV-cache attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code
with the CUDA library (``head_wise_kv_b200``) and imports nothing from it; the
library never imports this.

Plain, slow and meant to be checked by eye against the pages:

* "DuoAttention: Dual Retrieval & Streaming Heads Guide" (the DuoAttention
  guide below), sections 1 (KV-cache-size equation), 2 ("Retrieval Heads vs.
  Streaming Heads", "Cache Partitioning Mechanics" and its memory equation)
  and its Python simulation of the dual-head cache;
* "Attention Variants and KV-Cache Compression", sections "MHA and GQA"
  (size formula) and "When Is Reuse Exact?" (chunked-prefill mask rule,
  original positions kept after eviction);
* "Attention Variants and Memory Efficiency", sections "Multi-Query and
  Grouped-Query Attention" (``repeat_kv``) and "Sliding-Window and Mixed
  Attention" (window rule and ``SlidingKVCache`` ring).

Every bf16 input is widened exactly to float64; all arithmetic is float64.

Readings taken where the pages leave a step open (each listed in the design
notes of the repository):
  * the recent window includes the current token: keys t-W+1 .. t;
  * when fewer than S+W tokens exist, a streaming head sees every token
    (sinks and window overlap; union, no duplicates);
  * the ring slot of token p is p for p < S, else S + ((p - S) mod W): the
    sliding-window ring's "slot = appended-count mod W" rule applied to the
    tokens that come after the sinks;
  * query head h reads KV head h // (Hq / n_kv) (``repeat_interleave``);
  * a decode query sits at t = T - 1, the token just appended; prefill row i
    of a chunk that follows P cached tokens sits at t = P + i.

FP8 KV cache (DuoAttention guide, "Synergies with Low-Bit Quantization":
cache elements stored in 8 bits instead of 16, a 2x footprint reduction).
The pages fix neither the 8-bit format nor the scaling; readings taken:
  * the format is FP8 E4M3 (OCP 8-bit floating point: sign, 4 exponent bits
    with bias 7, 3 mantissa bits, subnormals, no infinities, code 0x7F/0xFF
    NaN, largest finite magnitude 448);
  * one scale per (layer, KV head) for keys and one for values, given by the
    caller (static, no per-token metadata: exactly 2x, as the pages state);
  * code = round-to-nearest-even E4M3 of fp32(x) / fp32(scale), computed in
    fp32 (IEEE division), magnitudes above 448 saturating to 448; the stored
    value stands for scale * E4M3(code);
  * attention reads every cached key and value dequantized (decode: all of
    them, the new token included, since it is appended first; chunked
    prefill: the cached prefix dequantized, the chunk's own keys and values
    as given, because they are attended before they are appended).

INT4 KV cache (the same passage: 4 bits per element, a 4x footprint
reduction).  The pages give no integer format or scaling either; readings:
  * a code is a signed 4-bit integer c in [-8, 7] (two's complement nibble);
  * the same caller scales as FP8, one per (layer, KV head) for keys and one
    for values (exactly 4x, as the pages state: no per-group metadata);
  * c = round-half-to-even of fp32(x) / fp32(scale), clamped to [-8, 7]; the
    stored value stands for scale * c;
  * two codes per byte, element 2i in the low nibble of byte i and element
    2i + 1 in the high nibble.

Parity pins for every function live in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "kv_cache_bytes", "duo_effective_context", "duo_cache_bytes", "duo_slots",
    "StreamingCache", "ring_positions", "keep_set", "key_mask", "kv_head_of",
    "attend", "decode_attention", "prefill_attention", "brute_force_attention", "blended_decode",
    "E4M3_MAX", "e4m3_decode", "e4m3_encode", "quantize_kv", "dequantize_kv",
    "INT4_MIN", "INT4_MAX", "int4_encode", "int4_pack", "int4_unpack", "quantize_kv_int4", "dequantize_kv_int4",
]


# ---------------------------------------------------------------- sizes
def kv_cache_bytes(layers: int, n_kv: int, d: int, tokens: int, elem_bytes: int = 2) -> int:
    """Dense KV-cache bytes: keys and values (x2), ``elem_bytes`` per element,
    for every layer, KV head, head-dim element and token.
    DuoAttention guide, section 1, KV-cache-size equation; the same product
    as the size formula of "Attention Variants and KV-Cache Compression",
    section "MHA and GQA"."""
    return 2 * elem_bytes * layers * n_kv * d * tokens


def duo_effective_context(tokens: int, sink: int, window: int, retrieval_frac: float) -> float:
    """Tokens held per KV head on average: R*T + (1-R)*(S+W).
    DuoAttention guide, section 2, memory equation and its 128k worked line."""
    return retrieval_frac * tokens + (1.0 - retrieval_frac) * (sink + window)


def duo_cache_bytes(layers: int, n_kv: int, d: int, tokens: int, sink: int, window: int,
                    n_retrieval, elem_bytes: int = 2) -> int:
    """Bytes of the DuoAttention cache for one sequence with ``tokens`` rows
    reserved per retrieval head: retrieval heads keep all T tokens, streaming
    heads keep S + W (DuoAttention guide, section 2, memory equation,
    with R = retrieval heads / n_kv).  ``n_retrieval`` is one count for all
    layers or a per-layer list; the result is exact integer arithmetic."""
    per_layer = list(n_retrieval) if hasattr(n_retrieval, "__len__") else [n_retrieval] * layers
    assert len(per_layer) == layers
    total = 0
    for n_r in per_layer:
        n_s = n_kv - int(n_r)
        total += 2 * elem_bytes * d * (int(n_r) * tokens + n_s * (sink + window))
    return total


def duo_slots(tokens: int, sink: int, window: int, n_retrieval: int, n_streaming: int) -> int:
    """Occupied cache rows after ``tokens`` appends: every token in each
    retrieval head, at most S + W in each streaming head (the DuoAttention
    guide's simulation counts slots this way in its memory statistics)."""
    return n_retrieval * tokens + n_streaming * min(tokens, sink + window)


# ---------------------------------------------------------------- ring
class StreamingCache:
    """Literal per-token model of one streaming head's cache.

    Tokens go to the sink region until it holds S tokens (DuoAttention guide,
    simulation, ``append_token``); every later token goes to the recent
    window, a W-slot ring that overwrites its oldest entry, its slot being the
    number of window appends so far modulo W ("Attention Variants and Memory
    Efficiency", ``SlidingKVCache.append``).  Slots 0..S-1 are the sinks, slots
    S..S+W-1 the ring.  ``pos[slot]`` keeps each token's original position
    (-1 = empty): "Attention Variants and KV-Cache Compression", section
    "When Is Reuse Exact?" -- positions are not renumbered after eviction."""

    def __init__(self, sink: int, window: int):
        assert sink >= 0 and window >= 1
        self.sink, self.window = sink, window
        self.pos = np.full(sink + window, -1, dtype=np.int64)
        self.items = [None] * (sink + window)
        self.n_sink = 0
        self.n_window = 0

    def append(self, position: int, item=None) -> int:
        if self.n_sink < self.sink:
            slot = self.n_sink
            self.n_sink += 1
        else:
            slot = self.sink + (self.n_window % self.window)
            self.n_window += 1
        self.pos[slot] = position
        self.items[slot] = item
        return slot

    def ordered(self):
        """Held (position, item) pairs, sinks first, then the window oldest to
        newest (the ring's ordered view)."""
        sinks = [(int(self.pos[s]), self.items[s]) for s in range(self.n_sink)]
        count = min(self.n_window, self.window)
        win = [(int(self.pos[self.sink + (k % self.window)]), self.items[self.sink + (k % self.window)])
               for k in range(self.n_window - count, self.n_window)]
        return sinks + win


def ring_positions(tokens: int, sink: int, window: int) -> np.ndarray:
    """pos table [S+W] after appending positions 0 .. tokens-1 one by one."""
    c = StreamingCache(sink, window)
    for p in range(tokens):
        c.append(p)
    return c.pos.copy()


# ---------------------------------------------------------------- key sets
def keep_set(t: int, sink: int, window: int) -> np.ndarray:
    """Key positions a streaming head attends from query position t: the
    attention sinks 0..S-1 and the recent window max(0, t-W+1) .. t
    (DuoAttention guide, section 2, streaming heads; window rule of
    "Attention Variants and Memory Efficiency", section "Sliding-Window and
    Mixed Attention")."""
    j = np.arange(t + 1)
    return j[(j < sink) | (j >= t - window + 1)]


def key_mask(rows_t: np.ndarray, n_keys: int, retrieval: bool, sink: int, window: int) -> np.ndarray:
    """bool [len(rows_t)][n_keys]: may the query at absolute position
    rows_t[i] read the key at absolute position j?  Retrieval heads: every
    j <= t (full causal).  Streaming heads: j <= t and j in keep_set(t)."""
    t = np.asarray(rows_t)[:, None]
    j = np.arange(n_keys)[None, :]
    m = j <= t
    if not retrieval:
        m &= (j < sink) | (j >= t - window + 1)
    return m


def kv_head_of(h: int, hq: int, n_kv: int) -> int:
    """KV head read by query head h: K/V repeated along the head axis with
    ``repeat_interleave(hq // n_kv)`` ("Attention Variants and Memory
    Efficiency", section "Multi-Query and Grouped-Query Attention")."""
    assert hq % n_kv == 0
    return h // (hq // n_kv)


# ---------------------------------------------------------------- attention
def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """Softmax attention of one query over the given keys (float64).
    Returns (o [d], lse) with lse = log sum_j exp(s_j)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    s = scale * (k @ q)
    m = s.max()
    e = np.exp(s - m)
    z = e.sum()
    return (e @ v) / z, m + math.log(z)


def decode_attention(q, k_hist, v_hist, lens_after, mask, sink, window, scale, pairs=None):
    """One decode step of one layer.

    q: [B][Hq][d] (the newest token's query per sequence);
    k_hist(b, g) / v_hist(b, g): callables returning the history of KV head g
    of sequence b as an array indexable by position (at least lens_after[b]
    rows: tokens 0 .. T_b-1);
    mask: [n_kv], 1 = retrieval head.  Query position t = T_b - 1.
    pairs: optional iterable of (b, h) to evaluate; the rest stay NaN.
    Returns out [B][Hq][d] and lse [B][Hq] (float64)."""
    q = np.asarray(q, dtype=np.float64)
    B, hq, d = q.shape
    n_kv = len(mask)
    out = np.full((B, hq, d), np.nan)
    lse = np.full((B, hq), np.nan)
    todo = {(b, h) for b in range(B) for h in range(hq)} if pairs is None else set(pairs)
    for b in range(B):
        t = int(lens_after[b]) - 1
        for g in range(n_kv):
            heads = [h for h in range(hq) if kv_head_of(h, hq, n_kv) == g and (b, h) in todo]
            if not heads:
                continue
            keys = np.arange(t + 1) if mask[g] else keep_set(t, sink, window)
            K = np.asarray(k_hist(b, g)[keys], dtype=np.float64)
            V = np.asarray(v_hist(b, g)[keys], dtype=np.float64)
            for h in heads:
                out[b, h], lse[b, h] = attend(q[b, h], K, V, scale)
    return out, lse


def blended_decode(q, k_hist, v_hist, lens_after, n_kv, alpha, sink, window, scale):
    """Gated attention of head identification (DuoAttention guide, section 3
    "Automated Head Identification", item 2): for each query head h,
    alpha[h] * FullAttn + (1 - alpha[h]) * StreamAttn, where FullAttn reads
    every key 0..t of the head's full history and StreamAttn only the sinks
    and the recent window of that same history.  Returns [B][Hq][d] float64."""
    alpha = np.asarray(alpha, dtype=np.float64)[None, :, None]
    full, _ = decode_attention(q, k_hist, v_hist, lens_after, np.ones(n_kv, np.uint8), sink, window, scale)
    strm, _ = decode_attention(q, k_hist, v_hist, lens_after, np.zeros(n_kv, np.uint8), sink, window, scale)
    return alpha * full + (1.0 - alpha) * strm


def prefill_attention(q, k_hist, v_hist, prefix, mask, sink, window, scale,
                      rows=None, row_block: int = 256):
    """Attention of a prefill chunk of C queries that follows ``prefix[b]``
    cached tokens ("Attention Variants and KV-Cache Compression", section
    "When Is Reuse Exact?": row i sits at absolute position P + i and may read
    keys through P + i, not an upper-left C x (P + C) triangle).

    q: [B][Hq][C][d]; k_hist(b, g) / v_hist(b, g): history [P_b + C][d]
    (cached prefix followed by the chunk's own keys); rows: optional list of
    chunk rows to evaluate (others are left as NaN).
    Returns out [B][Hq][C][d] (float64)."""
    q = np.asarray(q, dtype=np.float64)
    B, hq, C, d = q.shape
    n_kv = len(mask)
    rows = np.arange(C) if rows is None else np.asarray(sorted(rows))
    out = np.full((B, hq, C, d), np.nan)
    for b in range(B):
        P = int(prefix[b])
        for g in range(n_kv):
            K = np.asarray(k_hist(b, g), dtype=np.float64)
            V = np.asarray(v_hist(b, g), dtype=np.float64)
            assert K.shape[0] >= P + C
            for h in range(hq):
                if kv_head_of(h, hq, n_kv) != g:
                    continue
                for r0 in range(0, len(rows), row_block):
                    rr = rows[r0:r0 + row_block]
                    t = P + rr
                    n_keys = int(t.max()) + 1
                    allowed = key_mask(t, n_keys, bool(mask[g]), sink, window)
                    s = scale * (q[b, h, rr] @ K[:n_keys].T)
                    s = np.where(allowed, s, -np.inf)
                    m = s.max(axis=1, keepdims=True)
                    e = np.exp(s - m)
                    out[b, h, rr] = (e @ V[:n_keys]) / e.sum(axis=1, keepdims=True)
    return out


def brute_force_attention(q, k, v, keys, scale):
    """Pure-Python loops (tiny inputs only): softmax over the listed key
    positions of scale * <q, k_j>, weights applied to v_j."""
    d = len(q)
    scores = []
    for j in keys:
        acc = 0.0
        for x in range(d):
            acc += float(q[x]) * float(k[j][x])
        scores.append(scale * acc)
    m = max(scores)
    w = [math.exp(s - m) for s in scores]
    z = sum(w)
    o = [0.0] * d
    for wj, j in zip(w, keys):
        for x in range(d):
            o[x] += wj * float(v[j][x])
    return [ox / z for ox in o], m + math.log(z)


# ---------------------------------------------------------------- FP8 (E4M3) KV cache
E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """Value of each E4M3 byte, float64.  Bit 7 sign, bits 6..3 exponent e
    (bias 7), bits 2..0 mantissa m: e = 0 gives (m / 8) * 2^-6, otherwise
    (1 + m / 8) * 2^(e - 7); e = 15 with m = 7 is NaN (no infinities)."""
    c = np.asarray(codes, dtype=np.int64) & 0xFF
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


# the 127 non-negative finite values, codes 0x00 .. 0x7E, increasing
_E4M3_POS = e4m3_decode(np.arange(0x7F))


def e4m3_encode(x) -> np.ndarray:
    """E4M3 byte nearest to each value of x (round to nearest, ties to the
    code with an even mantissa), magnitudes beyond 448 saturating to 448;
    the sign is kept (a negative value that rounds to 0 gives 0x80); NaN
    gives 0x7F.  x is taken as float64 (pass fp32 values for fp32 inputs)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    hi = np.clip(np.searchsorted(_E4M3_POS, a, side="left"), 0, 0x7E)   # first value >= a
    lo = np.clip(hi - 1, 0, 0x7E)
    d_hi = np.abs(_E4M3_POS[hi] - a)
    d_lo = np.abs(a - _E4M3_POS[lo])
    pick = np.where(d_lo < d_hi, lo, hi)
    pick = np.where(d_lo == d_hi, np.where(lo % 2 == 0, lo, hi), pick)   # tie: even code = even mantissa
    pick = np.where(a >= E4M3_MAX, 0x7E, pick)
    code = pick.astype(np.int64) | np.where(np.signbit(x), 0x80, 0)
    code = np.where(np.isnan(x), 0x7F, code)
    return code.astype(np.uint8)


def quantize_kv(x, scale: float) -> np.ndarray:
    """Cache codes of K or V values x (bf16 values, any shape) under one
    scale: E4M3 of fp32(x) / fp32(scale), the quotient rounded once in fp32."""
    q = np.asarray(x, dtype=np.float32) / np.float32(scale)
    return e4m3_encode(q.astype(np.float64))


def dequantize_kv(codes, scale: float) -> np.ndarray:
    """Values the cache codes stand for: scale * E4M3(code), float64 (exact)."""
    return float(np.float32(scale)) * e4m3_decode(codes)


# ---------------------------------------------------------------- INT4 KV cache
INT4_MIN, INT4_MAX = -8, 7


def int4_encode(x) -> np.ndarray:
    """Signed 4-bit code of each value of x: the nearest integer (ties to the
    even one), clamped to [-8, 7]; NaN gives 0.  x as float64 (pass fp32
    quotients for fp32 inputs)."""
    x = np.asarray(x, dtype=np.float64)
    r = np.rint(np.where(np.isnan(x), 0.0, x))          # round half to even
    return np.clip(r, INT4_MIN, INT4_MAX).astype(np.int8)


def int4_pack(codes) -> np.ndarray:
    """Pack codes [..., d] (d even) two per byte: element 2i in the low
    nibble of byte i, element 2i + 1 in the high nibble (two's complement)."""
    c = np.asarray(codes, dtype=np.int64)
    lo = c[..., 0::2] & 0xF
    hi = c[..., 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def int4_unpack(packed) -> np.ndarray:
    """Codes [..., 2n] of packed bytes [..., n], sign-extended from 4 bits."""
    b = np.asarray(packed, dtype=np.int64) & 0xFF
    nib = np.stack([b & 0xF, b >> 4], axis=-1).reshape(*b.shape[:-1], 2 * b.shape[-1])
    return np.where(nib >= 8, nib - 16, nib).astype(np.int8)


def quantize_kv_int4(x, scale: float) -> np.ndarray:
    """Packed INT4 cache bytes [..., d/2] of K or V values x [..., d]: the
    code of fp32(x) / fp32(scale), the quotient rounded once in fp32."""
    q = np.asarray(x, dtype=np.float32) / np.float32(scale)
    return int4_pack(int4_encode(q.astype(np.float64)))


def dequantize_kv_int4(packed, scale: float) -> np.ndarray:
    """Values packed INT4 cache bytes stand for: scale * code, float64 (exact)."""
    return float(np.float32(scale)) * int4_unpack(packed).astype(np.float64)
