"""FP8 (E4M3) caches through the C ABI against the fp64 oracle.

* the cached bytes are the oracle's codes of value / scale, bit for bit
  (retrieval rows and ring slots), positions as for bf16 caches;
* decode equals attention over the dequantised history (scale * E4M3(code)),
  the new token included (it is appended, hence quantised, first), for every
  GQA group size, ragged lengths that cross the 256-key tiles, any split of
  the keys over CTAs, saturating scales and extreme query magnitudes, and the
  full 128K GQA workload (sampled heads) at the launch configuration the
  benchmark uses;
* chunked prefill attends to the cached prefix dequantised and to the
  chunk's own keys and values as given.
"""
import numpy as np
import pytest
import torch

import duo_workloads as W
from _harness import History, assert_close, fill, new_token_inputs
from oracle import duo_oracle as O

pytestmark = pytest.mark.gpu


def _dev():
    return torch.device("cuda", 0)


def _scales(w, seed, lo=0.25, hi=2.0):
    rng = np.random.default_rng(seed)
    return (rng.uniform(lo, hi, (w.layers, w.n_kv)).astype(np.float32),
            rng.uniform(lo, hi, (w.layers, w.n_kv)).astype(np.float32))


def _cache(w, cap, ks, vs, mask=None):
    from head_wise_kv_b200 import DuoKVCache
    masks = W.retrieval_masks(w) if mask is None else np.asarray(mask, np.uint8).reshape(w.layers, w.n_kv)
    return DuoKVCache(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, cap, masks, device=_dev(),
                      kv_dtype="fp8", k_scale=ks, v_scale=vs)


class DequantHistory:
    """Dequantised K/V streams: scale * E4M3(code of value / scale)."""

    def __init__(self, hist: History, ks, vs, layer=0):
        self.h, self.ks, self.vs, self.layer = hist, ks, vs, layer
        self._c = {}

    def get(self, b, g, kind, n):
        key = (b, g, kind)
        have = self._c.get(key)
        if have is None or have.shape[0] < n:
            x = self.h.kv(self.layer, b, g, kind, n).float().numpy()
            s = float((self.ks if kind == W.TENSOR_K else self.vs)[self.layer, g])
            self._c[key] = O.dequantize_kv(O.quantize_kv(x, s), s)
        return self._c[key][:n]


def _decode_step(cache, w, hist, lens0, ks, vs, q_mult=1.0, pairs=None):
    """Append token lens0[b] of every sequence, decode, compare with the oracle."""
    dev = _dev()
    q, k, v = new_token_inputs(w, 0, lens0)
    if q_mult != 1.0:
        q = (q.float() * q_mult).to(torch.bfloat16)
    cache.append(0, k.to(dev), v.to(dev), torch.from_numpy(lens0.astype(np.int32)).to(dev))
    lens = lens0 + 1
    out = cache.decode(0, q.to(dev), torch.from_numpy(lens.astype(np.int32)).to(dev), w.scale)
    dq = DequantHistory(hist, ks, vs)
    ref, _ = O.decode_attention(q.double().numpy(), lambda b, g: dq.get(b, g, W.TENSOR_K, int(lens[b])),
                                lambda b, g: dq.get(b, g, W.TENSOR_V, int(lens[b])), lens, W.retrieval_mask(w, 0),
                                w.sink, w.window, w.scale, pairs=pairs)
    got = out.cpu().double().numpy()
    if pairs is not None:
        got = np.stack([got[b, h] for b, h in pairs])
        ref = np.stack([ref[b, h] for b, h in pairs])
    return got, ref


def test_fp8_codes_bit_exact():
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=2, layers=1, t0_range=None, t0=700, sink=16, window=64)
    ks, vs = _scales(w, 5)
    dev = _dev()
    T0 = np.array([700, 513])
    cache = _cache(w, 720, ks, vs)
    hist = History(w)
    fill(cache, hist, 0, T0, dev)
    for s in range(3):                         # then single-token steps
        q, k, v = new_token_inputs(w, 0, T0 + s)
        cache.append(0, k.to(dev), v.to(dev), torch.from_numpy((T0 + s).astype(np.int32)).to(dev))
    T = T0 + 3
    torch.cuda.synchronize()
    assert cache.status() == 0
    views = cache.layer_views(0)
    mask = W.retrieval_mask(w, 0)
    for b in range(w.batch):
        pos = O.ring_positions(int(T[b]), w.sink, w.window)
        assert np.array_equal(views["positions"][b].cpu().numpy(), pos)
        for g in range(w.n_kv):
            r = views["head_rank"][g]
            for kind, name, sc in ((W.TENSOR_K, "k", ks), (W.TENSOR_V, "v", vs)):
                x = hist.kv(0, b, g, kind, int(T[b])).float().numpy()
                codes = O.quantize_kv(x, float(sc[0, g]))
                if mask[g]:
                    got = views[f"{name}_retrieval"][b, r, :T[b]].cpu().numpy()
                    assert np.array_equal(got, codes), f"b{b} g{g} {name} retrieval codes"
                else:
                    got = views[f"{name}_streaming"][b, r].cpu().numpy()
                    filled = pos >= 0
                    assert np.array_equal(got[filled], codes[pos[filled]]), f"b{b} g{g} {name} ring codes"
    cache.close()


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_fp8_decode_matches_oracle(G):
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=3, layers=1, hq=4 * G, n_kv=4, t0_range=None, t0=0,
                 sink=16, window=64)
    ks, vs = _scales(w, 6 + G)
    lens0 = np.array([900, 255, 70])           # three tiles + a tail, one short of a tile, inside the ring
    cache = _cache(w, 1000, ks, vs)
    hist = History(w)
    fill(cache, hist, 0, lens0, _dev())
    got, ref = _decode_step(cache, w, hist, lens0, ks, vs)
    assert cache.status() == 0
    assert_close(got, ref, f"fp8 decode G={G}")
    cache.close()


@pytest.mark.parametrize("ctas", [5, 37, 300])
def test_fp8_split_count_invariance(ctas):
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=2, layers=1, t0_range=None, t0=0, sink=16, window=64)
    ks, vs = _scales(w, 21)
    lens0 = np.array([1500, 777])
    cache = _cache(w, 1600, ks, vs)
    cache.set_decode_ctas(ctas)
    hist = History(w)
    fill(cache, hist, 0, lens0, _dev())
    got, ref = _decode_step(cache, w, hist, lens0, ks, vs)
    assert cache.status() == 0
    assert_close(got, ref, f"fp8 decode over {ctas} CTAs")
    cache.close()


@pytest.mark.parametrize("scale_lo,scale_hi,q_mult", [(1 / 256, 1 / 128, 1.0), (4.0, 16.0, 1.0),
                                                      (0.5, 1.0, 1e-3), (0.5, 1.0, 300.0)])
def test_fp8_saturating_scales_and_query_range(scale_lo, scale_hi, q_mult):
    """Small scales push |value / scale| past 448 (codes saturate, as in the
    oracle); large ones push values into the E4M3 subnormals; tiny and large
    queries exercise the power-of-two prescale of q."""
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=2, layers=1, t0_range=None, t0=0, sink=16, window=64)
    ks, vs = _scales(w, 31, scale_lo, scale_hi)
    lens0 = np.array([600, 333])
    cache = _cache(w, 700, ks, vs)
    hist = History(w)
    fill(cache, hist, 0, lens0, _dev())
    got, ref = _decode_step(cache, w, hist, lens0, ks, vs, q_mult=q_mult)
    assert_close(got, ref, f"fp8 scales [{scale_lo}, {scale_hi}], q x {q_mult}")
    cache.close()


def test_fp8_gqa128k_config_sampled():
    """The full 128K GQA workload (8 sequences, 16K-128K tokens) in an FP8
    cache, one decode step at the launch configuration the benchmark times;
    a seeded sample of (sequence, query head) pairs against the oracle."""
    w = W.WORKLOADS["gqa128k"]
    ks, vs = _scales(w, 41, 0.5, 1.5)
    lens0 = W.context_lengths(w)
    cache = _cache(w, int(lens0.max()) + 1, ks, vs)
    hist = History(w)
    fill(cache, hist, 0, lens0, _dev(), slab=16384)
    rng = np.random.default_rng(3)
    pairs = [(int(b), int(h)) for b, h in zip(rng.integers(0, w.batch, 12), rng.integers(0, w.hq, 12))]
    got, ref = _decode_step(cache, w, hist, lens0, ks, vs, pairs=pairs)
    assert cache.status() == 0
    assert_close(got, ref, "fp8 gqa128k sampled")
    cache.close()


# ------------------------------------------------------------------ prefill on an FP8 cache
def _chunk(w, prefix, C):
    q = torch.empty(w.batch, w.hq, C, w.d, dtype=torch.bfloat16)
    k = torch.empty(w.batch, w.n_kv, C, w.d, dtype=torch.bfloat16)
    v = torch.empty_like(k)
    for b in range(w.batch):
        P = int(prefix[b])
        for h in range(w.hq):
            q[b, h] = W.tokens(w, 0, b, h, W.TENSOR_Q, P, P + C)
        for g in range(w.n_kv):
            k[b, g] = W.tokens(w, 0, b, g, W.TENSOR_K, P, P + C)
            v[b, g] = W.tokens(w, 0, b, g, W.TENSOR_V, P, P + C)
    return q, k, v


@pytest.mark.parametrize("chunks,S,Wn", [([300, 700, 129], 16, 64), ([256, 384], 64, 1024)])
def test_fp8_prefill_matches_oracle(chunks, S, Wn):
    """Chunked prefill on an FP8 cache: each chunk attends to the cached
    prefix dequantised and to its own keys / values as given (they are
    appended, hence quantised, only afterwards)."""
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=2, layers=1, t0_range=None, t0=0, sink=S, window=Wn)
    ks, vs = _scales(w, 51)
    dev = _dev()
    cache = _cache(w, sum(chunks), ks, vs)
    hist = History(w)
    dq = DequantHistory(hist, ks, vs)
    mask = W.retrieval_mask(w, 0)
    prefix = np.zeros(w.batch, dtype=np.int64)
    for C in chunks:
        q, k, v = _chunk(w, prefix, C)
        pre = torch.from_numpy(prefix.astype(np.int32)).to(dev)
        out = cache.prefill(0, q.to(dev), k.to(dev), v.to(dev), pre, w.scale)
        cache.append(0, k.to(dev), v.to(dev), pre)

        def hist_of(kind):
            def f(b, g):
                P = int(prefix[b])
                cached = dq.get(b, g, kind, P) if P else np.zeros((0, w.d))
                own = hist.kv(0, b, g, kind, P + C)[P:].double().numpy()
                return np.concatenate([cached, own])
            return f
        ref = O.prefill_attention(q.double().numpy(), hist_of(W.TENSOR_K), hist_of(W.TENSOR_V), prefix, mask,
                                  w.sink, w.window, w.scale)
        assert_close(out.cpu().double().numpy(), ref, f"fp8 prefill chunk {C} after {prefix.tolist()}")
        prefix = prefix + C
    assert cache.status() == 0
    cache.close()


def test_fp8_prefill_rejects_value_scales_out_of_range():
    from head_wise_kv_b200 import _lib as L
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=1, layers=1, t0_range=None, t0=0, sink=16, window=64)
    ks, vs = _scales(w, 52)
    vs[0, 0] = 1000.0
    cache = _cache(w, 256, ks, vs)
    q, k, v = _chunk(w, np.zeros(1, np.int64), 128)
    dev = _dev()
    with pytest.raises(L.DuoError) as e:
        cache.prefill(0, q.to(dev), k.to(dev), v.to(dev), torch.zeros(1, dtype=torch.int32, device=dev), w.scale)
    assert e.value.code == L.DUO_ERR_UNSUPPORTED
    cache.close()
