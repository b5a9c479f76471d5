"""INT4 caches through the C ABI against the fp64 oracle.

* the cached bytes are the oracle's packed codes of value / scale, bit for
  bit (retrieval rows and ring slots);
* decode equals attention over the dequantised history (scale * code), the
  new token included, for every GQA group size, ragged lengths that cross
  the 256-key tiles, any split of the keys over CTAs, saturating scales,
  paged pools, and the full 128K GQA workload (sampled heads) at the launch
  configuration the benchmark uses;
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


def _scales(w, seed, lo=0.3, hi=1.0):
    rng = np.random.default_rng(seed)
    return (rng.uniform(lo, hi, (w.layers, w.n_kv)).astype(np.float32),
            rng.uniform(lo, hi, (w.layers, w.n_kv)).astype(np.float32))


def _cache(w, cap, ks, vs, **kw):
    from head_wise_kv_b200 import DuoKVCache
    return DuoKVCache(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, cap, W.retrieval_masks(w),
                      device=_dev(), kv_dtype="int4", k_scale=ks, v_scale=vs, **kw)


class DequantHistory:
    """Dequantised K/V streams: scale * INT4 code of value / scale."""

    def __init__(self, hist: History, ks, vs, layer=0):
        self.h, self.ks, self.vs, self.layer = hist, ks, vs, layer
        self._c = {}

    def get(self, b, g, kind, n):
        key = (b, g, kind)
        have = self._c.get(key)
        if have is None or have.shape[0] < n:
            x = self.h.kv(self.layer, b, g, kind, n).float().numpy()
            s = float((self.ks if kind == W.TENSOR_K else self.vs)[self.layer, g])
            self._c[key] = O.dequantize_kv_int4(O.quantize_kv_int4(x, s), s)
        return self._c[key][:n]


def _decode_step(cache, w, hist, lens0, ks, vs, pairs=None):
    dev = _dev()
    q, k, v = new_token_inputs(w, 0, lens0)
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


def test_int4_codes_bit_exact():
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=2, layers=1, t0_range=None, t0=700, sink=16, window=64)
    ks, vs = _scales(w, 5)
    dev = _dev()
    T0 = np.array([700, 513])
    cache = _cache(w, 720, ks, vs)
    hist = History(w)
    fill(cache, hist, 0, T0, dev)
    for s in range(3):
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
                packed = O.quantize_kv_int4(x, float(sc[0, g]))
                if mask[g]:
                    got = views[f"{name}_retrieval"][b, r, :T[b]].cpu().numpy()
                    assert np.array_equal(got, packed), f"b{b} g{g} {name} retrieval codes"
                else:
                    got = views[f"{name}_streaming"][b, r].cpu().numpy()
                    filled = pos >= 0
                    assert np.array_equal(got[filled], packed[pos[filled]]), f"b{b} g{g} {name} ring codes"
    cache.close()


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_int4_decode_matches_oracle(G):
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=3, layers=1, hq=4 * G, n_kv=4, t0_range=None, t0=0,
                 sink=16, window=64)
    ks, vs = _scales(w, 6 + G)
    lens0 = np.array([900, 255, 70])
    cache = _cache(w, 1000, ks, vs)
    hist = History(w)
    fill(cache, hist, 0, lens0, _dev())
    got, ref = _decode_step(cache, w, hist, lens0, ks, vs)
    assert cache.status() == 0
    assert_close(got, ref, f"int4 decode G={G}")
    cache.close()


@pytest.mark.parametrize("ctas", [5, 37, 300])
def test_int4_split_count_invariance(ctas):
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=2, layers=1, t0_range=None, t0=0, sink=16, window=64)
    ks, vs = _scales(w, 21)
    lens0 = np.array([1500, 777])
    cache = _cache(w, 1600, ks, vs)
    cache.set_decode_ctas(ctas)
    hist = History(w)
    fill(cache, hist, 0, lens0, _dev())
    got, ref = _decode_step(cache, w, hist, lens0, ks, vs)
    assert cache.status() == 0
    assert_close(got, ref, f"int4 decode over {ctas} CTAs")
    cache.close()


@pytest.mark.parametrize("scale_lo,scale_hi", [(0.02, 0.05), (3.0, 8.0)])
def test_int4_saturating_and_coarse_scales(scale_lo, scale_hi):
    """Small scales clamp most codes to -8 / 7; large ones leave most at 0."""
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=2, layers=1, t0_range=None, t0=0, sink=16, window=64)
    ks, vs = _scales(w, 31, scale_lo, scale_hi)
    lens0 = np.array([600, 333])
    cache = _cache(w, 700, ks, vs)
    hist = History(w)
    fill(cache, hist, 0, lens0, _dev())
    got, ref = _decode_step(cache, w, hist, lens0, ks, vs)
    assert_close(got, ref, f"int4 scales [{scale_lo}, {scale_hi}]")
    cache.close()


def test_int4_paged_decode_matches_oracle():
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=3, layers=1, t0_range=None, t0=0, sink=16, window=64)
    ks, vs = _scales(w, 61)
    lens0 = np.array([1300, 257, 90])
    page = 256
    per_seq = (1400 + page - 1) // page
    n_pages = w.batch * per_seq + 3
    cache = _cache(w, 1400, ks, vs, page_tokens=page, num_pages=n_pages)
    perm = np.random.default_rng(4).permutation(n_pages)[:w.batch * per_seq]
    cache.set_page_table(torch.from_numpy(perm.reshape(w.batch, per_seq).astype(np.int32)).to(_dev()))
    hist = History(w)
    fill(cache, hist, 0, lens0, _dev())
    got, ref = _decode_step(cache, w, hist, lens0, ks, vs)
    assert cache.status() == 0
    assert_close(got, ref, "paged int4 decode")
    cache.close()


def test_int4_gqa128k_config_sampled():
    """The full 128K GQA workload in an INT4 cache, one decode step at the
    launch configuration the benchmark times; a seeded sample of (sequence,
    query head) pairs against the oracle."""
    w = W.WORKLOADS["gqa128k"]
    ks, vs = _scales(w, 41, 0.4, 0.8)
    lens0 = W.context_lengths(w)
    cache = _cache(w, int(lens0.max()) + 1, ks, vs)
    hist = History(w)
    fill(cache, hist, 0, lens0, _dev(), slab=16384)
    rng = np.random.default_rng(3)
    pairs = [(int(b), int(h)) for b, h in zip(rng.integers(0, w.batch, 12), rng.integers(0, w.hq, 12))]
    got, ref = _decode_step(cache, w, hist, lens0, ks, vs, pairs=pairs)
    assert cache.status() == 0
    assert_close(got, ref, "int4 gqa128k sampled")
    cache.close()


@pytest.mark.parametrize("chunks,S,Wn", [([300, 700, 129], 16, 64), ([256, 384], 64, 1024)])
def test_int4_prefill_matches_oracle(chunks, S, Wn):
    """Chunked prefill on an INT4 cache: each chunk attends to the cached
    prefix dequantised and to its own keys and values as given."""
    from test_gpu_fp8 import _chunk
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=2, layers=1, t0_range=None, t0=0, sink=S, window=Wn)
    ks, vs = _scales(w, 71)
    cache = _cache(w, sum(chunks), ks, vs)
    hist = History(w)
    dq = DequantHistory(hist, ks, vs)
    mask = W.retrieval_mask(w, 0)
    dev = _dev()
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
        assert_close(out.cpu().double().numpy(), ref, f"int4 prefill chunk {C}")
        prefix = prefix + C
    assert cache.status() == 0
    cache.close()


def test_int4_fork_copies_codes():
    """Prefix sharing on an INT4 cache (64-byte rows): the fork's decode
    equals the oracle on the shared prefix + its own tokens."""
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=2, layers=1, t0_range=None, t0=0, sink=16, window=64)
    ks, vs = _scales(w, 91)
    L = 500
    cache = _cache(w, 800, ks, vs)
    hist = History(w)
    fill(cache, hist, 0, np.array([L, 0]), _dev())
    cache.fork(0, 1, L)
    dev = _dev()
    q, k, v = new_token_inputs(w, 0, np.array([L, L]))
    k[1] = k[0]
    v[1] = v[0]                                   # both sequences append the same token
    cache.append(0, k.to(dev), v.to(dev), torch.full((2,), L, dtype=torch.int32, device=dev))
    lens = np.array([L + 1, L + 1])
    out = cache.decode(0, q.to(dev), torch.from_numpy(lens.astype(np.int32)).to(dev), w.scale)
    dq = DequantHistory(hist, ks, vs)
    ref, _ = O.decode_attention(q.double().numpy(), lambda b, g: dq.get(0, g, W.TENSOR_K, L + 1),
                                lambda b, g: dq.get(0, g, W.TENSOR_V, L + 1), lens, W.retrieval_mask(w, 0),
                                w.sink, w.window, w.scale)
    assert_close(out.cpu().double().numpy(), ref, "int4 fork")
    assert cache.status() == 0
    cache.close()
