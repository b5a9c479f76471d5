"""Paged retrieval caches through the C ABI against the fp64 oracle.

Retrieval keys and values live in a per-layer pool of fixed-size pages
(paged attention: fixed-size blocks that need not be contiguous); a device
table maps each sequence's positions to pages.  Paging changes where bytes
are stored, not what attention computes, so:

* every appended row sits, bit for bit, at (page of its position, offset) of
  the pool, with the pages handed out in a shuffled order;
* decode and chunked prefill equal the oracle on the sequence's history,
  for bf16 and FP8 caches, any split of the keys over CTAs, and the full
  128K GQA workload (sampled heads);
* a position whose page is missing sets DUO_STATUS_NO_PAGE.
"""
import numpy as np
import pytest
import torch

import duo_workloads as W
from _harness import History, assert_close, fill, new_token_inputs
from oracle import duo_oracle as O

pytestmark = pytest.mark.gpu

PAGE = 256


def _dev():
    return torch.device("cuda", 0)


def _paged(w, cap, kv_dtype="bf16", extra_pages=3, seed=0, ks=None, vs=None):
    """Cache + a page table that hands the pool's pages out in a shuffled
    order (pool = exactly the pages the batch needs, plus a few spare)."""
    from head_wise_kv_b200 import DuoKVCache
    per_seq = (cap + PAGE - 1) // PAGE
    n_pages = w.batch * per_seq + extra_pages
    cache = DuoKVCache(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, cap, W.retrieval_masks(w),
                       device=_dev(), kv_dtype=kv_dtype, k_scale=ks, v_scale=vs, page_tokens=PAGE,
                       num_pages=n_pages)
    perm = np.random.default_rng(seed).permutation(n_pages)[:w.batch * per_seq]
    table = torch.from_numpy(perm.reshape(w.batch, per_seq).astype(np.int32)).to(_dev())
    cache.set_page_table(table)
    return cache, table.cpu().numpy()


def _decode_step(cache, w, hist, lens0, kh=None, vh=None, pairs=None):
    dev = _dev()
    q, k, v = new_token_inputs(w, 0, lens0)
    cache.append(0, k.to(dev), v.to(dev), torch.from_numpy(lens0.astype(np.int32)).to(dev))
    lens = lens0 + 1
    out = cache.decode(0, q.to(dev), torch.from_numpy(lens.astype(np.int32)).to(dev), w.scale)
    kh = kh or (lambda b, g: hist.kv(0, b, g, W.TENSOR_K, int(lens[b])).float().numpy())
    vh = vh or (lambda b, g: hist.kv(0, b, g, W.TENSOR_V, int(lens[b])).float().numpy())
    ref, _ = O.decode_attention(q.double().numpy(), kh, vh, lens, W.retrieval_mask(w, 0), w.sink, w.window,
                                w.scale, pairs=pairs)
    got = out.cpu().double().numpy()
    if pairs is not None:
        got = np.stack([got[b, h] for b, h in pairs])
        ref = np.stack([ref[b, h] for b, h in pairs])
    return got, ref


def test_paged_rows_land_in_their_pages():
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=3, layers=1, t0_range=None, t0=0, sink=16, window=64)
    lens = np.array([700, 256, 513])
    cache, table = _paged(w, 800, seed=1)
    hist = History(w)
    fill(cache, hist, 0, lens, _dev(), slab=300)       # slabs that cross page boundaries
    torch.cuda.synchronize()
    assert cache.status() == 0
    views = cache.layer_views(0)
    mask = W.retrieval_mask(w, 0)
    for b in range(w.batch):
        for g in np.nonzero(mask)[0]:
            r = views["head_rank"][g]
            for kind, name in ((W.TENSOR_K, "k"), (W.TENSOR_V, "v")):
                x = hist.kv(0, b, int(g), kind, int(lens[b]))
                for p0 in range(0, int(lens[b]), PAGE):
                    n = min(PAGE, int(lens[b]) - p0)
                    page = int(table[b, p0 // PAGE])
                    got = views[f"{name}_retrieval"][page, r, :n].cpu()
                    assert torch.equal(got.view(torch.int16), x[p0:p0 + n].view(torch.int16)), \
                        f"b{b} g{g} {name} positions {p0}..{p0 + n}"
    cache.close()


@pytest.mark.parametrize("G", [1, 4, 8])
def test_paged_decode_matches_oracle(G):
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=3, layers=1, hq=4 * G, n_kv=4, t0_range=None, t0=0,
                 sink=16, window=64)
    lens0 = np.array([1500, 255, 600])
    cache, _ = _paged(w, 1600, seed=2)
    hist = History(w)
    fill(cache, hist, 0, lens0, _dev())
    got, ref = _decode_step(cache, w, hist, lens0)
    assert cache.status() == 0
    assert_close(got, ref, f"paged decode G={G}")
    cache.close()


@pytest.mark.parametrize("ctas", [3, 64, 300])
def test_paged_split_count_invariance(ctas):
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=2, layers=1, t0_range=None, t0=0, sink=16, window=64)
    lens0 = np.array([2000, 900])
    cache, _ = _paged(w, 2100, seed=3)
    cache.set_decode_ctas(ctas)
    hist = History(w)
    fill(cache, hist, 0, lens0, _dev())
    got, ref = _decode_step(cache, w, hist, lens0)
    assert cache.status() == 0
    assert_close(got, ref, f"paged decode over {ctas} CTAs")
    cache.close()


def test_paged_fp8_decode_matches_oracle():
    from test_gpu_fp8 import DequantHistory, _scales
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=3, layers=1, t0_range=None, t0=0, sink=16, window=64)
    ks, vs = _scales(w, 61)
    lens0 = np.array([1300, 257, 90])
    cache, _ = _paged(w, 1400, kv_dtype="fp8", seed=4, ks=ks, vs=vs)
    hist = History(w)
    fill(cache, hist, 0, lens0, _dev())
    dq = DequantHistory(hist, ks, vs)
    lens = lens0 + 1
    got, ref = _decode_step(cache, w, hist, lens0, kh=lambda b, g: dq.get(b, g, W.TENSOR_K, int(lens[b])),
                            vh=lambda b, g: dq.get(b, g, W.TENSOR_V, int(lens[b])))
    assert cache.status() == 0
    assert_close(got, ref, "paged fp8 decode")
    cache.close()


def test_missing_page_sets_status():
    from head_wise_kv_b200 import _lib as L
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=2, layers=1, t0_range=None, t0=0, sink=16, window=64)
    cache, table = _paged(w, 800, seed=5)
    t = torch.from_numpy(table.copy()).to(_dev())
    t[1, 1] = -1                                  # sequence 1, positions 256..511
    cache.set_page_table(t)
    hist = History(w)
    fill(cache, hist, 0, np.array([300, 400]), _dev())
    torch.cuda.synchronize()
    assert cache.status() & L.DUO_STATUS_NO_PAGE
    cache.close()


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
def test_paged_prefill_matches_oracle(kv_dtype):
    from test_gpu_fp8 import DequantHistory, _chunk, _scales
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=2, layers=1, t0_range=None, t0=0, sink=16, window=64)
    ks, vs = _scales(w, 71) if kv_dtype == "fp8" else (None, None)
    chunks = [300, 500, 129]
    cache, _ = _paged(w, sum(chunks), kv_dtype=kv_dtype, seed=6, ks=ks, vs=vs)
    hist = History(w)
    dq = DequantHistory(hist, ks, vs) if kv_dtype == "fp8" else None
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
                if dq is not None:
                    cached = dq.get(b, g, kind, P) if P else np.zeros((0, w.d))
                    own = hist.kv(0, b, g, kind, P + C)[P:].double().numpy()
                    return np.concatenate([cached, own])
                return hist.kv(0, b, g, kind, P + C).double().numpy()
            return f
        ref = O.prefill_attention(q.double().numpy(), hist_of(W.TENSOR_K), hist_of(W.TENSOR_V), prefix, mask,
                                  w.sink, w.window, w.scale)
        assert_close(out.cpu().double().numpy(), ref, f"paged {kv_dtype} prefill chunk {C}")
        prefix = prefix + C
    assert cache.status() == 0
    cache.close()


def test_paged_gqa128k_config_sampled():
    """The full 128K GQA workload in a paged cache (shuffled pages), one
    decode step; a seeded sample of (sequence, query head) pairs."""
    w = W.WORKLOADS["gqa128k"]
    lens0 = W.context_lengths(w)
    cache, _ = _paged(w, int(lens0.max()) + 1, seed=7)
    hist = History(w)
    fill(cache, hist, 0, lens0, _dev(), slab=16384)
    rng = np.random.default_rng(8)
    pairs = [(int(b), int(h)) for b, h in zip(rng.integers(0, w.batch, 12), rng.integers(0, w.hq, 12))]
    got, ref = _decode_step(cache, w, hist, lens0, pairs=pairs)
    assert cache.status() == 0
    assert_close(got, ref, "paged gqa128k sampled")
    cache.close()
