"""Prefix sharing (duo_kv_fork) through the C ABI against the fp64 oracle.

After a fork, sequence dst holds sequence src's first L tokens and goes on
with its own; attention must equal the oracle on exactly that history
(shared prefix + own continuation), for both sequences, whichever pages are
shared ("Attention Variants and Memory Efficiency", "What the Inference
Runtime Can Change": paged blocks, prefix sharing).  Checked:

* paged caches: full prefix pages shared (same pool page in both tables),
  the partly filled last page copied, later pages private; the shared pages
  keep src's rows bit for bit after both sequences append;
* contiguous bf16 and FP8 caches (a wrapped streaming ring is copied);
* a chunked prefill continuing a forked sequence;
* status bits for a shared partial page and for a wrong prefix length.
"""
import numpy as np
import pytest
import torch

import duo_workloads as W
from _harness import assert_close, fill, History
from oracle import duo_oracle as O

pytestmark = pytest.mark.gpu

PAGE = 256


def _dev():
    return torch.device("cuda", 0)


def _w():
    # batch 2: sequence 0 is the source, sequence 1 the fork
    return W.scaled(W.WORKLOADS["gqa128k"], batch=2, layers=1, t0_range=None, t0=0, sink=16, window=64)


class ForkHistory:
    """Token streams of the two sequences: dst = src's first L tokens, then
    its own stream from position L."""

    def __init__(self, w, L):
        self.w, self.L = w, L

    def rows(self, b, g, kind, p0, p1):
        w, L = self.w, self.L
        if b == 0 or p1 <= L:
            return W.tokens(w, 0, 0, g, kind, p0, p1)
        if p0 >= L:
            return W.tokens(w, 0, 1, g, kind, p0, p1)
        return torch.cat([W.tokens(w, 0, 0, g, kind, p0, L), W.tokens(w, 0, 1, g, kind, L, p1)])

    def f64(self, b, g, kind, n):
        return self.rows(b, g, kind, 0, n).double().numpy()


def _append(cache, fh, p0, n):
    """Append positions p0 .. p0+n-1 of both sequences' streams."""
    w = fh.w
    k = torch.empty(w.batch, w.n_kv, n, w.d, dtype=torch.bfloat16)
    v = torch.empty_like(k)
    for b in range(w.batch):
        for g in range(w.n_kv):
            k[b, g] = fh.rows(b, g, W.TENSOR_K, p0, p0 + n)
            v[b, g] = fh.rows(b, g, W.TENSOR_V, p0, p0 + n)
    dev = _dev()
    cache.append(0, k.to(dev), v.to(dev), torch.full((w.batch,), p0, dtype=torch.int32, device=dev))


def _decode_vs_oracle(cache, fh, T, kh=None, vh=None, what=""):
    w = fh.w
    lens = np.full(w.batch, T)
    q = W.decode_q(w, 0, lens)
    out = cache.decode(0, q.to(_dev()), torch.from_numpy(lens.astype(np.int32)).to(_dev()), w.scale)
    kh = kh or (lambda b, g: fh.f64(b, g, W.TENSOR_K, T))
    vh = vh or (lambda b, g: fh.f64(b, g, W.TENSOR_V, T))
    ref, _ = O.decode_attention(q.double().numpy(), kh, vh, lens, W.retrieval_mask(w, 0), w.sink, w.window,
                                w.scale)
    assert_close(out.cpu().double().numpy(), ref, what)


def _fill_src(cache, w, L):
    fill(cache, History(w), 0, np.array([L, 0]), _dev())


def _paged_cache(w, cap, table_rows, n_pages):
    from head_wise_kv_b200 import DuoKVCache
    cache = DuoKVCache(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, cap, W.retrieval_masks(w),
                       device=_dev(), page_tokens=PAGE, num_pages=n_pages)
    table = torch.tensor(table_rows, dtype=torch.int32, device=_dev())
    cache.set_page_table(table)
    return cache


def test_fork_paged_shares_full_pages():
    w = _w()
    L, n = 700, 300                                   # pages 0, 1 full; page 2 partial
    # src pages 5, 2, 7, 0; the fork shares 5 and 2, gets 4 for the partial page, 1 for the next
    cache = _paged_cache(w, 1100, [[5, 2, 7, 0, 3], [5, 2, 4, 1, 6]], 8)
    fh = ForkHistory(w, L)
    _fill_src(cache, w, L)
    cache.fork(0, 1, L)
    assert cache.status() == 0
    _append(cache, fh, L, n)
    _decode_vs_oracle(cache, fh, L + n, what="paged fork")
    assert cache.status() == 0
    # the shared pages still hold src's rows exactly
    views = cache.layer_views(0)
    mask = W.retrieval_mask(w, 0)
    for g in np.nonzero(mask)[0]:
        r = views["head_rank"][g]
        for page, p0 in ((5, 0), (2, PAGE)):
            want = W.tokens(w, 0, 0, int(g), W.TENSOR_K, p0, p0 + PAGE)
            got = views["k_retrieval"][page, r].cpu()
            assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    cache.close()


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
def test_fork_contiguous(kv_dtype):
    from head_wise_kv_b200 import DuoKVCache
    from test_gpu_fp8 import _scales
    w = _w()
    L, n = 1000, 200                                  # L > S + W: the ring has wrapped
    ks, vs = _scales(w, 81) if kv_dtype == "fp8" else (None, None)
    cache = DuoKVCache(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, 1300, W.retrieval_masks(w),
                       device=_dev(), kv_dtype=kv_dtype, k_scale=ks, v_scale=vs)
    fh = ForkHistory(w, L)
    _fill_src(cache, w, L)
    cache.fork(0, 1, L)
    _append(cache, fh, L, n)
    kh = vh = None
    if kv_dtype == "fp8":
        def deq(kind):
            def f(b, g):
                s = float((ks if kind == W.TENSOR_K else vs)[0, g])
                return O.dequantize_kv(O.quantize_kv(fh.rows(b, g, kind, 0, L + n).float().numpy(), s), s)
            return f
        kh, vh = deq(W.TENSOR_K), deq(W.TENSOR_V)
    _decode_vs_oracle(cache, fh, L + n, kh, vh, what=f"{kv_dtype} contiguous fork")
    assert cache.status() == 0
    cache.close()


def test_fork_then_prefill():
    """A chunked prefill on both sequences after the fork: dst's chunk
    attends to the shared prefix plus its own chunk."""
    w = _w()
    L, C = 600, 333
    cache = _paged_cache(w, 1000, [[3, 0, 6, 2], [3, 0, 5, 1]], 7)
    fh = ForkHistory(w, L)
    _fill_src(cache, w, L)
    cache.fork(0, 1, L)
    dev = _dev()
    q = torch.empty(w.batch, w.hq, C, w.d, dtype=torch.bfloat16)
    k = torch.empty(w.batch, w.n_kv, C, w.d, dtype=torch.bfloat16)
    v = torch.empty_like(k)
    for b in range(w.batch):
        for h in range(w.hq):
            q[b, h] = W.tokens(w, 0, b, h, W.TENSOR_Q, L, L + C)
        for g in range(w.n_kv):
            k[b, g] = fh.rows(b, g, W.TENSOR_K, L, L + C)
            v[b, g] = fh.rows(b, g, W.TENSOR_V, L, L + C)
    prefix = np.full(w.batch, L)
    pre = torch.from_numpy(prefix.astype(np.int32)).to(dev)
    out = cache.prefill(0, q.to(dev), k.to(dev), v.to(dev), pre, w.scale)
    ref = O.prefill_attention(q.double().numpy(), lambda b, g: fh.f64(b, g, W.TENSOR_K, L + C),
                              lambda b, g: fh.f64(b, g, W.TENSOR_V, L + C), prefix, W.retrieval_mask(w, 0),
                              w.sink, w.window, w.scale)
    assert_close(out.cpu().double().numpy(), ref, "prefill after fork")
    assert cache.status() == 0
    cache.close()


def test_fork_shared_partial_page_sets_status():
    from head_wise_kv_b200 import _lib as L_
    w = _w()
    cache = _paged_cache(w, 800, [[1, 2, 3], [1, 2, 0]], 4)
    _fill_src(cache, w, 300)                          # page 1 (positions 256..299) partly filled
    cache.fork(0, 1, 300)
    assert cache.status() & L_.DUO_STATUS_SHARED_PAGE
    cache.close()


def test_fork_wrong_length_sets_status():
    from head_wise_kv_b200 import _lib as L_
    w = _w()
    cache = _paged_cache(w, 800, [[1, 2, 3], [1, 0, 3]], 4)
    _fill_src(cache, w, 300)
    cache.fork(0, 1, 299)                             # src holds 300 tokens
    assert cache.status() & L_.DUO_STATUS_BAD_LENGTH
    cache.close()
