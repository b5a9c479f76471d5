"""Chunked prefill (tcgen05 tensor cores) through the C ABI against the fp64
oracle.  Row i of a chunk after P cached tokens sits at position P + i:
retrieval heads attend causally over everything, streaming heads over the
sinks and the window.  Bar: max-abs 2e-3, relative L2 1e-3 (fp32 output)."""
import numpy as np
import pytest
import torch

import duo_workloads as W
from _harness import History, assert_close, errors
from oracle import duo_oracle as O

pytestmark = pytest.mark.gpu


def _dev():
    return torch.device("cuda", 0)


def _mk(w, cap):
    from head_wise_kv_b200 import DuoKVCache
    return DuoKVCache(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, cap, W.retrieval_masks(w),
                      device=_dev())


def _chunk_kv(w, layer, prefix, C):
    k = torch.empty(w.batch, w.n_kv, C, w.d, dtype=torch.bfloat16)
    v = torch.empty_like(k)
    for b in range(w.batch):
        P = int(prefix[b])
        for g in range(w.n_kv):
            k[b, g] = W.tokens(w, layer, b, g, W.TENSOR_K, P, P + C)
            v[b, g] = W.tokens(w, layer, b, g, W.TENSOR_V, P, P + C)
    return k, v


def _chunk_q(w, layer, prefix, C):
    q = torch.empty(w.batch, w.hq, C, w.d, dtype=torch.bfloat16)
    for b in range(w.batch):
        P = int(prefix[b])
        for h in range(w.hq):
            q[b, h] = W.tokens(w, layer, b, h, W.TENSOR_Q, P, P + C)
    return q


def _oracle(hist, layer, q, prefix, C, mask, rows=None):
    w = hist.w

    def kh(b, g):
        return hist.kv(layer, b, g, W.TENSOR_K, int(prefix[b]) + C).float().numpy()

    def vh(b, g):
        return hist.kv(layer, b, g, W.TENSOR_V, int(prefix[b]) + C).float().numpy()
    return O.prefill_attention(q.double().numpy(), kh, vh, prefix, mask, w.sink, w.window, w.scale, rows=rows)


def _run_chunks(w, chunks, layer=0, rows=None, check=None, cache=None):
    """Prefill the given chunk sizes in order (attend, then append) and
    compare each checked chunk with the oracle.  Returns the outputs."""
    dev = _dev()
    total = sum(chunks)
    own = cache is None
    if own:
        cache = _mk(w, total)
    hist = History(w)
    mask = W.retrieval_mask(w, layer)
    prefix = np.zeros(w.batch, dtype=np.int64)
    outs = []
    for ci, C in enumerate(chunks):
        q = _chunk_q(w, layer, prefix, C)
        k, v = _chunk_kv(w, layer, prefix, C)
        pre = torch.from_numpy(prefix.astype(np.int32)).to(dev)
        out = cache.prefill(layer, q.to(dev), k.to(dev), v.to(dev), pre, w.scale)
        cache.append(layer, k.to(dev), v.to(dev), pre)
        got = out.cpu().double().numpy()
        outs.append(got)
        if check is None or ci in check:
            ref = _oracle(hist, layer, q, prefix, C, mask, rows=rows)
            if rows is not None:
                got, ref = got[:, :, rows], ref[:, :, rows]
            assert_close(got, ref, f"chunk {ci} (P={int(prefix[0])}, C={C})")
        prefix += C
    torch.cuda.synchronize()
    assert cache.status() == 0
    if own:
        cache.close()
    return outs


def _small(**kw):
    base = dict(batch=1, hq=8, n_kv=4, d=128, sink=16, window=64, retrieval_frac=0.5, t0_range=None, t0=0,
                steps=0, fixed_retrieval=(0, 2), rope=False, prompt=0, chunk=0)
    base.update(kw)
    return W.scaled(W.WORKLOADS["prefill64k"], **base)


def test_single_chunk_mixed_heads():
    _run_chunks(_small(), [128])


@pytest.mark.parametrize("chunks", [[200, 200, 200], [1, 127, 129, 300], [64, 700]])
def test_chunked_ragged_sizes(chunks):
    _run_chunks(_small(), chunks)


def test_all_retrieval_and_all_streaming():
    _run_chunks(_small(fixed_retrieval=(0, 1, 2, 3)), [300, 300])
    _run_chunks(_small(fixed_retrieval=()), [300, 300])


@pytest.mark.parametrize("S,Wn", [(0, 64), (4, 1), (130, 200), (16, 300)])
def test_streaming_window_shapes(S, Wn):
    _run_chunks(_small(sink=S, window=Wn), [150, 250, 260])


def test_gqa_group_sizes():
    for hq, n_kv, ret in [(4, 4, (1, 3)), (16, 2, (1,)), (32, 4, (0, 3))]:
        _run_chunks(_small(hq=hq, n_kv=n_kv, fixed_retrieval=ret), [256, 130])


def test_chunked_equals_one_shot_and_last_row_equals_decode():
    """Cached against uncached ("When Is Reuse Exact?"): the rows of a chunked
    prefill equal the same rows of a one-shot prefill, and the last row equals
    decode attention at that position."""
    w = _small()
    one = _run_chunks(w, [600], check=[])[0]
    parts = _run_chunks(w, [256, 100, 244], check=[])
    m, r = errors(np.concatenate(parts, axis=2), one)
    assert m < 2e-3 and r < 1e-3
    # decode at position 599 over the same cache
    dev = _dev()
    cache = _mk(w, 600)
    hist = History(w)
    k, v = _chunk_kv(w, 0, np.zeros(1, np.int64), 600)
    cache.append(0, k.to(dev), v.to(dev), torch.zeros(1, dtype=torch.int32, device=dev))
    q = W.decode_q(w, 0, np.array([600]))
    dec = cache.decode(0, q.to(dev), torch.tensor([600], dtype=torch.int32, device=dev), w.scale)
    m, r = errors(dec.cpu().numpy(), one[:, :, 599])
    assert m < 2e-3 and r < 1e-3
    cache.close()


def test_ragged_prefixes_in_one_batch():
    """Two sequences with different cached prefixes in one call."""
    w = _small(batch=2)
    dev = _dev()
    cache = _mk(w, 900)
    hist = History(w)
    mask = W.retrieval_mask(w, 0)
    first = np.array([300, 517])
    # one bulk append with per-sequence counts (the cached prefixes differ)
    k, v = _chunk_kv(w, 0, np.zeros(2, np.int64), int(first.max()))
    cache.append(0, k.to(dev), v.to(dev), torch.zeros(2, dtype=torch.int32, device=dev),
                 torch.from_numpy(first.astype(np.int32)).to(dev))
    C = 200
    q = _chunk_q(w, 0, first, C)
    k, v = _chunk_kv(w, 0, first, C)
    out = cache.prefill(0, q.to(dev), k.to(dev), v.to(dev), torch.from_numpy(first.astype(np.int32)).to(dev),
                        w.scale)
    ref = _oracle(hist, 0, q, first, C, mask)
    assert_close(out.cpu().double().numpy(), ref, "ragged prefixes")
    cache.close()


def test_prefill64k_first_and_last_chunks_sampled():
    """The 64K-token prompt in 16 chunks of 4096 (4 retrieval / 4 streaming
    KV heads, S=64, W=1024): rows sampled on the first and last chunks and on
    one middle chunk, every query head."""
    w = W.WORKLOADS["prefill64k"]
    rng = np.random.default_rng(5)
    rows = sorted(set(rng.choice(w.chunk, 48, replace=False).tolist()) | {0, 1, 127, 128, 1022, 1023, 1024,
                                                                          4095})
    _run_chunks(w, [w.chunk] * (w.prompt // w.chunk), rows=rows, check=[0, 7, 15])


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
def test_long_prefix_split_query_tiles(kv_dtype):
    """A 17,000-token prefix makes every retrieval query tile long enough to be
    shared by two CTAs (their halves merged by log-sum-exp); two sequences
    with different prefixes, a ragged chunk of 333 rows (a partial last query
    tile), retrieval and streaming heads."""
    from head_wise_kv_b200 import DuoKVCache
    w = _small(batch=2)
    dev = _dev()
    first = np.array([17000, 16390])
    C = 333
    ks = vs = None
    if kv_dtype == "fp8":
        rng = np.random.default_rng(9)
        ks = rng.uniform(0.5, 2.0, (w.layers, w.n_kv)).astype(np.float32)
        vs = rng.uniform(0.5, 2.0, (w.layers, w.n_kv)).astype(np.float32)
    cache = DuoKVCache(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, int(first.max()) + C,
                       W.retrieval_masks(w), device=dev, kv_dtype=kv_dtype, k_scale=ks, v_scale=vs)
    hist = History(w)
    mask = W.retrieval_mask(w, 0)
    k, v = _chunk_kv(w, 0, np.zeros(2, np.int64), int(first.max()))
    cache.append(0, k.to(dev), v.to(dev), torch.zeros(2, dtype=torch.int32, device=dev),
                 torch.from_numpy(first.astype(np.int32)).to(dev))
    q = _chunk_q(w, 0, first, C)
    k, v = _chunk_kv(w, 0, first, C)
    out = cache.prefill(0, q.to(dev), k.to(dev), v.to(dev), torch.from_numpy(first.astype(np.int32)).to(dev),
                        w.scale)

    def hist_of(kind):
        def f(b, g):
            P = int(first[b])
            x = hist.kv(0, b, g, kind, P + C).float().numpy()
            if kv_dtype == "fp8":
                s = float((ks if kind == W.TENSOR_K else vs)[0, g])
                x = np.concatenate([O.dequantize_kv(O.quantize_kv(x[:P], s), s), x[P:]])
            return x
        return f
    ref = O.prefill_attention(q.double().numpy(), hist_of(W.TENSOR_K), hist_of(W.TENSOR_V), first, mask,
                              w.sink, w.window, w.scale)
    assert_close(out.cpu().double().numpy(), ref, f"{kv_dtype} long prefix, split query tiles")
    assert cache.status() == 0
    cache.close()
