"""Row-range decode, log-sum-exp merge and the gated (alpha-blended) forward
through the C ABI, against the fp64 oracle.

* Sequence split: R caches (one per device in a real deployment; here R
  independent caches on one GPU, none waiting on another) each hold a slice
  of every sequence's retrieval history; their partial (out, lse) merge to the
  single-device result.
* Gated forward: on a cache whose heads all keep full history, the streaming
  attention is two row ranges (sinks, recent window) merged, then blended
  with full attention per query head.
Both on bf16, FP8 and INT4 caches (the oracle reads the dequantised history).
"""
import numpy as np
import pytest
import torch

import duo_workloads as W
from _harness import History, assert_close
from oracle import duo_oracle as O

pytestmark = pytest.mark.gpu


def _dev():
    return torch.device("cuda", 0)


SCALES = {"bf16": None, "fp8": 0.25, "int4": 0.5}   # one K and V scale for every head


def _cache(w, cap, mask, kv_dtype="bf16"):
    from head_wise_kv_b200 import DuoKVCache
    sc = SCALES[kv_dtype]
    sc = None if sc is None else np.full((1, w.n_kv), sc, np.float32)
    return DuoKVCache(1, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, cap, mask[None], device=_dev(),
                      kv_dtype=kv_dtype, k_scale=sc, v_scale=sc)


def _history(w, T):
    k = torch.zeros(w.batch, w.n_kv, T, w.d, dtype=torch.bfloat16)
    v = torch.zeros_like(k)
    return k, v


def _fill_rows(cache, w, lens, lo, hi, dev):
    """Append tokens 0..lens[b]-1 of every sequence (one bulk call with
    per-sequence counts); retrieval rows keep positions [lo[b], hi[b])."""
    T = int(max(lens))
    k = torch.zeros(w.batch, w.n_kv, T, w.d, dtype=torch.bfloat16)
    v = torch.zeros_like(k)
    for b in range(w.batch):
        for g in range(w.n_kv):
            k[b, g, :lens[b]] = W.tokens(w, 0, b, g, W.TENSOR_K, 0, int(lens[b]))
            v[b, g, :lens[b]] = W.tokens(w, 0, b, g, W.TENSOR_V, 0, int(lens[b]))
    i32 = lambda a: torch.tensor(np.asarray(a, dtype=np.int32), device=dev)
    cache.append_rows(0, k.to(dev), v.to(dev), i32([0] * w.batch), i32(lo), i32(hi), n_new=i32(lens))


def _oracle_full(w, q, lens, mask, kv_dtype="bf16"):
    hist = History(w)
    sc = SCALES[kv_dtype]

    def read(x):
        if kv_dtype == "fp8":
            return O.dequantize_kv(O.quantize_kv(x, sc), sc)
        if kv_dtype == "int4":
            return O.dequantize_kv_int4(O.quantize_kv_int4(x, sc), sc)
        return x

    def kh(b, g):
        return read(hist.kv(0, b, g, W.TENSOR_K, int(lens[b])).float().numpy())

    def vh(b, g):
        return read(hist.kv(0, b, g, W.TENSOR_V, int(lens[b])).float().numpy())
    return kh, vh


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8", "int4"])
@pytest.mark.parametrize("R,cap", [(2, 1600), (3, 1100), (4, 1024)])
def test_sequence_split_decode_merges_to_full_result(R, cap, kv_dtype):
    from head_wise_kv_b200 import seqsplit
    from head_wise_kv_b200.cache import lse_merge
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=2, t0_range=None, t0=0, sink=16, window=64)
    dev = _dev()
    mask = W.retrieval_mask(w, 0)
    lens = np.array([2900, 1301])            # after this step's append
    caches = [_cache(w, cap, mask, kv_dtype) for _ in range(R)]
    for r, c in enumerate(caches):
        lo, hi = seqsplit.slice_bounds(cap, r)
        _fill_rows(c, w, lens, [lo] * w.batch, [hi] * w.batch, dev)
    q = W.decode_q(w, 0, lens)
    L = torch.from_numpy(lens.astype(np.int32)).to(dev)
    outs, lses = [], []
    for r, c in enumerate(caches):
        rows = seqsplit.local_rows(L, cap, r)
        s_len = L if r == R - 1 else torch.zeros_like(L)
        o, l = c.decode_rows(0, q.to(dev), rows, w.scale, s_len=s_len)
        outs.append(o)
        lses.append(l)
    out, lse = lse_merge(torch.stack(outs), torch.stack(lses))
    kh, vh = _oracle_full(w, q, lens, mask, kv_dtype)
    ref, ref_lse = O.decode_attention(q.double().numpy(), kh, vh, lens, mask, w.sink, w.window, w.scale)
    assert_close(out.cpu().double().numpy(), ref, f"{kv_dtype} split over {R}")
    assert np.abs(lse.cpu().double().numpy() - ref_lse).max() < 1e-3
    for c in caches:
        assert c.status() == 0
        c.close()


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8", "int4"])
@pytest.mark.parametrize("lens", [[700, 90], [79, 12], [5, 300]])
def test_gated_forward_matches_oracle(lens, kv_dtype):
    from head_wise_kv_b200.cache import alpha_blend, lse_merge
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=2, hq=8, n_kv=4, t0_range=None, t0=0, sink=16, window=64)
    dev = _dev()
    lens = np.array(lens)
    full_mask = np.ones(w.n_kv, np.uint8)         # identification keeps every head's full history
    cache = _cache(w, int(lens.max()), full_mask, kv_dtype)
    _fill_rows(cache, w, lens, [0] * w.batch, [1 << 30] * w.batch, dev)
    q = W.decode_q(w, 0, lens).to(dev)
    L = torch.from_numpy(lens.astype(np.int32)).to(dev)
    full = cache.decode(0, q, L, w.scale)
    S, Wn = w.sink, w.window
    sink_end = torch.clamp(L, max=S)
    win_begin = torch.clamp(L - Wn, min=S)
    o_s, l_s = cache.decode_rows(0, q, sink_end, w.scale)
    o_w, l_w = cache.decode_rows(0, q, L, w.scale, r_begin=win_begin)
    strm, _ = lse_merge(torch.stack([o_s, o_w]), torch.stack([l_s, l_w]))
    alpha = torch.from_numpy(np.random.default_rng(3).uniform(0, 1, w.hq).astype(np.float32)).to(dev)
    out = alpha_blend(alpha, full, strm)
    kh, vh = _oracle_full(w, q.cpu(), lens, full_mask, kv_dtype)
    ref = O.blended_decode(q.cpu().double().numpy(), kh, vh, lens, w.n_kv, alpha.cpu().double().numpy(), S, Wn,
                           w.scale)
    assert_close(out.cpu().double().numpy(), ref, f"{kv_dtype} gated forward")
    cache.close()


def test_lse_merge_ignores_empty_parts():
    from head_wise_kv_b200.cache import lse_merge
    dev = _dev()
    rng = np.random.default_rng(4)
    o = torch.from_numpy(rng.standard_normal((3, 5, 64)).astype(np.float32)).to(dev)
    l = torch.from_numpy(rng.standard_normal((3, 5)).astype(np.float32)).to(dev)
    l[1] = float("-inf")
    o[1] = float("nan")                            # an empty part's output is never read
    l[:, 4] = float("-inf")                        # a row no part saw
    out, lse = lse_merge(o, l)
    ll = l.cpu().double().numpy()
    oo = o.cpu().double().numpy()
    for row in range(4):
        wts = np.exp(ll[[0, 2], row] - np.logaddexp(ll[0, row], ll[2, row]))
        np.testing.assert_allclose(out[row].cpu().numpy(), wts[0] * oo[0, row] + wts[1] * oo[2, row], rtol=1e-5,
                                   atol=1e-6)
    assert torch.all(out[4] == 0) and lse[4].item() == float("-inf")


class _ThreadAllGather:
    """All-gather among R host threads of one process: a stand-in for the
    NCCL all-gather of gather_partials when the R ranks' caches share one
    GPU.  Kernels never wait on one another: the threads meet on the host
    after each has enqueued its own decode."""

    def __init__(self, world):
        import threading
        self.world = world
        self.slots = [None] * world
        self.barrier = threading.Barrier(world, timeout=120)

    def __call__(self, out, lse, rank):
        self.slots[rank] = (out, lse)
        self.barrier.wait()
        parts = (torch.stack([s[0] for s in self.slots]), torch.stack([s[1] for s in self.slots]))
        self.barrier.wait()
        return parts


@pytest.mark.parametrize("R,cap", [(2, 1600), (3, 1100), (4, 1024)])
def test_split_decode_step_on_every_rank(R, cap):
    """seqsplit.split_decode_step as R ranks call it (one host thread per
    rank, each with its own cache holding its slice): the rank-dependent row
    ranges (only the last rank reads the streaming rings), the exchange and
    the merge give every rank the oracle's result."""
    import threading
    from head_wise_kv_b200 import seqsplit
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=3, t0_range=None, t0=0, sink=16, window=64)
    dev = _dev()
    mask = W.retrieval_mask(w, 0)
    lens = np.array([2900, 1301, 40])        # the last sequence: fewer tokens than the ring holds
    lens = np.minimum(lens, R * cap)
    caches = [_cache(w, cap, mask) for _ in range(R)]
    for r, c in enumerate(caches):
        lo, hi = seqsplit.slice_bounds(cap, r)
        _fill_rows(c, w, lens, [lo] * w.batch, [hi] * w.batch, dev)
    q = W.decode_q(w, 0, lens).to(dev)
    L = torch.from_numpy(lens.astype(np.int32)).to(dev)
    torch.cuda.synchronize()
    gather = _ThreadAllGather(R)
    results, errors_ = [None] * R, []

    def rank_main(r):
        try:
            torch.cuda.set_device(dev)
            results[r] = seqsplit.split_decode_step(caches[r], 0, q, L, w.scale, cap, r, R, group=r,
                                                    gather=gather)
        except Exception as e:                 # reported below
            errors_.append(e)
            gather.barrier.abort()
    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(R)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors_, errors_
    torch.cuda.synchronize()
    kh, vh = _oracle_full(w, q.cpu(), lens, mask)
    ref, ref_lse = O.decode_attention(q.cpu().double().numpy(), kh, vh, lens, mask, w.sink, w.window, w.scale)
    for r, (out, lse) in enumerate(results):
        assert_close(out.cpu().double().numpy(), ref, f"rank {r} of {R}")
        assert np.abs(lse.cpu().double().numpy() - ref_lse).max() < 1e-3
        assert torch.equal(out, results[0][0]) and torch.equal(lse, results[0][1])
    for c in caches:
        assert c.status() == 0
        c.close()
