"""Append / evict through the C ABI: position tables and cache bytes must be
bit-identical to the oracle's literal per-token ring simulation."""
import numpy as np
import pytest
import torch

import duo_workloads as W
from oracle import duo_oracle as O

pytestmark = pytest.mark.gpu


def _dev():
    return torch.device("cuda", 0)


def _mk(w, cap):
    from head_wise_kv_b200 import DuoKVCache
    return DuoKVCache(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, cap,
                      W.retrieval_masks(w), device=_dev())


def _hist(w, layer, T):
    k = torch.stack([torch.stack([W.tokens(w, layer, b, g, W.TENSOR_K, 0, T) for g in range(w.n_kv)])
                     for b in range(w.batch)])
    v = torch.stack([torch.stack([W.tokens(w, layer, b, g, W.TENSOR_V, 0, T) for g in range(w.n_kv)])
                     for b in range(w.batch)])
    return k, v


def _check_layer(cache, w, layer, lens, k, v):
    """Every retrieval row and every streaming slot equals the oracle's ring
    content, bit for bit; positions equal the oracle's table."""
    views = cache.layer_views(layer)
    mask = W.retrieval_mask(w, layer)
    pos = views["positions"].cpu().numpy()
    kr, vr = views["k_retrieval"].cpu(), views["v_retrieval"].cpu()
    ks, vs = views["k_streaming"].cpu(), views["v_streaming"].cpu()
    for b in range(w.batch):
        T = int(lens[b])
        ring = O.StreamingCache(w.sink, w.window)
        for p in range(T):
            ring.append(p, p)
        assert np.array_equal(pos[b], ring.pos), f"positions b={b}"
        for g in range(w.n_kv):
            r = views["head_rank"][g]
            if mask[g]:
                assert torch.equal(kr[b, r, :T].view(torch.int16), k[b, g, :T].view(torch.int16))
                assert torch.equal(vr[b, r, :T].view(torch.int16), v[b, g, :T].view(torch.int16))
            else:
                held = [s for s in range(w.sink + w.window) if ring.pos[s] >= 0]
                src = torch.tensor([int(ring.items[s]) for s in held], dtype=torch.long)
                assert torch.equal(ks[b, r, held].view(torch.int16), k[b, g, src].view(torch.int16))
                assert torch.equal(vs[b, r, held].view(torch.int16), v[b, g, src].view(torch.int16))


@pytest.mark.parametrize("mode", ["one_by_one", "bulk", "ragged_slabs"])
def test_append_matches_ring_simulation(mode):
    w = W.scaled(W.WORKLOADS["tiny"], batch=3, t0=0)
    T = 200
    k, v = _hist(w, 0, T)
    cache = _mk(w, T)
    dev = _dev()
    if mode == "one_by_one":
        for p in range(T):
            cache.append(0, k[:, :, p:p + 1].contiguous().to(dev), v[:, :, p:p + 1].contiguous().to(dev),
                         torch.full((w.batch,), p, dtype=torch.int32, device=dev))
        lens = [T] * w.batch
    elif mode == "bulk":
        cache.append(0, k.to(dev), v.to(dev), torch.zeros(w.batch, dtype=torch.int32, device=dev))
        lens = [T] * w.batch
    else:
        lens = [T, 77, 5]
        done = np.zeros(w.batch, dtype=np.int64)
        for n in [3, 50, 1, 90, 56]:
            cnt = np.clip(np.array(lens) - done, 0, n).astype(np.int32)
            kk = torch.zeros(w.batch, w.n_kv, n, w.d, dtype=torch.bfloat16)
            vv = torch.zeros_like(kk)
            for b in range(w.batch):
                kk[b, :, :cnt[b]] = k[b, :, done[b]:done[b] + cnt[b]]
                vv[b, :, :cnt[b]] = v[b, :, done[b]:done[b] + cnt[b]]
            cache.append(0, kk.to(dev), vv.to(dev), torch.from_numpy(done.astype(np.int32)).to(dev),
                         torch.from_numpy(cnt).to(dev))
            done += cnt
        assert list(done) == lens
    torch.cuda.synchronize()
    assert cache.status() == 0
    _check_layer(cache, w, 0, lens, k, v)


def test_append_restart_resets_positions():
    """A sequence that starts over (len_before = 0) keeps no stale positions."""
    w = W.scaled(W.WORKLOADS["tiny"], batch=2, t0=0)
    k, v = _hist(w, 0, 150)
    cache = _mk(w, 150)
    dev = _dev()
    zero = torch.zeros(w.batch, dtype=torch.int32, device=dev)
    cache.append(0, k.to(dev), v.to(dev), zero)
    cache.append(0, k[:, :, :30].contiguous().to(dev), v[:, :, :30].contiguous().to(dev), zero)
    torch.cuda.synchronize()
    _check_layer(cache, w, 0, [30, 30], k, v)


def test_append_over_capacity_sets_status():
    w = W.scaled(W.WORKLOADS["tiny"], batch=1, t0=0)
    k, v = _hist(w, 0, 40)
    cache = _mk(w, 32)
    dev = _dev()
    cache.append(0, k.to(dev), v.to(dev), torch.zeros(1, dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    from head_wise_kv_b200 import _lib
    assert cache.status() & _lib.DUO_STATUS_OVER_CAPACITY
    assert cache.status() == 0   # cleared by the previous read


@pytest.mark.parametrize("S,Wn", [(0, 1), (0, 7), (5, 1), (16, 64), (3, 300)])
def test_append_window_shapes(S, Wn):
    w = W.scaled(W.WORKLOADS["tiny"], batch=2, t0=0, sink=S, window=Wn, d=128)
    T = 257
    k, v = _hist(w, 0, T)
    cache = _mk(w, T)
    dev = _dev()
    cache.append(0, k[:, :, :100].contiguous().to(dev), v[:, :, :100].contiguous().to(dev),
                 torch.zeros(w.batch, dtype=torch.int32, device=dev))
    for p in range(100, T):
        cache.append(0, k[:, :, p:p + 1].contiguous().to(dev), v[:, :, p:p + 1].contiguous().to(dev),
                     torch.full((w.batch,), p, dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    _check_layer(cache, w, 0, [T, T], k, v)
