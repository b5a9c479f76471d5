"""Decode attention through the C ABI against the fp64 oracle.

Bar (bf16 inputs, fp32 accumulation, fp32 output): max-abs error <= 2e-3 and
relative L2 error <= 1e-3 over the compared outputs; lse to 1e-3 absolute.
"""
import numpy as np
import pytest
import torch

import duo_workloads as W
from _harness import History, assert_close, errors, fill, new_token_inputs, oracle_decode

pytestmark = pytest.mark.gpu


def _dev():
    return torch.device("cuda", 0)


def _mk(w, cap):
    from head_wise_kv_b200 import DuoKVCache
    return DuoKVCache(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, cap,
                      W.retrieval_masks(w), device=_dev())


def _run_steps(w, steps, lens0=None, ctas=None, layer=0, pairs=None, check_every=1):
    """Fill, then `steps` decode steps (append + attend), each compared with
    the oracle.  Returns the worst (max-abs, rel-L2)."""
    dev = _dev()
    lens0 = W.context_lengths(w) if lens0 is None else np.asarray(lens0, dtype=np.int64)
    cache = _mk(w, int(lens0.max()) + steps)
    if ctas is not None:
        cache.set_decode_ctas(ctas)
    cache._ws.fill_(0xFF)   # NaN canary: a read of an unwritten workspace slot fails parity
    hist = History(w)
    fill(cache, hist, layer, lens0, dev)
    mask = W.retrieval_mask(w, layer)
    worst = (0.0, 0.0)
    for s in range(steps):
        lens_b = lens0 + s
        q, k, v = new_token_inputs(w, layer, lens_b)
        cache.append(layer, k.to(dev), v.to(dev), torch.from_numpy(lens_b.astype(np.int32)).to(dev))
        lens_a = torch.from_numpy((lens_b + 1).astype(np.int32)).to(dev)
        out, lse = cache.decode(layer, q.to(dev), lens_a, w.scale, want_lse=True)
        if s % check_every and s != steps - 1:
            continue
        ref, ref_lse = oracle_decode(hist, layer, q, lens_b + 1, mask, pairs=pairs)
        got, got_lse = out.cpu().double().numpy(), lse.cpu().double().numpy()
        if pairs is not None:
            idx = tuple(np.array(pairs).T)
            got, ref, got_lse, ref_lse = got[idx], ref[idx], got_lse[idx], ref_lse[idx]
        e = assert_close(got, ref, f"step {s}")
        assert np.abs(got_lse - ref_lse).max() < 1e-3, f"lse step {s}"
        worst = (max(worst[0], e[0]), max(worst[1], e[1]))
    torch.cuda.synchronize()
    assert cache.status() == 0
    cache.close()
    return worst


def test_tiny_config_all_steps():
    """Tiny: MHA 4 heads, d=64, T0=512, 16 steps, heads {0,2} retrieval, S=16, W=64."""
    _run_steps(W.WORKLOADS["tiny"], 16)


@pytest.mark.parametrize("d,G", [(64, 1), (64, 2), (64, 4), (64, 8), (128, 1), (128, 2), (128, 4), (128, 8)])
def test_shapes_ragged(d, G):
    n_kv = 4 if G < 8 else 2
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=3, hq=n_kv * G, n_kv=n_kv, d=d, sink=8, window=40,
                 t0_range=None, t0=0, steps=3)
    _run_steps(w, 3, lens0=[1000, 37, 3])


@pytest.mark.parametrize("ctas", [1, 2, 7, 148, 600])
def test_split_count_invariance(ctas):
    """The split of keys over CTAs changes only rounding."""
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=4, t0_range=(300, 3000), steps=2)
    _run_steps(w, 2, ctas=ctas)


def test_edge_lengths():
    """T = 1 (first token), T < S + W, T = S + W exactly, S = 0, W = 1."""
    for S, Wn, lens in [(16, 64, [0, 5, 79, 80]), (0, 1, [0, 1, 2, 100]), (0, 33, [7, 32, 33, 500]),
                        (4, 1, [3, 4, 5, 64])]:
        w = W.scaled(W.WORKLOADS["gqa128k"], batch=4, sink=S, window=Wn, t0_range=None, t0=0, steps=2,
                     d=64)
        _run_steps(w, 2, lens0=lens)


def test_streaming_slot_order_does_not_matter():
    """Permuting the ring slots (and their positions) leaves the output unchanged
    up to rounding: the streaming kernel reads the slots as an unordered set."""
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=2, t0_range=None, t0=900, steps=1, sink=16, window=48)
    dev = _dev()
    lens0 = np.array([900, 900])
    cache = _mk(w, 901)
    hist = History(w)
    fill(cache, hist, 0, lens0 + 1, dev)
    q = W.decode_q(w, 0, lens0 + 1).to(dev)
    lens = torch.tensor([901, 901], dtype=torch.int32, device=dev)
    a = cache.decode(0, q, lens, w.scale).clone()
    views = cache.layer_views(0)
    perm = torch.randperm(w.sink + w.window, generator=torch.Generator().manual_seed(0)).to(dev)
    for name in ("k_streaming", "v_streaming"):
        views[name].copy_(views[name][:, :, perm].clone())
    views["positions"].copy_(views["positions"][:, perm].clone())
    b = cache.decode(0, q, lens, w.scale)
    m, r = errors(b.cpu().numpy(), a.cpu().numpy())
    # Up to rounding: the probabilities enter the PV product as a sum of two
    # bf16 terms (~2^-16 relative), and the running max that scales them
    # depends on which keys the first tile holds.
    assert m < 1e-4 and r < 2e-5


def test_empty_and_over_capacity_status():
    from head_wise_kv_b200 import _lib
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=3, t0_range=None, t0=0, steps=1, d=64)
    dev = _dev()
    cache = _mk(w, 64)
    hist = History(w)
    fill(cache, hist, 0, [64, 64, 64], dev)
    q = W.decode_q(w, 0, np.array([64, 64, 64])).to(dev)
    out = cache.decode(0, q, torch.tensor([64, 0, 64], dtype=torch.int32, device=dev), w.scale)
    torch.cuda.synchronize()
    st = cache.status()
    assert st & _lib.DUO_STATUS_EMPTY_SEQUENCE
    assert torch.all(out[1] == 0)
    cache.decode(0, q, torch.tensor([64, 65, 64], dtype=torch.int32, device=dev), w.scale)
    torch.cuda.synchronize()
    assert cache.status() & _lib.DUO_STATUS_OVER_CAPACITY


def test_mha32k_config_sampled():
    """MHA 32 heads, T=32768, 8 retrieval heads, key rows 0..3 x4: 4 of 64
    steps checked in full (all 32 heads)."""
    w = W.scaled(W.WORKLOADS["mha32k"], steps=4)
    _run_steps(w, 4)


def test_gqa128k_config_sampled():
    """The full GQA 128K workload (B=8 ragged 16K..128K, 4 of 8 KV heads
    retrieval): two decode steps, every sequence and query head compared."""
    w = W.scaled(W.WORKLOADS["gqa128k"], steps=2)
    _run_steps(w, 2)


def test_timed_out_wait_is_reported_and_the_context_stays_usable():
    """A device wait that nothing completes gives up after its bound and sets
    DUO_STATUS_WAIT_TIMEOUT (the same routine and status path as every
    pipeline wait); reading the status with clear resets it, and decode then
    runs and matches the oracle."""
    import time
    from head_wise_kv_b200 import _lib as L
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=2, layers=1, t0_range=None, t0=0, sink=16, window=64)
    from head_wise_kv_b200 import DuoKVCache
    dev = torch.device("cuda", 0)
    cache = DuoKVCache(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, 700, W.retrieval_masks(w),
                       device=dev)
    lens0 = np.array([600, 333])
    hist = History(w)
    fill(cache, hist, 0, lens0, dev)
    torch.cuda.synchronize()
    assert cache.status() == 0
    t0 = time.perf_counter()
    cache.check_wait_timeout(2_000_000)           # 2 ms
    st = cache.status(clear=True)
    elapsed = time.perf_counter() - t0
    assert st & L.DUO_STATUS_WAIT_TIMEOUT
    assert 0.002 <= elapsed < 5.0
    assert cache.status() == 0
    q, k, v = new_token_inputs(w, 0, lens0)
    cache.append(0, k.to(dev), v.to(dev), torch.from_numpy(lens0.astype(np.int32)).to(dev))
    lens = lens0 + 1
    out = cache.decode(0, q.to(dev), torch.from_numpy(lens.astype(np.int32)).to(dev), w.scale)
    ref, _ = oracle_decode(hist, 0, q, lens, W.retrieval_mask(w, 0))
    assert_close(out.cpu().double().numpy(), ref, "decode after a reported timeout")
    assert cache.status() == 0
    with pytest.raises(L.DuoError):
        cache.check_wait_timeout(0)
    cache.close()
