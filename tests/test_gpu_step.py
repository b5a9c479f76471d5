"""duo_decode_step: append + decode in one call, the decode reading ahead of
the append, against the two separate calls and the fp64 oracle.

The step's attention kernel starts while the append of the new token is
still running and waits for it only before the tiles that can hold the new
row (the last tile of each retrieval head, the streaming rings).  If that
rule missed a tile, the kernel would read a stale row, which shows up as a
difference from append + decode.  So every step here runs on twin caches
(one with duo_decode_step, one with duo_kv_append then duo_decode_attn) and
requires identical output bits, identical lse bits and identical cache
buffers after each step, over many steps (rings small enough that every
step evicts a slot), for bf16, FP8, INT4 and paged caches and both head
dims.  One step of each is also checked against the oracle at the parity
bar, and a step whose lengths do not grow by exactly one (the kernel then
waits for the append before reading anything) must match as well.
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


def _twins(kind, w, cap):
    from head_wise_kv_b200 import DuoKVCache
    kv_dtype = kind.replace("paged_", "")
    ks = vs = None
    if kv_dtype != "bf16":
        rng = np.random.default_rng(5)
        ks = rng.uniform(0.3, 1.0, (w.layers, w.n_kv)).astype(np.float32)
        vs = rng.uniform(0.3, 1.0, (w.layers, w.n_kv)).astype(np.float32)
    kw = {}
    per_seq = (cap + PAGE - 1) // PAGE
    if kind.startswith("paged"):
        kw = dict(page_tokens=PAGE, num_pages=w.batch * per_seq + 1)
    caches = [DuoKVCache(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, cap, W.retrieval_masks(w),
                         device=_dev(), kv_dtype=kv_dtype, k_scale=ks, v_scale=vs, **kw) for _ in range(2)]
    caches[1].buf.copy_(caches[0].buf)   # the same starting bytes (rows not yet written included)
    if kw:
        perm = np.random.default_rng(9).permutation(w.batch * per_seq + 1)[:w.batch * per_seq]
        table = torch.from_numpy(perm.reshape(w.batch, per_seq).astype(np.int32)).to(_dev())
        for c in caches:
            c.set_page_table(table)
    return caches, ks, vs


def _value(hist, kv_dtype, ks, vs, b, g, tensor, n):
    x = hist.kv(0, b, g, tensor, n).float().numpy()
    if kv_dtype == "bf16":
        return x
    s = float((ks if tensor == W.TENSOR_K else vs)[0, g])
    if kv_dtype == "fp8":
        return O.dequantize_kv(O.quantize_kv(x, s), s)
    return O.dequantize_kv_int4(O.quantize_kv_int4(x, s), s)


@pytest.mark.parametrize("kind,d,sink,window,steps", [
    ("bf16", 128, 4, 8, 40), ("fp8", 128, 4, 8, 40), ("int4", 128, 4, 8, 40), ("paged_bf16", 128, 4, 8, 40),
    ("bf16", 128, 64, 256, 12), ("bf16", 64, 4, 8, 20),
])
def test_step_equals_append_then_decode(kind, d, sink, window, steps):
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=6, layers=1, t0_range=None, t0=0, sink=sink, window=window,
                 steps=steps, d=d)
    kv_dtype = kind.replace("paged_", "")
    lens0 = np.array([0, 1, sink + window - 1, sink + window, 700, 3000], dtype=np.int64)
    cap = int(lens0.max()) + steps + 1
    (a, b), ks, vs = _twins(kind, w, cap)
    dev = _dev()
    hist = History(w)
    for c in (a, b):
        fill(c, hist, 0, lens0, dev)
    mask = W.retrieval_mask(w, 0)
    for s in range(steps):
        lb = lens0 + s
        q, k, v = new_token_inputs(w, 0, lb)
        q, k, v = q.to(dev), k.to(dev), v.to(dev)
        lbt = torch.from_numpy(lb.astype(np.int32)).to(dev)
        lat = torch.from_numpy((lb + 1).astype(np.int32)).to(dev)
        a.append(0, k, v, lbt)
        ref_out, ref_lse = a.decode(0, q, lat, w.scale, want_lse=True)
        got_out, got_lse = b.step(0, q, k, v, lbt, lat, w.scale, want_lse=True)
        what = f"{kind} d={d} S={sink} W={window} step {s}"
        assert torch.equal(got_out, ref_out), f"out differs from append + decode: {what}"
        assert torch.equal(got_lse, ref_lse), f"lse differs from append + decode: {what}"
        assert torch.equal(a.buf, b.buf), f"cache contents differ: {what}"
        if s in (0, steps - 1):
            lens = lb + 1
            ref, rl = O.decode_attention(q.cpu().double().numpy(),
                                         lambda bb, g: _value(hist, kv_dtype, ks, vs, bb, g, W.TENSOR_K, int(lens[bb])),
                                         lambda bb, g: _value(hist, kv_dtype, ks, vs, bb, g, W.TENSOR_V, int(lens[bb])),
                                         lens, mask, w.sink, w.window, w.scale)
            assert_close(got_out.cpu().double().numpy(), ref, what)
            assert np.abs(got_lse.cpu().double().numpy() - rl).max() < 1e-3, f"lse vs oracle: {what}"
    torch.cuda.synchronize()
    assert a.status() == 0 and b.status() == 0
    a.close()
    b.close()


def test_step_lengths_not_one_more():
    """A sequence whose length does not grow by one (here: the lengths passed
    are those before the append for one sequence) turns the read-ahead off;
    the result still equals append + decode with the same arguments."""
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=4, layers=1, t0_range=None, t0=0, sink=4, window=8, steps=2)
    lens0 = np.array([30, 500, 9, 2000], dtype=np.int64)
    (a, b), _, _ = _twins("bf16", w, int(lens0.max()) + 4)
    dev = _dev()
    hist = History(w)
    for c in (a, b):
        fill(c, hist, 0, lens0, dev)
    q, k, v = new_token_inputs(w, 0, lens0)
    q, k, v = q.to(dev), k.to(dev), v.to(dev)
    lbt = torch.from_numpy(lens0.astype(np.int32)).to(dev)
    after = lens0 + 1
    after[2] = lens0[2]                     # sequence 2 decodes without its new token
    lat = torch.from_numpy(after.astype(np.int32)).to(dev)
    a.append(0, k, v, lbt)
    ref = a.decode(0, q, lat, w.scale)
    got = b.step(0, q, k, v, lbt, lat, w.scale)
    assert torch.equal(got, ref)
    assert torch.equal(a.buf, b.buf)
    torch.cuda.synchronize()
    assert a.status() == 0 and b.status() == 0
    a.close()
    b.close()


def test_step_checks_before_launching():
    """A rejected step (a misaligned output) appends nothing."""
    from head_wise_kv_b200 import _lib as L
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=2, layers=1, t0_range=None, t0=0, sink=4, window=8, steps=1)
    (a, _), _, _ = _twins("bf16", w, 64)
    dev = _dev()
    lens0 = np.array([5, 9])
    hist = History(w)
    fill(a, hist, 0, lens0, dev)
    torch.cuda.synchronize()
    before = a.buf.clone()
    q, k, v = new_token_inputs(w, 0, lens0)
    lbt = torch.from_numpy(lens0.astype(np.int32)).to(dev)
    lat = lbt + 1
    out = torch.empty(w.batch * w.hq * w.d + 1, dtype=torch.float32, device=dev)[1:]
    with pytest.raises(L.DuoError) as e:
        L.duo_decode_step(a.handle, 0, k.to(dev).data_ptr(), v.to(dev).data_ptr(), lbt.data_ptr(),
                          q.to(dev).data_ptr(), lat.data_ptr(), w.scale, out.data_ptr(), None, a._ws.data_ptr(),
                          a._ws.numel(), 0)
    assert e.value.code == L.DUO_ERR_ALIGNMENT
    torch.cuda.synchronize()
    assert torch.equal(a.buf, before)
    a.close()
