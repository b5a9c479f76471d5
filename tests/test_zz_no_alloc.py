"""duo_decode_attn_static_ws: decode for callers that cannot allocate device
memory (their host program owns it all, or they must not call cudaMalloc in
the serving loop).  It runs the same kernel as duo_decode_attn with the same
split of the keys, only on the library's built-in scratch, so its output and
log-sum-exp must equal duo_decode_attn's bit for bit, call after call; one
call is also compared with the fp64 oracle at the parity bar.

Collected last on purpose: if it fails, a run that stops at the first
failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import duo_workloads as W
from _harness import History, assert_close, fill, new_token_inputs, oracle_decode

pytestmark = pytest.mark.gpu


def _setup(w, lens0, steps=2):
    from head_wise_kv_b200 import DuoKVCache
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cache = DuoKVCache(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, int(max(lens0)) + steps,
                       W.retrieval_masks(w), device=dev)
    fill(cache, History(w), 0, lens0, dev)
    return cache, dev


def test_static_scratch_decode_matches_workspace_decode():
    from head_wise_kv_b200 import _lib as L
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=4, t0_range=(2000, 40000), steps=2)
    lens0 = W.context_lengths(w)
    cache, dev = _setup(w, lens0)
    hist = History(w)
    assert L.duo_decode_workspace_bytes(cache.handle) <= L.DUO_STATIC_WS_BYTES
    stream = torch.cuda.current_stream(dev).cuda_stream
    for s in range(2):   # two calls in a row, the second after another append
        lens_b = lens0 + s
        q, k, v = new_token_inputs(w, 0, lens_b)
        cache.append(0, k.to(dev), v.to(dev), torch.from_numpy(lens_b.astype(np.int32)).to(dev))
        qd = q.to(dev)
        lens = torch.from_numpy((lens_b + 1).astype(np.int32)).to(dev)
        ref = torch.empty(w.batch, w.hq, w.d, dtype=torch.float32, device=dev)
        ref_lse = torch.empty(w.batch, w.hq, dtype=torch.float32, device=dev)
        L.duo_decode_attn(cache.handle, 0, qd.data_ptr(), lens.data_ptr(), w.scale, ref.data_ptr(),
                          ref_lse.data_ptr(), cache._ws.data_ptr(), cache._ws.numel(), stream)
        got = torch.full_like(ref, float("nan"))
        got_lse = torch.full_like(ref_lse, float("nan"))
        L.duo_decode_attn_static_ws(cache.handle, 0, qd.data_ptr(), lens.data_ptr(), w.scale, got.data_ptr(),
                                    got_lse.data_ptr(), stream)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), f"call {s}: output differs from the workspace decode"
        assert torch.equal(got_lse, ref_lse), f"call {s}: lse differs from the workspace decode"
        if s == 1:
            o_ref, o_lse = oracle_decode(hist, 0, q, lens_b + 1, W.retrieval_mask(w, 0))
            assert_close(got.cpu().double().numpy(), o_ref, f"call {s} against the oracle")
            assert np.abs(got_lse.cpu().double().numpy() - o_lse).max() < 1e-3
    assert cache.status() == 0
    cache.close()


def test_static_scratch_rejects_problems_beyond_its_size():
    from head_wise_kv_b200 import _lib as L
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=64, hq=64, n_kv=8, t0_range=None, t0=64, steps=1)
    cache, dev = _setup(w, np.full(64, 64))
    cache.set_decode_ctas(8192)   # many partial slots: more scratch than the fixed array holds
    assert L.duo_decode_workspace_bytes(cache.handle) > L.DUO_STATIC_WS_BYTES
    q = torch.zeros(w.batch, w.hq, w.d, dtype=torch.bfloat16, device=dev)
    lens = torch.full((w.batch,), 64, dtype=torch.int32, device=dev)
    out = torch.empty(w.batch, w.hq, w.d, dtype=torch.float32, device=dev)
    with pytest.raises(L.DuoError) as e:
        L.duo_decode_attn_static_ws(cache.handle, 0, q.data_ptr(), lens.data_ptr(), w.scale, out.data_ptr(),
                                    None, torch.cuda.current_stream(dev).cuda_stream)
    assert e.value.code == L.DUO_ERR_WORKSPACE
    cache.close()
