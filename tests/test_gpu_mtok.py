"""Million-token GQA decode (32 layers x 32 query / 8 KV heads, d=128, B=1,
T = 1,048,576, 2 of 8 KV heads retrieval per layer, S=64, W=1024): one decode
step through all 32 layers, every query head of three sampled layers compared
with the fp64 oracle.  The caches of the sampled layers hold the seeded
history (streaming heads need only the tokens their rings keep, so the
evicted middle of their history is not generated); the other layers are
filled on the device with random values and only have to run."""
import numpy as np
import pytest
import torch

import duo_workloads as W
from _harness import assert_close, new_token_inputs
from oracle import duo_oracle as O

pytestmark = pytest.mark.gpu

CHECK_LAYERS = (0, 13, 31)


class _Rows:
    """History of one (layer, head, K or V) that draws only the positions the
    oracle indexes (contiguous runs), as float32 rows."""

    def __init__(self, w, layer, g, kind):
        self.w, self.layer, self.g, self.kind = w, layer, g, kind

    def __getitem__(self, keys):
        keys = np.asarray(keys)
        out = np.empty((len(keys), self.w.d), dtype=np.float32)
        start = 0
        while start < len(keys):
            end = start
            while end + 1 < len(keys) and keys[end + 1] == keys[end] + 1:
                end += 1
            out[start:end + 1] = W.tokens(self.w, self.layer, 0, self.g, self.kind, int(keys[start]),
                                          int(keys[end]) + 1).float().numpy()
            start = end + 1
        return out


def _fill_checked_layer(cache, w, layer, T, dev, slab=65536):
    """Bulk-append positions 0..T-1: retrieval heads get every seeded token,
    streaming heads only the ones their ring keeps (zeros elsewhere; the append
    kernel drops evicted positions anyway)."""
    mask = W.retrieval_mask(w, layer)
    keep = set(O.keep_set(T - 1, w.sink, w.window).tolist())
    keep_lo, keep_hi = w.sink, T - w.window     # positions outside [keep_lo, keep_hi) are kept
    assert all(p < keep_lo or p >= keep_hi for p in keep)
    for p0 in range(0, T, slab):
        n = min(slab, T - p0)
        k = torch.zeros(1, w.n_kv, n, w.d, dtype=torch.bfloat16)
        v = torch.zeros_like(k)
        for g in range(w.n_kv):
            if mask[g]:
                k[0, g] = W.tokens(w, layer, 0, g, W.TENSOR_K, p0, p0 + n)
                v[0, g] = W.tokens(w, layer, 0, g, W.TENSOR_V, p0, p0 + n)
            else:
                for a, e in [(p0, min(p0 + n, keep_lo)), (max(p0, keep_hi), p0 + n)]:
                    if a < e:
                        k[0, g, a - p0:e - p0] = W.tokens(w, layer, 0, g, W.TENSOR_K, a, e)
                        v[0, g, a - p0:e - p0] = W.tokens(w, layer, 0, g, W.TENSOR_V, a, e)
        cache.append(layer, k.to(dev), v.to(dev), torch.tensor([p0], dtype=torch.int32, device=dev))


def test_million_token_decode_step_through_32_layers():
    from head_wise_kv_b200 import DuoKVCache
    w = W.WORKLOADS["mtok"]
    dev = torch.device("cuda", 0)
    T0 = w.t0
    cache = DuoKVCache(w.layers, 1, w.hq, w.n_kv, w.d, w.sink, w.window, T0 + 1, W.retrieval_masks(w),
                       device=dev)
    gen = torch.Generator(device=dev).manual_seed(0)
    for layer in range(w.layers):
        if layer in CHECK_LAYERS:
            _fill_checked_layer(cache, w, layer, T0, dev)
        else:
            views = cache.layer_views(layer)
            for name in ("k_retrieval", "v_retrieval", "k_streaming", "v_streaming"):
                views[name].copy_(torch.randn(views[name].shape, generator=gen, device=dev,
                                              dtype=torch.float32).to(torch.bfloat16))
    torch.cuda.synchronize()
    lens_b = np.array([T0])
    lb = torch.tensor([T0], dtype=torch.int32, device=dev)
    la = torch.tensor([T0 + 1], dtype=torch.int32, device=dev)
    outs = {}
    for layer in range(w.layers):       # one decode step, layer after layer
        q, k, v = new_token_inputs(w, layer, lens_b)
        cache.append(layer, k.to(dev), v.to(dev), lb)
        out = cache.decode(layer, q.to(dev), la, w.scale)
        if layer in CHECK_LAYERS:
            outs[layer] = (q, out.clone())
    torch.cuda.synchronize()
    assert cache.status() == 0
    for layer, (q, out) in outs.items():
        ref, _ = O.decode_attention(q.double().numpy(), lambda b, g: _Rows(w, layer, g, W.TENSOR_K),
                                    lambda b, g: _Rows(w, layer, g, W.TENSOR_V), lens_b + 1,
                                    W.retrieval_mask(w, layer), w.sink, w.window, w.scale)
        assert_close(out.cpu().double().numpy(), ref, f"layer {layer}")
    cache.close()
