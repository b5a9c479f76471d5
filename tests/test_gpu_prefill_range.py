"""Values far beyond fp16's range in chunked prefill, against the fp64 oracle.

bf16 values reach 3.4e38; the prefill multiplies probabilities and values
in fp16 (largest finite value 65504) on per-head copies scaled by a power of
two, undone at the end.  Planted rows of +-1e5 and +-3e38 (in the chunk's
own values, in the retrieval cache and in the streaming ring, i.e. as a
later chunk's cached prefix) must give the oracle's result, for bf16, FP8
and INT4 caches.

The bar: attention is linear in V, so scaling every value of a head by c
scales the exact output, and the rounding error of any fixed-precision
evaluation, by c.  The parity bar (max-abs 2e-3, relative L2 1e-3 at unit
scale) is therefore applied to out / M, with M = max(1, largest |v| the
head can read); heads with no planted row (M of order 1) meet it unscaled.
"""
import numpy as np
import pytest
import torch

import duo_workloads as W
from _harness import assert_close
from oracle import duo_oracle as O

pytestmark = pytest.mark.gpu

CHUNKS = [200, 300]
# (sequence, KV head, position, magnitude): a row rescaled so that its largest
# element is the magnitude (sign kept).  With S = 16, W = 64: head 1 and 3
# stream, 0 and 2 are retrieval heads; positions < 200 are cached when the
# second chunk attends, and 3 / 10 / 30 are sinks of the ring.
PLANTS = [(0, 0, 5, 1e5), (0, 0, 150, -1e5), (0, 1, 3, 3e38), (0, 2, 250, -1e5), (0, 3, 460, 3e38),
          (1, 0, 420, -3e38), (1, 1, 10, 1e5), (1, 2, 30, 3e38), (1, 3, 470, 1e5)]


def _dev():
    return torch.device("cuda", 0)


def _workload():
    return W.scaled(W.WORKLOADS["prefill64k"], batch=2, hq=8, n_kv=4, d=128, sink=16, window=64,
                    retrieval_frac=0.5, t0_range=None, t0=0, steps=0, fixed_retrieval=(0, 2), rope=False,
                    prompt=0, chunk=0)


def _quant(kv_dtype, x, s):
    # x / scale overflows fp32 for the 3e38 rows: the code saturates (448 or 7)
    with np.errstate(over="ignore"):
        if kv_dtype == "fp8":
            return O.dequantize_kv(O.quantize_kv(x, s), s)
        if kv_dtype == "int4":
            return O.dequantize_kv_int4(O.quantize_kv_int4(x, s), s)
    return x


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8", "int4"])
def test_prefill_values_beyond_fp16(kv_dtype):
    from head_wise_kv_b200 import DuoKVCache
    w = _workload()
    total = sum(CHUNKS)
    dev = _dev()
    K = {(b, g): W.tokens(w, 0, b, g, W.TENSOR_K, 0, total) for b in range(w.batch) for g in range(w.n_kv)}
    V = {(b, g): W.tokens(w, 0, b, g, W.TENSOR_V, 0, total).clone()
         for b in range(w.batch) for g in range(w.n_kv)}
    for b, g, pos, mag in PLANTS:
        row = V[(b, g)][pos].double()
        V[(b, g)][pos] = (row / row.abs().max() * mag).to(torch.bfloat16)
    assert all(torch.isfinite(V[k].float()).all() for k in V)
    ones = np.ones((1, w.n_kv), np.float32)
    ks = vs = ones
    if kv_dtype != "bf16":
        rng = np.random.default_rng(77)
        ks = rng.uniform(0.3, 1.0, (1, w.n_kv)).astype(np.float32)
        vs = rng.uniform(0.3, 1.0, (1, w.n_kv)).astype(np.float32)
    cache = DuoKVCache(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, total, W.retrieval_masks(w),
                       device=dev, kv_dtype=kv_dtype, k_scale=ks, v_scale=vs)
    mask = W.retrieval_mask(w, 0)
    prefix = np.zeros(w.batch, dtype=np.int64)
    planted_heads = {(b, g) for b, g, _, _ in PLANTS}
    for C in CHUNKS:
        q = torch.empty(w.batch, w.hq, C, w.d, dtype=torch.bfloat16)
        k = torch.empty(w.batch, w.n_kv, C, w.d, dtype=torch.bfloat16)
        v = torch.empty_like(k)
        for b in range(w.batch):
            P = int(prefix[b])
            for h in range(w.hq):
                q[b, h] = W.tokens(w, 0, b, h, W.TENSOR_Q, P, P + C)
            for g in range(w.n_kv):
                k[b, g] = K[(b, g)][P:P + C]
                v[b, g] = V[(b, g)][P:P + C]
        pre = torch.from_numpy(prefix.astype(np.int32)).to(dev)
        out = cache.prefill(0, q.to(dev), k.to(dev), v.to(dev), pre, w.scale)
        cache.append(0, k.to(dev), v.to(dev), pre)

        # cached prefix as the cache stores it (dequantised codes), the chunk as given
        def hist(tensors, scales):
            def f(b, g):
                P = int(prefix[b])
                x = tensors[(b, g)][:P + C].double().numpy().copy()
                x[:P] = _quant(kv_dtype, tensors[(b, g)][:P].float().numpy(), float(scales[0, g]))
                return x
            return f
        kh, vh = hist(K, ks), hist(V, vs)
        ref = O.prefill_attention(q.double().numpy(), kh, vh, prefix, mask, w.sink, w.window, w.scale)
        got = out.cpu().double().numpy()
        assert np.all(np.isfinite(got)), f"{kv_dtype}: non-finite output, chunk {C}"
        for b in range(w.batch):
            for g in range(w.n_kv):
                M = max(1.0, float(np.abs(vh(b, g)).max()))
                hs = slice(g * w.group, (g + 1) * w.group)
                what = f"{kv_dtype} chunk {C} b{b} g{g} M={M:.3g}"
                if (b, g) in planted_heads:
                    assert_close(got[b, hs] / M, ref[b, hs] / M, what)
                else:
                    assert_close(got[b, hs], ref[b, hs], what)
        prefix = prefix + C
    torch.cuda.synchronize()
    assert cache.status() == 0
    cache.close()


def test_decode_values_beyond_fp16():
    """The decode multiplies bf16 values directly (fp32 accumulation): rows of
    +-1e5 in the retrieval cache, in the ring and in the new token give the
    oracle's result."""
    from head_wise_kv_b200 import DuoKVCache
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=2, layers=1, t0_range=None, t0=0, sink=16, window=64)
    dev = _dev()
    lens0 = np.array([700, 300])
    n = int(lens0.max()) + 1
    K = {(b, g): W.tokens(w, 0, b, g, W.TENSOR_K, 0, n) for b in range(w.batch) for g in range(w.n_kv)}
    V = {(b, g): W.tokens(w, 0, b, g, W.TENSOR_V, 0, n).clone() for b in range(w.batch) for g in range(w.n_kv)}
    for b, g, pos, mag in [(0, 0, 5, 1e5), (0, 1, 3, -1e5), (0, 5, 700, 1e5), (1, 2, 299, -1e5),
                           (1, 7, 300, 1e5), (1, 4, 100, 1e5), (0, 3, 690, -1e5)]:
        row = V[(b, g)][pos].double()
        V[(b, g)][pos] = (row / row.abs().max() * mag).to(torch.bfloat16)
    cache = DuoKVCache(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, 800, W.retrieval_masks(w),
                       device=dev)
    top = int(lens0.max())
    k = torch.zeros(w.batch, w.n_kv, top, w.d, dtype=torch.bfloat16)
    v = torch.zeros_like(k)
    for b in range(w.batch):
        for g in range(w.n_kv):
            k[b, g, :lens0[b]] = K[(b, g)][:lens0[b]]
            v[b, g, :lens0[b]] = V[(b, g)][:lens0[b]]
    zeros = torch.zeros(w.batch, dtype=torch.int32, device=dev)
    cache.append(0, k.to(dev), v.to(dev), zeros, torch.from_numpy(lens0.astype(np.int32)).to(dev))
    kn = torch.stack([torch.stack([K[(b, g)][lens0[b]] for g in range(w.n_kv)]) for b in range(w.batch)])
    vn = torch.stack([torch.stack([V[(b, g)][lens0[b]] for g in range(w.n_kv)]) for b in range(w.batch)])
    cache.append(0, kn.unsqueeze(2).to(dev), vn.unsqueeze(2).to(dev),
                 torch.from_numpy(lens0.astype(np.int32)).to(dev))
    lens = lens0 + 1
    q = W.decode_q(w, 0, lens)
    out = cache.decode(0, q.to(dev), torch.from_numpy(lens.astype(np.int32)).to(dev), w.scale)
    ref, _ = O.decode_attention(q.double().numpy(), lambda b, g: K[(b, g)].double().numpy(),
                                lambda b, g: V[(b, g)].double().numpy(), lens, W.retrieval_mask(w, 0),
                                w.sink, w.window, w.scale)
    got = out.cpu().double().numpy()
    assert np.all(np.isfinite(got))
    for b in range(w.batch):
        for g in range(w.n_kv):
            M = max(1.0, float(V[(b, g)][:lens[b]].float().abs().max()))
            hs = slice(g * w.group, (g + 1) * w.group)
            assert_close(got[b, hs] / M, ref[b, hs] / M, f"decode b{b} g{g} M={M:.3g}")
    torch.cuda.synchronize()
    assert cache.status() == 0
    cache.close()
