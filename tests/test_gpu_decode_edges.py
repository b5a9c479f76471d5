"""The window rule's own edge cases on the d = 128 decode (the tensor-core
kernel that serves every 128-dimension head), against the fp64 oracle.

The key set of a streaming head at query position t is the sinks j < S plus
the window max(0, t - W + 1) .. t ("Attention Variants and Memory
Efficiency", "Sliding-Window and Mixed Attention"; DuoAttention guide,
section 2, the sink + recent cache).  Its edge cases are the ones covered
here, each for five cache kinds (bf16, FP8 E4M3, INT4, and paged bf16 and
INT4 pools) and for one CTA (every segment whole) and 600 CTAs (more CTAs
than the keys need, so that one-key segments and short pieces land on
split ranges and go through the in-kernel merge):

* no sinks (S = 0), a one-token window (W = 1), both at once;
* lengths T = 1 (the first token: a segment of one key in a 128- or
  256-row tile), T < S + W (ring partly filled), T = S + W exactly (ring
  just full), T = S + W + 1 (first eviction) and T >> S + W.

Each case runs two decode steps (append, then attend) and compares every
sequence and query head with the oracle at the parity bar: max-abs error
<= 2e-3 and relative L2 error <= 1e-3, log-sum-exp within 1e-3, and the
status word clean.
"""
import numpy as np
import pytest
import torch

import duo_workloads as W
from _harness import History, assert_close, fill, new_token_inputs
from oracle import duo_oracle as O

pytestmark = pytest.mark.gpu

PAGE = 256
WINDOWS = [(0, 1), (0, 33), (4, 1), (16, 64)]
KINDS = ["bf16", "fp8", "int4", "paged_bf16", "paged_int4"]
LONG = 1500          # several 128- and 256-key tiles and a ragged tail


def _dev():
    return torch.device("cuda", 0)


def _lens0(S, Wn):
    """Lengths before the first step; the two steps then meet T = 1, 2;
    T < S + W; T = S + W and S + W + 1; S + W + 1 and S + W + 2; and a long
    history."""
    sw = S + Wn
    return np.array([0, max(0, sw // 2 - 1), sw - 1, sw, LONG], dtype=np.int64)


def _cache(w, cap, kind, ks, vs):
    from head_wise_kv_b200 import DuoKVCache
    kv_dtype = kind.replace("paged_", "")
    kw = {}
    n_pages = 0
    if kind.startswith("paged"):
        per_seq = (cap + PAGE - 1) // PAGE
        n_pages = w.batch * per_seq + 2
        kw = dict(page_tokens=PAGE, num_pages=n_pages)
    cache = DuoKVCache(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, cap, W.retrieval_masks(w),
                       device=_dev(), kv_dtype=kv_dtype, k_scale=ks, v_scale=vs, **kw)
    if n_pages:
        perm = np.random.default_rng(17).permutation(n_pages)[:w.batch * per_seq]
        cache.set_page_table(torch.from_numpy(perm.reshape(w.batch, per_seq).astype(np.int32)).to(_dev()))
    return cache


class _Values:
    """What attention reads for each cached token: the bf16 history, or its
    dequantised codes for FP8 / INT4 caches (scale * E4M3(code) or
    scale * code, with code the oracle's quantisation of value / scale)."""

    def __init__(self, hist, kv_dtype, ks, vs):
        self.h, self.kv_dtype, self.ks, self.vs = hist, kv_dtype, ks, vs
        self._c = {}

    def get(self, b, g, kind, n):
        key = (b, g, kind)
        have = self._c.get(key)
        if have is None or have.shape[0] < n:
            x = self.h.kv(0, b, g, kind, n).float().numpy()
            s = float((self.ks if kind == W.TENSOR_K else self.vs)[0, g])
            if self.kv_dtype == "fp8":
                x = O.dequantize_kv(O.quantize_kv(x, s), s)
            elif self.kv_dtype == "int4":
                x = O.dequantize_kv_int4(O.quantize_kv_int4(x, s), s)
            self._c[key] = x
        return self._c[key][:n]


@pytest.mark.parametrize("ctas", [1, 600])
@pytest.mark.parametrize("S,Wn", WINDOWS)
@pytest.mark.parametrize("kind", KINDS)
def test_d128_window_edges(kind, S, Wn, ctas):
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=5, layers=1, t0_range=None, t0=0, sink=S, window=Wn, steps=2)
    kv_dtype = kind.replace("paged_", "")
    rng = np.random.default_rng(1000 + 10 * S + Wn)
    if kv_dtype == "bf16":
        ks = vs = None
        ksa = vsa = np.ones((1, w.n_kv), np.float32)
    else:
        lo, hi = (0.25, 2.0) if kv_dtype == "fp8" else (0.3, 1.0)
        ksa = rng.uniform(lo, hi, (1, w.n_kv)).astype(np.float32)
        vsa = rng.uniform(lo, hi, (1, w.n_kv)).astype(np.float32)
        ks, vs = ksa, vsa
    lens0 = _lens0(S, Wn)
    dev = _dev()
    cache = _cache(w, LONG + 2, kind, ks, vs)
    cache.set_decode_ctas(ctas)
    cache._ws.fill_(0xFF)                 # NaN canary: reading an unwritten partial fails parity
    hist = History(w)
    if lens0.max() > 0:
        fill(cache, hist, 0, lens0, dev)
    vals = _Values(hist, kv_dtype, ksa, vsa)
    mask = W.retrieval_mask(w, 0)
    for s in range(2):
        lens_b = lens0 + s
        q, k, v = new_token_inputs(w, 0, lens_b)
        cache.append(0, k.to(dev), v.to(dev), torch.from_numpy(lens_b.astype(np.int32)).to(dev))
        lens = lens_b + 1
        out, lse = cache.decode(0, q.to(dev), torch.from_numpy(lens.astype(np.int32)).to(dev), w.scale,
                                want_lse=True)
        ref, ref_lse = O.decode_attention(q.double().numpy(),
                                          lambda b, g: vals.get(b, g, W.TENSOR_K, int(lens[b])),
                                          lambda b, g: vals.get(b, g, W.TENSOR_V, int(lens[b])),
                                          lens, mask, S, Wn, w.scale)
        got = out.cpu().double().numpy()
        what = f"{kind} S={S} W={Wn} ctas={ctas} step {s} T={lens.tolist()}"
        assert_close(got, ref, what)
        assert np.abs(lse.cpu().double().numpy() - ref_lse).max() < 1e-3, f"lse {what}"
    torch.cuda.synchronize()
    assert cache.status() == 0
    cache.close()
