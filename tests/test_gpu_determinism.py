"""Repeatability of the decode kernel: the same inputs must give the same
bits on every launch.  The split-K partition, the tile order of each CTA and
the log-sum-exp merge order are all fixed, so any difference between two
launches is a race (a buffer overwritten while it is still read, a barrier
phase taken for another).  Each case repeats one decode step many times on
bf16, FP8 and INT4 caches, with few CTAs (long pieces, deep pipelines) and
with the default persistent wave.
"""
import numpy as np
import pytest
import torch

import duo_workloads as W
from _harness import History, fill, new_token_inputs

pytestmark = pytest.mark.gpu

REPEATS = 60


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8", "int4"])
@pytest.mark.parametrize("ctas", [5, 0])
def test_decode_is_bitwise_repeatable(kv_dtype, ctas):
    from head_wise_kv_b200 import DuoKVCache
    dev = torch.device("cuda", 0)
    w = W.scaled(W.WORKLOADS["gqa128k"], batch=2, layers=1, t0_range=None, t0=0, sink=16, window=64)
    sc = np.full((1, w.n_kv), 0.5, np.float32) if kv_dtype != "bf16" else None
    lens0 = np.array([1500, 777])
    cache = DuoKVCache(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, 1600, W.retrieval_masks(w),
                       device=dev, kv_dtype=kv_dtype, k_scale=sc, v_scale=sc)
    if ctas:
        cache.set_decode_ctas(ctas)
    fill(cache, History(w), 0, lens0, dev)
    q, k, v = new_token_inputs(w, 0, lens0)
    cache.append(0, k.to(dev), v.to(dev), torch.from_numpy(lens0.astype(np.int32)).to(dev))
    lens = torch.from_numpy((lens0 + 1).astype(np.int32)).to(dev)
    qd = q.to(dev)
    first = cache.decode(0, qd, lens, w.scale).clone()
    differ = 0
    for _ in range(REPEATS):
        differ += int(not torch.equal(cache.decode(0, qd, lens, w.scale), first))
    assert cache.status() == 0
    assert differ == 0, f"{differ} of {REPEATS} launches differ from the first"
    cache.close()
