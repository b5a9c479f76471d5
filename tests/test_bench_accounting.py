"""The benchmark's algorithmic accounting (the numerators of its roofline
fractions), checked on CPU against brute-force counts and closed forms.

* Decode: KV bytes of a layer-step = full K and V rows of every retrieval
  head plus the filled ring slots of every streaming head, counted here by
  enumerating each query's key set.
* Chunked prefill: useful FLOPs = 4 d per mask-valid (query, key) pair, the
  pairs counted by enumerating keys; the 64K-prompt total against the closed
  form 4 d (16 * 2,147,516,416 + 16 * 70,711,840).
* Gated decode: its streaming part reads the sink rows and the window rows,
  a union that covers exactly min(T, S + W) positions.
"""
import numpy as np
import pytest

import bench
import duo_workloads as W


def _key_set(t, retrieval, S, Wn):
    """Positions query t reads, enumerated: the full history for a
    retrieval head; for a streaming head the first S tokens and the last W
    (DuoAttention guide, section 2, "Retrieval Heads vs. Streaming Heads";
    window rule of "Attention Variants and Memory Efficiency", section
    "Sliding-Window and Mixed Attention")."""
    if retrieval:
        return set(range(t + 1))
    return {j for j in range(t + 1) if j < S or j >= t - Wn + 1}


@pytest.mark.parametrize("S,Wn", [(4, 16), (0, 8), (16, 64)])
def test_decode_kv_bytes_equal_enumerated_key_sets(S, Wn):
    rng = np.random.default_rng(S + Wn)
    mask = np.array([1, 0, 1, 0, 0], np.uint8)
    d = 64
    lens = rng.integers(1, 200, size=3)
    want = 0
    for T in lens:
        for g, r in enumerate(mask):
            want += 4 * d * len(_key_set(int(T) - 1, bool(r), S, Wn))
    assert bench.kv_bytes(lens, mask, d, S, Wn, cap=10 ** 9) == want


def test_decode_kv_bytes_of_the_128k_workload_first_step():
    base = W.WORKLOADS["gqa128k"]
    lens = W.context_lengths(base) + 1             # after the first decode append
    mask = W.retrieval_mask(base, 0)
    n_r = int(mask.sum())
    closed = sum(n_r * 512 * int(T) + (base.n_kv - n_r) * 512 * (base.sink + base.window) for T in lens)
    assert bench.kv_bytes(lens, mask, base.d, base.sink, base.window, cap=10 ** 9) == closed
    assert 0.9e9 < closed < 1.3e9                   # ~1.1 GB per layer-step at d = 128


@pytest.mark.parametrize("prompt,chunk,S,Wn", [(300, 128, 4, 16), (257, 64, 0, 32), (90, 100, 8, 8)])
def test_prefill_pairs_equal_enumerated_masks(prompt, chunk, S, Wn):
    n_r_q, n_s_q = 3, 2
    want = 0
    for t in range(prompt):
        want += n_r_q * len(_key_set(t, True, S, Wn)) + n_s_q * len(_key_set(t, False, S, Wn))
    assert bench.prefill_pairs(prompt, chunk, n_r_q, n_s_q, S, Wn) == want


def test_prefill_flops_of_the_64k_prompt():
    pairs = bench.prefill_pairs(65536, 4096, 16, 16, 64, 1024)
    assert pairs == 16 * 2_147_516_416 + 16 * 70_711_840
    assert 4 * 128 * pairs == 18_171_725_873_152
    # per retrieval query head: chunk c holds 4096 c prefix keys per row plus its causal triangle
    assert bench.prefill_pairs(4096, 4096, 1, 0, 64, 1024) == 8_390_656
    assert (bench.prefill_pairs(65536, 4096, 1, 0, 64, 1024) -
            bench.prefill_pairs(61440, 4096, 1, 0, 64, 1024)) == 4096 * 61440 + 8_390_656


@pytest.mark.parametrize("S,Wn", [(64, 256), (16, 64), (0, 8)])
def test_gated_streaming_rows_cover_the_keep_set(S, Wn):
    for T in range(0, 3 * (S + Wn) + 5):
        sink_rows = set(range(min(T, S)))
        win_rows = set(range(max(T - Wn, S), T))
        assert not sink_rows & win_rows
        assert len(sink_rows) + len(win_rows) == min(T, S) + max(0, T - max(T - Wn, S))
        if T:
            assert sink_rows | win_rows == _key_set(T - 1, False, S, Wn)
        assert len(sink_rows | win_rows) == min(T, S + Wn)


def test_decode_kv_bytes_of_the_million_token_step():
    """One decode step of the 32-layer million-token workload: per layer 2
    retrieval heads over T + 1 = 1,048,577 keys and 6 streaming heads over
    S + W = 1,088 slots, 512 bytes per key (K and V, d = 128, bf16): 34.47 GB
    per step, 1.077 GB per layer."""
    w = W.WORKLOADS["mtok"]
    T = w.t0 + 1
    per_layer = 2 * 512 * T + 6 * 512 * 1088
    total = sum(bench.kv_bytes([T], W.retrieval_mask(w, l), w.d, w.sink, w.window, T) for l in range(w.layers))
    assert total == 32 * per_layer == 34_466_725_888
    assert round(per_layer / 1e9, 3) == 1.077


def test_decode_kv_bytes_of_the_mha32k_step():
    """MHA-32K, first decode step: 8 retrieval heads over 32,769 keys and 24
    streaming heads over 320 slots, 512 bytes per key: ~138.1 MB."""
    w = W.WORKLOADS["mha32k"]
    lens = W.context_lengths(w) + 1
    got = bench.kv_bytes(lens, W.retrieval_mask(w, 0), w.d, w.sink, w.window, 10 ** 9)
    assert got == 8 * 512 * 32769 + 24 * 512 * 320 == 138_153_984


def test_traffic_constants_match_their_workloads():
    """Each recorded DRAM traffic per launch (ncu, one launch of the leg's
    own workload) lies between the leg's algorithmic KV bytes and 5 % above
    them: reads cannot be fewer than the keys and values the launch must
    stream, and the excess is the partial outputs and tile tails.  A constant
    left over from another workload, cache type or kernel falls outside."""
    base = W.WORKLOADS["gqa128k"]
    lens = W.context_lengths(base) + 1                       # the captured (first timed) step
    mask = W.retrieval_mask(base, 0)
    bf16 = bench.kv_bytes(lens, mask, base.d, base.sink, base.window, cap=10 ** 9)
    full = bench.kv_bytes(lens, np.ones_like(mask), base.d, base.sink, base.window, cap=10 ** 9)
    mha = W.WORKLOADS["mha32k"]
    mha_b = bench.kv_bytes(W.context_lengths(mha) + 1, W.retrieval_mask(mha, 0), mha.d, mha.sink, mha.window,
                           cap=10 ** 9)
    mt = W.WORKLOADS["mtok"]
    mt_b = bench.kv_bytes([mt.t0 + 1], W.retrieval_masks(mt)[0], mt.d, mt.sink, mt.window, cap=10 ** 9)
    cases = {
        "bf16": (bench.DECODE_TRAFFIC_BYTES, bf16),
        "fp8": (bench.DECODE_FP8_TRAFFIC_BYTES, bf16 // 2),
        "int4": (bench.DECODE_INT4_TRAFFIC_BYTES, bf16 // 4),
        "paged": (bench.DECODE_PAGED_TRAFFIC_BYTES, bf16),
        "seqsplit (both slices)": (bench.DECODE_SEQSPLIT_TRAFFIC_BYTES, bf16),
        "gated (all heads full)": (bench.DECODE_GATED_TRAFFIC_BYTES, full),
        "mha32k": (bench.MHA32K_DECODE_TRAFFIC_BYTES, mha_b),
        "mtok (one layer)": (bench.MTOK_DECODE_TRAFFIC_BYTES, mt_b),
    }
    for name, (traffic, alg) in cases.items():
        assert traffic is not None, name
        assert alg <= traffic <= 1.05 * alg, f"{name}: traffic {traffic} against algorithmic {alg}"
