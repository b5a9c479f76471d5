"""The seeded input generator (duo_workloads) that both the oracle side and
the CUDA side draw from: every token's K, V and q are a fixed function of
(workload, layer, sequence, head, kind, position), whatever slice a caller
asks for; draws are N(0, 1) rounded to bf16 to nearest-even; the length mix,
head roles, RoPE and sink-key scaling follow the stated recipe."""
import math

import numpy as np
import pytest
import torch

import duo_workloads as W


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).numpy()


@pytest.mark.parametrize("name,kind,p0,p1", [
    ("gqa128k", W.TENSOR_K, 1000, 9000),     # crosses two 4096-token blocks
    ("gqa128k", W.TENSOR_V, 4095, 4097),
    ("gqa128k", W.TENSOR_Q, 60, 200),        # q blocks are 64 tokens
    ("tiny", W.TENSOR_K, 3, 300),            # rotated keys
    ("tiny", W.TENSOR_Q, 100, 130),          # rotated queries
    ("mha32k", W.TENSOR_K, 2, 70),           # starts inside the scaled sink rows
])
def test_a_slice_equals_the_same_rows_of_a_longer_draw(name, kind, p0, p1):
    w = W.WORKLOADS[name]
    whole = W.tokens(w, 0, 0, 1, kind, 0, p1 + 50)
    part = W.tokens(w, 0, 0, 1, kind, p0, p1)
    assert np.array_equal(_bits(whole[p0:p1]), _bits(part))


def test_draws_are_repeatable_and_streams_distinct():
    w = W.WORKLOADS["gqa128k"]
    a = W.tokens(w, 0, 3, 2, W.TENSOR_K, 500, 600)
    W._block.cache_clear()
    assert np.array_equal(_bits(a), _bits(W.tokens(w, 0, 3, 2, W.TENSOR_K, 500, 600)))
    others = [W.tokens(w, 0, 3, 2, W.TENSOR_V, 500, 600),     # kind
              W.tokens(w, 0, 3, 1, W.TENSOR_K, 500, 600),     # head
              W.tokens(w, 0, 2, 2, W.TENSOR_K, 500, 600),     # sequence
              W.tokens(W.WORKLOADS["mtok"], 1, 0, 2, W.TENSOR_K, 500, 600)]   # layer / workload
    for o in others:
        assert not torch.equal(a, o)


def test_bf16_rounding_is_to_nearest_even():
    w = W.WORKLOADS["gqa128k"]
    x = np.ascontiguousarray(W.tokens_f32(w, 0, 0, 0, W.TENSOR_K, 0, 4096))
    u = x.view(np.uint32).astype(np.uint64)
    # round to nearest, ties to even, on the upper 16 bits (finite inputs)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    got = W.tokens(w, 0, 0, 0, W.TENSOR_K, 0, 4096).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got.reshape(-1), r.reshape(-1))


def test_draws_are_standard_normal():
    w = W.WORKLOADS["gqa128k"]
    x = W.tokens_f32(w, 0, 5, 3, W.TENSOR_V, 0, 8192).astype(np.float64)
    assert abs(x.mean()) < 0.01
    assert abs(x.std() - 1.0) < 0.01
    assert abs(np.mean(x ** 4) / np.mean(x ** 2) ** 2 - 3.0) < 0.05     # Gaussian kurtosis


def test_rope_keeps_norms_and_leaves_position_zero():
    w = W.WORKLOADS["tiny"]
    plain = W.scaled(w, rope=False)
    for p0, p1 in [(0, 64), (200, 300)]:
        r = W.tokens_f32(w, 0, 0, 1, W.TENSOR_K, p0, p1).astype(np.float64)
        x = W.tokens_f32(plain, 0, 0, 1, W.TENSOR_K, p0, p1).astype(np.float64)
        np.testing.assert_allclose(np.linalg.norm(r, axis=1), np.linalg.norm(x, axis=1), rtol=1e-6)
        if p0 == 0:
            np.testing.assert_allclose(r[0], x[0], rtol=1e-7)
            assert not np.allclose(r[1], x[1])
    # values are not rotated
    np.testing.assert_array_equal(W.tokens_f32(w, 0, 0, 1, W.TENSOR_V, 5, 9),
                                  W.tokens_f32(plain, 0, 0, 1, W.TENSOR_V, 5, 9))


def test_sink_keys_scaled_by_four_only_in_rows_zero_to_three():
    w = W.WORKLOADS["mha32k"]
    plain = W.scaled(w, sink_boost=1.0)
    k = W.tokens_f32(w, 0, 0, 7, W.TENSOR_K, 0, 8)
    k0 = W.tokens_f32(plain, 0, 0, 7, W.TENSOR_K, 0, 8)
    np.testing.assert_array_equal(k[:4], 4.0 * k0[:4])
    np.testing.assert_array_equal(k[4:], k0[4:])
    np.testing.assert_array_equal(W.tokens_f32(w, 0, 0, 7, W.TENSOR_V, 0, 8),
                                  W.tokens_f32(plain, 0, 0, 7, W.TENSOR_V, 0, 8))


def test_lengths_head_roles_and_capacities():
    g = W.WORKLOADS["gqa128k"]
    lens = W.context_lengths(g)
    assert lens.shape == (8,) and lens.min() >= 16384 and lens.max() <= 131072
    assert len(set(lens.tolist())) == 8                     # ragged
    assert np.array_equal(lens, W.context_lengths(g))
    assert W.capacity(g) == int(lens.max()) + g.steps
    assert W.capacity(W.WORKLOADS["prefill64k"]) == 65536
    for name, want in [("gqa128k", 4), ("mha32k", 8), ("mtok", 2), ("prefill64k", 4)]:
        w = W.WORKLOADS[name]
        for layer in range(w.layers):
            m = W.retrieval_mask(w, layer)
            assert m.dtype == np.uint8 and int(m.sum()) == want == math.ceil(w.retrieval_frac * w.n_kv)
    assert W.retrieval_mask(W.WORKLOADS["tiny"], 0).tolist() == [1, 0, 1, 0]
    masks = W.retrieval_masks(W.WORKLOADS["mtok"])
    assert len({m.tobytes() for m in masks}) > 1             # drawn per layer
