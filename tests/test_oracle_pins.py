"""Pins for the fp64 oracle, against values the pages print, closed forms,
library routines and brute force -- never against the oracle itself.

The last section plants plausible mistakes in the oracle (monkeypatched, on
the CPU) and checks that some pin fails for each.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import duo_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def fixture(name):
    rows = []
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line)
    return rows


def fixture_kv(name):
    out = {}
    for r in fixture(name):
        k, v = r.split(None, 1)
        out[k] = v
    return out


# ------------------------------------------------------------------ sizes
def test_dense_sizes_match_printed_values():
    n = 0
    for row in fixture("kv_sizes.txt"):
        lhs, rhs = row.split("=")
        kind, L, n_kv, d, T = lhs.split()
        assert kind == "dense"
        assert O.kv_cache_bytes(int(L), int(n_kv), int(d), int(T)) == int(rhs)
        n += 1
    assert n == 3


def test_four_gqa_sequences_equal_one_mha_sequence():
    # "Attention Variants and KV-Cache Compression", MHA and GQA: four equal-length
    # GQA sequences use 2 GiB, as one MHA sequence does.
    assert 4 * O.kv_cache_bytes(32, 8, 128, 4096) == O.kv_cache_bytes(32, 32, 128, 4096) == 2 ** 31


def test_effective_context_printed_value():
    f = fixture_kv("duo_effective_context.txt")
    got = O.duo_effective_context(int(f["tokens"]), int(f["sink"]), int(f["window"]),
                                  float(f["retrieval_frac"]))
    assert got == pytest.approx(int(f["effective_context"]), abs=1e-9)


def test_duo_bytes_of_the_guides_example():
    # 80 layers, 8 KV heads, d=128, T=128,000, S=32, W=128 and R = 0.25 (2 of 8 heads):
    # the printed effective context (32,120 tokens per head) times the printed dense
    # bytes per token (41,943,040,000 / 128,000).
    f = fixture_kv("duo_effective_context.txt")
    dense_per_token = 41943040000 // 128000
    got = O.duo_cache_bytes(80, 8, 128, 128000, 32, 128, 2)
    assert got == int(f["effective_context"]) * dense_per_token == 10525081600


def test_duo_bytes_limits():
    # all heads retrieval: the dense formula; no retrieval heads: T replaced by S+W
    assert O.duo_cache_bytes(3, 4, 64, 1000, 16, 64, 4) == O.kv_cache_bytes(3, 4, 64, 1000)
    assert O.duo_cache_bytes(3, 4, 64, 1000, 16, 64, 0) == O.kv_cache_bytes(3, 4, 64, 80)
    assert O.duo_cache_bytes(2, 8, 128, 5000, 64, 256, [2, 5]) == \
        O.kv_cache_bytes(1, 7, 128, 5000) + O.kv_cache_bytes(1, 9, 128, 320)


# ------------------------------------------------------------------ ring
def test_sliding_window_printed_example():
    f = fixture_kv("sliding_window_ring.txt")
    c = O.StreamingCache(0, int(f["window"]))
    for p in range(int(f["appends"])):
        c.append(p, int(f["value_factor"]) * p)
    want = [tuple(int(x) for x in e.split(":")) for e in f["ordered"].split()]
    assert [(p, it) for p, it in c.ordered()] == want
    # slot layout: slot = appended count mod 3 -> positions 3, 4, 2 in slots 0, 1, 2
    assert list(c.pos) == [3, 4, 2]


def _list_simulation(T, S, W):
    """The guide's simulation: a sink list filled first, then a window list
    that drops its oldest entry once it holds more than W."""
    sinks, window = [], []
    for p in range(T):
        if len(sinks) < S:
            sinks.append(p)
        else:
            window.append(p)
            if len(window) > W:
                window.pop(0)
    return sinks, window


@pytest.mark.parametrize("seed", range(6))
def test_ring_matches_list_simulation(seed):
    rng = np.random.default_rng(seed)
    for _ in range(40):
        S, W = int(rng.integers(0, 9)), int(rng.integers(1, 12))
        T = int(rng.integers(0, 60))
        c = O.StreamingCache(S, W)
        for p in range(T):
            c.append(p)
        sinks, window = _list_simulation(T, S, W)
        assert [p for p, _ in c.ordered()] == sinks + window
        held = sorted(int(p) for p in c.pos if p >= 0)
        assert held == sorted(sinks + window)
        if T:
            # the keep set of the newest token is exactly what the cache holds
            assert held == list(O.keep_set(T - 1, S, W))


def test_needle_simulation_statements():
    f = fixture_kv("duo_simulation_needle.txt")
    L, H, S, W, T = (int(f[k]) for k in ("layers", "heads", "sink", "window", "tokens"))
    needle = int(f["needle"])
    # head assignment of the page's simulation: max(1, int(L*H*R)) retrieval heads,
    # taken from layers >= 1 at even head indices
    count = max(1, int(L * H * float(f["retrieval_frac"])))
    roles, taken = {}, 0
    for l in range(L):
        for h in range(H):
            r = taken < count and l >= 1 and h % 2 == 0
            roles[(l, h)] = r
            taken += r
    n_r = sum(roles.values())
    held = set(int(p) for p in O.ring_positions(T, S, W) if p >= 0)
    # every retrieval head keeps all T tokens (the needle included); streaming heads not
    assert f["needle_in_retrieval"] == "all" and needle < T
    assert f["needle_in_streaming"] == "none" and needle not in held
    assert O.duo_slots(T, S, W, n_r, L * H - n_r) == int(f["derived_duo_slots"])
    assert L * H * T == int(f["derived_dense_slots"])


def test_worked_positions_tiny_config():
    # S=16, W=64 after 513 and 528 appends (repository-derived worked values;
    # cross-checked against the list simulation above)
    pos = O.ring_positions(513, 16, 64)
    assert list(pos[:16]) == list(range(16))
    assert (pos[16], pos[64], pos[65], pos[79]) == (464, 512, 449, 463)
    pos = O.ring_positions(528, 16, 64)
    assert [pos[16 + k] for k in range(16)] == [464 + k for k in range(16)]
    pos = O.ring_positions(50, 16, 64)
    assert list(pos[:50]) == list(range(50)) and all(p == -1 for p in pos[50:])
    pos = O.ring_positions(32769, 64, 256)
    assert (pos[64], pos[256], pos[257]) == (32576, 32768, 32513)


# ------------------------------------------------------------------ attention
def _rand(rng, *shape):
    x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).to(torch.bfloat16)
    return x.double().numpy()


@pytest.mark.parametrize("seed", range(4))
def test_brute_force_matches_vectorised(seed):
    rng = np.random.default_rng(100 + seed)
    d, T = 8, 23
    q, k, v = _rand(rng, d), _rand(rng, T, d), _rand(rng, T, d)
    keys = sorted(rng.choice(T, size=9, replace=False).tolist())
    scale = float(rng.uniform(0.1, 1.0))
    o_ref, lse_ref = O.brute_force_attention(q, k, v, keys, scale)
    o, lse = O.attend(q, k[keys], v[keys], scale)
    np.testing.assert_allclose(o, o_ref, rtol=1e-13, atol=1e-13)
    assert lse == pytest.approx(lse_ref, rel=1e-13)


def test_weights_sum_to_one_and_closed_forms():
    rng = np.random.default_rng(7)
    d = 16
    q, k, v = _rand(rng, d), _rand(rng, 40, d), _rand(rng, 40, d)
    _, lse = O.attend(q, k, v, 0.25)
    assert np.exp(0.25 * (k @ q) - lse).sum() == pytest.approx(1.0, abs=1e-12)
    # one key: the output is that key's value
    o, _ = O.attend(q, k[:1], v[:1], 0.25)
    np.testing.assert_allclose(o, v[0], rtol=0, atol=1e-15)
    # identical keys: the plain mean of the values
    o, _ = O.attend(q, np.repeat(k[:1], 7, 0), v[:7], 0.25)
    np.testing.assert_allclose(o, v[:7].mean(0), rtol=1e-13, atol=1e-14)
    # two keys: logistic weights
    o, _ = O.attend(q, k[:2], v[:2], 0.5)
    s0, s1 = 0.5 * q @ k[0], 0.5 * q @ k[1]
    w0 = 1.0 / (1.0 + math.exp(s1 - s0))
    np.testing.assert_allclose(o, w0 * v[0] + (1 - w0) * v[1], rtol=1e-13, atol=1e-14)


def _hist(rng, B, n_kv, T, d):
    return _rand(rng, B, n_kv, T, d), _rand(rng, B, n_kv, T, d)


def _sdpa(q, k, v, mask, scale):
    """torch fp64 scaled_dot_product_attention, one query row set."""
    q = torch.from_numpy(q)[None, None]
    k = torch.from_numpy(k)[None, None]
    v = torch.from_numpy(v)[None, None]
    m = torch.from_numpy(mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=m, scale=scale)[0, 0].numpy()


@pytest.mark.parametrize("S,W,T", [(4, 8, 30), (0, 5, 17), (3, 1, 9), (16, 64, 513), (2, 40, 20)])
def test_decode_matches_sdpa_with_ring_contents(S, W, T):
    """Streaming heads: attention over exactly what a literal ring simulation
    holds after T appends, computed by torch's SDPA.  Retrieval heads: SDPA
    with every key."""
    rng = np.random.default_rng(S * 1000 + W * 10 + T)
    B, hq, n_kv, d = 2, 4, 2, 16
    K, V = _hist(rng, B, n_kv, T, d)
    q = _rand(rng, B, hq, d)
    mask = np.array([1, 0], dtype=np.uint8)
    lens = np.array([T, T])
    out, lse = O.decode_attention(q, lambda b, g: K[b, g], lambda b, g: V[b, g], lens, mask, S, W, 0.3)
    held = np.zeros(T, dtype=bool)
    held[[p for p in O.ring_positions(T, S, W) if p >= 0]] = True
    for b in range(B):
        for h in range(hq):
            g = h // (hq // n_kv)
            m = np.ones(T, dtype=bool) if mask[g] else held
            want = _sdpa(q[b, h][None], K[b, g], V[b, g], m[None], 0.3)[0]
            np.testing.assert_allclose(out[b, h], want, rtol=1e-12, atol=1e-12)


def test_streaming_equals_full_when_window_covers_context():
    rng = np.random.default_rng(3)
    B, hq, n_kv, d, T = 1, 4, 4, 8, 50
    K, V = _hist(rng, B, n_kv, T, d)
    q = _rand(rng, B, hq, d)
    kh, vh = (lambda b, g: K[b, g]), (lambda b, g: V[b, g])
    full, _ = O.decode_attention(q, kh, vh, [T], np.ones(4, np.uint8), 10, 40, 0.35)
    for S, W in [(10, 40), (0, 50), (50, 1), (20, 200)]:
        strm, _ = O.decode_attention(q, kh, vh, [T], np.zeros(4, np.uint8), S, W, 0.35)
        np.testing.assert_allclose(strm, full, rtol=1e-14, atol=1e-14)
    # one token short of covering: differs
    strm, _ = O.decode_attention(q, kh, vh, [T], np.zeros(4, np.uint8), 10, 39, 0.35)
    assert np.abs(strm - full).max() > 1e-6


def test_gqa_equals_mha_with_repeated_kv():
    """GQA with n_kv heads == MHA on K/V repeated with repeat_interleave
    ("Attention Variants and Memory Efficiency", repeat_kv)."""
    rng = np.random.default_rng(11)
    B, hq, n_kv, d, T = 2, 8, 2, 16, 40
    K, V = _hist(rng, B, n_kv, T, d)
    q = _rand(rng, B, hq, d)
    mask = np.array([0, 1], np.uint8)
    Kr = torch.from_numpy(K).repeat_interleave(hq // n_kv, dim=1).numpy()
    Vr = torch.from_numpy(V).repeat_interleave(hq // n_kv, dim=1).numpy()
    mask_r = np.repeat(mask, hq // n_kv)
    lens = np.array([T, T - 7])
    a, la = O.decode_attention(q, lambda b, g: K[b, g, :lens[b]], lambda b, g: V[b, g, :lens[b]],
                               lens, mask, 3, 6, 0.25)
    m, lm = O.decode_attention(q, lambda b, g: Kr[b, g, :lens[b]], lambda b, g: Vr[b, g, :lens[b]],
                               lens, mask_r, 3, 6, 0.25)
    np.testing.assert_allclose(a, m, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(la, lm, rtol=1e-14)


# ------------------------------------------------------------------ prefill
def _prefill_case(seed, T=96, d=16, hq=4, n_kv=2):
    rng = np.random.default_rng(seed)
    K, V = _hist(rng, 1, n_kv, T, d)
    Q = _rand(rng, 1, hq, T, d)
    return K, V, Q


def test_prefill_retrieval_rows_equal_causal_sdpa():
    """Chunk rows after a cached prefix P equal rows P.. of one-shot causal
    attention over the whole sequence (torch SDPA, is_causal) -- the
    offset-causal rule of "When Is Reuse Exact?"."""
    K, V, Q = _prefill_case(1)
    T, P, C = 96, 40, 56
    mask = np.array([1, 1], np.uint8)
    out = O.prefill_attention(Q[:, :, P:P + C], lambda b, g: K[b, g], lambda b, g: V[b, g],
                              [P], mask, 4, 8, 0.25)
    for h in range(4):
        g = h // 2
        full = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(Q[0, h])[None], torch.from_numpy(K[0, g])[None],
            torch.from_numpy(V[0, g])[None], is_causal=True, scale=0.25)[0].numpy()
        np.testing.assert_allclose(out[0, h], full[P:P + C], rtol=1e-12, atol=1e-12)
    # the naive upper-left C x (P+C) triangle hides cached keys and gives other rows
    naive = np.tril(np.ones((C, P + C), dtype=bool))
    got_naive = _sdpa(Q[0, 0, P:P + C], K[0, 0], V[0, 0], naive, 0.25)
    assert np.abs(got_naive - out[0, 0]).max() > 1e-3


def test_prefill_streaming_rows_equal_ring_contents():
    """Each streaming row reads exactly what a ring holds right after its own
    token was appended (literal simulation, then torch SDPA)."""
    K, V, Q = _prefill_case(2)
    T, P, C, S, W = 96, 30, 66, 5, 12
    mask = np.array([0, 0], np.uint8)
    out = O.prefill_attention(Q[:, :, P:P + C], lambda b, g: K[b, g], lambda b, g: V[b, g],
                              [P], mask, S, W, 0.3)
    ring = O.StreamingCache(S, W)
    rows = []
    for p in range(T):
        ring.append(p)
        if p >= P:
            m = np.zeros(T, dtype=bool)
            m[[x for x in ring.pos if x >= 0]] = True
            rows.append(m)
    rows = np.stack(rows)
    for h in range(4):
        want = _sdpa(Q[0, h, P:P + C], K[0, h // 2], V[0, h // 2], rows, 0.3)
        np.testing.assert_allclose(out[0, h], want, rtol=1e-12, atol=1e-12)


def test_chunked_equals_one_shot_and_last_row_equals_decode():
    K, V, Q = _prefill_case(3)
    T = 96
    mask = np.array([1, 0], np.uint8)
    kh, vh = (lambda b, g: K[b, g]), (lambda b, g: V[b, g])
    one = O.prefill_attention(Q, kh, vh, [0], mask, 4, 10, 0.25)
    parts = []
    for P, C in [(0, 32), (32, 40), (72, 24)]:
        parts.append(O.prefill_attention(Q[:, :, P:P + C], kh, vh, [P], mask, 4, 10, 0.25))
    np.testing.assert_allclose(np.concatenate(parts, axis=2), one, rtol=1e-13, atol=1e-13)
    dec, _ = O.decode_attention(Q[:, :, T - 1], kh, vh, [T], mask, 4, 10, 0.25)
    np.testing.assert_allclose(one[:, :, T - 1], dec, rtol=1e-13, atol=1e-13)
    # sampled rows equal the full evaluation
    some = O.prefill_attention(Q, kh, vh, [0], mask, 4, 10, 0.25, rows=[0, 5, 95])
    np.testing.assert_allclose(some[:, :, [0, 5, 95]], one[:, :, [0, 5, 95]], rtol=0, atol=0)


# ------------------------------------------------------------------ planted mistakes
def _fails(fn, *a, **kw):
    try:
        fn(*a, **kw)
    except AssertionError:
        return True
    return False


def test_planted_window_off_by_one_is_caught(monkeypatch):
    def bad_keep(t, sink, window):
        j = np.arange(t + 1)
        return j[(j < sink) | (j >= t - window)]
    monkeypatch.setattr(O, "keep_set", bad_keep)
    assert _fails(test_ring_matches_list_simulation, 0)
    assert _fails(test_decode_matches_sdpa_with_ring_contents, 4, 8, 30)


def test_planted_ring_slot_error_is_caught(monkeypatch):
    orig = O.StreamingCache.append

    def bad_append(self, position, item=None):
        if self.n_sink < self.sink:
            return orig(self, position, item)
        slot = self.sink + (position % self.window)   # forgets to count from the sinks
        self.n_window += 1
        self.pos[slot] = position
        self.items[slot] = item
        return slot
    monkeypatch.setattr(O.StreamingCache, "append", bad_append)
    assert _fails(test_worked_positions_tiny_config)
    monkeypatch.setattr(O.StreamingCache, "append", orig)


def test_planted_gqa_mapping_error_is_caught(monkeypatch):
    monkeypatch.setattr(O, "kv_head_of", lambda h, hq, n_kv: h % n_kv)
    assert _fails(test_gqa_equals_mha_with_repeated_kv)


def test_planted_causal_offset_error_is_caught(monkeypatch):
    orig = O.key_mask

    def upper_left(rows_t, n_keys, retrieval, sink, window):
        t = np.asarray(rows_t)
        return orig(t - t.min(), n_keys, retrieval, sink, window)
    monkeypatch.setattr(O, "key_mask", upper_left)
    assert _fails(test_prefill_retrieval_rows_equal_causal_sdpa)


def test_planted_missing_scale_is_caught(monkeypatch):
    orig = O.attend
    monkeypatch.setattr(O, "attend", lambda q, k, v, scale: orig(q, k, v, 1.0))
    assert _fails(test_decode_matches_sdpa_with_ring_contents, 4, 8, 30)


def test_planted_size_factor_error_is_caught(monkeypatch):
    monkeypatch.setattr(O, "kv_cache_bytes", lambda L, n, d, T, elem_bytes=2: elem_bytes * L * n * d * T)
    assert _fails(test_dense_sizes_match_printed_values)


# ------------------------------------------------------------------ gated forward, split sums
def test_blended_decode_reduces_to_full_and_streaming_and_is_linear():
    """alpha = 1 is full attention (every head retrieval), alpha = 0 is the
    sink + window attention (every head streaming), and the gate mixes the two
    linearly (DuoAttention guide, section 3, item 2)."""
    rng = np.random.default_rng(21)
    B, hq, n_kv, d, T = 2, 8, 4, 16, 70
    K, V = _hist(rng, B, n_kv, T, d)
    q = _rand(rng, B, hq, d)
    kh, vh = (lambda b, g: K[b, g]), (lambda b, g: V[b, g])
    lens = [T, T - 20]
    full, _ = O.decode_attention(q, kh, vh, lens, np.ones(n_kv, np.uint8), 4, 16, 0.3)
    strm, _ = O.decode_attention(q, kh, vh, lens, np.zeros(n_kv, np.uint8), 4, 16, 0.3)
    np.testing.assert_allclose(O.blended_decode(q, kh, vh, lens, n_kv, np.ones(hq), 4, 16, 0.3), full,
                               rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(O.blended_decode(q, kh, vh, lens, n_kv, np.zeros(hq), 4, 16, 0.3), strm,
                               rtol=1e-14, atol=1e-14)
    a = rng.uniform(0, 1, hq)
    mix = O.blended_decode(q, kh, vh, lens, n_kv, a, 4, 16, 0.3)
    np.testing.assert_allclose(mix, a[None, :, None] * full + (1 - a[None, :, None]) * strm, rtol=1e-13,
                               atol=1e-14)
    assert np.abs(full - strm).max() > 1e-3


def test_attention_over_a_union_is_the_lse_weighted_mix_of_its_parts():
    """The identity sequence-split decode and the two-range streaming
    attention rely on: softmax attention over disjoint key sets joined by
    their log-sum-exps equals attention over the union (brute force)."""
    rng = np.random.default_rng(22)
    d, T = 8, 40
    q, k, v = _rand(rng, d), _rand(rng, T, d), _rand(rng, T, d)
    cuts = [0, 7, 8, 25, 40]
    parts = [O.attend(q, k[a:b], v[a:b], 0.4) for a, b in zip(cuts[:-1], cuts[1:])]
    lse = np.array([p[1] for p in parts])
    LSE = np.log(np.exp(lse - lse.max()).sum()) + lse.max()
    mixed = sum(np.exp(l - LSE) * o for o, l in parts)
    want, want_lse = O.brute_force_attention(q, k, v, list(range(T)), 0.4)
    np.testing.assert_allclose(mixed, want, rtol=1e-12, atol=1e-13)
    assert LSE == pytest.approx(want_lse, rel=1e-13)


# ------------------------------------------------------------------ FP8 (E4M3) KV codes
def _torch_codes(x32):
    """E4M3 bytes from torch's float8_e4m3fn conversion (a library routine)."""
    return torch.from_numpy(np.asarray(x32, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_decode_closed_forms_and_library_table():
    v = O.e4m3_decode([0x00, 0x01, 0x07, 0x08, 0x38, 0x3F, 0x7E, 0x80, 0xB8, 0xFE])
    assert list(v) == [0.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 1.0, 1.875, 448.0, -0.0, -1.0, -448.0]
    assert np.signbit(v[7])
    assert np.isnan(O.e4m3_decode([0x7F, 0xFF])).all()
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = O.e4m3_decode(codes)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok]) and np.array_equal(np.signbit(ours[ok]), np.signbit(ref[ok]))


def test_e4m3_encode_matches_library_in_range():
    rng = np.random.default_rng(11)
    mag = np.exp2(rng.uniform(-13, np.log2(440.0), 20000))
    x = (mag * rng.choice([-1.0, 1.0], mag.size)).astype(np.float32)
    pos = O.e4m3_decode(np.arange(0x7E))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)            # every tie between neighbours
    x = np.concatenate([x, mids, -mids, np.float32([0.0, -0.0, 1e-30, -1e-30])])
    assert np.array_equal(O.e4m3_encode(x.astype(np.float64)), _torch_codes(x))


def test_e4m3_ties_saturation_nan_and_round_trip():
    # ties go to the even mantissa
    assert list(O.e4m3_encode([2.0 ** -10, 3 * 2.0 ** -10, 1.0625, 1.1875])) == [0x00, 0x02, 0x38, 0x3A]
    # magnitudes beyond the largest finite value saturate to it, sign kept
    assert list(O.e4m3_encode([448.0, 460.0, 464.0, 1e6, -1e6, np.inf])) == [0x7E] * 4 + [0xFE, 0x7E]
    assert O.e4m3_encode([np.nan])[0] == 0x7F
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)])
    assert np.array_equal(O.e4m3_encode(O.e4m3_decode(finite)), finite.astype(np.uint8))


def test_quantize_kv_is_one_fp32_division_then_e4m3():
    rng = np.random.default_rng(12)
    x = torch.randn(4096, dtype=torch.float32).to(torch.bfloat16).float().numpy()
    for s in (1.0, 0.37, 3.0, 1 / 64):
        q32 = (torch.from_numpy(x) / torch.tensor(s, dtype=torch.float32)).numpy()
        assert np.array_equal(O.quantize_kv(x, s), _torch_codes(q32))
        back = O.dequantize_kv(O.quantize_kv(x, s), s)
        # relative error of E4M3 (3 mantissa bits) is at most 2^-4 above the subnormal range
        big = np.abs(x / s) >= 2.0 ** -6
        assert np.all(np.abs(back[big] - x[big]) <= 2.0 ** -4 * np.abs(x[big]) + 1e-12)


def test_planted_e4m3_bias_error_is_caught(monkeypatch):
    def wrong(codes):
        c = np.asarray(codes, dtype=np.int64) & 0xFF
        e = (c >> 3) & 0xF
        m = (c & 0x7).astype(np.float64)
        mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 8.0))   # bias 8
        return np.where(c & 0x80, -1.0, 1.0) * np.where((e == 15) & (m == 7), np.nan, mag)
    monkeypatch.setattr(O, "e4m3_decode", wrong)
    with pytest.raises(AssertionError):
        test_e4m3_decode_closed_forms_and_library_table()


def test_planted_e4m3_ties_away_is_caught(monkeypatch):
    real = O.e4m3_encode

    def away(x):
        x = np.asarray(x, dtype=np.float64)
        nudged = x * (1 + 2.0 ** -40)          # ties resolve away from zero
        return real(nudged)
    monkeypatch.setattr(O, "e4m3_encode", away)
    with pytest.raises(AssertionError):
        test_e4m3_ties_saturation_nan_and_round_trip()


# ------------------------------------------------------------------ INT4 KV codes
def test_int4_encode_closed_forms():
    # nearest integer, ties to the even one, clamped to [-8, 7]
    x = [0.0, 0.49, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.51, 6.5, 7.4, 7.5, 100.0, -7.5, -8.4, -8.5, -100.0, np.nan]
    assert list(O.int4_encode(x)) == [0, 0, 0, 2, 2, 0, -2, -2, 4, 6, 7, 7, 7, -8, -8, -8, -8, 0]
    # every code is reached exactly by its own value
    assert list(O.int4_encode(np.arange(-8, 8))) == list(range(-8, 8))


def test_int4_encode_matches_library_rounding():
    """torch.round rounds half to even (a library routine); clamp is a clamp."""
    rng = np.random.default_rng(21)
    x = np.concatenate([rng.uniform(-10, 10, 20000), np.arange(-10.5, 10.5, 0.5)]).astype(np.float32)
    lib = torch.from_numpy(x).round().clamp(-8, 7).to(torch.int8).numpy()
    assert np.array_equal(O.int4_encode(x.astype(np.float64)), lib)


def test_int4_pack_layout_and_round_trip():
    # element 2i in the low nibble, 2i+1 in the high nibble, two's complement
    assert list(O.int4_pack([1, -1, -8, 7, 0, 3])) == [0xF1, 0x78, 0x30]
    assert list(O.int4_unpack([0xF1, 0x78, 0x30])) == [1, -1, -8, 7, 0, 3]
    every = np.array([[a, b] for a in range(-8, 8) for b in range(-8, 8)])      # all 256 bytes
    packed = O.int4_pack(every)[:, 0]
    assert sorted(packed.tolist()) == list(range(256))
    assert np.array_equal(O.int4_unpack(packed[:, None]), every)


def test_quantize_kv_int4_is_one_fp32_division_then_rounding():
    x = torch.randn(4096, dtype=torch.float32).to(torch.bfloat16).float().numpy().reshape(32, 128)
    for s in (1.0, 0.37, 0.3, 1 / 64):
        q32 = (torch.from_numpy(x) / torch.tensor(s, dtype=torch.float32)).round().clamp(-8, 7).to(torch.int64)
        codes = q32.numpy()
        want = ((codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)).astype(np.uint8)
        assert np.array_equal(O.quantize_kv_int4(x, s), want)
        back = O.dequantize_kv_int4(O.quantize_kv_int4(x, s), s)
        inside = (x / s >= -8.5) & (x / s <= 7.5)
        # within the grid the error is at most half a step (plus the fp32 division's rounding)
        assert np.all(np.abs(back[inside] - x[inside]) <= 0.5 * np.float32(s) * (1 + 1e-6) + 1e-12)
    # a value whose fp32 quotient is an exact tie while the fp64 quotient is
    # above it: 1.75 / fp32(0.7) is 2.5 in fp32 (code 2), 2.50000004 in fp64 (3)
    s = np.float32(0.7)
    v = np.float32(1.75)
    assert np.float32(v / s) == np.float32(2.5) and float(v) / float(s) > 2.5
    assert O.int4_unpack(O.quantize_kv_int4(np.array([v, v]), float(s)))[0] == 2


def test_planted_int4_ties_away_is_caught(monkeypatch):
    def wrong(x):
        x = np.asarray(x, dtype=np.float64)
        x = np.where(np.isnan(x), 0.0, x)
        r = np.sign(x) * np.floor(np.abs(x) + 0.5)                       # half away from zero
        return np.clip(r, -8, 7).astype(np.int8)
    monkeypatch.setattr(O, "int4_encode", wrong)
    with pytest.raises(AssertionError):
        test_int4_encode_closed_forms()


def test_planted_int4_nibble_swap_is_caught(monkeypatch):
    def wrong(codes):
        c = np.asarray(codes, dtype=np.int64)
        return ((c[..., 1::2] & 0xF) | ((c[..., 0::2] & 0xF) << 4)).astype(np.uint8)
    monkeypatch.setattr(O, "int4_pack", wrong)
    with pytest.raises(AssertionError):
        test_int4_pack_layout_and_round_trip()
