"""C ABI checks that need no GPU: the library loads, exports every function
include/duo_kv.h declares, sizes caches by the method's memory equation, and
rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import numpy as np
import pytest

import duo_workloads as W
from oracle import duo_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lib():
    from head_wise_kv_b200 import _lib as L
    return L


def declared_functions():
    names = []
    for f in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            names += re.findall(r"^DUO_API\s+[\w\s\*]*?\b(duo_\w+)\s*\(", src, flags=re.M)
    return names


def test_library_exports_every_declared_function():
    L = _lib()
    names = declared_functions()
    assert len(names) >= 12
    raw = ctypes.CDLL(L.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), f"{n} declared in include/ but not exported"
    assert set(L.EXPORTED) <= set(names)


def _desc(L, layers=2, B=3, hq=32, n_kv=8, d=128, S=64, Wn=256, cap=1000, mask=None):
    if mask is None:
        mask = np.zeros((layers, n_kv), np.uint8)
        mask[:, ::2] = 1
    return L.make_desc(layers, B, hq, n_kv, d, S, Wn, cap, np.asarray(mask, np.uint8).tobytes())


@pytest.mark.parametrize("cfg", ["tiny", "mha32k", "gqa128k", "mtok", "prefill64k"])
def test_cache_bytes_follow_memory_equation(cfg):
    """The K/V bytes the library lays out equal the batch times the Duo memory
    equation (oracle) with T = capacity and the per-layer retrieval counts."""
    L = _lib()
    w = W.WORKLOADS[cfg]
    masks = W.retrieval_masks(w)
    cap = W.capacity(w)
    d, keep = L.make_desc(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, cap, masks.tobytes())
    total, cache = L.duo_kv_required_bytes(d)
    want = w.batch * O.duo_cache_bytes(w.layers, w.n_kv, w.d, cap, w.sink, w.window, masks.sum(1).tolist())
    assert cache == want
    pos_bytes = w.layers * w.batch * (w.sink + w.window) * 4
    assert want + pos_bytes <= total <= want + pos_bytes + 256 * (6 * w.layers + 1)


def test_guide_example_bytes():
    """80 layers, 8 KV heads (2 retrieval), d=128, T=128,000, S=32, W=128:
    the guide's 32,120-token effective context times the dense bytes per token."""
    L = _lib()
    mask = np.zeros((80, 8), np.uint8)
    mask[:, :2] = 1
    d, keep = _desc(L, layers=80, B=1, hq=64, n_kv=8, d=128, S=32, Wn=128, cap=128000, mask=mask)
    assert L.duo_kv_required_bytes(d)[1] == 10525081600


@pytest.mark.parametrize("field,value,code", [
    ("head_dim", 96, -2), ("head_dim", 256, -2), ("window", 0, -1), ("sink", -1, -1),
    ("num_q_heads", 24, -2), ("num_q_heads", 30, -1), ("capacity", 0, -1), ("num_kv_heads", 0, -1),
    ("batch", 0, -1), ("num_layers", 0, -1), ("capacity", 1 << 40, -1),
])
def test_rejects_bad_shapes(field, value, code):
    L = _lib()
    d, keep = _desc(L)
    setattr(d, field, value)
    with pytest.raises(L.DuoError) as e:
        L.duo_kv_required_bytes(d)
    assert e.value.code == code


def test_rejects_more_than_64_kv_heads():
    L = _lib()
    d, keep = _desc(L, hq=128, n_kv=128, mask=np.zeros((2, 128), np.uint8))
    with pytest.raises(L.DuoError) as e:
        L.duo_kv_required_bytes(d)
    assert e.value.code == L.DUO_ERR_UNSUPPORTED


def test_alloc_argument_checks_before_cuda():
    L = _lib()
    d, keep = _desc(L)
    total, _ = L.duo_kv_required_bytes(d)
    with pytest.raises(L.DuoError) as e:
        L.duo_kv_alloc(d, 0, total, 0)
    assert e.value.code == L.DUO_ERR_INVALID_ARG
    with pytest.raises(L.DuoError) as e:
        L.duo_kv_alloc(d, 0x1000 + 16, total, 0)        # not 256-byte aligned
    assert e.value.code == L.DUO_ERR_ALIGNMENT
    with pytest.raises(L.DuoError) as e:
        L.duo_kv_alloc(d, 0x100000, total - 1, 0)       # too small
    assert e.value.code == L.DUO_ERR_BUFFER_TOO_SMALL


def test_null_handle_calls_fail_cleanly():
    L = _lib()
    for fn, args in [(L.duo_kv_append, (None, 0, 16, 16, 16, None, 1, None)),
                     (L.duo_decode_attn, (None, 0, 16, 16, 0.1, 16, None, 16, 1 << 20, None)),
                     (L.duo_prefill_attn, (None, 0, 16, 16, 16, 16, 8, 0.1, 16, None, 0, None)),
                     (L.duo_kv_fork, (None, 0, 1, 10, None)),
                     # step: null handle, then a null len_before / len (checked before any launch)
                     (L.duo_decode_step, (None, 0, 16, 16, 16, 16, 16, 0.1, 16, None, 16, 1 << 20, None)),
                     (L.duo_decode_step, (None, 0, 16, 16, None, 16, 16, 0.1, 16, None, 16, 1 << 20, None)),
                     (L.duo_decode_step, (None, 0, 16, 16, 16, 16, None, 0.1, 16, None, 16, 1 << 20, None))]:
        with pytest.raises(L.DuoError) as e:
            fn(*args)
        assert e.value.code == L.DUO_ERR_INVALID_ARG
    with pytest.raises(L.DuoError) as e:   # len_before not 4-byte aligned
        L.duo_decode_step(None, 0, 16, 16, 18, 16, 16, 0.1, 16, None, 16, 1 << 20, None)
    assert e.value.code == L.DUO_ERR_ALIGNMENT
    assert L._c_free(None) == 0


def test_strerror_covers_codes():
    L = _lib()
    for c in range(0, -7, -1):
        assert L.duo_strerror(c) != "unknown error"
    assert L.duo_strerror(-99) == "unknown error"


@pytest.mark.parametrize("cfg", ["mha32k", "gqa128k", "mtok"])
def test_fp8_cache_bytes_follow_memory_equation_at_one_byte(cfg):
    """FP8 caches: the same memory equation with one byte per element
    (the guide's 8 instead of 16 bits), i.e. half the bf16 bytes."""
    L = _lib()
    w = W.WORKLOADS[cfg]
    masks = W.retrieval_masks(w)
    cap = W.capacity(w)
    d, keep = L.make_desc(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, cap, masks.tobytes(),
                          L.DUO_KV_FP8_E4M3)
    _, cache = L.duo_kv_required_bytes(d)
    want = w.batch * O.duo_cache_bytes(w.layers, w.n_kv, w.d, cap, w.sink, w.window, masks.sum(1).tolist(),
                                       elem_bytes=1)
    assert cache == want
    d16, keep16 = L.make_desc(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, cap, masks.tobytes())
    assert 2 * cache == L.duo_kv_required_bytes(d16)[1]


def test_fp8_descriptor_checks():
    L = _lib()
    n = 2 * 8
    d, keep = _desc(L)
    d.kv_dtype = 7
    with pytest.raises(L.DuoError) as e:
        L.duo_kv_required_bytes(d)
    assert e.value.code == L.DUO_ERR_INVALID_ARG
    d, keep = _desc(L, d=64, hq=8)
    d.kv_dtype = L.DUO_KV_FP8_E4M3
    with pytest.raises(L.DuoError) as e:
        L.duo_kv_required_bytes(d)
    assert e.value.code == L.DUO_ERR_UNSUPPORTED
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        mask = np.zeros((2, 8), np.uint8)
        d, keep = L.make_desc(2, 3, 32, 8, 128, 64, 256, 1000, mask.tobytes(), L.DUO_KV_FP8_E4M3,
                              [1.0] * (n - 1) + [bad], None)
        with pytest.raises(L.DuoError) as e:
            L.duo_kv_required_bytes(d)
        assert e.value.code == L.DUO_ERR_INVALID_ARG
    d, keep = L.make_desc(2, 3, 32, 8, 128, 64, 256, 1000, np.zeros((2, 8), np.uint8).tobytes(),
                          L.DUO_KV_FP8_E4M3, [0.5] * n, [2.0] * n)
    assert L.duo_kv_required_bytes(d)[1] > 0


@pytest.mark.parametrize("cfg", ["mha32k", "gqa128k", "mtok"])
def test_int4_cache_bytes_follow_memory_equation_at_half_a_byte(cfg):
    """INT4 caches: the memory equation with 4 bits per element (the guide's
    4x cut), i.e. a quarter of the bf16 bytes."""
    L = _lib()
    w = W.WORKLOADS[cfg]
    masks = W.retrieval_masks(w)
    cap = W.capacity(w)
    d, keep = L.make_desc(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, cap, masks.tobytes(),
                          L.DUO_KV_INT4)
    _, cache = L.duo_kv_required_bytes(d)
    want = w.batch * O.duo_cache_bytes(w.layers, w.n_kv, w.d, cap, w.sink, w.window, masks.sum(1).tolist(),
                                       elem_bytes=0.5)
    assert cache == want
    d16, keep16 = L.make_desc(w.layers, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, cap, masks.tobytes())
    assert 4 * cache == L.duo_kv_required_bytes(d16)[1]


def test_int4_descriptor_checks():
    L = _lib()
    n = 2 * 8
    d, keep = _desc(L, d=64, hq=8)
    d.kv_dtype = L.DUO_KV_INT4
    with pytest.raises(L.DuoError) as e:
        L.duo_kv_required_bytes(d)
    assert e.value.code == L.DUO_ERR_UNSUPPORTED
    mask = np.zeros((2, 8), np.uint8)
    d, keep = L.make_desc(2, 3, 32, 8, 128, 64, 256, 1000, mask.tobytes(), L.DUO_KV_INT4, None,
                          [1.0] * (n - 1) + [0.0])
    with pytest.raises(L.DuoError) as e:
        L.duo_kv_required_bytes(d)
    assert e.value.code == L.DUO_ERR_INVALID_ARG


def test_paged_cache_bytes_and_checks():
    """Paged retrieval caches: each layer's retrieval part is a pool of
    num_pages pages of n_r x page_tokens rows (streaming rings unchanged)."""
    L = _lib()
    layers, B, n_kv, d, S, Wn = 2, 3, 8, 128, 64, 256
    mask = np.zeros((layers, n_kv), np.uint8)
    mask[:, ::2] = 1                              # 4 retrieval heads per layer
    d0, k0 = L.make_desc(layers, B, 32, n_kv, d, S, Wn, 1000, mask.tobytes(), L.DUO_KV_BF16, None, None, 256, 10)
    _, cache = L.duo_kv_required_bytes(d0)
    want = layers * (2 * 2 * d * (10 * 4 * 256) + B * 2 * 2 * d * 4 * (S + Wn))
    assert cache == want
    d8, k8 = L.make_desc(layers, B, 32, n_kv, d, S, Wn, 1000, mask.tobytes(), L.DUO_KV_FP8_E4M3, None, None, 256,
                         10)
    assert L.duo_kv_required_bytes(d8)[1] * 2 == want
    for pt, npg, code in ((100, 10, L.DUO_ERR_INVALID_ARG), (256, 0, L.DUO_ERR_INVALID_ARG),
                          (-256, 10, L.DUO_ERR_INVALID_ARG)):
        dd, kk = L.make_desc(layers, B, 32, n_kv, d, S, Wn, 1000, mask.tobytes(), L.DUO_KV_BF16, None, None, pt,
                             npg)
        with pytest.raises(L.DuoError) as e:
            L.duo_kv_required_bytes(dd)
        assert e.value.code == code
    dd, kk = L.make_desc(layers, B, 8, n_kv, 64, S, Wn, 1000, mask.tobytes(), L.DUO_KV_BF16, None, None, 256, 10)
    with pytest.raises(L.DuoError) as e:
        L.duo_kv_required_bytes(dd)
    assert e.value.code == L.DUO_ERR_UNSUPPORTED


def test_merge_blend_and_row_calls_check_arguments_before_cuda():
    """Argument errors come back as codes before any launch; empty work is a
    no-op that succeeds (fake, never dereferenced addresses stand in for
    device pointers)."""
    L = _lib()
    P = 0x100000          # 256-byte aligned stand-in address
    bad = [
        (L.duo_lse_merge, (0, 4, 64, P, P, P, P, None), L.DUO_ERR_INVALID_ARG),      # no parts
        (L.duo_lse_merge, (2, -1, 64, P, P, P, P, None), L.DUO_ERR_INVALID_ARG),     # negative rows
        (L.duo_lse_merge, (2, 4, 0, P, P, P, P, None), L.DUO_ERR_INVALID_ARG),       # d = 0
        (L.duo_lse_merge, (2, 4, 64, None, P, P, P, None), L.DUO_ERR_INVALID_ARG),   # no partial outputs
        (L.duo_lse_merge, (2, 4, 64, P, P, None, P, None), L.DUO_ERR_INVALID_ARG),   # no output
        (L.duo_lse_merge, (2, 4, 64, P + 2, P, P, P, None), L.DUO_ERR_ALIGNMENT),    # fp32 misaligned
        (L.duo_alpha_blend, (-1, 8, 64, P, P, P, P, None), L.DUO_ERR_INVALID_ARG),
        (L.duo_alpha_blend, (2, 0, 64, P, P, P, P, None), L.DUO_ERR_INVALID_ARG),
        (L.duo_alpha_blend, (2, 8, 64, None, P, P, P, None), L.DUO_ERR_INVALID_ARG),
        (L.duo_alpha_blend, (2, 8, 64, P, P, P + 1, P, None), L.DUO_ERR_ALIGNMENT),
        (L.duo_decode_attn_rows, (None, 0, P, None, P, None, 0.1, P, P, P, 1 << 20, None), L.DUO_ERR_INVALID_ARG),
        (L.duo_kv_append_rows, (None, 0, P, P, P, None, 1, P, P, None), L.DUO_ERR_INVALID_ARG),
        (L.duo_kv_set_page_table, (None, P, 4), L.DUO_ERR_INVALID_ARG),
        (L.duo_kv_check_wait_timeout, (None, 1000, None), L.DUO_ERR_INVALID_ARG),
    ]
    for fn, args, code in bad:
        with pytest.raises(L.DuoError) as e:
            fn(*args)
        assert e.value.code == code, (fn.__name__, args)
    L.duo_lse_merge(3, 0, 64, P, P, P, P, None)          # no rows: nothing to launch
    L.duo_alpha_blend(0, 8, 64, P, P, P, P, None)        # no sequences: nothing to launch


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "duo_kv.h"

int main(void) {
    /* 2 layers, batch 3, 32 query / 8 KV heads, d = 128, S = 64, W = 256,
       capacity 1000, even KV heads retrieval, bf16 */
    uint8_t mask[2 * 8];
    for (int i = 0; i < 16; ++i) mask[i] = (i % 2) == 0;
    duo_kv_desc d;
    memset(&d, 0, sizeof d);
    d.num_layers = 2; d.batch = 3; d.num_q_heads = 32; d.num_kv_heads = 8; d.head_dim = 128;
    d.sink = 64; d.window = 256; d.capacity = 1000; d.retrieval_mask = mask; d.kv_dtype = DUO_KV_BF16;
    size_t total = 0, cache = 0;
    int rc = duo_kv_required_bytes(&d, &total, &cache);
    d.head_dim = 96;
    int bad = duo_kv_required_bytes(&d, &total, NULL);
    duo_kv* h = NULL;
    int nul = duo_kv_alloc(NULL, NULL, 0, NULL, &h);
    printf("%d %zu %zu %d %d %s\n", rc, total, cache, bad, nul, duo_strerror(bad));
    return 0;
}
"""


def test_header_is_plain_c_and_links(tmp_path):
    """include/duo_kv.h compiles as C99 and a C program linked to
    libduo_kv.so sizes a cache exactly as the Python binding does."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc") or shutil.which("cc")
    if gcc is None:
        pytest.skip("no C compiler")
    L = _lib()
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(L.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", libdir, "-lduo_kv", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    d, keep = _desc(L)
    total, cache = L.duo_kv_required_bytes(d)
    assert [int(x) for x in out[:5]] == [0, total, cache, L.DUO_ERR_UNSUPPORTED, L.DUO_ERR_INVALID_ARG]
    assert " ".join(out[5:]) == L.duo_strerror(L.DUO_ERR_UNSUPPORTED)
