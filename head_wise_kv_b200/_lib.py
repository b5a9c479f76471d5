"""ctypes binding of libduo_kv.so (include/duo_kv.h), argument marshalling only.

Every function keeps the C name and takes plain integers for device
pointers and streams; ``DuoKVCache`` below adds a torch-owned buffer and
tensor checks on top.  There is no fallback: if the shared library is
missing this module raises on import.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libduo_kv.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m head_wise_kv_b200.build` "
        "(there is no CPU or Python fallback for the CUDA path)")

_lib = ctypes.CDLL(LIB_PATH)

DUO_OK = 0
DUO_ERR_INVALID_ARG = -1
DUO_ERR_UNSUPPORTED = -2
DUO_ERR_BUFFER_TOO_SMALL = -3
DUO_ERR_WORKSPACE = -4
DUO_ERR_CUDA = -5
DUO_ERR_ALIGNMENT = -6

DUO_KV_BF16 = 0
DUO_KV_FP8_E4M3 = 1
DUO_KV_INT4 = 2

DUO_STATUS_OVER_CAPACITY = 1
DUO_STATUS_EMPTY_SEQUENCE = 2
DUO_STATUS_WAIT_TIMEOUT = 4
DUO_STATUS_BAD_LENGTH = 8
DUO_STATUS_NO_PAGE = 16
DUO_STATUS_SHARED_PAGE = 32

# C entry points declared in include/duo_kv.h (checked by the CPU tests)
EXPORTED = (
    "duo_kv_required_bytes", "duo_kv_alloc", "duo_kv_free", "duo_kv_layer_view_get",
    "duo_kv_append", "duo_decode_workspace_bytes", "duo_decode_attn",
    "duo_prefill_workspace_bytes", "duo_prefill_attn", "duo_kv_read_status",
    "duo_kv_set_decode_ctas", "duo_strerror", "duo_decode_attn_static_ws",
    "duo_kv_append_rows", "duo_decode_attn_rows", "duo_lse_merge", "duo_alpha_blend", "duo_kv_set_page_table",
    "duo_kv_fork", "duo_kv_check_wait_timeout", "duo_decode_step",
)
DUO_STATIC_WS_BYTES = 4 << 20


class duo_kv_desc(ctypes.Structure):
    _fields_ = [
        ("num_layers", ctypes.c_int32),
        ("batch", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("sink", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("capacity", ctypes.c_int64),
        ("retrieval_mask", ctypes.POINTER(ctypes.c_uint8)),
        ("kv_dtype", ctypes.c_int32),
        ("k_scale", ctypes.POINTER(ctypes.c_float)),
        ("v_scale", ctypes.POINTER(ctypes.c_float)),
        ("page_tokens", ctypes.c_int32),
        ("num_pages", ctypes.c_int64),
    ]


class duo_kv_layer_view(ctypes.Structure):
    _fields_ = [
        ("k_retrieval", ctypes.c_void_p),
        ("v_retrieval", ctypes.c_void_p),
        ("k_streaming", ctypes.c_void_p),
        ("v_streaming", ctypes.c_void_p),
        ("positions", ctypes.c_void_p),
        ("n_retrieval", ctypes.c_int32),
        ("n_streaming", ctypes.c_int32),
        ("head_rank", ctypes.c_int32 * 64),
        ("is_retrieval", ctypes.c_uint8 * 64),
    ]


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_SZ = ctypes.c_size_t


def _sig(name, args, res=ctypes.c_int):
    f = getattr(_lib, name)
    f.argtypes = args
    f.restype = res
    return f


_c_required = _sig("duo_kv_required_bytes", [ctypes.POINTER(duo_kv_desc), ctypes.POINTER(_SZ), ctypes.POINTER(_SZ)])
_c_alloc = _sig("duo_kv_alloc", [ctypes.POINTER(duo_kv_desc), _P, _SZ, _P, ctypes.POINTER(_P)])
_c_free = _sig("duo_kv_free", [_P])
_c_view = _sig("duo_kv_layer_view_get", [_P, _I32, ctypes.POINTER(duo_kv_layer_view)])
_c_append = _sig("duo_kv_append", [_P, _I32, _P, _P, _P, _P, _I32, _P])
_c_dec_ws = _sig("duo_decode_workspace_bytes", [_P, ctypes.POINTER(_SZ)])
_c_decode = _sig("duo_decode_attn", [_P, _I32, _P, _P, ctypes.c_float, _P, _P, _P, _SZ, _P])
_c_decode_static = _sig("duo_decode_attn_static_ws", [_P, _I32, _P, _P, ctypes.c_float, _P, _P, _P])
_c_append_rows = _sig("duo_kv_append_rows", [_P, _I32, _P, _P, _P, _P, _I32, _P, _P, _P])
_c_decode_rows = _sig("duo_decode_attn_rows", [_P, _I32, _P, _P, _P, _P, ctypes.c_float, _P, _P, _P, _SZ, _P])
_c_lse_merge = _sig("duo_lse_merge", [_I32, _I32, _I32, _P, _P, _P, _P, _P])
_c_blend = _sig("duo_alpha_blend", [_I32, _I32, _I32, _P, _P, _P, _P, _P])
_c_pre_ws = _sig("duo_prefill_workspace_bytes", [_P, _I32, ctypes.POINTER(_SZ)])
_c_prefill = _sig("duo_prefill_attn", [_P, _I32, _P, _P, _P, _P, _I32, ctypes.c_float, _P, _P, _SZ, _P])
_c_status = _sig("duo_kv_read_status", [_P, ctypes.POINTER(_I32), _I32, _P])
_c_set_ctas = _sig("duo_kv_set_decode_ctas", [_P, _I32])
_c_set_pages = _sig("duo_kv_set_page_table", [_P, _P, _I32])
_c_fork = _sig("duo_kv_fork", [_P, _I32, _I32, _I32, _P])
_c_waitcheck = _sig("duo_kv_check_wait_timeout", [_P, ctypes.c_uint64, _P])
_c_step = _sig("duo_decode_step", [_P, _I32, _P, _P, _P, _P, _P, ctypes.c_float, _P, _P, _P, _SZ, _P])
_c_strerror = _sig("duo_strerror", [ctypes.c_int], ctypes.c_char_p)


class DuoError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {duo_strerror(code)} ({code})")


def _check(code: int, what: str) -> None:
    if code != DUO_OK:
        raise DuoError(code, what)


def duo_strerror(code: int) -> str:
    return _c_strerror(code).decode()


def make_desc(num_layers, batch, num_q_heads, num_kv_heads, head_dim, sink, window, capacity, mask_u8,
              kv_dtype=DUO_KV_BF16, k_scale=None, v_scale=None, page_tokens=0, num_pages=0):
    """Build a duo_kv_desc; ``mask_u8`` is a host bytes-like [layers][n_kv];
    k_scale / v_scale optional float sequences [layers * n_kv] (FP8).  The
    host arrays are kept alive by the returned pair."""
    buf = (ctypes.c_uint8 * len(mask_u8)).from_buffer_copy(bytes(mask_u8))
    keep = [buf]

    def floats(x):
        if x is None:
            return None
        arr = (ctypes.c_float * len(x))(*[float(v) for v in x])
        keep.append(arr)
        return ctypes.cast(arr, ctypes.POINTER(ctypes.c_float))
    d = duo_kv_desc(num_layers, batch, num_q_heads, num_kv_heads, head_dim, sink, window, capacity,
                    ctypes.cast(buf, ctypes.POINTER(ctypes.c_uint8)), kv_dtype, floats(k_scale), floats(v_scale),
                    page_tokens, num_pages)
    return d, keep


def duo_kv_required_bytes(desc) -> tuple[int, int]:
    total, cache = _SZ(0), _SZ(0)
    _check(_c_required(ctypes.byref(desc), ctypes.byref(total), ctypes.byref(cache)), "duo_kv_required_bytes")
    return total.value, cache.value


def duo_kv_alloc(desc, dev_buf: int, buf_bytes: int, stream: int) -> int:
    h = _P()
    _check(_c_alloc(ctypes.byref(desc), dev_buf, buf_bytes, stream, ctypes.byref(h)), "duo_kv_alloc")
    return h.value


def duo_kv_free(handle: int) -> None:
    _check(_c_free(handle), "duo_kv_free")


def duo_kv_layer_view_get(handle: int, layer: int) -> duo_kv_layer_view:
    v = duo_kv_layer_view()
    _check(_c_view(handle, layer, ctypes.byref(v)), "duo_kv_layer_view_get")
    return v


def duo_kv_append(handle, layer, k_new, v_new, len_before, n_new, n_new_max, stream) -> None:
    _check(_c_append(handle, layer, k_new, v_new, len_before, n_new, n_new_max, stream), "duo_kv_append")


def duo_decode_workspace_bytes(handle) -> int:
    n = _SZ(0)
    _check(_c_dec_ws(handle, ctypes.byref(n)), "duo_decode_workspace_bytes")
    return n.value


def duo_decode_attn(handle, layer, q, length, scale, out, lse, workspace, workspace_bytes, stream) -> None:
    _check(_c_decode(handle, layer, q, length, scale, out, lse, workspace, workspace_bytes, stream),
           "duo_decode_attn")


def duo_decode_attn_static_ws(handle, layer, q, length, scale, out, lse, stream) -> None:
    _check(_c_decode_static(handle, layer, q, length, scale, out, lse, stream), "duo_decode_attn_static_ws")


def duo_kv_append_rows(handle, layer, k_new, v_new, len_before, n_new, n_new_max, r_pos_begin, r_pos_end,
                       stream) -> None:
    _check(_c_append_rows(handle, layer, k_new, v_new, len_before, n_new, n_new_max, r_pos_begin, r_pos_end,
                          stream), "duo_kv_append_rows")


def duo_decode_attn_rows(handle, layer, q, r_begin, r_end, s_len, scale, out, lse, workspace, workspace_bytes,
                         stream) -> None:
    _check(_c_decode_rows(handle, layer, q, r_begin, r_end, s_len, scale, out, lse, workspace, workspace_bytes,
                          stream), "duo_decode_attn_rows")


def duo_lse_merge(parts, rows, d, part_out, part_lse, out, lse, stream) -> None:
    _check(_c_lse_merge(parts, rows, d, part_out, part_lse, out, lse, stream), "duo_lse_merge")


def duo_alpha_blend(batch, num_q_heads, d, alpha, full_out, stream_out, out, stream) -> None:
    _check(_c_blend(batch, num_q_heads, d, alpha, full_out, stream_out, out, stream), "duo_alpha_blend")


def duo_prefill_workspace_bytes(handle, chunk) -> int:
    n = _SZ(0)
    _check(_c_pre_ws(handle, chunk, ctypes.byref(n)), "duo_prefill_workspace_bytes")
    return n.value


def duo_prefill_attn(handle, layer, q, k_chunk, v_chunk, prefix_len, chunk, scale, out, workspace,
                     workspace_bytes, stream) -> None:
    _check(_c_prefill(handle, layer, q, k_chunk, v_chunk, prefix_len, chunk, scale, out, workspace,
                      workspace_bytes, stream), "duo_prefill_attn")


def duo_kv_read_status(handle, clear: bool, stream: int) -> int:
    s = _I32(0)
    _check(_c_status(handle, ctypes.byref(s), int(bool(clear)), stream), "duo_kv_read_status")
    return s.value


def duo_kv_set_decode_ctas(handle, ctas: int) -> None:
    _check(_c_set_ctas(handle, ctas), "duo_kv_set_decode_ctas")


def duo_kv_set_page_table(handle, d_table: int, max_pages: int) -> None:
    _check(_c_set_pages(handle, d_table, max_pages), "duo_kv_set_page_table")


def duo_kv_fork(handle, src: int, dst: int, length: int, stream: int) -> None:
    _check(_c_fork(handle, src, dst, length, stream), "duo_kv_fork")


def duo_kv_check_wait_timeout(handle, limit_ns: int, stream: int) -> None:
    _check(_c_waitcheck(handle, limit_ns, stream), "duo_kv_check_wait_timeout")


def duo_decode_step(handle, layer, k_new, v_new, len_before, q, length, scale, out, lse, workspace,
                    workspace_bytes, stream) -> None:
    _check(_c_step(handle, layer, k_new, v_new, len_before, q, length, scale, out, lse, workspace, workspace_bytes,
                   stream), "duo_decode_step")
