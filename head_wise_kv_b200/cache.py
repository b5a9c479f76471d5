"""Torch-facing wrapper of the C ABI: owns the cache buffer and workspace as
torch tensors and passes their device pointers and the current stream to
libduo_kv.  Shape / dtype / device checks and pointer marshalling only --
every step of the path runs in the library's CUDA kernels."""
from __future__ import annotations

import numpy as np
import torch

from . import _lib as L


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _need(t: torch.Tensor, name: str, dtype, shape, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


class DuoKVCache:
    """Mixed-head KV cache for ``num_layers`` layers and ``batch`` sequences.

    retrieval_mask: [num_layers][num_kv_heads] (1 = retrieval KV head).
    kv_dtype: "bf16", "fp8" (E4M3 codes) or "int4" (signed 4-bit codes, two
    per byte); k_scale / v_scale per [num_layers][num_kv_heads], default 1.0.
    page_tokens > 0: paged retrieval caches, a pool of num_pages pages per
    layer; the page table (int32 [batch][max_pages] on the device) is given
    with set_page_table.
    """

    def __init__(self, num_layers, batch, num_q_heads, num_kv_heads, head_dim, sink, window, capacity,
                 retrieval_mask, device="cuda", kv_dtype="bf16", k_scale=None, v_scale=None, page_tokens=0,
                 num_pages=0):
        self.device = torch.device(device)
        if self.device.type != "cuda":
            raise ValueError("DuoKVCache lives on a CUDA device")
        if self.device.index is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        mask = np.asarray(retrieval_mask, dtype=np.uint8).reshape(num_layers, num_kv_heads)
        self.mask = mask.copy()
        self.L, self.B, self.hq, self.n_kv, self.d = num_layers, batch, num_q_heads, num_kv_heads, head_dim
        self.S, self.W, self.cap = sink, window, capacity
        if kv_dtype not in ("bf16", "fp8", "int4"):
            raise ValueError("kv_dtype must be 'bf16', 'fp8' or 'int4'")
        self.kv_dtype = kv_dtype
        self.fp8 = kv_dtype == "fp8"
        self.int4 = kv_dtype == "int4"

        def scales(x):
            if x is None:
                return np.ones((num_layers, num_kv_heads), dtype=np.float32)
            return np.asarray(x, dtype=np.float32).reshape(num_layers, num_kv_heads)
        self.k_scale, self.v_scale = scales(k_scale), scales(v_scale)
        self._desc, self._mask_buf = L.make_desc(
            num_layers, batch, num_q_heads, num_kv_heads, head_dim, sink, window, capacity, mask.tobytes(),
            {"bf16": L.DUO_KV_BF16, "fp8": L.DUO_KV_FP8_E4M3, "int4": L.DUO_KV_INT4}[kv_dtype],
            self.k_scale.ravel().tolist(),
            self.v_scale.ravel().tolist(), page_tokens, num_pages)
        self.page_tokens, self.num_pages = page_tokens, num_pages
        self._page_table = None
        self.total_bytes, self.cache_bytes = L.duo_kv_required_bytes(self._desc)
        with torch.cuda.device(self.device):
            self.buf = torch.empty(self.total_bytes, dtype=torch.uint8, device=self.device)
            self.handle = L.duo_kv_alloc(self._desc, self.buf.data_ptr(), self.total_bytes, _stream(self.device))
        self._ws = None
        self._alloc_workspace()

    # ------------------------------------------------------------ housekeeping
    def _alloc_workspace(self):
        n = L.duo_decode_workspace_bytes(self.handle)
        self._ws = torch.empty(max(n, 256), dtype=torch.uint8, device=self.device)

    def set_page_table(self, table):
        """table: int32 [batch][max_pages] on the cache's device (kept
        referenced; its contents may change between calls)."""
        if table.dtype != torch.int32 or table.dim() != 2 or table.shape[0] != self.B:
            raise ValueError("page table must be int32 [batch][max_pages]")
        if table.device != self.device or not table.is_contiguous():
            raise ValueError("page table must be a contiguous tensor on the cache's device")
        L.duo_kv_set_page_table(self.handle, table.data_ptr(), table.shape[1])
        self._page_table = table

    def fork(self, src: int, dst: int, length: int):
        """Sequence dst continues from the first ``length`` tokens of
        sequence src (every layer).  Paged caches share the pages that the
        page table maps to the same pool page for both; see duo_kv_fork."""
        L.duo_kv_fork(self.handle, src, dst, length, _stream(self.device))

    def check_wait_timeout(self, limit_ns: int):
        """Make one bounded device wait run out (see duo_kv_check_wait_timeout)."""
        L.duo_kv_check_wait_timeout(self.handle, limit_ns, _stream(self.device))

    def set_decode_ctas(self, ctas: int):
        L.duo_kv_set_decode_ctas(self.handle, ctas)
        self._alloc_workspace()

    def close(self):
        if getattr(self, "handle", None):
            L.duo_kv_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def status(self, clear: bool = True) -> int:
        return L.duo_kv_read_status(self.handle, clear, _stream(self.device))

    def layer_views(self, layer: int) -> dict:
        """Torch views of one layer's cache regions (see duo_kv_layer_view):
        bf16 tensors, uint8 E4M3 codes for an FP8 cache, or uint8 bytes of
        two INT4 codes each (last dimension d / 2) for an INT4 cache."""
        v = L.duo_kv_layer_view_get(self.handle, layer)
        base = self.buf.data_ptr()
        B, d, SW, cap = self.B, self.d, self.S + self.W, self.cap

        def region(ptr, nbytes):
            off = ptr - base
            return self.buf[off:off + nbytes]
        nr, ns = v.n_retrieval, v.n_streaming
        quant = self.fp8 or self.int4
        eb = 1 if quant else 2
        dl = d // 2 if self.int4 else d          # last dimension of a row in its element type

        def typed(t):
            return t if quant else t.view(torch.bfloat16)
        if self.page_tokens > 0:   # the pool [num_pages][n_r][page_tokens][d]
            shape = (self.num_pages, nr, self.page_tokens, dl)
        else:
            shape = (B, nr, cap, dl)
        n_el = shape[0] * shape[1] * shape[2] * shape[3]
        kr = typed(region(v.k_retrieval, n_el * eb)).view(*shape)
        vr = typed(region(v.v_retrieval, n_el * eb)).view(*shape)
        ks = typed(region(v.k_streaming, B * ns * SW * dl * eb)).view(B, ns, SW, dl)
        vs = typed(region(v.v_streaming, B * ns * SW * dl * eb)).view(B, ns, SW, dl)
        pos = region(v.positions, B * SW * 4).view(torch.int32).view(B, SW)
        rank = [v.head_rank[g] for g in range(self.n_kv)]
        is_r = [bool(v.is_retrieval[g]) for g in range(self.n_kv)]
        return dict(k_retrieval=kr, v_retrieval=vr, k_streaming=ks, v_streaming=vs, positions=pos,
                    head_rank=rank, is_retrieval=is_r)

    # ------------------------------------------------------------ the path
    def append(self, layer: int, k_new, v_new, len_before, n_new=None):
        """k_new, v_new: bf16 [B][n_kv][n][d]; len_before: int32 [B] (device);
        n_new: optional int32 [B] per-sequence counts (<= n)."""
        n = k_new.shape[2]
        shp = (self.B, self.n_kv, n, self.d)
        kp = _need(k_new, "k_new", torch.bfloat16, shp, self.device)
        vp = _need(v_new, "v_new", torch.bfloat16, shp, self.device)
        lp = _need(len_before, "len_before", torch.int32, (self.B,), self.device)
        np_ = _need(n_new, "n_new", torch.int32, (self.B,), self.device) if n_new is not None else None
        L.duo_kv_append(self.handle, layer, kp, vp, lp, np_, n, _stream(self.device))

    def append_rows(self, layer: int, k_new, v_new, len_before, r_pos_begin, r_pos_end, n_new=None):
        """append() for a cache whose retrieval rows hold positions
        [r_pos_begin[b], r_pos_end[b]) (int32 [B] each) from row 0."""
        n = k_new.shape[2]
        shp = (self.B, self.n_kv, n, self.d)
        kp = _need(k_new, "k_new", torch.bfloat16, shp, self.device)
        vp = _need(v_new, "v_new", torch.bfloat16, shp, self.device)
        lp = _need(len_before, "len_before", torch.int32, (self.B,), self.device)
        bp = _need(r_pos_begin, "r_pos_begin", torch.int32, (self.B,), self.device)
        ep = _need(r_pos_end, "r_pos_end", torch.int32, (self.B,), self.device)
        np_ = _need(n_new, "n_new", torch.int32, (self.B,), self.device) if n_new is not None else None
        L.duo_kv_append_rows(self.handle, layer, kp, vp, lp, np_, n, bp, ep, _stream(self.device))

    def decode_rows(self, layer: int, q, r_end, scale: float, r_begin=None, s_len=None, out=None, lse=None):
        """Decode over retrieval rows [r_begin, r_end) and streaming slots
        [0, s_len) (int32 [B] each; r_begin / s_len optional).  Returns
        (out [B][Hq][d], lse [B][Hq]) fp32."""
        qp = _need(q, "q", torch.bfloat16, (self.B, self.hq, self.d), self.device)
        ep = _need(r_end, "r_end", torch.int32, (self.B,), self.device)
        bp = _need(r_begin, "r_begin", torch.int32, (self.B,), self.device) if r_begin is not None else None
        sp = _need(s_len, "s_len", torch.int32, (self.B,), self.device) if s_len is not None else None
        if out is None:
            out = torch.empty(self.B, self.hq, self.d, dtype=torch.float32, device=self.device)
        if lse is None:
            lse = torch.empty(self.B, self.hq, dtype=torch.float32, device=self.device)
        op = _need(out, "out", torch.float32, (self.B, self.hq, self.d), self.device)
        lp = _need(lse, "lse", torch.float32, (self.B, self.hq), self.device)
        L.duo_decode_attn_rows(self.handle, layer, qp, bp, ep, sp, float(scale), op, lp, self._ws.data_ptr(),
                               self._ws.numel(), _stream(self.device))
        return out, lse

    def decode(self, layer: int, q, lengths, scale: float, out=None, lse=None, want_lse=False):
        """q: bf16 [B][Hq][d]; lengths: int32 [B] after this step's append.
        Returns fp32 out [B][Hq][d] (and lse [B][Hq] if asked)."""
        qp = _need(q, "q", torch.bfloat16, (self.B, self.hq, self.d), self.device)
        lp = _need(lengths, "lengths", torch.int32, (self.B,), self.device)
        if out is None:
            out = torch.empty(self.B, self.hq, self.d, dtype=torch.float32, device=self.device)
        op = _need(out, "out", torch.float32, (self.B, self.hq, self.d), self.device)
        if want_lse and lse is None:
            lse = torch.empty(self.B, self.hq, dtype=torch.float32, device=self.device)
        sp = _need(lse, "lse", torch.float32, (self.B, self.hq), self.device) if lse is not None else None
        L.duo_decode_attn(self.handle, layer, qp, lp, float(scale), op, sp, self._ws.data_ptr(),
                          self._ws.numel(), _stream(self.device))
        return (out, lse) if lse is not None else out

    def step(self, layer: int, q, k_new, v_new, len_before, lengths, scale: float, out=None, lse=None,
             want_lse=False):
        """One decode step: append the new token (k_new, v_new: bf16 [B][n_kv][1][d]
        at positions len_before) and decode q (bf16 [B][Hq][d]) over lengths
        (int32 [B], = len_before + 1); see duo_decode_step.  Returns fp32 out
        [B][Hq][d] (and lse [B][Hq] if asked)."""
        shp = (self.B, self.n_kv, 1, self.d)
        kp = _need(k_new, "k_new", torch.bfloat16, shp, self.device)
        vp = _need(v_new, "v_new", torch.bfloat16, shp, self.device)
        bp = _need(len_before, "len_before", torch.int32, (self.B,), self.device)
        qp = _need(q, "q", torch.bfloat16, (self.B, self.hq, self.d), self.device)
        lp = _need(lengths, "lengths", torch.int32, (self.B,), self.device)
        if out is None:
            out = torch.empty(self.B, self.hq, self.d, dtype=torch.float32, device=self.device)
        op = _need(out, "out", torch.float32, (self.B, self.hq, self.d), self.device)
        if want_lse and lse is None:
            lse = torch.empty(self.B, self.hq, dtype=torch.float32, device=self.device)
        sp = _need(lse, "lse", torch.float32, (self.B, self.hq), self.device) if lse is not None else None
        L.duo_decode_step(self.handle, layer, kp, vp, bp, qp, lp, float(scale), op, sp, self._ws.data_ptr(),
                          self._ws.numel(), _stream(self.device))
        return (out, lse) if lse is not None else out

    def prefill(self, layer: int, q, k_chunk, v_chunk, prefix_len, scale: float, out=None):
        """q: bf16 [B][Hq][C][d]; k_chunk, v_chunk: bf16 [B][n_kv][C][d];
        prefix_len: int32 [B].  Returns fp32 out [B][Hq][C][d]."""
        C = q.shape[2]
        qp = _need(q, "q", torch.bfloat16, (self.B, self.hq, C, self.d), self.device)
        kp = _need(k_chunk, "k_chunk", torch.bfloat16, (self.B, self.n_kv, C, self.d), self.device)
        vp = _need(v_chunk, "v_chunk", torch.bfloat16, (self.B, self.n_kv, C, self.d), self.device)
        pp = _need(prefix_len, "prefix_len", torch.int32, (self.B,), self.device)
        if out is None:
            out = torch.empty(self.B, self.hq, C, self.d, dtype=torch.float32, device=self.device)
        op = _need(out, "out", torch.float32, (self.B, self.hq, C, self.d), self.device)
        n = L.duo_prefill_workspace_bytes(self.handle, C)
        ws = torch.empty(max(n, 256), dtype=torch.uint8, device=self.device)
        L.duo_prefill_attn(self.handle, layer, qp, kp, vp, pp, C, float(scale), op, ws.data_ptr(), ws.numel(),
                           _stream(self.device))
        return out


def lse_merge(part_out, part_lse, out=None, lse=None):
    """Combine attention over disjoint key sets: part_out fp32 [R][..., d],
    part_lse fp32 [R][...] (same leading shape) -> (out [..., d], lse [...])."""
    R = part_out.shape[0]
    d = part_out.shape[-1]
    rows = part_lse[0].numel()
    dev = part_out.device
    if part_out.dtype != torch.float32 or part_lse.dtype != torch.float32:
        raise TypeError("lse_merge takes fp32 tensors")
    if not (part_out.is_contiguous() and part_lse.is_contiguous()):
        raise ValueError("lse_merge takes contiguous tensors")
    if part_out.numel() != R * rows * d or part_lse.shape[0] != R:
        raise ValueError("part_out must be [R][rows][d] and part_lse [R][rows]")
    if out is None:
        out = torch.empty(part_out.shape[1:], dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty(part_lse.shape[1:], dtype=torch.float32, device=dev)
    L.duo_lse_merge(R, rows, d, part_out.data_ptr(), part_lse.data_ptr(), out.data_ptr(), lse.data_ptr(),
                    _stream(dev))
    return out, lse


def alpha_blend(alpha, full_out, stream_out, out=None):
    """out = alpha[h] * full_out + (1 - alpha[h]) * stream_out, tensors
    [B][Hq][d] fp32, alpha fp32 [Hq]."""
    B, hq, d = full_out.shape
    dev = full_out.device
    ap = _need(alpha, "alpha", torch.float32, (hq,), dev)
    fp = _need(full_out, "full_out", torch.float32, (B, hq, d), dev)
    sp = _need(stream_out, "stream_out", torch.float32, (B, hq, d), dev)
    if out is None:
        out = torch.empty_like(full_out)
    op = _need(out, "out", torch.float32, (B, hq, d), dev)
    L.duo_alpha_blend(B, hq, d, ap, fp, sp, op, _stream(dev))
    return out
