"""ctypes binding of liblvq (include/lvq.h), same names as the C ABI.

Argument marshalling only: every step of the codec and the attention runs in
the library's CUDA kernels.  torch supplies device memory and streams.  If the
library is missing, or the device is not sm_100, calls raise: there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblvq.so")

LVQ_OK, LVQ_EINVAL, LVQ_EUNSUPPORTED, LVQ_ECAPACITY, LVQ_ECUDA, LVQ_ETIMEOUT, LVQ_EDEVICE = range(7)


class LvqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class lvq_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "n_layers", "n_kv_heads", "n_q_heads", "head_dim", "T", "Tc", "G", "K", "n_sink", "n_recent",
        "page_tokens", "max_batch", "max_ctx", "max_splits")] + [("rope_base", ctypes.c_float)] + [
        ("pool_pages", ctypes.c_int32), ("reserved_", ctypes.c_int32), ("page_table", ctypes.c_void_p)]


class lvq_layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "c", "n_groups", "n_blocks", "ring_tokens", "max_pages", "page_bytes", "rope_coarse",
        "page_table_stride")] + [
        ("idx_bytes", ctypes.c_size_t), ("idx_strides", ctypes.c_int64 * 8), ("page_table_bytes", ctypes.c_size_t),
        ("cb_bytes", ctypes.c_size_t), ("cb_strides", ctypes.c_int64 * 7),
        ("cbp_bytes", ctypes.c_size_t), ("cbp_strides", ctypes.c_int64 * 8),
        ("cb_norm_bytes", ctypes.c_size_t),
        ("sink_bytes", ctypes.c_size_t), ("sink_strides", ctypes.c_int64 * 7),
        ("ring_bytes", ctypes.c_size_t), ("ring_strides", ctypes.c_int64 * 7),
        ("rope_bytes", ctypes.c_size_t), ("workspace_bytes", ctypes.c_size_t)]


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_SIGS = {
    "lvq_cache_layout": [ctypes.POINTER(lvq_config), ctypes.POINTER(lvq_layout)],
    "lvq_pack_codebooks": [ctypes.POINTER(lvq_config), ctypes.POINTER(lvq_layout), _P, _P, _P, _P],
    "lvq_rope_table": [ctypes.POINTER(lvq_config), ctypes.POINTER(lvq_layout), _P, _P],
    "lvq_encode_prefill": [ctypes.POINTER(lvq_config), ctypes.POINTER(lvq_layout), _I32, _I32, _P,
                           ctypes.c_int64, _I32, _I32, _I32, _I32, _P, _P, _P, _P],
    "lvq_encode_page": [ctypes.POINTER(lvq_config), ctypes.POINTER(lvq_layout), _I32, _P, _P, _P, _P, _P,
                        _P, _P, _P],
    "lvq_decode_attention": [ctypes.POINTER(lvq_config), ctypes.POINTER(lvq_layout), _I32, _I32, _I32, _P,
                             _P, _P, _P, _P, _P, _P, _P, _I32, _P, _P, _P, _P, _P, _P],
    "lvq_dequantize": [ctypes.POINTER(lvq_config), ctypes.POINTER(lvq_layout), _I32, _I32, _I32, _I32, _P,
                       _P, _I32, _I32, _P, _P],
    "lvq_kmeans_update": [ctypes.POINTER(lvq_config), ctypes.POINTER(lvq_layout), _I32, _I32, _P,
                          ctypes.c_int64, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _P],
    "lvq_status_string": [_I32],
    "lvq_debug_faults": [ctypes.c_int64, _I32],
    "lvq_decode_max_ctas": [_I32],
    "lvq_decode_attention_noalloc": [ctypes.POINTER(lvq_config), ctypes.POINTER(lvq_layout), _I32, _I32, _I32,
                                     _P, _P, _P, _P, _P, _P, _P, _P, _I32, _P, _P, _P, _P, _P],
    "lvq_pool_create": [_I32, ctypes.POINTER(_P)],
    "lvq_pool_destroy": [_P],
    "lvq_pool_alloc": [_P, _I32, ctypes.POINTER(_I32)],
    "lvq_pool_free": [_P, ctypes.POINTER(_I32), _I32],
    "lvq_pool_available": [_P],
}
EXPORTED = tuple(_SIGS)

_lib = None


def lib():
    """Loads liblvq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m sub_bit_kv_b200._build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            fn = getattr(h, name)
            fn.argtypes = args
            fn.restype = {"lvq_status_string": ctypes.c_char_p, "lvq_pool_destroy": None}.get(name, ctypes.c_int)
        _lib = h
    return _lib


def status_string(s: int) -> str:
    return lib().lvq_status_string(int(s)).decode()


def _check(s: int, where: str):
    if s != LVQ_OK:
        raise LvqError(s, where)


def make_config(n_layers, n_kv_heads, n_q_heads, head_dim, T, Tc, G, n_sink, n_recent, max_batch, max_ctx,
                max_splits=64, rope_base=10000.0, K=256, page_tokens=8, pool_pages=0) -> lvq_config:
    """pool_pages > 0: pool mode (CodedCache allocates the page table and sets page_table)."""
    return lvq_config(n_layers, n_kv_heads, n_q_heads, head_dim, T, Tc, G, K, n_sink, n_recent, page_tokens,
                      max_batch, max_ctx, max_splits, rope_base, pool_pages, 0, None)


class PagePool:
    """The library's host-side page allocator (lvq_pool): physical page ids of a pool, handed
    out lowest first and taken back when a request ends."""

    def __init__(self, n_pages: int):
        h = _P()
        _check(lib().lvq_pool_create(int(n_pages), ctypes.byref(h)), "lvq_pool_create")
        self._h = h

    def alloc(self, n: int) -> list:
        ids = (_I32 * max(1, n))()
        _check(lib().lvq_pool_alloc(self._h, int(n), ids), "lvq_pool_alloc")
        return list(ids[:n])

    def free(self, ids) -> None:
        arr = (_I32 * max(1, len(ids)))(*ids)
        _check(lib().lvq_pool_free(self._h, arr, len(ids)), "lvq_pool_free")

    def available(self) -> int:
        return int(lib().lvq_pool_available(self._h))

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and _lib is not None:
            _lib.lvq_pool_destroy(h)
            self._h = None


def lvq_cache_layout(cfg: lvq_config) -> lvq_layout:
    lay = lvq_layout()
    _check(lib().lvq_cache_layout(ctypes.byref(cfg), ctypes.byref(lay)), "lvq_cache_layout")
    return lay


def _ptr(t: Optional[torch.Tensor], name: str, dtype=None, min_bytes: int = 0, optional=False):
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.numel() * t.element_size() < min_bytes:
        raise ValueError(f"{name} holds {t.numel() * t.element_size()} bytes, needs {min_bytes}")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def lvq_pack_codebooks(cfg, lay, cb, cbp, cb_norm=None, stream=None):
    _check(lib().lvq_pack_codebooks(
        ctypes.byref(cfg), ctypes.byref(lay), _ptr(cb, "cb", torch.bfloat16, lay.cb_bytes),
        _ptr(cbp, "cbp", torch.bfloat16, lay.cbp_bytes),
        _ptr(cb_norm, "cb_norm", torch.float32, lay.cb_norm_bytes, optional=True), _stream(stream)),
        "lvq_pack_codebooks")


def lvq_rope_table(cfg, lay, rope, stream=None):
    _check(lib().lvq_rope_table(ctypes.byref(cfg), ctypes.byref(lay), _ptr(rope, "rope", torch.float32,
                                                                           lay.rope_bytes), _stream(stream)),
           "lvq_rope_table")


def lvq_encode_prefill(cfg, lay, layer, req, kv, tok_begin, n_tok, coded_offset, cb, idx, dev_status,
                       kv_tok_stride=None, stream=None):
    """kv: bf16 [2][T][N][Hkv][d] of one layer and request (contiguous); with layer = -1
    (every layer in one call) [n_layers][2][T][N][Hkv][d]."""
    if layer == -1:
        if kv.dim() != 6 or kv.shape[0] != cfg.n_layers:
            raise ValueError("layer = -1 takes kv as [n_layers][2][T][N][Hkv][d]")
        kv1 = kv[0]
    else:
        kv1 = kv
    if kv1.dim() != 5 or kv1.shape[0] != 2 or kv1.shape[1] != cfg.T:
        raise ValueError("kv must be [2][T][N][Hkv][d]")
    n_total = kv1.shape[2]
    stride = kv_tok_stride if kv_tok_stride is not None else kv1.shape[3] * kv1.shape[4]
    _check(lib().lvq_encode_prefill(
        ctypes.byref(cfg), ctypes.byref(lay), layer, req, _ptr(kv, "kv", torch.bfloat16), stride, n_total,
        tok_begin, n_tok, coded_offset, _ptr(cb, "cb", torch.bfloat16, lay.cb_bytes),
        _ptr(idx, "idx", torch.uint8, lay.idx_bytes), _ptr(dev_status, "dev_status", torch.int32, 4),
        _stream(stream)), "lvq_encode_prefill")


def lvq_kmeans_update(cfg, lay, layer, req, kv, tok_begin, n_tok, coded_offset, idx, cb, counts, dev_status,
                      kv_tok_stride=None, stream=None):
    """Update step of one k-means iteration after lvq_encode_prefill wrote the codes.
    kv: bf16 [2][T][N][Hkv][d] of one layer and request (contiguous); cb is updated in
    place; counts: None or int32 [2][n_blk][Hkv][n_g][256] (the library writes uint32)."""
    if kv.dim() != 5 or kv.shape[0] != 2 or kv.shape[1] != cfg.T:
        raise ValueError("kv must be [2][T][N][Hkv][d]")
    n_total = kv.shape[2]
    stride = kv_tok_stride if kv_tok_stride is not None else kv.shape[3] * kv.shape[4]
    n_counts = 2 * lay.n_blocks * cfg.n_kv_heads * lay.n_groups * 256
    _check(lib().lvq_kmeans_update(
        ctypes.byref(cfg), ctypes.byref(lay), layer, req, _ptr(kv, "kv", torch.bfloat16), stride, n_total,
        tok_begin, n_tok, coded_offset, _ptr(idx, "idx", torch.uint8, lay.idx_bytes),
        _ptr(cb, "cb", torch.bfloat16, lay.cb_bytes),
        _ptr(counts, "counts", torch.int32, 4 * n_counts, optional=True),
        _ptr(dev_status, "dev_status", torch.int32, 4), _stream(stream)), "lvq_kmeans_update")


def lvq_debug_faults(wait_iters: int = 0, fault_mask: int = 0):
    """Test hook: bound of every device-side wait (0: the normal bound) and copies that never
    happen (bit 0: decode's first code chunk, bit 1: k-means' first tile).  Process-global."""
    _check(lib().lvq_debug_faults(int(wait_iters), int(fault_mask)), "lvq_debug_faults")


def lvq_decode_max_ctas(max_ctas: int = 0):
    """Caps the CTAs of later lvq_decode_attention calls (0: one per work item); with more work
    items than the cap each CTA walks a run of them.  Process-global."""
    _check(lib().lvq_decode_max_ctas(int(max_ctas)), "lvq_decode_max_ctas")


def lvq_encode_page(cfg, lay, batch, ctx_len, coded_len, ring, cb, cb_norm, idx, dev_status, stream=None):
    _check(lib().lvq_encode_page(
        ctypes.byref(cfg), ctypes.byref(lay), batch, _ptr(ctx_len, "ctx_len", torch.int32, 4 * batch),
        _ptr(coded_len, "coded_len", torch.int32, 4 * batch), _ptr(ring, "ring", torch.bfloat16, lay.ring_bytes),
        _ptr(cb, "cb", torch.bfloat16, lay.cb_bytes), _ptr(cb_norm, "cb_norm", torch.float32, lay.cb_norm_bytes),
        _ptr(idx, "idx", torch.uint8, lay.idx_bytes),
        _ptr(dev_status, "dev_status", torch.int32, 4), _stream(stream)), "lvq_encode_page")


def lvq_decode_attention(cfg, lay, layer, step, batch, q, ctx_len, coded_len, sink, ring, idx, cbp, rope,
                         num_splits, workspace, out, lse, dev_status, split_lse=None, stream=None):
    d = cfg.head_dim
    _check(lib().lvq_decode_attention(
        ctypes.byref(cfg), ctypes.byref(lay), layer, step, batch,
        _ptr(q, "q", torch.bfloat16, 2 * batch * cfg.n_q_heads * d),
        _ptr(ctx_len, "ctx_len", torch.int32, 4 * batch), _ptr(coded_len, "coded_len", torch.int32, 4 * batch),
        _ptr(sink, "sink", torch.bfloat16, lay.sink_bytes), _ptr(ring, "ring", torch.bfloat16, lay.ring_bytes),
        _ptr(idx, "idx", torch.uint8, lay.idx_bytes), _ptr(cbp, "cbp", torch.bfloat16, lay.cbp_bytes),
        _ptr(rope, "rope", torch.float32, lay.rope_bytes), num_splits,
        _ptr(workspace, "workspace", torch.float32, lay.workspace_bytes),
        _ptr(out, "out", torch.float32, 4 * batch * cfg.n_q_heads * d),
        _ptr(lse, "lse", torch.float32, 4 * batch * cfg.n_q_heads),
        _ptr(split_lse, "split_lse", torch.float32, 4 * batch * cfg.n_q_heads * (num_splits + 1), optional=True),
        _ptr(dev_status, "dev_status", torch.int32, 4), _stream(stream)), "lvq_decode_attention")


def lvq_decode_attention_noalloc(cfg, lay, layer, step, batch, q, ctx_len, coded_len, sink, ring, idx, cbp, rope,
                                 num_splits, out, lse, dev_status, split_lse=None, stream=None):
    """lvq_decode_attention with the library's own 4 MiB device workspace (no workspace argument)."""
    d = cfg.head_dim
    _check(lib().lvq_decode_attention_noalloc(
        ctypes.byref(cfg), ctypes.byref(lay), layer, step, batch,
        _ptr(q, "q", torch.bfloat16, 2 * batch * cfg.n_q_heads * d),
        _ptr(ctx_len, "ctx_len", torch.int32, 4 * batch), _ptr(coded_len, "coded_len", torch.int32, 4 * batch),
        _ptr(sink, "sink", torch.bfloat16, lay.sink_bytes), _ptr(ring, "ring", torch.bfloat16, lay.ring_bytes),
        _ptr(idx, "idx", torch.uint8, lay.idx_bytes), _ptr(cbp, "cbp", torch.bfloat16, lay.cbp_bytes),
        _ptr(rope, "rope", torch.float32, lay.rope_bytes), num_splits,
        _ptr(out, "out", torch.float32, 4 * batch * cfg.n_q_heads * d),
        _ptr(lse, "lse", torch.float32, 4 * batch * cfg.n_q_heads),
        _ptr(split_lse, "split_lse", torch.float32, 4 * batch * cfg.n_q_heads * (num_splits + 1), optional=True),
        _ptr(dev_status, "dev_status", torch.int32, 4), _stream(stream)), "lvq_decode_attention_noalloc")


def lvq_dequantize(cfg, lay, layer, step, req, kv, idx, cbp, tok_begin, n_tok, out, stream=None):
    _check(lib().lvq_dequantize(
        ctypes.byref(cfg), ctypes.byref(lay), layer, step, req, kv, _ptr(idx, "idx", torch.uint8, lay.idx_bytes),
        _ptr(cbp, "cbp", torch.bfloat16, lay.cbp_bytes), tok_begin, n_tok,
        _ptr(out, "out", torch.bfloat16, 2 * n_tok * cfg.n_kv_heads * cfg.head_dim), _stream(stream)),
        "lvq_dequantize")


class CodedCache:
    """Device buffers of one configuration, allocated with torch to the sizes
    lvq_cache_layout gives (plumbing: the library itself allocates nothing)."""

    def __init__(self, cfg: lvq_config, device="cuda"):
        self.cfg = cfg
        self.lay = lay = lvq_cache_layout(cfg)
        dev = torch.device(device)
        self.idx = torch.zeros(lay.idx_bytes, dtype=torch.uint8, device=dev)
        self.cb = torch.zeros(lay.cb_bytes // 2, dtype=torch.bfloat16, device=dev)
        self.cbp = torch.zeros(lay.cbp_bytes // 2, dtype=torch.bfloat16, device=dev)
        self.cb_norm = torch.zeros(lay.cb_norm_bytes // 4, dtype=torch.float32, device=dev)
        self.sink = torch.zeros(lay.sink_bytes // 2, dtype=torch.bfloat16, device=dev)
        self.ring = torch.zeros(lay.ring_bytes // 2, dtype=torch.bfloat16, device=dev)
        self.rope = torch.zeros(lay.rope_bytes // 4, dtype=torch.float32, device=dev)
        self.workspace = torch.zeros(lay.workspace_bytes // 4, dtype=torch.float32, device=dev)
        self.ctx_len = torch.zeros(cfg.max_batch, dtype=torch.int32, device=dev)
        self.coded_len = torch.zeros(cfg.max_batch, dtype=torch.int32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.pool = None
        if cfg.pool_pages > 0:
            # pool mode: the page table (every entry unassigned) and the host allocator; the
            # config carries the table's device address from here on
            self.page_table = torch.full((lay.page_table_bytes // 4,), -1, dtype=torch.int32, device=dev)
            cfg.page_table = self.page_table.data_ptr()
            self.pool = PagePool(cfg.pool_pages)
            self.pages = [[] for _ in range(cfg.max_batch)]       # host copy: physical page of logical page i

    # pool mode: pages of a request
    def assign_pages(self, b: int, n_pages: int) -> list:
        """Makes request b hold at least n_pages logical pages (new ones from the pool) and writes
        its page-table row.  Returns the request's physical pages."""
        have = self.pages[b]
        if n_pages > len(have):
            have += self.pool.alloc(n_pages - len(have))
            row = torch.tensor(have, dtype=torch.int32)
            self.page_table[b * self.lay.page_table_stride: b * self.lay.page_table_stride + len(have)].copy_(row)
        return list(have)

    def release(self, b: int) -> None:
        """Request b ends: its pages go back to the pool and its page-table row is cleared."""
        if self.pages[b]:
            self.pool.free(self.pages[b])
            self.pages[b] = []
            self.page_table[b * self.lay.page_table_stride:(b + 1) * self.lay.page_table_stride].fill_(-1)

    # shaped views of the caller-owned buffers (layouts from lvq_cache_layout)
    def cb_view(self):
        c = self.cfg
        return self.cb.view(c.n_layers, 2, self.lay.n_blocks, c.n_kv_heads, self.lay.n_groups, 256, c.G)

    def sink_view(self):
        c = self.cfg
        return self.sink.view(c.n_layers, 2, c.T, c.max_batch, c.n_kv_heads, c.n_sink, c.head_dim)

    def ring_view(self):
        c = self.cfg
        return self.ring.view(c.n_layers, 2, c.T, c.max_batch, c.n_kv_heads, self.lay.ring_tokens, c.head_dim)

    def idx_view(self):
        c, l = self.cfg, self.lay
        if c.pool_pages > 0:       # [layer][n_blk][Hkv][kv][pool page][n_g][8]
            return self.idx.view(c.n_layers, l.n_blocks, c.n_kv_heads, 2, c.pool_pages, l.n_groups, 8)
        return self.idx.view(c.n_layers, l.n_blocks, c.max_batch, c.n_kv_heads, 2, l.max_pages, l.n_groups, 8)

    def check_status(self, where="device"):
        s = int(self.status.item())
        if s != LVQ_OK:
            self.status.zero_()
            raise LvqError(s, where)
