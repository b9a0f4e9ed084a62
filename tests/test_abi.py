"""The C-ABI library loads, exports every declared symbol, and its host-side
layout arithmetic matches the closed forms (CPU only; no compute calls)."""
import os
import re

import pytest
import torch

from oracle import lvq_oracle as O
from sub_bit_kv_b200 import lvq, synth
from tests._helpers import make_cfg

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "lvq.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    from sub_bit_kv_b200 import _build
    _build.build()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:LVQ_API\s+)?(?:lvq_status|const char\*|void|int32_t)\s+(lvq_\w+)\s*\(",
                                 text, re.M)))


def test_exports_every_declared_symbol():
    names = declared_functions()
    assert "lvq_decode_attention" in names and "lvq_cache_layout" in names
    lib = lvq.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(lvq.EXPORTED)


def test_status_strings():
    for s in range(7):
        assert lvq.status_string(s)
    assert lvq.status_string(0) == "ok"


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_layout_closed_forms(name):
    w = synth.WORKLOADS[name]
    cfg = make_cfg(w)
    lay = lvq.lvq_cache_layout(cfg)
    c, ng, nblk = O.geometry(w.head_dim, w.T, w.Tc, w.G)
    assert (lay.c, lay.n_groups, lay.n_blocks) == (c, ng, nblk)
    assert lay.page_bytes == ng * 8
    assert lay.ring_tokens == w.n_recent + 8
    # code bytes per token, head and K/V: one row of n_g bytes per block ("one index row per Tc block")
    per_token = lay.idx_bytes / (cfg.n_layers * cfg.max_batch * cfg.n_kv_heads * lay.max_pages * 8 * 2)
    assert per_token == nblk * ng
    # bits per cached element = 8/G
    assert per_token * 8 / (w.T * w.head_dim) == 8 / w.G
    assert lay.cb_bytes == cfg.n_layers * 2 * nblk * cfg.n_kv_heads * ng * 256 * w.G * 2
    assert lay.cbp_bytes == lay.cb_bytes
    assert list(lay.idx_strides)[-3:] == [ng * 8, 8, 1]
    assert list(lay.ring_strides)[-2:] == [w.head_dim, 1]


def test_ouro_row_bytes():
    rows = {}
    for name, want in (("ouro14_g16_32k", (1, 32)), ("ouro14_g32_b32", (1, 16)), ("ouro14_tc2_64k", (2, 16))):
        lay = lvq.lvq_cache_layout(make_cfg(synth.WORKLOADS[name]))
        rows[name] = (lay.n_blocks, lay.n_groups)
        assert rows[name] == want
    # index storage for 24 layers x 16 heads at 32K context, B = 1: 24.6 KB per token
    w = synth.WORKLOADS["ouro14_g16_32k"]
    per_tok = w.n_layers * w.n_kv_heads * 2 * 32
    assert per_tok == 24576


@pytest.mark.parametrize("field,value,status", [
    ("Tc", 3, lvq.LVQ_EINVAL),           # Tc does not divide T = 4
    ("G", 18, lvq.LVQ_EINVAL),           # Tc = 4 does not divide G
    ("K", 128, lvq.LVQ_EUNSUPPORTED),
    ("page_tokens", 16, lvq.LVQ_EUNSUPPORTED),
    ("head_dim", 96, lvq.LVQ_EUNSUPPORTED),
    ("n_q_heads", 24, lvq.LVQ_EINVAL),    # not a multiple of 16 KV heads
    ("max_splits", 0, lvq.LVQ_EINVAL),
    ("n_layers", 0, lvq.LVQ_EINVAL),
])
def test_invalid_configs_rejected(field, value, status):
    cfg = make_cfg(synth.WORKLOADS["ouro14_g16_32k"])
    setattr(cfg, field, value)
    with pytest.raises(lvq.LvqError) as e:
        lvq.lvq_cache_layout(cfg)
    assert e.value.status == status


def test_layout_mismatch_is_rejected_before_any_device_work():
    """A caller's layout that does not match its config fails with EINVAL on the host."""
    import ctypes
    w = synth.WORKLOADS["tiny"]
    cfg = make_cfg(w)
    lay = lvq.lvq_cache_layout(cfg)
    lay.idx_bytes += 1
    st = lvq.lib().lvq_rope_table(ctypes.byref(cfg), ctypes.byref(lay), None, None)
    assert st == lvq.LVQ_EINVAL
    lay = lvq.lvq_cache_layout(cfg)
    st = lvq.lib().lvq_rope_table(ctypes.byref(cfg), ctypes.byref(lay), None, None)
    assert st == lvq.LVQ_EINVAL          # null table pointer
    st = lvq.lib().lvq_decode_attention(ctypes.byref(cfg), ctypes.byref(lay), 0, 4, 1, *([None] * 8), 1,
                                        None, None, None, None, None, None)
    assert st == lvq.LVQ_EINVAL          # step 4 out of range for T = 4


def test_kmeans_update_argument_checks_on_the_host():
    """lvq_kmeans_update rejects bad arguments before any device work (no GPU needed)."""
    import ctypes
    w = synth.WORKLOADS["tiny"]
    cfg = make_cfg(w)
    lay = lvq.lvq_cache_layout(cfg)
    L = lvq.lib()
    fake = 1 << 20                       # a 16-byte-aligned address that is never touched

    def call(layer=0, req=0, kv=fake, stride=w.n_kv_heads * w.head_dim, kv_tokens=64, tok_begin=0, n_tok=64,
             coded_offset=0, idx=fake, cb=fake, counts=None):
        return L.lvq_kmeans_update(ctypes.byref(cfg), ctypes.byref(lay), layer, req, kv, stride, kv_tokens,
                                   tok_begin, n_tok, coded_offset, idx, cb, counts, None, None)

    assert call(layer=cfg.n_layers) == lvq.LVQ_EINVAL
    assert call(req=cfg.max_batch) == lvq.LVQ_EINVAL
    assert call(n_tok=65) == lvq.LVQ_EINVAL                 # past the K/V buffer's tokens
    assert call(kv=None) == lvq.LVQ_EINVAL
    assert call(cb=fake + 8) == lvq.LVQ_EINVAL              # misaligned codebooks
    assert call(stride=w.n_kv_heads * w.head_dim - 1) == lvq.LVQ_EINVAL
    assert call(stride=w.n_kv_heads * w.head_dim + 4) == lvq.LVQ_EUNSUPPORTED   # rows TMA cannot read
    big = lay.idx_bytes                                      # coded slots past the capacity
    assert call(coded_offset=big) == lvq.LVQ_EINVAL


def test_debug_fault_hook_host_side():
    """The failure-detection test hook checks its bits on the host and restores cleanly."""
    with pytest.raises(lvq.LvqError) as e:
        lvq.lvq_debug_faults(0, 1 << 5)
    assert e.value.status == lvq.LVQ_EINVAL
    lvq.lvq_debug_faults(1 << 10, 3)
    lvq.lvq_debug_faults(0, 0)


def test_decode_max_ctas_host_side():
    with pytest.raises(lvq.LvqError) as e:
        lvq.lvq_decode_max_ctas(-1)
    assert e.value.status == lvq.LVQ_EINVAL
    lvq.lvq_decode_max_ctas(3)
    lvq.lvq_decode_max_ctas(0)


def test_encode_prefill_layer_argument_on_the_host():
    """layer = -1 (every layer in one call) passes the host checks -- on a machine without a
    GPU it then stops at the device check -- while anything below -1 or past the last layer
    is rejected first."""
    import ctypes
    w = synth.WORKLOADS["tiny"]
    cfg = make_cfg(w)
    lay = lvq.lvq_cache_layout(cfg)
    L = lvq.lib()
    fake = 1 << 20

    def call(layer):
        return L.lvq_encode_prefill(ctypes.byref(cfg), ctypes.byref(lay), layer, 0, fake,
                                    w.n_kv_heads * w.head_dim, 64, 0, 64, 0, fake, fake, None, None)

    assert call(-2) == lvq.LVQ_EINVAL
    assert call(cfg.n_layers) == lvq.LVQ_EINVAL
    if not torch.cuda.is_available():
        assert call(-1) == lvq.LVQ_EDEVICE
        assert call(0) == lvq.LVQ_EDEVICE


def test_pool_allocator_hands_out_lowest_ids_and_takes_them_back():
    pool = lvq.PagePool(10)
    assert pool.available() == 10
    assert pool.alloc(4) == [0, 1, 2, 3]
    assert pool.alloc(3) == [4, 5, 6]
    pool.free([1, 2])
    assert pool.available() == 5
    assert pool.alloc(2) == [1, 2]                  # lowest first: runs of consecutive ids
    with pytest.raises(lvq.LvqError) as e:
        pool.alloc(4)                               # only 3 left: nothing taken
    assert e.value.status == lvq.LVQ_ECAPACITY and pool.available() == 3
    for bad in ([10], [-1], [7], [0, 0]):           # out of range, out of range, free, repeated
        with pytest.raises(lvq.LvqError) as e:
            pool.free(bad)
        assert e.value.status == lvq.LVQ_EINVAL
    assert pool.available() == 3                    # all or nothing
    pool.free([0, 3, 4])
    assert pool.available() == 6


def test_pool_layout_closed_forms_and_table_checks():
    """Pool mode: codes live in pool_pages pages per (layer, block, head, K/V); the page table is
    [max_batch][stride] with the stride the request's page capacity rounded up to 4."""
    import ctypes
    w = synth.WORKLOADS["ouro14_tc2_64k"]
    cfg = make_cfg(w, n_layers=2, max_batch=3, max_ctx=1000)
    plain = lvq.lvq_cache_layout(cfg)
    cfg.pool_pages = 77
    lay = lvq.lvq_cache_layout(cfg)                 # the table's address is not needed for the layout
    c, ng, nblk = O.geometry(w.head_dim, w.T, w.Tc, w.G)
    assert lay.idx_bytes == 2 * nblk * w.n_kv_heads * 2 * 77 * ng * 8
    assert lay.page_table_stride == (plain.max_pages + 3) // 4 * 4
    assert lay.page_table_bytes == 3 * lay.page_table_stride * 4
    assert list(lay.idx_strides)[4:] == [ng * 8, 8, 1, 0]
    assert plain.page_table_bytes == 0 and plain.page_table_stride == 0
    L = lvq.lib()
    # any call that reads or writes codes needs the table (host check, before any device work)
    st = L.lvq_decode_attention(ctypes.byref(cfg), ctypes.byref(lay), 0, 0, 1, *([None] * 8), 1,
                                None, None, None, None, None, None)
    assert st == lvq.LVQ_EINVAL
    cfg.page_table = 1 << 20
    fake = 1 << 20
    st = L.lvq_kmeans_update(ctypes.byref(cfg), ctypes.byref(lay), 0, 0, fake, w.n_kv_heads * w.head_dim, 64, 0,
                             64, 0, fake, fake, None, None, None)
    assert st == lvq.LVQ_EUNSUPPORTED                # codebooks are built on per-request streams
    cfg.page_table = (1 << 20) + 4                   # misaligned table
    assert lvq.lib().lvq_cache_layout(ctypes.byref(cfg), ctypes.byref(lvq.lvq_layout())) == lvq.LVQ_EINVAL
