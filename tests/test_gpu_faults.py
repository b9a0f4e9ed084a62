"""Failure detection on the GPU without a GPU fault: the test hook shortens every
device-side wait and makes one copy never happen, so a bounded wait runs out; the kernel
reports LVQ_ETIMEOUT through the status word and returns (no trap, nothing left in
flight), and the same context then computes correct results again."""
import numpy as np
import pytest
import torch

from sub_bit_kv_b200 import lvq, synth
from tests import _helpers as Hl

pytestmark = pytest.mark.gpu

SHORT_WAIT = 1 << 12


@pytest.fixture(scope="module", autouse=True)
def built():
    from sub_bit_kv_b200 import _build
    _build.build()
    assert torch.cuda.is_available()
    yield
    lvq.lvq_debug_faults(0, 0)
    lvq.lvq_decode_max_ctas(0)


def test_decode_wait_runs_out_then_context_recovers():
    w = synth.WORKLOADS["tiny"]
    case = Hl.build_case(w, layers=1, ctx=[512])
    c = case.cache
    q = synth.queries(w, 0, 1).cuda()
    out = torch.empty(1, w.n_q_heads, w.head_dim, dtype=torch.float32, device="cuda")
    lse = torch.empty(1, w.n_q_heads, dtype=torch.float32, device="cuda")
    lvq.lvq_debug_faults(SHORT_WAIT, 1)           # every CTA's first code chunk is never copied
    try:
        lvq.lvq_decode_attention(case.cfg, c.lay, 0, 1, 1, q, c.ctx_len, c.coded_len, c.sink, c.ring, c.idx,
                                 c.cbp, c.rope, 4, c.workspace, out, lse, c.status)
        torch.cuda.synchronize()
    finally:
        lvq.lvq_debug_faults(0, 0)
    assert int(c.status.item()) == lvq.LVQ_ETIMEOUT
    c.status.zero_()
    got, gl, _ = Hl.run_decode(case, 0, 1, q, 4, split_lse=False)
    ro, rl, _ = Hl.oracle_decode(case, 0, 1, 0, 0, q, n_splits=4)
    assert float(np.abs(got[0, 0].numpy() - ro).max()) <= Hl.OUT_ATOL
    Hl.assert_lse_close(float(gl[0, 0]), rl)


def test_decode_wait_runs_out_with_several_items_per_cta():
    """Two CTAs walking 24 items each: the first item's missing chunk aborts the CTA; the items
    left are written as failed partials (so the merge counters stay exact) and the next call,
    on the same capped grid, is correct."""
    import dataclasses
    w = dataclasses.replace(synth.WORKLOADS["ouro14_g16_32k"], n_layers=1, n_kv_heads=2, n_q_heads=4, batch=3)
    ctx = [w.n_sink + 700 + w.n_recent, w.n_sink + 1300 + w.n_recent, w.n_sink + 90 + w.n_recent]
    case = Hl.build_case(w, layers=1, ctx=ctx, max_splits=8)
    c = case.cache
    q = synth.queries(w, 0, 1, batch=3).cuda()
    out = torch.empty(3, w.n_q_heads, w.head_dim, dtype=torch.float32, device="cuda")
    lse = torch.empty(3, w.n_q_heads, dtype=torch.float32, device="cuda")
    lvq.lvq_decode_max_ctas(2)
    try:
        lvq.lvq_debug_faults(SHORT_WAIT, 1)       # each CTA's first code chunk is never copied
        try:
            lvq.lvq_decode_attention(case.cfg, c.lay, 0, 1, 3, q, c.ctx_len, c.coded_len, c.sink, c.ring, c.idx,
                                     c.cbp, c.rope, 4, c.workspace, out, lse, c.status)
            torch.cuda.synchronize()
        finally:
            lvq.lvq_debug_faults(0, 0)
        assert int(c.status.item()) == lvq.LVQ_ETIMEOUT
        c.status.zero_()
        got, gl, _ = Hl.run_decode(case, 0, 1, q, 4, split_lse=False)
    finally:
        lvq.lvq_decode_max_ctas(0)
    for b, hq in ((0, 0), (1, 3), (2, 1)):
        ro, rl, _ = Hl.oracle_decode(case, 0, 1, b, hq, q, n_splits=4)
        assert float(np.abs(got[b, hq].numpy() - ro).max()) <= Hl.OUT_ATOL
        Hl.assert_lse_close(float(gl[b, hq]), rl)


def test_kmeans_wait_runs_out_then_context_recovers():
    import dataclasses
    w = dataclasses.replace(synth.WORKLOADS["ouro14_g16_32k"], n_layers=1, n_kv_heads=1, n_q_heads=1)
    ntok = 600
    case = Hl.build_case(w, layers=1, ctx=[w.n_sink + ntok + w.n_recent], coded=[ntok], codes_from="none")
    c, cfg = case.cache, case.cfg
    kv = synth.loop_kv(w, 0, ntok, stream="kmeans").cuda()
    lvq.lvq_encode_prefill(cfg, c.lay, 0, 0, kv, 0, ntok, 0, c.cb, c.idx, c.status)
    torch.cuda.synchronize()
    c.check_status()
    before = c.cb_view()[0].clone()
    lvq.lvq_debug_faults(SHORT_WAIT, 2)           # every CTA's first tile is never copied
    try:
        lvq.lvq_kmeans_update(cfg, c.lay, 0, 0, kv, 0, ntok, 0, c.idx, c.cb, None, c.status)
        torch.cuda.synchronize()
    finally:
        lvq.lvq_debug_faults(0, 0)
    assert int(c.status.item()) == lvq.LVQ_ETIMEOUT
    assert torch.equal(c.cb_view()[0], before)    # a CTA that gave up writes no entry
    c.status.zero_()
    lvq.lvq_kmeans_update(cfg, c.lay, 0, 0, kv, 0, ntok, 0, c.idx, c.cb, None, c.status)
    torch.cuda.synchronize()
    c.check_status()
    assert not torch.equal(c.cb_view()[0], before)
