"""The allocation-free decode entry point (runs last: a failure here leaves every
other test already run).

lvq_decode_attention_noalloc serves callers that cannot allocate device memory
for the decode workspace -- a plugin inside a serving engine whose memory pool
owns the device, or a deployment that forbids allocations after start-up.  Its
workspace is a 4 MiB device array inside the library.  Two calls in a row must
give what lvq_decode_attention gives with a caller-owned workspace.
"""
import dataclasses

import numpy as np
import pytest
import torch

from sub_bit_kv_b200 import _build, lvq, synth
from tests import _helpers as Hl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    _build.build()


def _call(case, fn, layer, step, q, ns, **extra):
    c = case.cache
    B = len(case.ctx)
    out = torch.empty(B, case.w.n_q_heads, case.w.head_dim, dtype=torch.float32, device="cuda")
    lse = torch.empty(B, case.w.n_q_heads, dtype=torch.float32, device="cuda")
    fn(case.cfg, c.lay, layer, step, B, q, c.ctx_len, c.coded_len, c.sink, c.ring, c.idx, c.cbp, c.rope, ns,
       *extra.get("ws", ()), out, lse, c.status)
    torch.cuda.synchronize()
    c.check_status()
    return out.cpu(), lse.cpu()


def test_noalloc_decode_matches_workspace_decode_twice():
    w = dataclasses.replace(synth.WORKLOADS["ouro14_g16_32k"], n_layers=2, n_kv_heads=2, n_q_heads=2)
    case = Hl.build_case(w, layers=2, ctx=[1900, 700], max_splits=16)
    assert case.cache.lay.workspace_bytes <= 4 << 20
    for call in range(2):                       # two calls in a row share the library's array
        layer, step, ns = call, 1 + call, 5 + 3 * call
        q = synth.queries(w, layer, step, batch=2, token=call).cuda()
        ref_out, ref_lse = _call(case, lvq.lvq_decode_attention, layer, step, q, ns, ws=(case.cache.workspace,))
        out, lse = _call(case, lvq.lvq_decode_attention_noalloc, layer, step, q, ns)
        assert float((out - ref_out).abs().max()) <= Hl.OUT_ATOL
        assert float((lse - ref_lse).abs().max()) <= Hl.LSE_REL * max(1.0, float(ref_lse.abs().max()))
        # and directly against the fp64 oracle, every request and head
        for b in range(2):
            for hq in range(w.n_q_heads):
                ro, rl, _ = Hl.oracle_decode(case, layer, step, b, hq, q.cpu())
                assert float(np.abs(out[b, hq].numpy() - ro).max()) <= Hl.OUT_ATOL
                Hl.assert_lse_close(float(lse[b, hq]), rl, (b, hq))


def test_noalloc_clears_the_counters_of_each_layout():
    """The merge counters sit after the partials, so their place in the shared array moves
    with the layout.  A call with many splits fills the array's start with partials; a
    following call whose layout puts its counters inside that region must clear them
    before its kernel runs (else the last CTA of a head is never recognised)."""
    w = dataclasses.replace(synth.WORKLOADS["ouro14_g16_32k"], n_layers=1, n_kv_heads=4, n_q_heads=4)
    big = Hl.build_case(w, layers=1, ctx=[3000], max_splits=96)
    small = Hl.build_case(w, layers=1, ctx=[2500], max_splits=4)
    # the small layout's counters lie inside the big layout's partial region
    assert small.cache.lay.workspace_bytes < big.cache.lay.workspace_bytes <= 4 << 20
    for rnd in range(2):
        q = synth.queries(w, 0, 2, batch=1, token=rnd).cuda()
        _call(big, lvq.lvq_decode_attention_noalloc, 0, 2, q, 96)
        out, lse = _call(small, lvq.lvq_decode_attention_noalloc, 0, 2, q, 3)
        ref_out, ref_lse = _call(small, lvq.lvq_decode_attention, 0, 2, q, 3, ws=(small.cache.workspace,))
        assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)


def test_noalloc_after_a_timed_out_call():
    """A noalloc call whose bounded waits run out (test hook: a copy that never happens) reports
    LVQ_ETIMEOUT and leaves the shared array's counters exact: the next noalloc call matches the
    workspace path bit for bit."""
    w = dataclasses.replace(synth.WORKLOADS["ouro14_g16_32k"], n_layers=1, n_kv_heads=2, n_q_heads=2)
    case = Hl.build_case(w, layers=1, ctx=[1500], max_splits=8)
    c = case.cache
    q = synth.queries(w, 0, 3, batch=1).cuda()
    out = torch.empty(1, w.n_q_heads, w.head_dim, dtype=torch.float32, device="cuda")
    lse = torch.empty(1, w.n_q_heads, dtype=torch.float32, device="cuda")
    lvq.lvq_debug_faults(1 << 12, 1)
    try:
        lvq.lvq_decode_attention_noalloc(case.cfg, c.lay, 0, 3, 1, q, c.ctx_len, c.coded_len, c.sink, c.ring, c.idx,
                                         c.cbp, c.rope, 4, out, lse, c.status)
        torch.cuda.synchronize()
    finally:
        lvq.lvq_debug_faults(0, 0)
    assert int(c.status.item()) == lvq.LVQ_ETIMEOUT
    c.status.zero_()
    got_out, got_lse = _call(case, lvq.lvq_decode_attention_noalloc, 0, 3, q, 4)
    ref_out, ref_lse = _call(case, lvq.lvq_decode_attention, 0, 3, q, 4, ws=(c.workspace,))
    assert torch.equal(got_out, ref_out) and torch.equal(got_lse, ref_lse)


def test_noalloc_rejects_a_layout_beyond_its_array():
    """Checked on the host before anything is launched."""
    w = dataclasses.replace(synth.WORKLOADS["ouro14_g16_32k"], n_layers=1)
    cfg = Hl.make_cfg(w, max_batch=64, max_ctx=1024, max_splits=256)
    lay = lvq.lvq_cache_layout(cfg)
    assert lay.workspace_bytes > 4 << 20
    import ctypes
    st = lvq.lib().lvq_decode_attention_noalloc(ctypes.byref(cfg), ctypes.byref(lay), 0, 0, 1, *([None] * 8), 1,
                                                None, None, None, None, None)
    assert st == lvq.LVQ_ECAPACITY
