"""The allocation-free decode entry point (runs last: a failure here leaves every
other test already run).

lvq_decode_attention_noalloc serves callers that cannot allocate device memory
for the decode workspace -- a plugin inside a serving engine whose memory pool
owns the device, or a deployment that forbids allocations after start-up.  Its
workspace is a 4 MiB device array inside the library.  Two calls in a row must
give what lvq_decode_attention gives with a caller-owned workspace.
"""
import dataclasses

import pytest
import torch

from sub_bit_kv_b200 import lvq, synth
from tests import _helpers as Hl

pytestmark = pytest.mark.gpu


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
    from sub_bit_kv_b200 import _build
    _build.build()
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


def test_noalloc_rejects_a_layout_beyond_its_array():
    w = dataclasses.replace(synth.WORKLOADS["ouro14_g16_32k"], n_layers=1)
    cfg = Hl.make_cfg(w, max_batch=64, max_ctx=1024, max_splits=256)
    lay = lvq.lvq_cache_layout(cfg)
    assert lay.workspace_bytes > 4 << 20
    import ctypes
    st = lvq.lib().lvq_decode_attention_noalloc(ctypes.byref(cfg), ctypes.byref(lay), 0, 0, 1, *([None] * 8), 1,
                                                None, None, None, None, None)
    assert st == lvq.LVQ_ECAPACITY
