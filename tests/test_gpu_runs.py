"""Decode launches with fewer CTAs than work items (request, query head, split): every CTA walks
a contiguous, cost-balanced run of items in (KV head, request, split, query head) order, keeping
the step slices of a KV head in shared memory across its items and streaming the next item's
code pages while it finishes the current one; the compute warps compute each item's bf16 share.
The CTA cap (lvq_decode_max_ctas) selects that path.  Any two such grids give the same
bits (the per-item arithmetic does not depend on the CTA); against one CTA per item (whose
producer warp computes the bf16 share in another fp32 order) they agree to the fp32 reordering
bound, and both match the oracle."""
import dataclasses

import numpy as np
import pytest
import torch

from sub_bit_kv_b200 import lvq, synth
from tests import _helpers as Hl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from sub_bit_kv_b200 import _build
    _build.build()
    assert torch.cuda.is_available()
    yield
    lvq.lvq_decode_max_ctas(0)


def _reduced(name, **kw):
    return dataclasses.replace(synth.WORKLOADS[name], **kw)


def _run(case, layer, step, q, ns, cap):
    lvq.lvq_decode_max_ctas(cap)
    try:
        return Hl.run_decode(case, layer, step, q, ns)
    finally:
        lvq.lvq_decode_max_ctas(0)


def _equal(a, b):
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def _close(case, a, b):
    """Two decodes of one case computed in different fp32 orders: outputs are convex combinations
    of value elements, so they agree to 2^-15 of the largest value magnitude (the bound of the
    split-count sweep); LSEs and split LSEs to the LSE tolerance."""
    vmax = 0.0
    for key in case.sink_kv:
        vmax = max(vmax, float(case.sink_kv[key][1].abs().max()), float(case.ring_kv[key][1].abs().max()))
    for cb in case.cb:
        vmax = max(vmax, float(cb[1].abs().max()))
    assert float((a[0] - b[0]).abs().max()) <= 2.0 ** -15 * vmax
    for x, y in ((a[1], b[1]), (a[2], b[2])):
        fin = torch.isfinite(y)
        assert torch.equal(torch.isfinite(x), fin)
        assert bool(((x[fin] - y[fin]).abs() <= Hl.LSE_REL * torch.clamp(y[fin].abs(), min=1.0)).all())


@pytest.mark.parametrize("name", ["ouro14_g16_32k", "ouro14_g32_b32", "ouro14_tc2_64k"])
def test_capped_grid_matches_one_cta_per_item_and_the_oracle(name):
    """GQA (2 query heads per KV head), ragged requests, one with no coded tokens at all: 60
    items on 1, 3 and 7 CTAs (KV-head changes inside a CTA's run) against one CTA per item."""
    w = _reduced(name, n_layers=1, n_kv_heads=2, n_q_heads=4, batch=3)
    S, R = w.n_sink, w.n_recent
    ctx = [S + 2333 + R, S + 37, S + 901 + R]           # request 1: sink and recent tokens only
    coded = [2333, 0, 901]
    case = Hl.build_case(w, layers=1, ctx=ctx, coded=coded, max_splits=16)
    ns = 5
    for step in (0, w.T - 1):
        q = synth.queries(w, 0, step, batch=3).cuda()
        single = _run(case, 0, step, q, ns, 0)
        ref = _run(case, 0, step, q, ns, 1)
        for cap in (3, 7, 3):                          # the last repeat: the merge counters came back to zero
            _equal(ref, _run(case, 0, step, q, ns, cap))
        _close(case, ref, single)
        out, lse, sl = ref
        for b, hq in ((0, 0), (0, 3), (1, 1), (2, 2)):
            ro, rl, rsl = Hl.oracle_decode(case, 0, step, b, hq, q, n_splits=ns)
            assert float(np.abs(out[b, hq].numpy() - ro).max()) <= Hl.OUT_ATOL
            Hl.assert_lse_close(float(lse[b, hq]), rl)
            for j in range(ns + 1):
                Hl.assert_lse_close(float(sl[b, hq, j]), float(rsl[j]), f"split {j}")


def test_gqa_with_more_items_than_sms():
    """Two query heads per KV head and 320 items: on 148 CTAs (one per SM) and on 11 the runs give
    the same bits, agree with one CTA per item to the fp32 reordering bound, and sampled heads
    match the oracle."""
    w = _reduced("ouro14_g16_32k", n_layers=1, n_kv_heads=8, n_q_heads=16, batch=4)
    S, R = w.n_sink, w.n_recent
    coded = [1500, 333, 2800, 64]
    ctx = [S + c + R for c in coded]
    case = Hl.build_case(w, layers=1, ctx=ctx, coded=coded, max_splits=8)
    ns = 5
    assert 4 * 16 * ns > 148
    q = synth.queries(w, 0, 2, batch=4).cuda()
    ref = _run(case, 0, 2, q, ns, 148)
    _equal(ref, _run(case, 0, 2, q, ns, 11))
    _close(case, ref, _run(case, 0, 2, q, ns, 0))
    out, lse, _ = ref
    for b, hq in ((0, 0), (1, 15), (2, 6), (3, 9)):
        ro, rl, _ = Hl.oracle_decode(case, 0, 2, b, hq, q, n_splits=ns)
        assert float(np.abs(out[b, hq].numpy() - ro).max()) <= Hl.OUT_ATOL
        Hl.assert_lse_close(float(lse[b, hq]), rl)


def test_capped_grid_through_a_page_table():
    from tests.test_gpu_pool import _pool_case, _scatter_codes
    w = _reduced("ouro14_g32_b32", n_layers=1, n_kv_heads=2, n_q_heads=2, batch=3)
    S, R = w.n_sink, w.n_recent
    ctx = [S + 1901 + R, S + 777 + R, S + 35 + R]
    case = Hl.build_case(w, layers=1, ctx=ctx, max_splits=16)
    need = [(cd + 7) // 8 for cd in case.coded]
    cfg, pc = _pool_case(case, pool_pages=sum(need) * 2 + 40, need=need)
    _scatter_codes(case, pc, need)
    pcase = dataclasses.replace(case, cfg=cfg, cache=pc)
    q = synth.queries(w, 0, 1, batch=3).cuda()
    for cap in (2, 5):
        _equal(_run(case, 0, 1, q, 4, cap), _run(pcase, 0, 1, q, 4, cap))
