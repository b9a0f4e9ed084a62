"""Pool mode (an 8-token page table over shared per-(layer, block, head, K/V) page pools) on
the GPU: decode, prefill encode and page encode through fragmented page tables give exactly
what the per-request streams give, and the oracle's results; an out-of-range page-table entry
is reported, not followed."""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import lvq_oracle as O
from sub_bit_kv_b200 import lvq, synth
from tests import _helpers as Hl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from sub_bit_kv_b200 import _build
    _build.build()
    assert torch.cuda.is_available()


def _reduced(name, **kw):
    return dataclasses.replace(synth.WORKLOADS[name], **kw)


def _pool_case(case, pool_pages, need, seed=3):
    """A pool-mode copy of `case` (same codebooks, bf16 tokens, counters), request b holding
    need[b] logical pages.  Request 0 takes its pages from the allocator in bites of 3,
    interleaved with the other requests' bites and with short-lived pages freed again (so its
    pages are runs with holes); request 1's pages are a random permutation of free ids written
    straight into the table (no two consecutive); the rest come from the allocator."""
    cfg = lvq.lvq_config.from_buffer_copy(case.cfg)
    cfg.pool_pages = pool_pages
    cfg.page_table = None
    pc = lvq.CodedCache(cfg)
    src = case.cache
    for name in ("cb", "cbp", "cb_norm", "sink", "ring", "rope", "ctx_len", "coded_len"):
        getattr(pc, name).copy_(getattr(src, name))
    B = len(need)
    scratch = []
    left = list(need)
    while any(left[b] > 0 for b in range(B) if b != 1):
        for b in range(B):
            if b == 1 or left[b] <= 0:
                continue
            k = min(3, left[b])
            pc.assign_pages(b, len(pc.pages[b]) + k)
            left[b] -= k
            scratch += pc.pool.alloc(1)             # a hole after every bite
    pc.pool.free(scratch)
    if B > 1 and need[1] > 0:
        rng = np.random.default_rng(seed)
        ids = pc.pool.alloc(need[1] * 2)
        mine = [int(i) for i in rng.permutation(ids)[:need[1]]]
        pc.pool.free([i for i in ids if i not in mine])
        pc.pages[1] = mine
        stride = pc.lay.page_table_stride
        pc.page_table[stride:stride + need[1]].copy_(torch.tensor(mine, dtype=torch.int32))
    torch.cuda.synchronize()
    return cfg, pc


def _scatter_codes(case, pc, need):
    """The case's per-request code pages, copied to their physical pages."""
    sv = case.cache.idx_view()                      # [L][n_blk][B][H][2][P][n_g][8]
    dv = pc.idx_view()                              # [L][n_blk][H][2][pool][n_g][8]
    for b, n in enumerate(need):
        for i in range(n):
            dv[:, :, :, :, pc.pages[b][i]] = sv[:, :, b, :, :, i]


def _pool_codes(pc, layer, b, kv, offset, N):
    """Logical codes [n_blk][N][H][n_g] of request b read back through its pages."""
    dv = pc.idx_view()
    pages = [dv[layer, :, :, kv, pc.pages[b][i]] for i in range((offset + N + 7) // 8)]   # [n_blk][H][n_g][8]
    flat = torch.stack(pages, dim=2)                # [n_blk][H][pages][n_g][8]
    flat = flat.permute(0, 1, 2, 4, 3).reshape(flat.shape[0], flat.shape[1], -1, flat.shape[3])
    return flat[:, :, offset:offset + N].permute(0, 2, 1, 3).cpu()


@pytest.mark.parametrize("name", ["ouro14_g16_32k", "ouro14_tc2_64k"])
def test_decode_through_a_fragmented_page_table(name):
    w = _reduced(name, n_layers=1, n_kv_heads=2, n_q_heads=2, batch=3)
    ctx = [w.n_sink + 2901 + w.n_recent, w.n_sink + 1203 + w.n_recent, w.n_sink + 517 + w.n_recent]
    case = Hl.build_case(w, layers=1, ctx=ctx, max_splits=16)
    need = [(cd + 7) // 8 for cd in case.coded]
    cfg, pc = _pool_case(case, pool_pages=sum(need) * 2 + 40, need=need)
    _scatter_codes(case, pc, need)
    pcase = dataclasses.replace(case, cfg=cfg, cache=pc)
    for step in (0, w.T - 1):
        q = synth.queries(w, 0, step, batch=3).cuda()
        for ns in (1, 5):
            ref = Hl.run_decode(case, 0, step, q, ns)
            got = Hl.run_decode(pcase, 0, step, q, ns)
            for a, b in zip(ref, got):
                assert torch.equal(a, b)            # the same tokens, read through the page table
        out, lse, _ = got
        for b, hq in ((0, 0), (1, 1), (2, 0)):
            ro, rl, _ = Hl.oracle_decode(case, 0, step, b, hq, q)
            assert float(np.abs(out[b, hq].numpy() - ro).max()) <= Hl.OUT_ATOL
            Hl.assert_lse_close(float(lse[b, hq]), rl)


@pytest.mark.parametrize("name", ["ouro14_g16_32k", "ouro14_tc2_64k"])
def test_prefill_and_page_encode_write_through_the_page_table(name):
    w = _reduced(name, n_layers=2, n_kv_heads=2, n_q_heads=2, batch=2, n_recent=16)
    R = w.n_recent + 8
    coded = [301, 77]
    ctx = [w.n_sink + coded[0] + R, w.n_sink + coded[1] + R - 1]     # request 0 due, request 1 not
    case = Hl.build_case(w, layers=2, ctx=ctx, coded=coded, codes_from="none")
    need = [(coded[0] + 8 + 7) // 8, (coded[1] + 8 + 7) // 8]       # room for the page encode
    cfg, pc = _pool_case(case, pool_pages=200, need=need)
    for layer in range(2):
        for b in range(2):
            kv = synth.loop_kv(w, layer, coded[b], stream="pool-enc", request=b).cuda()
            lvq.lvq_encode_prefill(cfg, pc.lay, layer, b, kv, 0, coded[b], 0, pc.cb, pc.idx, pc.status)
    torch.cuda.synchronize()
    pc.check_status()
    for layer in range(2):
        cbl = Hl.f64(case.cb[layer])
        for b in range(2):
            x = Hl.f64(synth.loop_kv(w, layer, coded[b], stream="pool-enc", request=b))
            for kvi in range(2):
                got = _pool_codes(pc, layer, b, kvi, 0, coded[b]).numpy()
                X = O.joint_vectors(x[kvi], w.Tc, w.G)
                for blk in range(X.shape[0]):
                    for h in range(X.shape[2]):
                        for g in range(X.shape[3]):
                            ref, a1, a2 = O.nearest_entry(X[blk, :, h, g], cbl[kvi, blk, h, g])
                            ok = (got[blk, :, h, g] == ref) | O.near_tie(a1, a2)
                            assert ok.all()
    # the page encode: request 0's 8 oldest recent tokens go to its logical page 37 .. (offset 301)
    lvq.lvq_encode_page(cfg, pc.lay, 2, pc.ctx_len, pc.coded_len, pc.ring, pc.cb, pc.cb_norm, pc.idx, pc.status)
    torch.cuda.synchronize()
    pc.check_status()
    assert pc.coded_len.cpu().tolist()[:2] == [coded[0] + 8, coded[1]]
    for layer in range(2):
        rk = Hl.f64(case.ring_kv[(layer, 0)])
        ck, cv = O.page_encode(rk[0], rk[1], Hl.f64(case.cb[layer][0]), Hl.f64(case.cb[layer][1]), w.Tc, w.G)
        for kvi, ref in ((0, ck), (1, cv)):
            got = _pool_codes(pc, layer, 0, kvi, coded[0], 8).numpy()
            assert (got == ref).mean() > 0.999      # near-ties aside (checked in the per-request tests)


def test_out_of_range_page_entry_is_reported():
    """A page-table entry past the pool: the decode reports LVQ_ECAPACITY (reading page 0 in
    its place, in bounds) and the context stays usable."""
    w = _reduced("ouro14_g16_32k", n_layers=1, n_kv_heads=2, n_q_heads=2, batch=1)
    case = Hl.build_case(w, layers=1, ctx=[w.n_sink + 700 + w.n_recent])
    need = [(case.coded[0] + 7) // 8]
    cfg, pc = _pool_case(case, pool_pages=2 * need[0] + 8, need=need)
    _scatter_codes(case, pc, need)
    pcase = dataclasses.replace(case, cfg=cfg, cache=pc)
    q = synth.queries(w, 0, 1, batch=1).cuda()
    good = Hl.run_decode(pcase, 0, 1, q, 3)
    pc.page_table[5] = cfg.pool_pages              # out of range
    out = torch.empty(1, w.n_q_heads, w.head_dim, dtype=torch.float32, device="cuda")
    lse = torch.empty(1, w.n_q_heads, dtype=torch.float32, device="cuda")
    lvq.lvq_decode_attention(cfg, pc.lay, 0, 1, 1, q, pc.ctx_len, pc.coded_len, pc.sink, pc.ring, pc.idx, pc.cbp,
                             pc.rope, 3, pc.workspace, out, lse, pc.status)
    torch.cuda.synchronize()
    assert int(pc.status.item()) == lvq.LVQ_ECAPACITY
    pc.status.zero_()
    pc.page_table[5] = pc.pages[0][5]
    again = Hl.run_decode(pcase, 0, 1, q, 3)
    assert torch.equal(good[0], again[0])


def test_released_pages_are_reused():
    w = _reduced("ouro14_g16_32k", n_layers=1, n_kv_heads=1, n_q_heads=1, batch=2)
    cfg = Hl.make_cfg(w, n_layers=1, max_batch=2, max_ctx=4096)
    cfg.pool_pages = 10
    pc = lvq.CodedCache(cfg)
    assert pc.assign_pages(0, 4) == [0, 1, 2, 3]
    assert pc.assign_pages(1, 3) == [4, 5, 6]
    pc.release(0)
    assert pc.pool.available() == 7
    assert int((pc.page_table[:pc.lay.page_table_stride] == -1).sum()) == pc.lay.page_table_stride
    assert pc.assign_pages(0, 2) == [0, 1]
