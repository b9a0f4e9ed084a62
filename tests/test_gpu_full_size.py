"""Decode parity at the full sizes of the workloads, in the launch configuration bench.py
times (its choice of num_splits for one GPU): sampled (request, head) outputs against the
fp64 oracle, computed one by one, and for every head a property that holds at any size --
the result does not depend on the number of splits.  Codes are seeded random bytes
written from the host (never produced by the CUDA path)."""
import numpy as np
import pytest
import torch

import _helpers as Hl
import bench
from sub_bit_kv_b200 import synth

pytestmark = pytest.mark.gpu


def _n_sm():
    return torch.cuda.get_device_properties(0).multi_processor_count


@pytest.mark.parametrize("name,samples", [
    ("ouro14_g16_32k", [(0, 0), (0, 7), (0, 15)]),         # 32K context, batch 1, G=16 (c=4)
    ("ouro14_g32_b32", [(0, 3), (13, 9), (31, 15)]),       # 32 ragged requests, G=32 (c=8)
    ("ouro14_tc2_64k", [(0, 0), (5, 11), (7, 15)]),        # 64K context, batch 8, Tc=2 (two blocks)
    ("ouro14_tc1_32k", [(0, 2), (0, 13)]),                 # 32K context, per-step coding (Tc=1, c=16)
])
def test_decode_full_size_sampled(name, samples):
    w = synth.WORKLOADS[name]
    ctx = synth.ctx_lengths(w)
    ns = bench.choose_splits(w, _n_sm())
    ns2 = 2 * ns + 1
    case = Hl.build_case(w, layers=1, ctx=ctx, max_splits=max(32, ns2))
    for step in sorted({0, w.T - 1}):
        q = synth.queries(w, 0, step).cuda()
        out, lse, sl = Hl.run_decode(case, 0, step, q, ns)
        assert torch.isfinite(out).all() and torch.isfinite(lse).all()
        for b, hq in samples:
            ro, rl, rs = Hl.oracle_decode(case, 0, step, b, hq, q, n_splits=ns)
            err = float(np.abs(out[b, hq].numpy() - ro).max())
            assert err <= Hl.OUT_ATOL, (name, step, b, hq, err)
            Hl.assert_lse_close(float(lse[b, hq]), rl, "lse")
            for j in range(ns + 1):
                Hl.assert_lse_close(float(sl[b, hq, j]), float(rs[j]), f"split {j}")
        out2, lse2, _ = Hl.run_decode(case, 0, step, q, ns2, split_lse=False)
        assert float((out - out2).abs().max()) <= 1e-4
        assert float((lse - lse2).abs().max()) <= 1e-4


def test_encode_prefill_full_layer_sampled():
    """One Ouro-2.6B-shaped prefill layer (32768 tokens x 16 heads x K/V x 32 groups = 33.5 M
    joint vectors), encoded as bench.py encodes it; 8192 sampled vectors checked against the
    oracle's brute-force nearest entry (exact except near-ties, where the entry must lie within
    the tie gap)."""
    from oracle import lvq_oracle as O
    from sub_bit_kv_b200 import lvq
    wc = synth.WORKLOADS["ouro26_prefill_32k"]
    cfg = lvq.make_config(1, wc.n_kv_heads, wc.n_q_heads, wc.head_dim, wc.T, wc.Tc, wc.G, 0, 0, 1, wc.ctx,
                          max_splits=1, rope_base=wc.rope_base)
    c = lvq.CodedCache(cfg, "cuda")
    cb = synth.codebooks(wc, 0)
    c.cb_view()[0] = cb.cuda()
    kv = synth.loop_kv(wc, 0, wc.ctx, stream="coded", device="cuda")      # [2][T][N][H][d] bf16
    lvq.lvq_encode_prefill(cfg, c.lay, 0, 0, kv, 0, wc.ctx, 0, c.cb, c.idx, c.status)
    torch.cuda.synchronize()
    c.check_status()
    lay = c.lay
    g = torch.Generator().manual_seed(7)
    M = 8192
    kvi = torch.randint(0, 2, (M,), generator=g)
    n = torch.randint(0, wc.ctx, (M,), generator=g)
    h = torch.randint(0, wc.n_kv_heads, (M,), generator=g)
    grp = torch.randint(0, lay.n_groups, (M,), generator=g)
    blk = torch.randint(0, lay.n_blocks, (M,), generator=g)
    idx = c.idx_view()                                      # [L][n_blk][B][H][2][P][n_g][8]
    got = idx[0, blk, 0, h, kvi, n // 8, grp, n % 8].cpu().numpy()
    xs = kv[kvi, :, n, h].cpu()                              # [M][T][d]
    cbf = Hl.f64(cb)                                         # [2][n_blk][H][n_g][256][G]
    cc = wc.G // wc.Tc
    ties = 0
    for m in range(M):
        x = Hl.f64(xs[m])                                    # [T][d]
        b_, g_ = int(blk[m]), int(grp[m])
        X = np.concatenate([x[b_ * wc.Tc + s, g_ * cc:(g_ + 1) * cc] for s in range(wc.Tc)])[None]
        C = cbf[int(kvi[m]), b_, int(h[m]), g_]
        ref, d1, d2 = O.nearest_entry(X, C)
        if got[m] != ref[0]:
            assert O.near_tie(d1, d2)[0], (m, int(got[m]), int(ref[0]))
            dg = float(((X[0] - C[int(got[m])]) ** 2).sum())
            assert dg - d1[0] <= O.NEAR_TIE_REL * d1[0]
            ties += 1
    assert ties <= M // 100


def test_page_encode_full_heads():
    """The decode-time page encode at the Ouro-1.4B shapes (16 heads, 32 groups, 128-token
    window, 32K context; two of the 24 layers): every code of the page against the oracle."""
    from oracle import lvq_oracle as O
    from sub_bit_kv_b200 import lvq
    w = synth.WORKLOADS["ouro14_g16_32k"]
    R = w.n_recent + 8
    coded = w.ctx - w.n_sink - R
    case = Hl.build_case(w, layers=2, ctx=[w.ctx], coded=[coded], max_splits=16)
    c = case.cache
    lvq.lvq_encode_page(case.cfg, c.lay, 1, c.ctx_len, c.coded_len, c.ring, c.cb, c.cb_norm, c.idx, c.status)
    torch.cuda.synchronize()
    c.check_status()
    assert c.coded_len.cpu().tolist() == [coded + 8]
    for layer in range(2):
        rk = Hl.f64(case.ring_kv[(layer, 0)])                 # [2][T][R][H][d], oldest first
        ck, cv = O.page_encode(rk[0], rk[1], Hl.f64(case.cb[layer][0]), Hl.f64(case.cb[layer][1]), w.Tc, w.G)
        for kvi, ref in enumerate((ck, cv)):
            got = Hl.get_codes(c, layer, 0, kvi, coded, 8).numpy()      # [n_blk][8][H][n_g]
            diff = got != ref
            if diff.any():                                    # only near-ties may differ
                X = O.joint_vectors(rk[kvi][:, :8], w.Tc, w.G)
                cbk = Hl.f64(case.cb[layer][kvi])
                for blk_, t, h, g in zip(*np.nonzero(diff)):
                    _, d1, d2 = O.nearest_entry(X[blk_, t, h, g][None], cbk[blk_, h, g])
                    assert O.near_tie(d1, d2)[0]
            assert diff.mean() <= 0.001
