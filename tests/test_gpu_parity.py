"""CUDA path against the fp64 oracle on the same seeded inputs (needs a B200).

Tolerances: code indices bit-exact except counted near-ties (oracle top-2 gap
<= 1e-6 relative), which must pick an entry within that gap; dequantized bf16
bit-exact; attention output max-abs <= 2e-3; LSEs within 1e-4 * max(1, |lse|).
"""
import math

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
    import dataclasses
    return dataclasses.replace(synth.WORKLOADS[name], **kw)


def check_codes(gpu_codes: np.ndarray, X: np.ndarray, cb: np.ndarray):
    """gpu_codes [M], X [M][G] joint vectors, cb [256][G]: exact except near-ties."""
    idx, d1, d2 = O.nearest_entry(X, cb)
    tie = O.near_tie(d1, d2)
    diff = gpu_codes != idx
    assert not (diff & ~tie).any(), np.nonzero(diff & ~tie)[0][:10]
    for m in np.nonzero(diff)[0]:                       # a tie: the GPU's entry is within the gap
        dg = float(((X[m] - cb[gpu_codes[m]]) ** 2).sum())
        assert dg - d1[m] <= O.NEAR_TIE_REL * d1[m]
    return int(tie.sum()), int(diff.sum())


# ----------------------------------------------------------------------------------- encode

@pytest.mark.parametrize("name,ntok,offset,extra", [
    ("tiny", 492, 0, {}),
    ("ouro14_g16_32k", 333, 5, {}),
    ("ouro14_g16_32k", 2100, 0, {"n_kv_heads": 2, "n_q_heads": 2}),     # several token tiles and items
    ("ouro14_g32_b32", 130, 8, {}),
    ("ouro14_tc2_64k", 77, 3, {}),
    ("ouro14_g16_32k", 200, 1, {"Tc": 1, "n_kv_heads": 2, "n_q_heads": 2}),   # c = 16: fp64 direct form
])
def test_encode_prefill_matches_oracle(name, ntok, offset, extra):
    w = _reduced(name, n_layers=1, **extra) if name != "tiny" else synth.WORKLOADS[name]
    case = Hl.build_case(w, layers=1, ctx=[w.n_sink + ntok + offset + w.n_recent], coded=[ntok + offset],
                         codes_from="none")
    c = case.cache
    kv = synth.loop_kv(w, 0, ntok + 10, stream="enc")
    lvq.lvq_encode_prefill(case.cfg, c.lay, 0, 0, kv.cuda(), 10, ntok, offset, c.cb, c.idx, c.status)
    torch.cuda.synchronize()
    c.check_status()
    cb = Hl.f64(case.cb[0])                              # [2][n_blk][H][n_g][256][G]
    x = Hl.f64(kv[:, :, 10:10 + ntok])                   # [2][T][N][H][d]
    ties = 0
    for kvi in range(2):
        got = Hl.get_codes(c, 0, 0, kvi, offset, ntok).numpy()   # [n_blk][N][H][n_g]
        X = O.joint_vectors(x[kvi], w.Tc, w.G)                    # [n_blk][N][H][n_g][G]
        for blk in range(X.shape[0]):
            for h in range(X.shape[2]):
                for g in range(X.shape[3]):
                    t, _ = check_codes(got[blk, :, h, g], X[blk, :, h, g], cb[kvi, blk, h, g])
                    ties += t
    print(f"{name}: near-ties {ties}")


@pytest.mark.parametrize("name,extra", [
    ("ouro14_g16_32k", {"n_kv_heads": 2, "n_q_heads": 2}),                 # tensor-core encoder, one launch
    ("ouro14_tc2_64k", {"n_kv_heads": 2, "n_q_heads": 2}),                 # c = 8, two blocks per token
    ("ouro14_g16_32k", {"Tc": 1, "n_kv_heads": 1, "n_q_heads": 1}),        # c = 16: direct form, per layer
])
def test_encode_prefill_all_layers_in_one_call(name, extra):
    """layer = -1: the K/V of every layer back to back, encoded by one call; every layer's codes
    equal the oracle's nearest entries (near-ties excepted), and none spill into another layer."""
    w = _reduced(name, n_layers=3, **extra)
    ntok, offset = 1500, 3
    case = Hl.build_case(w, layers=3, ctx=[w.n_sink + ntok + offset + w.n_recent], coded=[ntok + offset],
                         codes_from="none")
    c = case.cache
    kvs = [synth.loop_kv(w, layer, ntok, stream="enc-all") for layer in range(3)]   # [2][T][N][H][d] each
    kv_all = torch.stack(kvs).cuda()                                                # [L][2][T][N][H][d]
    c.idx.zero_()
    lvq.lvq_encode_prefill(case.cfg, c.lay, -1, 0, kv_all, 0, ntok, offset, c.cb, c.idx, c.status)
    torch.cuda.synchronize()
    c.check_status()
    for layer in range(3):
        cb = Hl.f64(case.cb[layer])
        x = Hl.f64(kvs[layer])
        for kvi in range(2):
            got = Hl.get_codes(c, layer, 0, kvi, offset, ntok).numpy()
            assert not Hl.get_codes(c, layer, 0, kvi, 0, offset).numpy().any()   # slots before the offset
            X = O.joint_vectors(x[kvi], w.Tc, w.G)
            for blk in range(X.shape[0]):
                for h in range(X.shape[2]):
                    for g in range(X.shape[3]):
                        check_codes(got[blk, :, h, g], X[blk, :, h, g], cb[kvi, blk, h, g])


@pytest.mark.parametrize("name,extra", [
    ("ouro14_g16_32k", {"n_kv_heads": 2, "n_q_heads": 2}),     # G = 16, c = 4 (tensor-core encoder)
    ("ouro14_g32_b32", {"n_kv_heads": 2, "n_q_heads": 2}),     # G = 32, c = 8
])
def test_encode_prefill_duplicate_entries_lowest_index(name, extra):
    """Exact ties: entries 128..191 repeat entries 0..63 (the twin lies four 32-entry blocks
    later) and entry 64+2j+1 repeats entry 64+2j (twins inside one block).  The direct form
    ranks twins equal, so the code is the lower index of the pair wherever a twin is nearest
    (the nearest-entry rule of the method, lowest index on ties)."""
    w = _reduced(name, n_layers=1, **extra)
    ntok = 700
    case = Hl.build_case(w, layers=1, ctx=[w.n_sink + ntok + w.n_recent], coded=[ntok], codes_from="none")
    c = case.cache
    cb = case.cb[0].clone()                                  # [2][n_blk][H][n_g][256][G]
    cb[..., 128:192, :] = cb[..., 0:64, :]
    cb[..., 65:128:2, :] = cb[..., 64:128:2, :]
    c.cb_view()[0] = cb.cuda()
    kv = synth.loop_kv(w, 0, ntok, stream="enc")
    lvq.lvq_encode_prefill(case.cfg, c.lay, 0, 0, kv.cuda(), 0, ntok, 0, c.cb, c.idx, c.status)
    torch.cuda.synchronize()
    c.check_status()
    cbf = Hl.f64(cb)
    x = Hl.f64(kv)
    exact_ties = 0
    for kvi in range(2):
        got = Hl.get_codes(c, 0, 0, kvi, 0, ntok).numpy()    # [n_blk][N][H][n_g]
        X = O.joint_vectors(x[kvi], w.Tc, w.G)
        for blk in range(X.shape[0]):
            for h in range(X.shape[2]):
                for g in range(X.shape[3]):
                    ref, d1, d2 = O.nearest_entry(X[blk, :, h, g], cbf[kvi, blk, h, g])
                    twin = d2 == d1
                    assert (got[blk, twin, h, g] == ref[twin]).all()
                    exact_ties += int(twin.sum())
                    check_codes(got[blk, :, h, g], X[blk, :, h, g], cbf[kvi, blk, h, g])
    assert exact_ties > 0


def test_codebook_entries_reencode_to_own_index():
    w = synth.WORKLOADS["tiny"]
    case = Hl.build_case(w, layers=1, ctx=[w.n_sink + 256 + w.n_recent], coded=[256], codes_from="none")
    c = case.cache
    cb = case.cb[0]                                       # [2][1][1][n_g][256][G]
    # tokens whose joint vectors are exactly entry k of every group: x[t][n][h][g*c+e] = cb[..g][n][t*c+e]
    kv = torch.empty(2, w.T, 256, 1, w.head_dim, dtype=torch.bfloat16)
    for g in range(w.n_groups):
        for t in range(w.T):
            kv[:, t, :, 0, g * w.c:(g + 1) * w.c] = cb[:, 0, 0, g, :, t * w.c:(t + 1) * w.c]
    lvq.lvq_encode_prefill(case.cfg, c.lay, 0, 0, kv.cuda(), 0, 256, 0, c.cb, c.idx, c.status)
    torch.cuda.synchronize()
    for kvi in range(2):
        got = Hl.get_codes(c, 0, 0, kvi, 0, 256)[0, :, 0, :]    # [256][n_g]
        assert (got.long() == torch.arange(256)[:, None]).all()


# ----------------------------------------------------------------------------------- dequant

@pytest.mark.parametrize("name", ["tiny", "ouro14_tc2_64k", "ouro14_g32_b32", "ouro14_tc1_32k"])
def test_dequantize_bit_exact(name):
    w = synth.WORKLOADS[name] if name == "tiny" else _reduced(name, n_layers=2, n_kv_heads=3, n_q_heads=3)
    case = Hl.build_case(w, layers=2, ctx=[w.n_sink + 300 + w.n_recent])
    c = case.cache
    L = case.coded[0]
    for layer in range(2):
        cb = Hl.f64(case.cb[layer])
        for kvi in range(2):
            codes = case.codes[(layer, 0)][kvi].numpy()
            for t in range(w.T):
                out = torch.empty(L - 3, w.n_kv_heads, w.head_dim, dtype=torch.bfloat16, device="cuda")
                lvq.lvq_dequantize(case.cfg, c.lay, layer, t, 0, kvi, c.idx, c.cbp, 3, L - 3, out)
                torch.cuda.synchronize()
                ref = O.dequant_step(codes[:, 3:], cb[kvi], t, w.Tc, w.G)
                np.testing.assert_array_equal(Hl.f64(out), ref)


# ----------------------------------------------------------------------------------- decode

def _check_decode(case, layer, step, q, ns, hq_list=None):
    out, lse, sl = Hl.run_decode(case, layer, step, q, ns)
    worst = 0.0
    for b in range(len(case.ctx)):
        for hq in (hq_list or range(case.w.n_q_heads)):
            ro, rl, rs = Hl.oracle_decode(case, layer, step, b, hq, q, n_splits=ns)
            err = float(np.abs(out[b, hq].numpy() - ro).max())
            worst = max(worst, err)
            assert err <= Hl.OUT_ATOL, (b, hq, err)
            Hl.assert_lse_close(float(lse[b, hq]), rl, "lse")
            for j in range(ns + 1):
                Hl.assert_lse_close(float(sl[b, hq, j]), float(rs[j]), f"split {j}")
    return worst


@pytest.mark.parametrize("ns", [1, 2, 3, 4, 16, 64])
def test_decode_tiny_all_steps(ns):
    w = synth.WORKLOADS["tiny"]
    case = Hl.build_case(w, layers=1, ctx=[512])
    assert case.coded == [492]
    for step in range(w.T):
        q = synth.queries(w, 0, step).cuda()
        _check_decode(case, 0, step, q, ns)


@pytest.mark.parametrize("name,ctx,ns", [
    ("ouro14_g16_32k", [4 + 1000 + 128], 16),
    ("ouro14_g16_32k", [4 + 777 + 131], 5),                 # ragged tail, recent window of 131
    ("ouro14_g32_b32", [2000, 1437, 133, 4, 3, 600], 8),     # ragged batch, tiny contexts
    ("ouro14_tc2_64k", [3000, 2321], 16),
    ("ouro14_tc1_32k", [4 + 901 + 128, 700], 8),             # per-step coding: Tc = 1, c = 16
])
def test_decode_reduced_shapes(name, ctx, ns):
    w = _reduced(name, n_layers=2, n_kv_heads=2, n_q_heads=2)
    case = Hl.build_case(w, layers=2, ctx=ctx)
    for layer in range(2):
        for step in range(w.T):
            q = synth.queries(w, layer, step, batch=len(ctx)).cuda()
            _check_decode(case, layer, step, q, ns)


def test_decode_gqa_two_query_heads_per_kv_head():
    w = _reduced("ouro14_g16_32k", n_layers=1, n_kv_heads=2, n_q_heads=4)
    case = Hl.build_case(w, layers=1, ctx=[900])
    q = synth.queries(w, 0, 1).cuda()
    _check_decode(case, 0, 1, q, 4)


@pytest.mark.parametrize("ns", [1, 2])
def test_decode_long_split_several_super_chunks(ns):
    """A split longer than one CTA's score array (5280 tokens at head_dim 128, c = 4) is
    processed as several super-chunks, each with its own maximum and fixed-point scale."""
    w = _reduced("ouro14_g16_32k", n_layers=1, n_kv_heads=2, n_q_heads=2)
    case = Hl.build_case(w, layers=1, ctx=[4 + 12000 + 128], max_splits=4)
    for step in (0, 3):
        q = synth.queries(w, 0, step).cuda()
        _check_decode(case, 0, step, q, ns)


def test_split_count_sweep_agrees():
    w = _reduced("ouro14_g16_32k", n_layers=1, n_kv_heads=2, n_q_heads=2)
    case = Hl.build_case(w, layers=1, ctx=[4000])
    q = synth.queries(w, 0, 2).cuda()
    outs = [Hl.run_decode(case, 0, 2, q, ns)[0] for ns in (1, 2, 7, 16, 33, 64)]
    # Every output is a convex combination of value elements, computed per split count in
    # another fp32 order: a split's contraction sums 256 histogram-weighted entries (worst
    # case 256 * 2^-24 of max|V|), its fixed-point weights are exact to n * 2^-31 of their sum,
    # and the merge adds at most 2 * 64 + 1 weighted partials.  So any two split counts agree
    # to (256 + 129 + 2) * 2^-24 + 4000 * 2^-31 < 2^-15 of the largest value magnitude.
    vmax = max(float(case.cb[0][1].abs().max()), float(case.sink_kv[(0, 0)][1].abs().max()),
               float(case.ring_kv[(0, 0)][1].abs().max()))
    for o in outs[1:]:
        assert float((o - outs[0]).abs().max()) <= 2.0 ** -15 * vmax


def test_step_slice_isolation_on_gpu():
    """NaN in every packed codebook slice except step t's leaves step-t attention unchanged."""
    w = _reduced("ouro14_tc2_64k", n_layers=1, n_kv_heads=2, n_q_heads=2)
    case = Hl.build_case(w, layers=1, ctx=[1500])
    c = case.cache
    for step in range(w.T):
        q = synth.queries(w, 0, step).cuda()
        clean = Hl.run_decode(case, 0, step, q, 8)
        saved = c.cbp.clone()
        cbp = c.cbp.view(1, 2, c.lay.n_blocks, w.n_kv_heads, w.Tc, -1)
        blk, s = step // w.Tc, step % w.Tc
        mask = torch.ones(c.lay.n_blocks, w.Tc, dtype=torch.bool)
        mask[blk, s] = False
        for bb in range(c.lay.n_blocks):
            for ss in range(w.Tc):
                if mask[bb, ss]:
                    cbp[:, :, bb, :, ss] = float("nan")
        poisoned = Hl.run_decode(case, 0, step, q, 8)
        c.cbp.copy_(saved)
        assert torch.isfinite(poisoned[0]).all()
        # same inputs in the same order (the weight histogram is integer): bit-identical
        assert torch.equal(clean[0], poisoned[0]) and torch.equal(clean[1], poisoned[1])
        assert torch.equal(clean[2], poisoned[2])


def test_identical_codes_zero_key_share_uniform_attention():
    """Every coded key uses entry 42, whose step-t key share is zero, and the bf16 keys are
    zero: every score is 0 after RoPE, so the weights are uniform, lse = ln n and out is the
    mean of all values (sink, dequantized coded, recent)."""
    w = synth.WORKLOADS["tiny"]
    case = Hl.build_case(w, layers=1, ctx=[512])
    c = case.cache
    step = 1
    c.cb_view()[0, 0, :, :, :, 42, step * w.c:(step + 1) * w.c] = 0
    lvq.lvq_pack_codebooks(case.cfg, c.lay, c.cb, c.cbp, c.cb_norm)
    c.idx.view(c.idx_view().shape)[:, :, :, :, 0] = 42      # every K code -> 42
    c.sink_view()[:, 0].zero_()
    c.ring_view()[:, 0].zero_()
    q = synth.queries(w, 0, step).cuda()
    out, lse, _ = Hl.run_decode(case, 0, step, q, 4)
    n = 512
    Hl.assert_lse_close(float(lse[0, 0]), math.log(n))
    sk, rk = Hl.f64(case.sink_kv[(0, 0)]), Hl.f64(case.ring_kv[(0, 0)])
    codes_v = case.codes[(0, 0)][1].numpy()                   # [n_blk][L][H][n_g]
    vh = O.dequant_step(codes_v, Hl.f64(case.cb[0])[1], step, w.Tc, w.G)[:, 0]
    ref = np.concatenate([sk[1, step, :, 0], vh, rk[1, step, :, 0]]).mean(axis=0)
    assert float(np.abs(out[0, 0].numpy() - ref).max()) <= Hl.OUT_ATOL


# ----------------------------------------------------------------------------------- page encode

@pytest.mark.parametrize("name", ["ouro14_tc2_64k", "ouro14_g16_32k", "ouro14_g32_b32", "ouro14_tc1_32k"])
def test_page_encode_matches_oracle_and_advances(name):
    """Requests 0 and 2 have a full recent window and are encoded (several due requests share
    each codebook read); request 1 is one token short and is left untouched."""
    w = _reduced(name, n_layers=2, n_kv_heads=2, n_q_heads=2, n_recent=16)
    R = w.n_recent + 8
    ctx = [w.n_sink + 100 + R, w.n_sink + 50 + R - 1, w.n_sink + 64 + R]
    case = Hl.build_case(w, layers=2, ctx=ctx, coded=[100, 50, 64])
    c = case.cache
    before = c.idx.clone()
    lvq.lvq_encode_page(case.cfg, c.lay, 3, c.ctx_len, c.coded_len, c.ring, c.cb, c.cb_norm, c.idx, c.status)
    torch.cuda.synchronize()
    c.check_status()
    assert c.coded_len.cpu().tolist() == [108, 50, 72]
    for b, off in ((0, 100), (2, 64)):
        for layer in range(2):
            rk = Hl.f64(case.ring_kv[(layer, b)])                 # [2][T][R][H][d], oldest first
            ck, cv = O.page_encode(rk[0], rk[1], Hl.f64(case.cb[layer][0]), Hl.f64(case.cb[layer][1]), w.Tc, w.G)
            got_k = Hl.get_codes(c, layer, b, 0, off, 8).numpy()
            got_v = Hl.get_codes(c, layer, b, 1, off, 8).numpy()
            # compare through the near-tie rule
            for kvi, (got, ref) in enumerate(((got_k, ck), (got_v, cv))):
                X = O.joint_vectors(rk[kvi][:, :8], w.Tc, w.G)
                cbk = Hl.f64(case.cb[layer][kvi])
                for blk in range(X.shape[0]):
                    for h in range(X.shape[2]):
                        for g in range(X.shape[3]):
                            check_codes(got[blk, :, h, g], X[blk, :, h, g], cbk[blk, h, g])
                assert (got == ref).mean() > 0.999
    # request 1's codes and the other pages of requests 0 and 2 are untouched
    after = c.idx.view(c.idx_view().shape)
    b4 = before.view(c.idx_view().shape)
    assert torch.equal(after[:, :, 1], b4[:, :, 1])
    assert torch.equal(after[:, :, 0, :, :, :12], b4[:, :, 0, :, :, :12])
    assert torch.equal(after[:, :, 0, :, :, 14:], b4[:, :, 0, :, :, 14:])
    assert torch.equal(after[:, :, 2, :, :, :8], b4[:, :, 2, :, :, :8])
    assert torch.equal(after[:, :, 2, :, :, 9:], b4[:, :, 2, :, :, 9:])


def test_decode_large_score_range():
    """Keys of one entry are scaled by 100 and used only outside the first page of every
    4-page run: scores then spread far beyond the exponent range of a float weight, most
    weights underflow to zero against the exact maximum, and the result must still match
    the oracle."""
    w = synth.WORKLOADS["tiny"]
    case = Hl.build_case(w, layers=1, ctx=[512])
    c = case.cache
    cbv = c.cb_view()
    cbv[0, 0, :, :, :, 7, :] = (cbv[0, 0, :, :, :, 7, :].float() * 100).to(torch.bfloat16)
    case.cb[0][0, :, :, :, 7, :] = cbv[0, 0, :, :, :, 7, :].cpu()
    lvq.lvq_pack_codebooks(case.cfg, c.lay, c.cb, c.cbp, c.cb_norm)
    ck, cv = case.codes[(0, 0)]
    ck = ck.clone()
    n = torch.arange(ck.shape[1])
    first_pages = ((n // 8) % 4) == 0          # the first page of every warp's 4-page run
    sel = ck[:, first_pages]
    sel[sel == 7] = 8
    ck[:, first_pages] = sel
    Hl.put_codes(c, 0, 0, 0, ck.cuda())
    case.codes[(0, 0)] = (ck, cv)
    for step in range(w.T):
        q = synth.queries(w, 0, step).cuda()
        _check_decode(case, 0, step, q, 1)


@pytest.mark.parametrize("cap", [0, 2])
def test_decode_reports_counters_outside_the_layout(cap):
    """A request whose counters the layout cannot hold (its recent window longer than the ring)
    is reported as LVQ_ECAPACITY and left empty (output 0, lse -inf); the other requests of
    the launch are computed as usual.  cap = 2: two CTAs walking runs of items."""
    w = _reduced("ouro14_g16_32k", n_layers=1, n_kv_heads=2, n_q_heads=2)
    ctx = [4 + 900 + 128, 4 + 500 + 128, 4 + 300 + 128]
    case = Hl.build_case(w, layers=1, ctx=ctx, max_splits=8)
    c = case.cache
    c.coded_len[1] = case.coded[1] - (c.lay.ring_tokens + 5)       # recent window > ring
    q = synth.queries(w, 0, 1, batch=3).cuda()
    out = torch.empty(3, w.n_q_heads, w.head_dim, dtype=torch.float32, device="cuda")
    lse = torch.empty(3, w.n_q_heads, dtype=torch.float32, device="cuda")
    lvq.lvq_decode_max_ctas(cap)
    try:
        lvq.lvq_decode_attention(case.cfg, c.lay, 0, 1, 3, q, c.ctx_len, c.coded_len, c.sink, c.ring, c.idx, c.cbp,
                                 c.rope, 4, c.workspace, out, lse, c.status)
        torch.cuda.synchronize()
    finally:
        lvq.lvq_decode_max_ctas(0)
    assert int(c.status.item()) == lvq.LVQ_ECAPACITY
    out, lse = out.cpu(), lse.cpu()
    assert torch.equal(out[1], torch.zeros_like(out[1])) and bool(torch.isneginf(lse[1]).all())
    for b in (0, 2):
        for hq in range(w.n_q_heads):
            ro, rl, _ = Hl.oracle_decode(case, 0, 1, b, hq, q)
            assert float(np.abs(out[b, hq].numpy() - ro).max()) <= Hl.OUT_ATOL
            Hl.assert_lse_close(float(lse[b, hq]), rl)
    c.status.zero_()
