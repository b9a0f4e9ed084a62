"""Codebook construction on the GPU (one plain k-means iteration: the prefill encoder as
the assignment step, lvq_kmeans_update as the update step) against the fp64 oracle.

The oracle assigns and updates on its own.  Where its codes and the GPU's differ (only
near-ties may), the two entries involved are not compared; every other entry must be
bit-identical in bf16 and every count equal."""
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


def _gpu_step(cfg, c, kv, ntok):
    """One iteration on the GPU: codes into the cache's index rows, entries updated in place."""
    counts = torch.zeros(2 * c.lay.n_blocks * cfg.n_kv_heads * c.lay.n_groups * 256, dtype=torch.int32,
                         device="cuda")
    lvq.lvq_encode_prefill(cfg, c.lay, 0, 0, kv, 0, ntok, 0, c.cb, c.idx, c.status)
    lvq.lvq_kmeans_update(cfg, c.lay, 0, 0, kv, 0, ntok, 0, c.idx, c.cb, counts, c.status)
    torch.cuda.synchronize()
    c.check_status()
    return counts.view(2, c.lay.n_blocks, cfg.n_kv_heads, c.lay.n_groups, 256).cpu().numpy()


def _compare(w, cb_old, cb_new_gpu, counts_gpu, codes_gpu, x, kvi, blk, h, g):
    """One codebook: the oracle's iteration against the GPU's.  Returns entries compared."""
    X = O.joint_vectors(x[kvi], w.Tc, w.G)[blk, :, h, g]              # [N][G]
    C = cb_old[kvi, blk, h, g]
    codes, C_new, counts = O.kmeans_step(X, C)
    got = codes_gpu[kvi][blk, :, h, g].astype(np.int64)
    skip = np.zeros(256, dtype=bool)
    for m in np.nonzero(got != codes)[0]:                              # near-ties only
        _, d1, d2 = O.nearest_entry(X[m][None], C)
        assert O.near_tie(d1, d2)[0], (kvi, blk, h, g, m)
        skip[got[m]] = skip[codes[m]] = True
    keep = ~skip
    np.testing.assert_array_equal(cb_new_gpu[kvi, blk, h, g][keep], C_new[keep])
    np.testing.assert_array_equal(counts_gpu[kvi, blk, h, g][keep], counts[keep])
    return int(keep.sum())


@pytest.mark.parametrize("name,ntok,extra", [
    ("ouro14_g16_32k", 1500, {"n_kv_heads": 2, "n_q_heads": 2}),     # G = 16, c = 4
    ("ouro14_g32_b32", 700, {"n_kv_heads": 2, "n_q_heads": 2}),      # G = 32, c = 8
    ("ouro14_tc2_64k", 900, {"n_kv_heads": 1, "n_q_heads": 1}),      # Tc = 2: two codebooks per group
    ("ouro14_tc1_32k", 1100, {"n_kv_heads": 2, "n_q_heads": 2}),     # Tc = 1, c = 16
])
def test_kmeans_iteration_matches_oracle(name, ntok, extra):
    w = _reduced(name, n_layers=1, **extra)
    case = Hl.build_case(w, layers=1, ctx=[w.n_sink + ntok + w.n_recent], coded=[ntok], codes_from="none")
    c = case.cache
    cb_old = case.cb[0].clone()
    # a duplicated entry: its higher copy loses every vector to the lower one (exact tie, lowest
    # index), so it must keep its value with a count of 0
    cb_old[..., 7, :] = cb_old[..., 3, :]
    c.cb_view()[0] = cb_old.cuda()
    kv = synth.loop_kv(w, 0, ntok, stream="kmeans")
    counts = _gpu_step(case.cfg, c, kv.cuda(), ntok)
    cb_new = Hl.f64(c.cb_view()[0].cpu())
    codes_gpu = [Hl.get_codes(c, 0, 0, kvi, 0, ntok).numpy() for kvi in range(2)]
    x = Hl.f64(kv)
    cbo = Hl.f64(cb_old)
    compared = 0
    for kvi in range(2):
        for blk in range(c.lay.n_blocks):
            for h in range(w.n_kv_heads):
                for g in range(c.lay.n_groups):
                    compared += _compare(w, cbo, cb_new, counts, codes_gpu, x, kvi, blk, h, g)
    total = 2 * c.lay.n_blocks * w.n_kv_heads * c.lay.n_groups * 256
    assert compared >= total - total // 100
    assert (counts[..., 7] == 0).all()
    np.testing.assert_array_equal(cb_new[..., 7, :], cbo[..., 7, :])


def test_kmeans_offsets_and_ragged_tail():
    """Tokens taken from inside the K/V buffer (tok_begin = 5) and coded at an offset that is
    not a page boundary (coded_offset = 3), with a ragged last tile: the update reads the same
    vectors and codes the encoder used."""
    w = _reduced("ouro14_g16_32k", n_layers=1, n_kv_heads=1, n_q_heads=1)
    ntok, tb, co = 1000, 5, 3
    case = Hl.build_case(w, layers=1, ctx=[w.n_sink + co + ntok + w.n_recent], coded=[co + ntok],
                         codes_from="none")
    c, cfg = case.cache, case.cfg
    cb_old = case.cb[0].clone()
    kv = synth.loop_kv(w, 0, tb + ntok + 7, stream="kmeans").cuda()
    counts = torch.zeros(2 * c.lay.n_blocks * cfg.n_kv_heads * c.lay.n_groups * 256, dtype=torch.int32,
                         device="cuda")
    lvq.lvq_encode_prefill(cfg, c.lay, 0, 0, kv, tb, ntok, co, c.cb, c.idx, c.status)
    lvq.lvq_kmeans_update(cfg, c.lay, 0, 0, kv, tb, ntok, co, c.idx, c.cb, counts, c.status)
    torch.cuda.synchronize()
    c.check_status()
    counts = counts.view(2, c.lay.n_blocks, cfg.n_kv_heads, c.lay.n_groups, 256).cpu().numpy()
    cb_new = Hl.f64(c.cb_view()[0].cpu())
    codes_gpu = [Hl.get_codes(c, 0, 0, kvi, co, ntok).numpy() for kvi in range(2)]
    x = Hl.f64(kv.cpu()[:, :, tb:tb + ntok])
    cbo = Hl.f64(cb_old)
    for kvi in range(2):
        for g in range(c.lay.n_groups):
            _compare(w, cbo, cb_new, counts, codes_gpu, x, kvi, 0, 0, g)
    assert counts.sum() == 2 * c.lay.n_groups * ntok


def test_kmeans_two_iterations_lower_the_objective():
    """Lloyd descent on the GPU path: the second iteration's codes fit at least as well."""
    w = _reduced("ouro14_g16_32k", n_layers=1, n_kv_heads=1, n_q_heads=1)
    ntok = 2000
    case = Hl.build_case(w, layers=1, ctx=[w.n_sink + ntok + w.n_recent], coded=[ntok], codes_from="none")
    c = case.cache
    kv = synth.loop_kv(w, 0, ntok, stream="kmeans")
    X = O.joint_vectors(Hl.f64(kv[0]), w.Tc, w.G)[0, :, 0, 5]
    sse = []
    for _ in range(3):
        C = Hl.f64(c.cb_view()[0, 0, 0, 0, 5].cpu())
        _, d1, _ = O.nearest_entry(X, C)
        sse.append(d1.sum())
        _gpu_step(case.cfg, c, kv.cuda(), ntok)
    assert sse[1] <= sse[0] and sse[2] <= sse[1] * (1 + 1e-3)      # bf16 storage may add a hair
    assert sse[2] < sse[0]


def test_kmeans_full_layer_sampled_codebooks():
    """One Ouro-2.6B-shaped layer (32768 tokens, 16 heads, K and V, 32 groups): a full GPU
    iteration; 6 codebooks checked against the oracle's own iteration."""
    wc = synth.WORKLOADS["ouro26_prefill_32k"]
    cfg = lvq.make_config(1, wc.n_kv_heads, wc.n_q_heads, wc.head_dim, wc.T, wc.Tc, wc.G, 0, 0, 1, wc.ctx,
                          max_splits=1, rope_base=wc.rope_base)
    c = lvq.CodedCache(cfg, "cuda")
    cb = synth.codebooks(wc, 0)
    c.cb_view()[0] = cb.cuda()
    kv = synth.loop_kv(wc, 0, wc.ctx, stream="coded", device="cuda")
    counts = _gpu_step(cfg, c, kv, wc.ctx)
    assert counts.sum() == 2 * 16 * 32 * wc.ctx
    cb_new = Hl.f64(c.cb_view()[0].cpu())
    lay = c.lay
    rng = np.random.default_rng(4)
    picks = [(int(rng.integers(2)), 0, int(rng.integers(16)), int(rng.integers(32))) for _ in range(6)]
    kv_c = kv.cpu()
    for kvi, blk, h, g in picks:
        xg = Hl.f64(kv_c[kvi, :, :, h:h + 1, g * lay.c:(g + 1) * lay.c])      # [T][N][1][c]
        X = np.concatenate([xg[s, :, 0] for s in range(wc.Tc)], axis=1)       # [N][G], step-major
        C = Hl.f64(cb[kvi, blk, h, g])
        codes, C_new, cnt = O.kmeans_step(X, C)
        got = Hl.get_codes(c, 0, 0, kvi, 0, wc.ctx)[blk, :, h, g].numpy().astype(np.int64)
        skip = np.zeros(256, dtype=bool)
        for m in np.nonzero(got != codes)[0]:
            skip[got[m]] = skip[codes[m]] = True
        assert skip.sum() <= 8
        np.testing.assert_array_equal(cb_new[kvi, blk, h, g][~skip], C_new[~skip])
        np.testing.assert_array_equal(counts[kvi, blk, h, g][~skip], cnt[~skip])
