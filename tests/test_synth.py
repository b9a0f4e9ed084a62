"""The seeded generator draws what its docstring promises (CPU, no GPU)."""
import math

import numpy as np
import torch

from sub_bit_kv_b200 import synth


def _tiny(**kw):
    base = dict(name="t", n_layers=1, n_kv_heads=2, n_q_heads=2, head_dim=64, T=4, Tc=4, G=16,
                batch=1, n_sink=4, n_recent=16, ctx=512, key_outliers=True)
    base.update(kw)
    return synth.Workload(**base)


def test_rho_schedule_rises_from_069_to_094():
    assert synth.rho_schedule(4) == [0.69, 0.815, 0.94]
    assert synth.rho_schedule(2) == [0.69]


def test_adjacent_step_correlation_matches_schedule():
    w = _tiny(n_kv_heads=4, head_dim=64)
    x = synth.loop_kv(w, 0, 4096).float()                 # [2][T][N][H][d]
    sc = synth.channel_scales(w, 0)
    z = x / sc[:, None, None]                              # undo the channel scale
    for t, rho in enumerate(synth.rho_schedule(w.T), start=1):
        a, b = z[:, t - 1].reshape(-1).double(), z[:, t].reshape(-1).double()
        r = torch.corrcoef(torch.stack([a, b]))[0, 1].item()
        assert abs(r - rho) < 0.01, (t, r, rho)
    # different channels of the same step are uncorrelated
    r = torch.corrcoef(torch.stack([z[0, 1, :, :, 0].reshape(-1), z[0, 1, :, :, 1].reshape(-1)]))[0, 1]
    assert abs(r.item()) < 0.05


def test_channel_scales_lognormal_and_outliers():
    w = _tiny(n_kv_heads=64, head_dim=128)
    s = synth.channel_scales(w, 3)
    logv = torch.log(s[1]).reshape(-1)                   # values carry no outliers
    assert abs(logv.mean().item()) < 0.03 and abs(logv.std().item() - 0.5) < 0.03
    g = synth.generator("cpu", w.seed, "scale", 3)
    z = torch.randn(2, w.n_kv_heads, w.head_dim, generator=g)
    plain = torch.exp(0.5 * z)
    big = (s[0] / plain[0])
    assert torch.allclose(s[1], plain[1])
    for h in range(w.n_kv_heads):
        vals = sorted(set(round(v, 5) for v in big[h].tolist()))
        assert vals == [1.0, 8.0]
        assert int((big[h] > 4).sum()) == 2


def test_bf16_and_determinism():
    w = _tiny()
    a = synth.loop_kv(w, 0, 64)
    b = synth.loop_kv(w, 0, 64)
    assert a.dtype == torch.bfloat16 and torch.equal(a, b)
    assert not torch.equal(a, synth.loop_kv(w, 0, 64, stream="other"))
    cb = synth.codebooks(w, 0)
    assert cb.shape == (2, 1, 2, 16, 256, 16) and cb.dtype == torch.bfloat16
    # no duplicate entries inside any codebook
    flat = cb.view(-1, 256, 16).float()
    for i in range(flat.shape[0]):
        assert torch.unique(flat[i], dim=0).shape[0] == 256


def test_codebook_entries_follow_the_loop_law():
    """Entry element s*c+e is step s of the block: its steps correlate like the data's."""
    w = _tiny(n_kv_heads=8, head_dim=64, Tc=2, G=16)
    cb = synth.codebooks(w, 0).float()                    # [2][2][H][n_g][256][G]
    sc = synth.channel_scales(w, 0).view(2, 8, w.n_groups, w.c)
    c = w.c
    blk1 = cb[:, 1] / torch.cat([sc, sc], dim=-1)[:, :, :, None, :]
    a, b = blk1[..., :c].reshape(-1).double(), blk1[..., c:].reshape(-1).double()
    r = torch.corrcoef(torch.stack([a, b]))[0, 1].item()
    assert abs(r - synth.rho_schedule(4)[2]) < 0.02


def test_ctx_lengths_uniform_range_and_seeded():
    w = synth.WORKLOADS["ouro14_g32_b32"]
    L = synth.ctx_lengths(w)
    assert len(L) == 32 and all(8192 <= x <= 32768 for x in L)
    assert L == synth.ctx_lengths(w)
    assert synth.ctx_lengths(synth.WORKLOADS["ouro14_g16_32k"]) == [32768]


def test_workload_geometry():
    w = synth.WORKLOADS["ouro14_tc2_64k"]
    assert (w.c, w.n_groups, w.n_blocks) == (8, 16, 2)
    w = synth.WORKLOADS["ouro14_g16_32k"]
    assert (w.c, w.n_groups, w.n_blocks) == (4, 32, 1)
    assert math.isclose(8 * w.n_blocks * w.n_groups / (w.T * w.head_dim), 0.5)
    np.testing.assert_equal(synth.WORKLOADS["tiny"].ctx - 4 - 16, 492)
