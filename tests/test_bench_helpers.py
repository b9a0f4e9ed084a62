"""Host-side helpers of bench.py: the split choice and the algorithmic byte model that the
roofline line divides by (closed forms of the cache layout)."""
import dataclasses

import bench
from sub_bit_kv_b200 import synth


class _Lay:
    def __init__(self, n_groups):
        self.n_groups = n_groups


def test_decode_bytes_closed_form_32k():
    w = synth.WORKLOADS["ouro14_g16_32k"]
    coded, recent = 32636, 128
    got = bench.decode_bytes_per_launch(w, _Lay(32), [coded], [recent])
    idx = coded * 16 * 2 * 32                 # 32 code bytes per token, head and K/V
    slices = 16 * 2 * 256 * 128 * 2           # step-t K/V slices of the 16 heads
    bf16 = (4 + 128) * 16 * 2 * 128 * 2       # sink + recent tokens, K and V
    qo = 16 * 128 * (2 + 4) + 16 * 4          # bf16 query in, fp32 output and lse out
    assert got == idx + slices + bf16 + qo == 36_610_112


def test_decode_bytes_per_step_coding_reads_one_block():
    """Tc = 1 (c = 16): a step reads only its own block's 8 code bytes per token, head and K/V."""
    w = synth.WORKLOADS["ouro14_tc1_32k"]
    coded, recent = 32636, 128
    got = bench.decode_bytes_per_launch(w, _Lay(8), [coded], [recent])
    idx = coded * 16 * 2 * 8
    slices = 16 * 2 * 256 * 128 * 2
    bf16 = (4 + 128) * 16 * 2 * 128 * 2
    qo = 16 * 128 * (2 + 4) + 16 * 4
    assert got == idx + slices + bf16 + qo


def test_decode_bytes_two_blocks_read_only_this_steps_block():
    """Tc = 2 (c = 8): two index rows per token, a step reads the 16 bytes of its own block."""
    w = synth.WORKLOADS["ouro14_tc2_64k"]
    got = bench.decode_bytes_per_launch(w, _Lay(16), [65276], [256])
    idx = 65276 * 16 * 2 * 16
    slices = 16 * 2 * 256 * 128 * 2
    bf16 = (4 + 256) * 16 * 2 * 128 * 2
    qo = 16 * 128 * (2 + 4) + 16 * 4
    assert got == idx + slices + bf16 + qo


def test_decode_bytes_batch_counts_slices_once():
    w = synth.WORKLOADS["ouro14_g32_b32"]
    one = bench.decode_bytes_per_launch(w, _Lay(16), [1000], [128])
    two = bench.decode_bytes_per_launch(w, _Lay(16), [1000, 1000], [128, 128])
    slices = 16 * 2 * 256 * 128 * 2
    assert two - one == one - slices


def test_choose_splits():
    ws = synth.WORKLOADS
    assert bench.choose_splits(ws["ouro14_g16_32k"], 148) == 9         # 16 heads fill one wave
    assert bench.choose_splits(ws["ouro14_tc2_64k"], 148) == 8         # 1024 CTAs: 7 nearly full waves
    assert bench.choose_splits(ws["ouro14_g32_b32"], 148) == 3         # 512 heads: ~6K-token splits
    tiny = dataclasses.replace(ws["tiny"], batch=1)
    assert bench.choose_splits(tiny, 148) == 128                        # capped


def test_decode_issue_ceiling(monkeypatch):
    """Warp instructions issued at one per scheduler per cycle, 4 schedulers per SM: 148 SMs at
    1000 MHz issue 5.92e11 per second, so 5.92e6 instructions take 10 us."""
    monkeypatch.setattr(bench, "_decode_ncu", lambda: {"warp_inst_per_launch": 5.92e6})
    got = bench.decode_issue(launch_ms=0.020, sm_mhz=1000, n_sm=148, token_heads=1000)
    assert abs(got["ceiling_us"] - 10.0) < 1e-9
    assert abs(got["frac"] - 0.5) < 1e-12
    assert got["per_coded_token_head"] == 5.92e3
    assert bench.decode_issue(0.02, None, 148, 1000) is None            # no clock sample
    monkeypatch.setattr(bench, "_decode_ncu", lambda: None)              # another decode source
    assert bench.decode_issue(0.02, 1000, 148, 1000) is None
