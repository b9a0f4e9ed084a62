"""Seeded synthetic inputs shaped like a looped transformer's KV cache.

This module only draws random numbers and lays them out; it holds none of the
codec's or the attention's arithmetic (no nearest-entry search, no
dequantisation, no RoPE, no softmax).  Tests and the benchmark draw their inputs
here and hand the same tensors to both the CUDA library and the fp64 oracle.

What the numbers look like follows the LoopVQ pages:
  * "LoopVQ summary" (onedev.kr), section "how it works": adjacent loop steps of
    the same layer are strongly correlated (0.69 between the first two steps,
    rising to 0.94 between the last two; same-channel correlation about 0.85).
    Here each channel follows an AR(1) process along the loop axis,
    x_t = rho_t * x_{t-1} + sqrt(1 - rho_t^2) * eps_t with x_0 ~ N(0, 1), and
    rho rises linearly from 0.69 to 0.94 over the T-1 transitions.
  * Per-channel lognormal(0, 0.5) scales, one per (layer, K/V, head, channel),
    shared by every loop step and token.
  * Keys (not values) of the Ouro-shaped workloads carry two outlier channels
    per (layer, head), scaled by 8.
  * Everything is rounded to bf16 with round-to-nearest-even.
Tokens are independent of one another (the pages are silent on correlation
along the sequence).

Codebooks are 256 further samples of the same process per codebook, drawn
directly in the codebook's logical layout: entry k of the codebook for
(layer, K/V, block b, head h, group g) holds, at element s*c + e, a sample of
step b*Tc + s, channel g*c + e.  No codec arithmetic is needed to draw them.

Every draw is keyed by (seed, stream name, layer, ...) through its own
torch.Generator, so a layer's data does not depend on which other layers were
drawn, or in which order.
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import Optional, Sequence

import torch

RHO_FIRST = 0.69
RHO_LAST = 0.94
SCALE_LOG_SIGMA = 0.5
OUTLIER_CHANNELS = 2
OUTLIER_FACTOR = 8.0
CODEBOOK_ENTRIES = 256


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and seeds of one synthetic workload.

    n_layers, n_kv_heads, n_q_heads, head_dim: model shape.
    T: loop steps; Tc: loop steps per block; G: joint-vector length.
    ctx: context length per request (tokens, including the newest one), or
         None when lengths are drawn per request (see ctx_lengths()).
    batch: number of requests; n_sink / n_recent: bf16 sink and recent tokens.
    key_outliers: whether keys carry the two x8 outlier channels.
    """

    name: str
    n_layers: int
    n_kv_heads: int
    n_q_heads: int
    head_dim: int
    T: int
    Tc: int
    G: int
    batch: int
    n_sink: int
    n_recent: int
    ctx: Optional[int]
    key_outliers: bool
    rope_base: float = 10000.0
    seed: int = 0
    len_seed: int = 2
    ctx_low: int = 0
    ctx_high: int = 0
    gen_tokens: int = 0

    @property
    def c(self) -> int:
        return self.G // self.Tc

    @property
    def n_groups(self) -> int:
        return self.head_dim // self.c

    @property
    def n_blocks(self) -> int:
        return self.T // self.Tc


# The five workloads: a tiny one the oracle finishes in seconds, then the
# Ouro-shaped decode and encode cases.
WORKLOADS = {
    "tiny": Workload("tiny", n_layers=1, n_kv_heads=1, n_q_heads=1, head_dim=64, T=4, Tc=4, G=16,
                     batch=1, n_sink=4, n_recent=16, ctx=512, key_outliers=False),
    "ouro14_g16_32k": Workload("ouro14_g16_32k", n_layers=24, n_kv_heads=16, n_q_heads=16,
                               head_dim=128, T=4, Tc=4, G=16, batch=1, n_sink=4, n_recent=128,
                               ctx=32768, key_outliers=True),
    "ouro14_g32_b32": Workload("ouro14_g32_b32", n_layers=24, n_kv_heads=16, n_q_heads=16,
                               head_dim=128, T=4, Tc=4, G=32, batch=32, n_sink=4, n_recent=128,
                               ctx=None, key_outliers=True, ctx_low=8192, ctx_high=32768),
    "ouro26_prefill_32k": Workload("ouro26_prefill_32k", n_layers=48, n_kv_heads=16, n_q_heads=16,
                                   head_dim=128, T=4, Tc=4, G=16, batch=1, n_sink=4, n_recent=128,
                                   ctx=32768, key_outliers=True),
    "ouro14_tc2_64k": Workload("ouro14_tc2_64k", n_layers=24, n_kv_heads=16, n_q_heads=16,
                               head_dim=128, T=4, Tc=2, G=16, batch=8, n_sink=4, n_recent=256,
                               ctx=65536, key_outliers=True, gen_tokens=256),
    # per-step coding (Tc = 1, c = G = 16) at the same 0.5 bits per element: the degenerate
    # case without a loop axis, a per-step baseline beside the joint coding of ouro14_g16_32k
    "ouro14_tc1_32k": Workload("ouro14_tc1_32k", n_layers=24, n_kv_heads=16, n_q_heads=16,
                               head_dim=128, T=4, Tc=1, G=16, batch=1, n_sink=4, n_recent=128,
                               ctx=32768, key_outliers=True),
}


def rho_schedule(T: int) -> list:
    """Correlation of step t with step t-1, for t = 1..T-1 (linear 0.69 -> 0.94)."""
    if T < 2:
        return []
    if T == 2:
        return [RHO_FIRST]
    return [RHO_FIRST + (RHO_LAST - RHO_FIRST) * i / (T - 2) for i in range(T - 1)]


def _seed_of(*keys) -> int:
    h = hashlib.sha256(repr(keys).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def generator(device, *keys) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed_of(*keys))
    return g


def channel_scales(w: Workload, layer: int, device="cpu") -> torch.Tensor:
    """[2][Hkv][d] float32: lognormal(0, 0.5) per channel, keys' outliers x8."""
    g = generator(device, w.seed, "scale", layer)
    z = torch.randn(2, w.n_kv_heads, w.head_dim, generator=g, device=device)
    s = torch.exp(SCALE_LOG_SIGMA * z)
    if w.key_outliers:
        for h in range(w.n_kv_heads):
            ch = torch.randperm(w.head_dim, generator=g, device=device)[:OUTLIER_CHANNELS]
            s[0, h, ch] *= OUTLIER_FACTOR
    return s


def _ar_steps(shape_tail, steps: Sequence[int], rhos, g, device) -> torch.Tensor:
    """AR(1) along the loop axis for the given consecutive steps (fp32).

    Returns [len(steps), *shape_tail].  The first listed step is drawn from the
    stationary N(0, 1) law, so any window of consecutive steps has the same
    joint law as in the full T-step chain.
    """
    out = torch.empty((len(steps),) + tuple(shape_tail), device=device, dtype=torch.float32)
    x = torch.randn(shape_tail, generator=g, device=device)
    out[0] = x
    for i in range(1, len(steps)):
        r = rhos[steps[i] - 1]
        eps = torch.randn(shape_tail, generator=g, device=device)
        x = r * x + math.sqrt(1.0 - r * r) * eps
        out[i] = x
    return out


def loop_kv(w: Workload, layer: int, n_tok: int, stream: str = "kv", request: int = 0,
            device="cpu", scales: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Pre-RoPE keys and values of n_tok tokens: [2][T][n_tok][Hkv][d] bf16."""
    if scales is None:
        scales = channel_scales(w, layer, device)
    g = generator(device, w.seed, stream, layer, request)
    rhos = rho_schedule(w.T)
    x = _ar_steps((2, n_tok, w.n_kv_heads, w.head_dim), list(range(w.T)), rhos, g, device)
    x = x.permute(1, 0, 2, 3, 4)  # [2][T][N][H][d]
    x = x * scales[:, None, None, :, :]
    return x.to(torch.bfloat16).contiguous()


def codebooks(w: Workload, layer: int, device="cpu",
              scales: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Logical codebooks of one layer: [2][n_blk][Hkv][n_g][256][G] bf16.

    Element s*c + e of entry k is a draw of loop step b*Tc + s, channel g*c + e.
    """
    if scales is None:
        scales = channel_scales(w, layer, device)
    g = generator(device, w.seed, "cb", layer)
    rhos = rho_schedule(w.T)
    c, ng, nb = w.c, w.n_groups, w.n_blocks
    out = torch.empty(2, nb, w.n_kv_heads, ng, CODEBOOK_ENTRIES, w.Tc, c, device=device)
    sc = scales.view(2, w.n_kv_heads, ng, c)
    for b in range(nb):
        steps = list(range(b * w.Tc, (b + 1) * w.Tc))
        x = _ar_steps((2, w.n_kv_heads, ng, CODEBOOK_ENTRIES, c), steps, rhos, g, device)
        # x: [Tc][2][H][n_g][256][c] -> [2][H][n_g][256][Tc][c]
        out[:, b] = x.permute(1, 2, 3, 4, 0, 5) * sc[:, :, :, None, None, :]
    return out.reshape(2, nb, w.n_kv_heads, ng, CODEBOOK_ENTRIES, w.G).to(torch.bfloat16).contiguous()


def queries(w: Workload, layer: int, step: int, batch: Optional[int] = None, token: int = 0,
            device="cpu") -> torch.Tensor:
    """Pre-RoPE decode queries: [B][Hq][d] bf16, N(0, 1)."""
    b = w.batch if batch is None else batch
    g = generator(device, w.seed, "q", layer, step, token)
    return torch.randn(b, w.n_q_heads, w.head_dim, generator=g, device=device).to(torch.bfloat16)


def random_codes(shape, seed: int, device="cpu") -> torch.Tensor:
    """Uniform 8-bit codes (for decode-only tests that bypass the encoder)."""
    g = generator(device, seed, "codes")
    return torch.randint(0, CODEBOOK_ENTRIES, tuple(shape), generator=g, device=device,
                         dtype=torch.int32).to(torch.uint8)


def ctx_lengths(w: Workload) -> list:
    """Per-request context lengths.  Fixed-length workloads repeat w.ctx;
    otherwise lengths are uniform integers in [ctx_low, ctx_high] drawn with
    w.len_seed."""
    if w.ctx is not None:
        return [w.ctx] * w.batch
    g = generator("cpu", w.len_seed, "len")
    u = torch.rand(w.batch, generator=g, dtype=torch.float64)
    span = w.ctx_high - w.ctx_low + 1
    return [int(w.ctx_low + math.floor(float(v) * span)) for v in u]
