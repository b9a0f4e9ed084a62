"""Test infrastructure: builds coded caches through the C ABI, converts the
library's physical layouts to the oracle's logical arrays, and runs the oracle
on the same seeded inputs.  Used by the GPU tests and __graft_entry__.smoke().
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

from oracle import lvq_oracle as O
from sub_bit_kv_b200 import lvq, synth

OUT_ATOL = 2e-3      # attention output, max-abs against the fp64 oracle
LSE_REL = 1e-4       # split LSE: |d| <= 1e-4 * max(1, |lse|)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def make_cfg(w: synth.Workload, n_layers=None, max_batch=None, max_ctx=None, max_splits=64):
    return lvq.make_config(
        n_layers=n_layers or w.n_layers, n_kv_heads=w.n_kv_heads, n_q_heads=w.n_q_heads, head_dim=w.head_dim,
        T=w.T, Tc=w.Tc, G=w.G, n_sink=w.n_sink, n_recent=w.n_recent, max_batch=max_batch or w.batch,
        max_ctx=max_ctx or (w.ctx or w.ctx_high), max_splits=max_splits, rope_base=w.rope_base)


# --------------------------------------------------------------------------- code layout conversion

def put_codes(cache: lvq.CodedCache, layer: int, b: int, kv: int, codes: torch.Tensor, offset: int = 0):
    """codes: uint8 [n_blk][N][H][n_g] (logical) -> coded slots offset..offset+N of request b."""
    n_blk, N, H, ng = codes.shape
    view = cache.idx_view()                               # [L][n_blk][B][H][2][P][n_g][8]
    flat = view[layer, :, b, :, kv]                       # [n_blk][H][P][n_g][8]
    flat = flat.permute(0, 1, 2, 4, 3).reshape(n_blk, H, -1, ng)   # [n_blk][H][P*8][n_g]
    flat[:, :, offset:offset + N, :] = codes.permute(0, 2, 1, 3).to(flat.device)
    view[layer, :, b, :, kv] = flat.reshape(n_blk, H, -1, 8, ng).permute(0, 1, 2, 4, 3)


def get_codes(cache: lvq.CodedCache, layer: int, b: int, kv: int, offset: int, N: int) -> torch.Tensor:
    """Inverse of put_codes: uint8 [n_blk][N][H][n_g] on the CPU."""
    view = cache.idx_view()
    flat = view[layer, :, b, :, kv]
    n_blk, H, P, ng, _ = flat.shape
    flat = flat.permute(0, 1, 2, 4, 3).reshape(n_blk, H, P * 8, ng)
    return flat[:, :, offset:offset + N, :].permute(0, 2, 1, 3).cpu()


# --------------------------------------------------------------------------- cache construction

@dataclasses.dataclass
class Case:
    w: synth.Workload
    cfg: lvq.lvq_config
    cache: lvq.CodedCache
    ctx: list                       # per request
    coded: list                     # per request
    layers: int
    cb: list                        # per layer: [2][n_blk][H][n_g][256][G] bf16 (cpu)
    sink_kv: dict                   # (layer, b) -> [2][T][S][H][d] bf16 (cpu)
    ring_kv: dict                   # (layer, b) -> [2][T][R'][H][d] recent tokens, oldest first (cpu)
    codes: dict                     # (layer, b) -> (codes_k, codes_v) [n_blk][L][H][n_g] uint8 (cpu)


def build_case(w: synth.Workload, layers: int, ctx: list, coded: Optional[list] = None, code_seed=0,
               device="cuda", max_ctx=None, max_splits=64, codes_from="random") -> Case:
    """A coded cache for `layers` layers and len(ctx) requests.

    codes_from="random": uniform codes from the generator (decode-only tests);
    "encode": codes written by lvq_encode_prefill from generated K/V."""
    B = len(ctx)
    cfg = make_cfg(w, n_layers=layers, max_batch=B, max_ctx=max_ctx or max(ctx) + 8, max_splits=max_splits)
    cache = lvq.CodedCache(cfg, device)
    lay = cache.lay
    S, R = w.n_sink, lay.ring_tokens
    if coded is None:
        coded = [max(0, c - S - w.n_recent) for c in ctx]
    cbs, sink_kv, ring_kv, codes = [], {}, {}, {}
    cbv, sv, rv = cache.cb_view(), cache.sink_view(), cache.ring_view()
    for layer in range(layers):
        scales = synth.channel_scales(w, layer)
        cb = synth.codebooks(w, layer, scales=scales)
        cbs.append(cb)
        cbv[layer] = cb.to(device)
        for b in range(B):
            n_sink = min(S, ctx[b])
            n_rec = ctx[b] - n_sink - coded[b]
            assert 0 <= n_rec <= R
            sk = synth.loop_kv(w, layer, n_sink, stream="sink", request=b, scales=scales)
            rk = synth.loop_kv(w, layer, n_rec, stream="recent", request=b, scales=scales)
            sink_kv[(layer, b)] = sk
            ring_kv[(layer, b)] = rk
            # sink[layer][kv][t][b][h][i][d] <- sk[kv][t][i][h][d]
            sv[layer, :, :, b, :, :n_sink, :] = sk.permute(0, 1, 3, 2, 4).to(device)
            for i in range(n_rec):
                slot = (coded[b] + i) % R            # position S + coded + i
                rv[layer, :, :, b, :, slot, :] = rk[:, :, i].to(device)
            if codes_from == "random":
                shape = (lay.n_blocks, coded[b], w.n_kv_heads, lay.n_groups)
                ck = synth.random_codes(shape, seed=(code_seed, layer, b, 0))
                cv = synth.random_codes(shape, seed=(code_seed, layer, b, 1))
                put_codes(cache, layer, b, 0, ck.to(device))
                put_codes(cache, layer, b, 1, cv.to(device))
                codes[(layer, b)] = (ck, cv)
    lvq.lvq_pack_codebooks(cfg, lay, cache.cb, cache.cbp, cache.cb_norm)
    lvq.lvq_rope_table(cfg, lay, cache.rope)
    if codes_from == "encode":
        for layer in range(layers):
            for b in range(B):
                kvt = synth.loop_kv(w, layer, coded[b], stream="coded", request=b).to(device)
                lvq.lvq_encode_prefill(cfg, lay, layer, b, kvt, 0, coded[b], 0, cache.cb, cache.idx, cache.status)
    cache.ctx_len.copy_(torch.tensor(ctx, dtype=torch.int32))
    cache.coded_len.copy_(torch.tensor(coded, dtype=torch.int32))
    torch.cuda.synchronize()
    cache.check_status("build_case")
    return Case(w, cfg, cache, list(ctx), list(coded), layers, cbs, sink_kv, ring_kv, codes)


def oracle_decode(case: Case, layer: int, step: int, b: int, hq: int, q: torch.Tensor, n_splits=None,
                  codes=None):
    """fp64 oracle for one (layer, step, request, query head); codes default to the case's."""
    w = case.w
    h = hq // (w.n_q_heads // w.n_kv_heads)
    sk = f64(case.sink_kv[(layer, b)])            # [2][T][S][H][d]
    rk = f64(case.ring_kv[(layer, b)])
    ck, cv = codes if codes is not None else case.codes[(layer, b)]
    cb = f64(case.cb[layer])                      # [2][n_blk][H][n_g][256][G]
    return O.decode_attention(
        f64(q[b, hq]), step, w.Tc, w.G, sk[0, step, :, h], sk[1, step, :, h],
        ck[:, :, h].numpy(), cv[:, :, h].numpy(), cb[0, :, h], cb[1, :, h], rk[0, step, :, h], rk[1, step, :, h],
        base=w.rope_base, n_splits=n_splits)


def run_decode(case: Case, layer: int, step: int, q: torch.Tensor, num_splits: int, split_lse=True):
    c = case.cache
    B = len(case.ctx)
    out = torch.empty(B, case.w.n_q_heads, case.w.head_dim, dtype=torch.float32, device=q.device)
    lse = torch.empty(B, case.w.n_q_heads, dtype=torch.float32, device=q.device)
    sl = torch.empty(B, case.w.n_q_heads, num_splits + 1, dtype=torch.float32, device=q.device) if split_lse else None
    lvq.lvq_decode_attention(case.cfg, c.lay, layer, step, B, q, c.ctx_len, c.coded_len, c.sink, c.ring, c.idx,
                             c.cbp, c.rope, num_splits, c.workspace, out, lse, c.status, split_lse=sl)
    torch.cuda.synchronize()
    c.check_status("lvq_decode_attention")
    return out.cpu(), lse.cpu(), (sl.cpu() if sl is not None else None)


def assert_lse_close(got: float, ref: float, what=""):
    if ref == -np.inf:
        assert got == -np.inf, (what, got)
        return
    assert abs(got - ref) <= LSE_REL * max(1.0, abs(ref)), (what, got, ref)
