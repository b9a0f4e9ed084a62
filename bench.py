"""LoopVQ hot-path benchmark: decode attention over the coded cache, with the
decode-time page encode, on the Ouro-1.4B-shaped 0.5-bit workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lvq|reference]

Workload (one GPU, per rank): 24 layers x 16 KV heads, head_dim 128, T = 4
loop steps, Tc = 4, G = 16 (c = 4, 32 code bytes per token, head and K/V),
context 32768 (4 bf16 sink tokens, 128-token bf16 recent window, the rest
coded in 8-token pages), batch 1, synthetic loop-correlated K/V with two x8
outlier key channels per head, codes written by the library's own encoder.

One step = 8 generated tokens: per token the context grows by one and the
96 attentions (loop step t outer, layer inner, as a looped model runs them)
read the cache; after the 8th token the oldest page of the recent window is
encoded for every layer and loop step.  The step is captured once in a CUDA
graph and replayed.  Each token reads ~3.5 GB of codes, far more than the
126 MB L2, so no flush is needed between steps.

value  = decode tokens/s over all ranks (weak scaling: each rank its own request).
e2e    = the same with the step's queries copied from pinned host memory and
         its attention outputs copied back inside the timed region.
roofline: the decode kernel's algorithmic bytes per launch (coded rows of the
         step's block + the step's codebook slices + bf16 tokens + q/out) over
         its CUDA-event-timed average launch duration, against the measured
         HBM peak.
cpu_baseline / --impl reference: the fp64 oracle timed on a bounded sample
         of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn tokens/s and code-stream HBM GB/s vs peak; encode vectors/s"
WORKLOAD = "ouro14_g16_32k"
TOKENS_PER_STEP = 8


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="lvq", choices=["lvq", "reference"])
    ap.add_argument("--splits", type=int, default=0, help="split count (0: choose)")
    ap.add_argument("--workload", default=WORKLOAD, choices=["ouro14_g16_32k", "ouro14_g32_b32", "ouro14_tc2_64k", "ouro14_tc1_32k"],
                    help="decode workload (the headline line uses the default)")
    ap.add_argument("--no-encode", action="store_true", help="skip the prefill-encode measurement")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-sample", type=int, default=2,
                    help="single-head attentions per step of the reference (oracle) arm")
    ap.add_argument("--profile", default="", choices=["", "decode", "encode", "kmeans"],
                    help="build the workload, run 3 launches of one kernel and exit (for ncu captures)")
    return ap.parse_args()


# DRAM bytes (read + write) of one decode_kernel<128,4> launch of this workload, from one ncu
# capture (`python bench.py --profile decode` under ncu), valid only for the decode source it was
# taken on: the bench reports it when the file's hash still matches, else null.
DECODE_TRAFFIC = {"source_sha256": "e9422eb0c0c52da9d84373c6bdacf44bd53c0350259b6b29ed0d4d54ef5ada21",
                  "bytes_per_launch": 36771200}


def decode_traffic():
    src = os.path.join(ROOT, "sub_bit_kv_b200", "csrc", "lvq_decode.cu")
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    return DECODE_TRAFFIC["bytes_per_launch"] if sha == DECODE_TRAFFIC["source_sha256"] else None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def bf16_peak():
    """Dense bf16 TFLOP/s for a kernel timed on its own (burst figure)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


# ------------------------------------------------------------------------------ oracle baseline

class _OracleDecode:
    """The fp64 oracle on single-head decode attentions of the headline workload (32K
    context, 1 thread): inputs built once, then any number of head-attentions timed."""

    def __init__(self):
        import numpy as np  # noqa: F401
        from oracle import lvq_oracle as O
        from sub_bit_kv_b200 import synth
        self.O, self.synth = O, synth
        w = self.w = synth.WORKLOADS[WORKLOAD]
        L = w.ctx - w.n_sink - w.n_recent
        f = lambda t: t.to(dtype=__import__("torch").float64).numpy()
        self.cbf = f(synth.codebooks(w, 0))
        self.skf = f(synth.loop_kv(w, 0, w.n_sink, stream="sink"))
        self.rkf = f(synth.loop_kv(w, 0, w.n_recent, stream="recent"))
        self.codes = synth.random_codes((2, 1, L, w.n_groups), seed=7).numpy()
        self.n = 0
        self.per_token = w.n_layers * w.T * w.n_q_heads          # head-attentions per decode token

    def run(self, count: int) -> float:
        """Runs `count` head-attentions; returns the elapsed seconds."""
        w, O, cbf, skf, rkf = self.w, self.O, self.cbf, self.skf, self.rkf
        t0 = time.perf_counter()
        for _ in range(count):
            h, step = self.n % w.n_kv_heads, self.n % w.T
            q = self.synth.queries(w, 0, step)[0, h].to(dtype=__import__("torch").float64).numpy()
            O.decode_attention(q, step, w.Tc, w.G, skf[0, step, :, h], skf[1, step, :, h], self.codes[0],
                               self.codes[1], cbf[0, :, h], cbf[1, :, h], rkf[0, step, :, h], rkf[1, step, :, h],
                               base=w.rope_base)
            self.n += 1
        return time.perf_counter() - t0


def _one_thread():
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(limits=1)
    except Exception:  # pragma: no cover
        return None


def cpu_baseline(seconds: float):
    """Times the fp64 oracle on whole head-attentions of the workload (32K context) for
    about `seconds`."""
    limiter = _one_thread()
    od = _OracleDecode()
    n, el = 0, 0.0
    while el < seconds:
        el += od.run(1)
        n += 1
    if limiter is not None:
        limiter.unregister()
    return {"value": n / el / od.per_token, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} single-head decode attentions at {od.w.ctx} context (fp64 numpy, 1 thread), "
                      f"scaled by {od.per_token} head-attentions per token"}


def reference_arm(args):
    """The oracle on the host: W untimed steps, then K timed steps, each step a bounded sample
    of the workload (args.ref_sample single-head attentions, scaled to decode tokens)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    limiter = _one_thread()
    od = _OracleDecode()
    for _ in range(args.warmup):
        od.run(args.ref_sample)
    el = sum(od.run(args.ref_sample) for _ in range(args.steps))
    if limiter is not None:
        limiter.unregister()
    value = args.steps * args.ref_sample / el / od.per_token
    cb = {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
          "sample": f"{args.steps} steps of {args.ref_sample} single-head decode attentions at {od.w.ctx} "
                    f"context (fp64 numpy, 1 thread), scaled by {od.per_token} head-attentions per token"}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": TOKENS_PER_STEP / value * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch": 1, "seq_len": 32768, "parallelism": "cpu"},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ GPU arm

class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        # the raw samples go to $LVQ_CLOCKS_DIR (default: the temporary directory); the JSON
        # line carries their summary
        out_dir = os.environ.get("LVQ_CLOCKS_DIR", tempfile.gettempdir())
        self.path = os.path.join(out_dir, f"lvq_clocks_rank{index}_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].isdigit():
                    rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [int(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": int(rows[0][2]), "reasons": reasons,
                "samples": len(rows)}


def build_cache(w, lvq, synth, torch, extra_tokens: int, device, request_seed: int):
    """Coded cache at the workload's per-request contexts, codes from the library's encoder."""
    ctx = synth.ctx_lengths(w)
    B = len(ctx)
    cfg = lvq.make_config(w.n_layers, w.n_kv_heads, w.n_q_heads, w.head_dim, w.T, w.Tc, w.G, w.n_sink,
                          w.n_recent, B, max(ctx) + extra_tokens, max_splits=128, rope_base=w.rope_base)
    cache = lvq.CodedCache(cfg, device)
    lay = cache.lay
    coded = [c - w.n_sink - w.n_recent for c in ctx]
    cbv, sv, rv = cache.cb_view(), cache.sink_view(), cache.ring_view()
    for layer in range(w.n_layers):
        sc = synth.channel_scales(w, layer, device=device)
        cbv[layer] = synth.codebooks(w, layer, device=device, scales=sc)
        for b in range(B):
            seed = request_seed * B + b
            sk = synth.loop_kv(w, layer, w.n_sink, stream="sink", request=seed, device=device, scales=sc)
            rk = synth.loop_kv(w, layer, lay.ring_tokens, stream="recent", request=seed, device=device, scales=sc)
            sv[layer, :, :, b] = sk.permute(0, 1, 3, 2, 4)
            rv[layer, :, :, b] = rk.permute(0, 1, 3, 2, 4)
    lvq.lvq_pack_codebooks(cfg, lay, cache.cb, cache.cbp, cache.cb_norm)
    lvq.lvq_rope_table(cfg, lay, cache.rope)
    for layer in range(w.n_layers):
        for b in range(B):
            kv = synth.loop_kv(w, layer, coded[b], stream="coded", request=request_seed * B + b, device=device)
            lvq.lvq_encode_prefill(cfg, lay, layer, b, kv, 0, coded[b], 0, cache.cb, cache.idx, cache.status)
            del kv
    cache.ctx_len.copy_(torch.tensor(ctx, dtype=torch.int32))
    cache.coded_len.copy_(torch.tensor(coded, dtype=torch.int32))
    torch.cuda.synchronize()
    cache.check_status("cache build")
    return cfg, cache


def reduce_max(value: float, device) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_plan(rank: int, world: int, batch_per_rank: int) -> dict:
    """Weak scaling by request: rank r serves requests [r*B, (r+1)*B) with its own seeds;
    no data crosses ranks."""
    return {"first_request": rank * batch_per_rank, "requests": batch_per_rank,
            "seed": rank, "global_batch": world * batch_per_rank}


def choose_splits(w, n_sm: int) -> int:
    """Splits per (request, head).  One CTA per SM: when the batch's heads fit in one wave,
    as many splits as fill it; otherwise splits of about 6K coded tokens, which balance the
    waves of a ragged batch against each CTA's fixed cost (measured on the 32-request
    workload: 3-4 splits beat 1, 2 and 6)."""
    heads = w.batch * w.n_q_heads
    if heads <= n_sm:
        return max(1, min(128, n_sm // heads))
    mean_ctx = w.ctx if w.ctx else (w.ctx_low + w.ctx_high) / 2
    return max(1, min(16, round(mean_ctx / 6144)))


def decode_bytes_per_launch(w, lay, coded, recent) -> int:
    """Algorithmic bytes of one decode attention (one layer, one loop step) over the batch:
    per request its coded rows of this step's block (K and V), its bf16 tokens and its
    query/output; the step-t codebook slices once per launch."""
    slices = w.n_kv_heads * 2 * 256 * w.head_dim * 2              # step-t codebook slices, K and V
    total = slices
    for cd, rc in zip(coded, recent):
        total += cd * w.n_kv_heads * 2 * lay.n_groups             # this step's block rows, K and V
        total += (min(w.n_sink, cd + rc) + rc) * w.n_kv_heads * 2 * w.head_dim * 2
        total += w.n_q_heads * w.head_dim * (2 + 4) + w.n_q_heads * 4
    return total


def profile_kmeans(lvq, synth, torch, device):
    """One Ouro-2.6B-shaped layer (32768 tokens): one encode, then the k-means update 3 times."""
    wc = synth.WORKLOADS["ouro26_prefill_32k"]
    cfg4 = lvq.make_config(1, wc.n_kv_heads, wc.n_q_heads, wc.head_dim, wc.T, wc.Tc, wc.G, 0, 0, 1, wc.ctx,
                           max_splits=1, rope_base=wc.rope_base)
    c4 = lvq.CodedCache(cfg4, device)
    c4.cb_view()[0] = synth.codebooks(wc, 0, device=device)
    kv4 = synth.loop_kv(wc, 0, wc.ctx, stream="coded", device=device)
    lvq.lvq_encode_prefill(cfg4, c4.lay, 0, 0, kv4, 0, wc.ctx, 0, c4.cb, c4.idx, c4.status)
    for _ in range(3):
        lvq.lvq_kmeans_update(cfg4, c4.lay, 0, 0, kv4, 0, wc.ctx, 0, c4.idx, c4.cb, None, c4.status)
    torch.cuda.synchronize()
    c4.check_status("profile kmeans")


def profile_encode(lvq, synth, torch, device):
    """One Ouro-2.6B-shaped layer (32768 tokens), encoded 3 times."""
    wc = synth.WORKLOADS["ouro26_prefill_32k"]
    cfg4 = lvq.make_config(1, wc.n_kv_heads, wc.n_q_heads, wc.head_dim, wc.T, wc.Tc, wc.G, 0, 0, 1, wc.ctx,
                           max_splits=1, rope_base=wc.rope_base)
    c4 = lvq.CodedCache(cfg4, device)
    c4.cb_view()[0] = synth.codebooks(wc, 0, device=device)
    kv4 = synth.loop_kv(wc, 0, wc.ctx, stream="coded", device=device)
    for _ in range(3):
        lvq.lvq_encode_prefill(cfg4, c4.lay, 0, 0, kv4, 0, wc.ctx, 0, c4.cb, c4.idx, c4.status)
    torch.cuda.synchronize()
    c4.check_status("profile encode")


def gpu_arm(args):
    import torch
    import torch.distributed as dist

    from sub_bit_kv_b200 import _build, lvq, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=300))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if rank == 0:
        _build.build()
    if world > 1:
        dist.barrier()
    lvq.lib()

    if args.profile == "encode":
        profile_encode(lvq, synth, torch, device)
        return
    if args.profile == "kmeans":
        profile_kmeans(lvq, synth, torch, device)
        return
    w = synth.WORKLOADS[args.workload]
    replays = 2 * args.steps + args.warmup + 3          # every graph replay adds 8 tokens
    cfg, cache = build_cache(w, lvq, synth, torch, TOKENS_PER_STEP * (replays + 4), device,
                             replica_plan(rank, world, w.batch)["seed"])
    lay = cache.lay
    n_sm = torch.cuda.get_device_properties(device).multi_processor_count
    ns = args.splits or choose_splits(w, n_sm)
    B, Hq, d = w.batch, w.n_q_heads, w.head_dim
    if args.profile == "decode":
        q = torch.randn(B, Hq, d, device=device).to(torch.bfloat16)
        o = torch.empty(B, Hq, d, device=device)
        l = torch.empty(B, Hq, device=device)
        for layer in range(3):
            lvq.lvq_decode_attention(cfg, lay, layer, 0, B, q, cache.ctx_len, cache.coded_len, cache.sink,
                                     cache.ring, cache.idx, cache.cbp, cache.rope, ns, cache.workspace, o, l,
                                     cache.status)
        torch.cuda.synchronize()
        cache.check_status("profile")
        return
    NL = w.n_layers * w.T                                            # attentions per token
    q_all = torch.randn(TOKENS_PER_STEP, w.T, w.n_layers, B, Hq, d, device=device,
                        generator=synth.generator(device, w.seed, "bench-q", rank)).to(torch.bfloat16)
    out_all = torch.empty(TOKENS_PER_STEP, w.T, w.n_layers, B, Hq, d, device=device, dtype=torch.float32)
    lse_all = torch.empty(TOKENS_PER_STEP, w.T, w.n_layers, B, Hq, device=device, dtype=torch.float32)

    def step_body(stream):
        for tok in range(TOKENS_PER_STEP):
            cache.ctx_len.add_(1)
            for t in range(w.T):
                for layer in range(w.n_layers):
                    lvq.lvq_decode_attention(cfg, lay, layer, t, B, q_all[tok, t, layer], cache.ctx_len,
                                             cache.coded_len, cache.sink, cache.ring, cache.idx, cache.cbp,
                                             cache.rope, ns, cache.workspace, out_all[tok, t, layer],
                                             lse_all[tok, t, layer], cache.status, stream=stream)
        lvq.lvq_encode_page(cfg, lay, B, cache.ctx_len, cache.coded_len, cache.ring, cache.cb, cache.cb_norm,
                            cache.idx, cache.status, stream=stream)

    launches_per_step = TOKENS_PER_STEP * NL + 2
    stream = torch.cuda.Stream(device)
    # one eager step to check everything runs, then capture the step
    with torch.cuda.stream(stream):
        step_body(stream)
    torch.cuda.synchronize()
    cache.check_status("eager step")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step_body(stream)
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    cache.check_status("warmup")

    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(local) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            t_start.record(stream)
            for _ in range(args.steps):
                graph.replay()
            t_end.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    ms = reduce_max(t_start.elapsed_time(t_end), device)
    cache.check_status("timed")
    plan = replica_plan(rank, world, B)
    tokens = TOKENS_PER_STEP * args.steps * plan["global_batch"]
    value = tokens / (ms / 1e3)

    # ---- decode kernel timing: a graph of the 96 attentions of one token, event-timed
    coded_now = [int(v) for v in cache.coded_len[:B].tolist()]
    ctx_now = [int(v) for v in cache.ctx_len[:B].tolist()]
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2, stream=stream):
        for t in range(w.T):
            for layer in range(w.n_layers):
                lvq.lvq_decode_attention(cfg, lay, layer, t, B, q_all[0, t, layer], cache.ctx_len,
                                         cache.coded_len, cache.sink, cache.ring, cache.idx, cache.cbp,
                                         cache.rope, ns, cache.workspace, out_all[0, t, layer],
                                         lse_all[0, t, layer], cache.status, stream=stream)
    reps = 5
    g2.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            g2.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    per_call_ms = e0.elapsed_time(e1) / (reps * NL)
    recent_now = [c - w.n_sink - cd for c, cd in zip(ctx_now, coded_now)]
    bpl = decode_bytes_per_launch(w, lay, coded_now, recent_now)
    hbm_peak, peak_kind = peaks()
    achieved = bpl / (per_call_ms / 1e3) / 1e9
    code_stream = sum(coded_now) * w.n_kv_heads * 2 * lay.n_groups / (per_call_ms / 1e3) / 1e9

    # ---- e2e: queries in from pinned host memory, outputs back, every step
    q_host = torch.empty(q_all.shape, dtype=q_all.dtype).pin_memory()
    q_host.copy_(q_all.cpu())
    out_host = torch.empty(out_all.shape, dtype=out_all.dtype).pin_memory()
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(args.steps):
            q_all.copy_(q_host, non_blocking=True)
            graph.replay()
            out_host.copy_(out_all, non_blocking=True)
        t1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(t0.elapsed_time(t1), device)
    e2e_value = tokens / (e2e_ms / 1e3)
    cache.check_status("e2e")

    # ---- prefill encode (secondary): one Ouro-2.6B-shaped layer, 32768 tokens
    enc = None
    if not args.no_encode:
        wc = synth.WORKLOADS["ouro26_prefill_32k"]
        cfg4 = lvq.make_config(1, wc.n_kv_heads, wc.n_q_heads, wc.head_dim, wc.T, wc.Tc, wc.G, 0, 0, 1,
                               wc.ctx, max_splits=1, rope_base=wc.rope_base)
        c4 = lvq.CodedCache(cfg4, device)
        c4.cb_view()[0] = synth.codebooks(wc, 0, device=device)
        kv4 = synth.loop_kv(wc, 0, wc.ctx, stream="coded", device=device)
        args4 = (cfg4, c4.lay, 0, 0, kv4, 0, wc.ctx, 0, c4.cb, c4.idx, c4.status)
        lvq.lvq_encode_prefill(*args4)
        torch.cuda.synchronize()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(3):
            lvq.lvq_encode_prefill(*args4)
        b_.record()
        torch.cuda.synchronize()
        enc_ms = a.elapsed_time(b_) / 3
        vectors = wc.ctx * wc.n_kv_heads * 2 * (wc.head_dim // (wc.G // wc.Tc)) * (wc.T // wc.Tc)
        # useful distance GEMM work: 256 entries x G dims x 2 flops per vector
        tflops = vectors * 256 * wc.G * 2 / (enc_ms / 1e3) / 1e12
        tpk, tpk_kind = bf16_peak()
        enc = {"vectors_per_s": vectors / (enc_ms / 1e3), "ms_per_layer": enc_ms,
               "distance_gemm_tflops": tflops, "frac_of_bf16_peak": tflops / tpk, "bf16_peak": tpk,
               "peak_kind": tpk_kind,
               "workload": "ouro26_prefill_32k (one of 48 layers)", "kernel": "encode_tc (tcgen05 distance GEMM + argmin)"}
        # codebook construction: the k-means update step over the codes the encoder just wrote
        # (one Lloyd iteration = this encode + this update); it reads the layer's bf16 K/V and
        # its codes once
        argsk = (cfg4, c4.lay, 0, 0, kv4, 0, wc.ctx, 0, c4.idx, c4.cb, None, c4.status)
        lvq.lvq_kmeans_update(*argsk)
        torch.cuda.synchronize()
        a.record()
        for _ in range(3):
            lvq.lvq_kmeans_update(*argsk)
        b_.record()
        torch.cuda.synchronize()
        c4.check_status("kmeans update")
        upd_ms = a.elapsed_time(b_) / 3
        upd_bytes = kv4.numel() * 2 + vectors + c4.lay.cb_bytes
        enc["kmeans"] = {"update_ms": upd_ms, "iteration_ms": enc_ms + upd_ms,
                         "iteration_vectors_per_s": vectors / ((enc_ms + upd_ms) / 1e3),
                         "update_gbps": upd_bytes / (upd_ms / 1e3) / 1e9,
                         "update_frac_of_hbm": upd_bytes / (upd_ms / 1e3) / 1e9 / peaks()[0],
                         "kernel": "kmeans_update (fp64 shared-memory sums per entry)"}
        del kv4, c4

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return
    cb = cpu_baseline(args.cpu_seconds)
    clocks = clk.summary()
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": args.workload, "global_batch": B * world,
                   "seq_len": w.ctx if w.ctx else f"{w.ctx_low}-{w.ctx_high}", "layers": w.n_layers,
                   "loop_steps": w.T, "Tc": w.Tc, "G": w.G, "kv_heads": w.n_kv_heads, "head_dim": d,
                   "num_splits": ns, "tokens_per_step": TOKENS_PER_STEP,
                   "l2": f"inputs larger than L2 ({NL * bpl / 1e9:.1f} GB read per generated token)",
                   "parallelism": f"replicas{world}"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak,
                     "traffic": decode_traffic() if args.workload == WORKLOAD else None,
                     "kernel": f"decode_kernel<{d},{lay.c}>",
                     "peak_kind": peak_kind, "bytes_per_launch": bpl, "launch_ms": per_call_ms},
        "code_stream_GBps": code_stream,
        "cpu_baseline": cb,
        "e2e": {"value": e2e_value, "unit": "tokens/s",
                "h2d_bytes_per_step": q_all.numel() * q_all.element_size() * world,
                "d2h_bytes_per_step": out_all.numel() * out_all.element_size() * world},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "encode": enc,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        reference_arm(args)
    else:
        gpu_arm(args)


if __name__ == "__main__":
    main()
