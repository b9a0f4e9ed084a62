"""LoopVQ hot-path benchmark: decode attention over the coded cache (with the decode-time
page encode) and the prefill encoder, on the Ouro-shaped workloads.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lvq|reference] [--workload NAME]

Workloads (one GPU, per rank; synthetic loop-correlated K/V with two x8 outlier key
channels per head, codes written by the library's own encoder):

  ouro14_g16_32k (default, the headline line): 24 layers x 16 KV heads, head_dim 128,
      T = 4 loop steps, Tc = 4, G = 16 (c = 4, 32 code bytes per token, head and K/V),
      context 32768 (4 bf16 sink tokens, 128-token bf16 recent window, the rest coded in
      8-token pages), batch 1.
  ouro14_g32_b32: the same model at G = 32 (0.25 bit), 32 requests with contexts drawn
      uniformly from [8192, 32768].
  ouro14_tc2_64k: Tc = 2 (two index rows per token), context 65536, batch 8, 256-token
      recent window; the timed region is the 256 generated tokens from that context, with
      the oldest page encoded every 8 tokens as the cache grows.
  ouro14_tc1_32k: per-step coding (Tc = 1, c = G = 16), otherwise the headline shape.
  ouro26_prefill_32k: prefill encode of a 32768-token prompt for 48 layers x 16 KV heads
      (1.61e9 joint vectors) as one call over every layer (layer = -1).

Decode: one step = 8 generated tokens per request: per token the context grows by one
and the 96 attentions (loop step t outer, layer inner, as a looped model runs them) read
the cache; after the 8th token the oldest page of the recent window is encoded for every
layer and loop step.  The step is captured once in a CUDA graph and replayed; the cache
counters are reset after the warm-up so that the timed tokens start at the workload's
context.  Each token reads gigabytes of codes, far more than the 126 MB L2, so no flush is
needed between steps.  Encode: one step = one call encoding all 48 layers (51.5 GB of
bf16 K/V read, also far above L2).

value  = decode tokens/s (encode: vectors/s) over all ranks (weak scaling: each rank
         its own requests).
e2e    = the same with each step's inputs copied from pinned host memory and its results
         copied back inside the timed region (decode: queries in, outputs out; encode: the
         K/V of every layer in, the codes out).
roofline: the dominant kernel's algorithmic bytes per launch over its CUDA-event-timed
         average launch duration, against the measured HBM peak.
cpu_baseline / --impl reference: the fp64 oracle timed on a bounded sample of the same
         workload on the host cores, scaled to the metric's unit.
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
DECODE_WORKLOADS = ("ouro14_g16_32k", "ouro14_g32_b32", "ouro14_tc2_64k", "ouro14_tc1_32k")
ENCODE_WORKLOAD = "ouro26_prefill_32k"
TOKENS_PER_STEP = 8
# timed steps when --steps is not given: the headline's 20 steps (160 tokens) take under a
# second; the 64K workload's 32 steps are its 256 generated tokens; the 48-layer encode takes
# ~0.1 s a step
DEFAULT_STEPS = {"ouro14_g16_32k": 20, "ouro14_g32_b32": 6, "ouro14_tc2_64k": 32, "ouro14_tc1_32k": 20,
                 "ouro26_prefill_32k": 5}


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="timed steps (default: per workload)")
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="lvq", choices=["lvq", "reference"])
    ap.add_argument("--splits", type=int, default=0, help="split count (0: choose)")
    ap.add_argument("--workload", default=WORKLOAD, choices=list(DECODE_WORKLOADS) + [ENCODE_WORKLOAD])
    ap.add_argument("--no-encode", action="store_true", help="skip the one-layer prefill-encode measurement")
    ap.add_argument("--max-ctas", type=int, default=0,
                    help="decode workloads: cap the decode's CTAs (lvq_decode_max_ctas); below the work-item "
                         "count each CTA walks a run of items")
    ap.add_argument("--pool", action="store_true",
                    help="decode workloads: codes in a shared page pool behind an 8-token page table")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--oracle-procs", type=int, default=0,
                    help="host processes timing the oracle (0: every usable core, at most %d)" % ORACLE_MAX_PROCS)
    ap.add_argument("--ref-sample", type=int, default=2,
                    help="units (head-attentions, or encode batches) per step of the reference (oracle) arm")
    ap.add_argument("--profile", default="", choices=["", "decode", "encode", "kmeans"],
                    help="build the workload, run 3 launches of one kernel and exit (for ncu captures)")
    args = ap.parse_args(argv)
    if args.steps is None:
        args.steps = DEFAULT_STEPS[args.workload]
    return args


# One ncu capture of a decode_kernel<128,4> launch of the headline workload
# (`python bench.py --profile decode` under ncu): its DRAM bytes (read + write) and its warp
# instructions (smsp__inst_executed.sum), valid only for the decode source they were taken on:
# the bench reports them when the file's hash still matches, else null.
DECODE_NCU = {"source_sha256": "3d24c45237a893e6b9f0d88fdb2b00c9fd52fe726cf3de34b51dd97015c8fed9",
              "dram_bytes_per_launch": 36983296, "warp_inst_per_launch": 15338781}


def _decode_ncu():
    src = os.path.join(ROOT, "sub_bit_kv_b200", "csrc", "lvq_decode.cu")
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    return DECODE_NCU if sha == DECODE_NCU["source_sha256"] else None


def decode_traffic():
    n = _decode_ncu()
    return n["dram_bytes_per_launch"] if n else None


def decode_issue(launch_ms, sm_mhz, n_sm, token_heads):
    """The issue ceiling of one decode launch: its warp instructions (ncu) issued at one per
    scheduler per cycle (4 per SM) at the SM clock sampled during the timed region; `frac` is
    that ceiling's duration over the measured one."""
    n = _decode_ncu()
    if not n or not sm_mhz:
        return None
    inst = n["warp_inst_per_launch"]
    ceiling_ms = inst / (n_sm * 4 * sm_mhz * 1e6) * 1e3
    return {"warp_inst_per_launch": inst, "per_coded_token_head": inst / token_heads, "sm_mhz": sm_mhz,
            "ceiling_us": ceiling_ms * 1e3, "frac": ceiling_ms / launch_ms}


def _peaks_file():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f)
    return None


def peaks():
    d = _peaks_file()
    if d is not None:
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def bf16_peak():
    """Dense bf16 TFLOP/s for a kernel timed on its own (burst figure)."""
    d = _peaks_file()
    if d is not None:
        return float(d["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:  # pragma: no cover
        return os.cpu_count() or 1


# ------------------------------------------------------------------------------ timing across ranks

class EventClock:
    """Marks on a CUDA stream (device time)."""

    def __init__(self, stream):
        self.stream = stream

    def mark(self):
        import torch
        e = torch.cuda.Event(enable_timing=True)
        e.record(self.stream)
        return e

    @staticmethod
    def elapsed_ms(a, b) -> float:
        return a.elapsed_time(b)


class HostClock:
    """Marks on the host clock (for the CPU oracle and for tests without a GPU)."""

    @staticmethod
    def mark():
        return time.perf_counter()

    @staticmethod
    def elapsed_ms(a, b) -> float:
        return (b - a) * 1e3


def reduce_max(value: float, device) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def time_region(body, clock, device, sync=lambda: None) -> float:
    """Times body() (all the timed steps) on `clock`, bracketed on both sides by a barrier over
    the ranks and a synchronize; returns the maximum over ranks, in ms.  Every rank takes the
    same collective steps."""
    import torch.distributed as dist
    multi = dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1
    if multi:
        dist.barrier()
    sync()
    a = clock.mark()
    body()
    b = clock.mark()
    sync()
    if multi:
        dist.barrier()
    return reduce_max(clock.elapsed_ms(a, b), device)


def replica_plan(rank: int, world: int, batch_per_rank: int) -> dict:
    """Weak scaling by request: rank r serves requests [r*B, (r+1)*B) with its own seeds;
    no data crosses ranks."""
    return {"first_request": rank * batch_per_rank, "requests": batch_per_rank,
            "seed": rank, "global_batch": world * batch_per_rank}


# ------------------------------------------------------------------------------ workload configs

def decode_config(w, world: int, ns: int) -> dict:
    """The `config` of a decode workload's line (both arms)."""

    class _Groups:
        n_groups = w.n_groups

    ctx = [c for c in __import__("sub_bit_kv_b200.synth", fromlist=["synth"]).ctx_lengths(w)]
    coded = [c - w.n_sink - w.n_recent for c in ctx]
    gb = w.n_layers * w.T * decode_bytes_per_launch(w, _Groups, coded, [w.n_recent] * len(ctx)) / 1e9
    return {"workload": w.name, "global_batch": w.batch * world,
            "seq_len": w.ctx if w.ctx else f"{w.ctx_low}-{w.ctx_high}", "layers": w.n_layers,
            "loop_steps": w.T, "Tc": w.Tc, "G": w.G, "kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
            "num_splits": ns, "tokens_per_step": TOKENS_PER_STEP * w.batch * world,
            "l2": f"inputs larger than L2 ({gb:.1f} GB read per generated token of every request)",
            "parallelism": f"replicas{world}"}


def encode_config(w, world: int) -> dict:
    """The `config` of the prefill-encode line (both arms)."""
    return {"workload": w.name, "global_batch": world, "seq_len": w.ctx, "layers": w.n_layers,
            "loop_steps": w.T, "Tc": w.Tc, "G": w.G, "kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
            "vectors_per_step": encode_vectors(w, w.n_layers, w.ctx),
            "call": "lvq_encode_prefill(layer = -1): all layers in one launch",
            "l2": "inputs larger than L2 (51.5 GB of K/V read per step)", "parallelism": f"replicas{world}"}


# ------------------------------------------------------------------------------ oracle baselines

ORACLE_MAX_PROCS = 32      # host processes of the oracle baselines (each one thread)


def oracle_procs(requested: int = 0) -> int:
    """Host processes for the oracle: `requested`, else every core this process may use, at most
    ORACLE_MAX_PROCS (each holds its own copy of the inputs)."""
    if requested > 0:
        return requested
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        n = os.cpu_count() or 1
    return max(1, min(n, ORACLE_MAX_PROCS))


def _one_thread():
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(limits=1)
    except Exception:  # pragma: no cover
        return None


class _OracleDecode:
    """The fp64 oracle on single-head decode attentions of a decode workload (numpy, one
    thread): inputs built per request on first use, then any number of head-attentions timed,
    the requests taken in turn (so that a ragged batch is sampled evenly).  For the workload
    with a growing cache it also times page-encode units (one codebook's nearest entries for
    8 tokens), in proportion to the attentions a generated token needs."""

    def __init__(self, name: str):
        import torch
        from oracle import lvq_oracle as O
        from sub_bit_kv_b200 import synth
        self.O, self.synth, self.torch = O, synth, torch
        w = self.w = synth.WORKLOADS[name]
        self.ctx = synth.ctx_lengths(w)
        self.f = lambda t: t.to(dtype=torch.float64).numpy()
        self.cbf = self.f(synth.codebooks(w, 0))
        self.skf = self.f(synth.loop_kv(w, 0, w.n_sink, stream="sink"))
        self.rkf = self.f(synth.loop_kv(w, 0, w.n_recent, stream="recent"))
        self.codes = {}
        self.n = 0
        self.per_token = w.n_layers * w.T * w.n_q_heads          # head-attentions per generated token
        # page-encode units per generated token of one request: every (layer, K/V, block, head,
        # group) codebook encodes 8 tokens once per 8 tokens
        self.units_per_token = w.n_layers * 2 * w.n_blocks * w.n_kv_heads * w.n_groups / TOKENS_PER_STEP
        self.page_kv = self.f(synth.loop_kv(w, 0, TOKENS_PER_STEP, stream="page"))   # [2][T][8][H][d]

    def _codes(self, b):
        if b not in self.codes:
            L = self.ctx[b] - self.w.n_sink - self.w.n_recent
            self.codes[b] = self.synth.random_codes((2, self.w.n_blocks, L, self.w.n_groups), seed=(7, b)).numpy()
        return self.codes[b]

    def run(self, count: int) -> float:
        """Runs `count` head-attentions; returns the elapsed seconds."""
        w, O, cbf, skf, rkf = self.w, self.O, self.cbf, self.skf, self.rkf
        el = 0.0
        for _ in range(count):
            b = self.n % len(self.ctx)
            h, step = (self.n // len(self.ctx)) % w.n_kv_heads, self.n % w.T
            codes = self._codes(b)
            q = self.synth.queries(w, 0, step, batch=1)[0, h].to(dtype=self.torch.float64).numpy()
            t0 = time.perf_counter()
            O.decode_attention(q, step, w.Tc, w.G, skf[0, step, :, h], skf[1, step, :, h], codes[0], codes[1],
                               cbf[0, :, h], cbf[1, :, h], rkf[0, step, :, h], rkf[1, step, :, h],
                               base=w.rope_base)
            el += time.perf_counter() - t0
            self.n += 1
        return el

    def page_units(self, count: int) -> float:
        """Runs `count` page-encode units; returns the elapsed seconds."""
        w, O = self.w, self.O
        X = O.joint_vectors(self.page_kv[0], w.Tc, w.G)          # [n_blk][8][H][n_g][G]
        t0 = time.perf_counter()
        for i in range(count):
            blk, h, g = i % w.n_blocks, (i // w.n_blocks) % w.n_kv_heads, i % w.n_groups
            O.nearest_entry(X[blk, :, h, g], self.cbf[0, blk, h, g])
        return time.perf_counter() - t0

    def tokens_per_s(self, attn_s: float, n_attn: int, unit_s: float, n_units: int) -> float:
        per_token = self.per_token * attn_s / n_attn
        if self.w.gen_tokens and n_units:
            per_token += self.units_per_token * unit_s / n_units
        return 1.0 / per_token


class _OracleEncode:
    """The fp64 oracle's brute-force nearest entries on joint vectors of the prefill workload
    (numpy, one thread): batches of 1024 vectors of one layer, each against its codebook (the
    K/V sides, heads and groups taken in turn)."""

    BATCH = 1024

    def __init__(self):
        import torch
        from oracle import lvq_oracle as O
        from sub_bit_kv_b200 import synth
        self.O = O
        w = self.w = synth.WORKLOADS[ENCODE_WORKLOAD]
        self.cbf = synth.codebooks(w, 0).to(torch.float64).numpy()          # [2][n_blk][H][n_g][256][G]
        kv = synth.loop_kv(w, 0, self.BATCH, stream="coded").to(torch.float64).numpy()   # [2][T][N][H][d]
        self.X = [O.joint_vectors(kv[kvi], w.Tc, w.G) for kvi in range(2)]  # [n_blk][N][H][n_g][G]
        self.i = 0

    def run(self, count: int) -> float:
        """Runs `count` batches; returns the elapsed seconds."""
        w = self.w
        el = 0.0
        for _ in range(count):
            i = self.i
            kvi, h, g = i % 2, (i // 2) % w.n_kv_heads, (i // (2 * w.n_kv_heads)) % w.n_groups
            t0 = time.perf_counter()
            self.O.nearest_entry(self.X[kvi][0, :, h, g], self.cbf[kvi, 0, h, g])
            el += time.perf_counter() - t0
            self.i += 1
        return el


def _oracle_proc(name, seconds, count, warm, offset, barrier, queue):
    """One host process of an oracle baseline (spawned, one thread): builds the workload's oracle
    inputs, runs `warm` untimed units, waits for every process at `barrier`, then runs units until
    `seconds` of oracle time have passed (or `count` units); puts (units, oracle seconds, rate in
    the workload's unit, description) on `queue`."""
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[var] = "1"
    _one_thread()
    if name == ENCODE_WORKLOAD:
        o = _OracleEncode()
        o.i = offset
        o.run(max(warm, 1))
        barrier.wait(timeout=900)
        n, el = 0, 0.0
        while (n < count) if count else (el < seconds):
            el += o.run(1)
            n += 1
        queue.put((n * o.BATCH, el, n * o.BATCH / el, ""))
        return
    o = _OracleDecode(name)
    for b in range(len(o.ctx)):
        o._codes(b)                                    # every request's inputs exist before the clock
    o.n = offset
    o.run(max(warm, 1))
    barrier.wait(timeout=900)
    n, el = 0, 0.0
    while (n < count) if count else (el < seconds):
        el += o.run(1)
        n += 1
    nu = 8 if o.w.gen_tokens else 0
    ue = o.page_units(nu) if nu else 0.0
    extra = f" plus {nu} page-encode units ({o.units_per_token:.0f} per token)" if nu else ""
    queue.put((n, el + ue, o.tokens_per_s(el, n, ue, nu),
               f"(requests in turn, contexts {min(o.ctx)}-{max(o.ctx)}){extra}, scaled by {o.per_token} "
               f"head-attentions per generated token"))


def oracle_parallel(name: str, procs: int, seconds: float = 0.0, count: int = 0, warm: int = 0):
    """The oracle on `procs` host processes at once (spawned, one thread each, each sampling other
    heads and requests); returns the per-process results of _oracle_proc."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    barrier, queue = ctx.Barrier(procs), ctx.Queue()
    ps = [ctx.Process(target=_oracle_proc, args=(name, seconds, count, warm, 7 * i, barrier, queue))
          for i in range(procs)]
    for p in ps:
        p.start()
    try:
        res = [queue.get(timeout=1800) for _ in ps]
    finally:
        for p in ps:
            p.join(timeout=60)
    return res


def cpu_baseline(name: str, seconds: float, procs: int = 0):
    """The oracle on a bounded sample of workload `name`: one single-threaded process per usable
    host core (at most ORACLE_MAX_PROCS), all timed at once; the rate is their sum."""
    P = oracle_procs(procs)
    res = oracle_parallel(name, P, seconds=seconds)
    value = sum(r[2] for r in res)
    units = sum(r[0] for r in res)
    if name == ENCODE_WORKLOAD:
        return {"value": value, "unit": "vectors/s", "cores": P, "kind": "oracle",
                "sample": f"{units} joint vectors of one layer over {P} processes (~{seconds:.0f} s each), "
                          f"brute-force nearest of 256 entries (fp64 numpy, 1 thread per process), per vector; "
                          f"the workload has 48 layers x 33.5 M vectors"}
    return {"value": value, "unit": "tokens/s", "cores": P, "kind": "oracle",
            "sample": f"{units} single-head decode attentions over {P} processes (~{seconds:.0f} s each) "
                      f"{res[0][3]} (fp64 numpy, 1 thread per process)"}


def reference_arm(args):
    """The oracle on the host: one single-threaded process per usable core (at most
    ORACLE_MAX_PROCS), each running W untimed steps then K timed steps of a bounded sample of the
    workload (args.ref_sample head-attentions, or encode batches of 1024 vectors); the rate, in the
    metric's unit, is the processes' sum."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from sub_bit_kv_b200 import synth
    P = oracle_procs(args.oracle_procs)
    res = oracle_parallel(args.workload, P, count=args.steps * args.ref_sample, warm=args.warmup * args.ref_sample)
    value = sum(r[2] for r in res)
    el = max(r[1] for r in res)                 # host seconds of the slowest process over the K steps
    if args.workload == ENCODE_WORKLOAD:
        unit = "vectors/s"
        sample = (f"{P} processes x {args.steps} steps of {args.ref_sample} batches of {_OracleEncode.BATCH} joint "
                  f"vectors of one layer, brute-force nearest entry (fp64 numpy, 1 thread per process), per vector")
        config = encode_config(synth.WORKLOADS[ENCODE_WORKLOAD], args.gpus)
    else:
        w = synth.WORKLOADS[args.workload]
        unit = "tokens/s"
        sample = (f"{P} processes x {args.steps} steps of {args.ref_sample} single-head decode attentions "
                  f"{res[0][3]} (fp64 numpy, 1 thread per process)")
        config = decode_config(w, args.gpus, choose_splits(w, 148))
    cb = {"value": value, "unit": unit, "cores": P, "kind": "oracle", "sample": sample}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            # the host time of one sampled step (the rate above is scaled to the workload's unit)
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
            "cpu_baseline": cb, "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
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


POOL_BITE = 64      # pages a request takes from the pool at a time in pool mode (512 tokens)


def build_cache(w, lvq, synth, torch, extra_tokens: int, device, request_seed: int, max_splits: int = 128,
                pool: bool = False):
    """Coded cache at the workload's per-request contexts, codes from the library's encoder.
    pool: codes in a shared page pool; every request holds the pages of its context plus
    extra_tokens, taken from the pool in round-robin bites of POOL_BITE pages (as requests that
    grow side by side would take them), so its pages are runs of POOL_BITE consecutive ids."""
    ctx = synth.ctx_lengths(w)
    B = len(ctx)
    coded = [c - w.n_sink - w.n_recent for c in ctx]
    need = [(cd + extra_tokens + 7) // 8 for cd in coded]
    cfg = lvq.make_config(w.n_layers, w.n_kv_heads, w.n_q_heads, w.head_dim, w.T, w.Tc, w.G, w.n_sink,
                          w.n_recent, B, max(ctx) + extra_tokens, max_splits=max_splits, rope_base=w.rope_base,
                          pool_pages=sum(need) if pool else 0)
    cache = lvq.CodedCache(cfg, device)
    lay = cache.lay
    if pool:
        left = list(need)
        while any(left):
            for b in range(B):
                k = min(POOL_BITE, left[b])
                if k:
                    cache.assign_pages(b, len(cache.pages[b]) + k)
                    left[b] -= k
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


SPLIT_FIXED_TOKENS = 850    # a CTA's fixed cost (slices, prologue, merge) in coded tokens of work


def choose_splits(w, n_sm: int) -> int:
    """Splits per (request, head), one CTA per SM.  Requests of equal length: the count (up to
    128) that minimises waves x (coded tokens per CTA + a CTA's fixed cost), the waves being
    whole -- at the 32K workload 9 splits fill one wave (144 of 148 SMs; 10 would spill into a
    second wave: 46 us against 27 us), at the 8-request 64K workload 8 splits give 7 nearly full
    waves (327 us per launch, against 410 us for 1 split and 372 us for 7).  A ragged batch:
    splits of about 6K coded tokens, which balance its waves against the fixed cost (measured on
    the 32-request workload: 3 splits, 486 us, against 521 for 2 and 496 for 4)."""
    heads = w.batch * w.n_q_heads
    if w.ctx:
        L = max(0, w.ctx - w.n_sink - w.n_recent)
        cost = {ns: -(-heads * ns // n_sm) * (L / ns + SPLIT_FIXED_TOKENS) for ns in range(1, 129)}
        return min(cost, key=lambda ns: (cost[ns], ns))
    mean_ctx = (w.ctx_low + w.ctx_high) / 2
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


def encode_bytes_per_call(w, n_layers: int, n_tok: int, cb_bytes: int) -> int:
    """Algorithmic bytes of a prefill encode over n_layers layers: the bf16 keys and values of
    every loop step read once, one code byte written per joint vector, the codebooks read once."""
    kv = n_layers * 2 * w.T * n_tok * w.n_kv_heads * w.head_dim * 2
    vectors = encode_vectors(w, n_layers, n_tok)
    return kv + vectors + cb_bytes


def encode_vectors(w, n_layers: int, n_tok: int) -> int:
    return n_layers * 2 * w.n_blocks * n_tok * w.n_kv_heads * w.n_groups


def page_encode_us(lvq, torch, cfg, cache, stream, B: int, calls: int = 10) -> float:
    """Event-timed lvq_encode_page calls (each with every request due: the contexts advanced
    by a page first, outside the timed interval).  The cache counters are restored after."""
    ctx0, coded0 = cache.ctx_len.clone(), cache.coded_len.clone()
    # make every request due once: its recent window full
    due = cache.coded_len[:B] + cfg.n_sink + cache.lay.ring_tokens
    cache.ctx_len[:B].copy_(due)
    ts = []
    with torch.cuda.stream(stream):
        for i in range(calls + 2):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            lvq.lvq_encode_page(cfg, cache.lay, B, cache.ctx_len, cache.coded_len, cache.ring, cache.cb,
                                cache.cb_norm, cache.idx, cache.status, stream=stream)
            b.record(stream)
            cache.ctx_len[:B].add_(TOKENS_PER_STEP)
            torch.cuda.synchronize()
            if i >= 2:
                ts.append(a.elapsed_time(b) * 1e3)
    cache.ctx_len.copy_(ctx0)
    cache.coded_len.copy_(coded0)
    torch.cuda.synchronize()
    cache.check_status("page encode")
    return statistics.median(ts)


def profile_kmeans(lvq, synth, torch, device):
    """One Ouro-2.6B-shaped layer (32768 tokens): one encode, then the k-means update 3 times."""
    wc = synth.WORKLOADS[ENCODE_WORKLOAD]
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
    wc = synth.WORKLOADS[ENCODE_WORKLOAD]
    cfg4 = lvq.make_config(1, wc.n_kv_heads, wc.n_q_heads, wc.head_dim, wc.T, wc.Tc, wc.G, 0, 0, 1, wc.ctx,
                           max_splits=1, rope_base=wc.rope_base)
    c4 = lvq.CodedCache(cfg4, device)
    c4.cb_view()[0] = synth.codebooks(wc, 0, device=device)
    kv4 = synth.loop_kv(wc, 0, wc.ctx, stream="coded", device=device)
    for _ in range(3):
        lvq.lvq_encode_prefill(cfg4, c4.lay, 0, 0, kv4, 0, wc.ctx, 0, c4.cb, c4.idx, c4.status)
    torch.cuda.synchronize()
    c4.check_status("profile encode")


def one_layer_encode(lvq, synth, torch, device):
    """The prefill encoder and the k-means update on one Ouro-2.6B-shaped layer (33.5 M joint
    vectors): the secondary measurements of the headline line."""
    wc = synth.WORKLOADS[ENCODE_WORKLOAD]
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
    vectors = encode_vectors(wc, 1, wc.ctx)
    bytes_ = encode_bytes_per_call(wc, 1, wc.ctx, c4.lay.cb_bytes)
    # useful distance GEMM work: 256 entries x G dims x 2 flops per vector
    tflops = vectors * 256 * wc.G * 2 / (enc_ms / 1e3) / 1e12
    tpk, tpk_kind = bf16_peak()
    hbm, hbm_kind = peaks()
    enc = {"vectors_per_s": vectors / (enc_ms / 1e3), "ms_per_layer": enc_ms,
           "hbm_gbps": bytes_ / (enc_ms / 1e3) / 1e9, "frac_of_hbm": bytes_ / (enc_ms / 1e3) / 1e9 / hbm,
           "distance_gemm_tflops": tflops, "frac_of_bf16_peak": tflops / tpk, "bf16_peak": tpk,
           "peak_kind": tpk_kind, "workload": f"{ENCODE_WORKLOAD} (one of 48 layers)",
           "kernel": "encode_tc (tcgen05 distance GEMM + argmin)"}
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
                     "update_frac_of_hbm": upd_bytes / (upd_ms / 1e3) / 1e9 / hbm,
                     "kernel": "kmeans_update (fp64 shared-memory sums per entry)"}
    del kv4, c4
    torch.cuda.empty_cache()
    return enc


def _setup(args):
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
    if getattr(args, "max_ctas", 0):
        lvq.lvq_decode_max_ctas(args.max_ctas)
    return torch, dist, lvq, synth, world, rank, local, device


def decode_arm(args, torch, dist, lvq, synth, world, rank, local, device):
    w = synth.WORKLOADS[args.workload]
    replays = 2 * args.steps + args.warmup + 3          # every graph replay adds 8 tokens
    n_sm = torch.cuda.get_device_properties(device).multi_processor_count
    ns = args.splits or choose_splits(w, n_sm)
    cfg, cache = build_cache(w, lvq, synth, torch, TOKENS_PER_STEP * (replays + 4), device,
                             replica_plan(rank, world, w.batch)["seed"], max_splits=max(128, ns), pool=args.pool)
    lay = cache.lay
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
        return None
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
    ctx0, coded0 = cache.ctx_len.clone(), cache.coded_len.clone()      # the workload's context
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
    # the timed tokens start at the workload's context
    cache.ctx_len.copy_(ctx0)
    cache.coded_len.copy_(coded0)
    torch.cuda.synchronize()

    def timed_steps():
        for _ in range(args.steps):
            graph.replay()

    with Clocks(local) as clk:
        with torch.cuda.stream(stream):
            ms = time_region(timed_steps, EventClock(stream), device, sync=torch.cuda.synchronize)
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
    page_us = page_encode_us(lvq, torch, cfg, cache, stream, B)

    # ---- e2e: queries in from pinned host memory, outputs back, every step
    cache.ctx_len.copy_(ctx0)
    cache.coded_len.copy_(coded0)
    q_host = torch.empty(q_all.shape, dtype=q_all.dtype).pin_memory()
    q_host.copy_(q_all.cpu())
    out_host = torch.empty(out_all.shape, dtype=out_all.dtype).pin_memory()
    graph.replay()
    torch.cuda.synchronize()

    def e2e_steps():
        for _ in range(args.steps):
            q_all.copy_(q_host, non_blocking=True)
            graph.replay()
            out_host.copy_(out_all, non_blocking=True)

    with torch.cuda.stream(stream):
        e2e_ms = time_region(e2e_steps, EventClock(stream), device, sync=torch.cuda.synchronize)
    e2e_value = tokens / (e2e_ms / 1e3)
    cache.check_status("e2e")
    del cache, graph, g2
    torch.cuda.empty_cache()

    enc = None
    if not args.no_encode and args.workload == WORKLOAD:
        enc = one_layer_encode(lvq, synth, torch, device)

    if rank != 0:
        return None
    cb = cpu_baseline(args.workload, args.cpu_seconds, args.oracle_procs)
    clocks = clk.summary()
    # the launch's kernel: with a CTA cap below the work items, CTAs walk runs of items
    runs = bool(args.max_ctas) and B * Hq * ns > min(args.max_ctas, n_sm)
    headline_kernel = args.workload == WORKLOAD and not runs      # the kernel the ncu counters describe
    extra_cfg = {}
    if args.pool:
        extra_cfg["codes"] = f"page pool, {POOL_BITE}-page bites"
    if args.max_ctas:
        extra_cfg["max_ctas"] = args.max_ctas
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": dict(decode_config(w, world, ns), **extra_cfg),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak,
                     "traffic": decode_traffic() if headline_kernel else None,
                     "kernel": f"decode_runs_kernel<{d},{lay.c}>" if runs else f"decode_kernel<{d},{lay.c}>",
                     "peak_kind": peak_kind, "bytes_per_launch": bpl, "launch_ms": per_call_ms},
        "issue": (decode_issue(per_call_ms, clocks.get("sm_mhz"), n_sm, sum(coded_now) * w.n_q_heads)
                  if headline_kernel else None),
        "code_stream_GBps": code_stream,
        "page_encode_us": page_us,
        "cpu_baseline": cb,
        "e2e": {"value": e2e_value, "unit": "tokens/s",
                "h2d_bytes_per_step": q_all.numel() * q_all.element_size() * world,
                "d2h_bytes_per_step": out_all.numel() * out_all.element_size() * world},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "encode": enc,
    }


def encode_arm(args, torch, dist, lvq, synth, world, rank, local, device):
    """The 48-layer prefill encode of one request as one call (layer = -1)."""
    wc = synth.WORKLOADS[ENCODE_WORKLOAD]
    L, N = wc.n_layers, wc.ctx
    cfg = lvq.make_config(L, wc.n_kv_heads, wc.n_q_heads, wc.head_dim, wc.T, wc.Tc, wc.G, 0, 0, 1, N,
                          max_splits=1, rope_base=wc.rope_base)
    cache = lvq.CodedCache(cfg, device)
    lay = cache.lay
    kv = torch.empty(L, 2, wc.T, N, wc.n_kv_heads, wc.head_dim, dtype=torch.bfloat16, device=device)
    cbv = cache.cb_view()
    seed = replica_plan(rank, world, 1)["seed"]
    for layer in range(L):
        sc = synth.channel_scales(wc, layer, device=device)
        cbv[layer] = synth.codebooks(wc, layer, device=device, scales=sc)
        kv[layer] = synth.loop_kv(wc, layer, N, stream="coded", request=seed, device=device, scales=sc)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device)

    def call():
        lvq.lvq_encode_prefill(cfg, lay, -1, 0, kv, 0, N, 0, cache.cb, cache.idx, cache.status, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            call()
    torch.cuda.synchronize()
    cache.check_status("encode warm-up")

    def timed_steps():
        for _ in range(args.steps):
            call()

    with Clocks(local) as clk:
        with torch.cuda.stream(stream):
            ms = time_region(timed_steps, EventClock(stream), device, sync=torch.cuda.synchronize)
    cache.check_status("encode timed")
    vectors = encode_vectors(wc, L, N)
    value = vectors * args.steps * world / (ms / 1e3)
    per_call_ms = ms / args.steps
    bytes_ = encode_bytes_per_call(wc, L, N, lay.cb_bytes)
    hbm_peak, peak_kind = peaks()
    achieved = bytes_ / (per_call_ms / 1e3) / 1e9
    tflops = vectors * 256 * wc.G * 2 / (per_call_ms / 1e3) / 1e12
    tpk, tpk_kind = bf16_peak()

    # ---- the decode-time page encode at this model's shape (48 layers): every codebook streamed
    # once per call for the 8 oldest recent tokens of a request
    w48 = synth.WORKLOADS[ENCODE_WORKLOAD]
    cfgp = lvq.make_config(L, w48.n_kv_heads, w48.n_q_heads, w48.head_dim, w48.T, w48.Tc, w48.G, w48.n_sink,
                           w48.n_recent, 1, 4096, max_splits=8, rope_base=w48.rope_base)
    cp = lvq.CodedCache(cfgp, device)
    cp.cb.copy_(cache.cb)
    rvp = cp.ring_view()
    for layer in range(L):
        rk = synth.loop_kv(w48, layer, cp.lay.ring_tokens, stream="recent", device=device)
        rvp[layer, :, :, 0] = rk.permute(0, 1, 3, 2, 4)
    lvq.lvq_pack_codebooks(cfgp, cp.lay, cp.cb, cp.cbp, cp.cb_norm)
    cp.ctx_len.fill_(0)
    cp.coded_len.fill_(0)
    torch.cuda.synchronize()
    page_us = page_encode_us(lvq, torch, cfgp, cp, stream, 1)
    del cp

    # ---- e2e: every step copies every layer's K/V from pinned host memory (one layer's buffer,
    # reused) and the codes back
    kv_host = torch.empty(kv.shape[1:], dtype=kv.dtype).pin_memory()
    kv_host.copy_(kv[0].cpu())
    idx_host = torch.empty(cache.idx.shape, dtype=cache.idx.dtype).pin_memory()

    def e2e_steps():
        for _ in range(args.steps):
            for layer in range(L):
                kv[layer].copy_(kv_host, non_blocking=True)
            call()
            idx_host.copy_(cache.idx, non_blocking=True)

    with torch.cuda.stream(stream):
        e2e_ms = time_region(e2e_steps, EventClock(stream), device, sync=torch.cuda.synchronize)
    cache.check_status("encode e2e")
    e2e_value = vectors * args.steps * world / (e2e_ms / 1e3)

    if rank != 0:
        return None
    cb = cpu_baseline(ENCODE_WORKLOAD, args.cpu_seconds, args.oracle_procs)
    return {
        "metric": METRIC, "value": value, "unit": "vectors/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": per_call_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": encode_config(wc, world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": None, "kernel": f"encode_tc_kernel<{wc.G},{wc.c}>",
                     "peak_kind": peak_kind, "bytes_per_launch": bytes_, "launch_ms": per_call_ms,
                     "tensor": {"distance_gemm_tflops": tflops, "frac_of_bf16_peak": tflops / tpk,
                                "peak_kind": tpk_kind}},
        "page_encode_us": page_us,
        "cpu_baseline": cb,
        "e2e": {"value": e2e_value, "unit": "vectors/s", "h2d_bytes_per_step": kv.numel() * kv.element_size() * world,
                "d2h_bytes_per_step": cache.idx.numel() * world},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
    }


def gpu_arm(args):
    torch, dist, lvq, synth, world, rank, local, device = _setup(args)
    if args.profile == "encode":
        profile_encode(lvq, synth, torch, device)
        return
    if args.profile == "kmeans":
        profile_kmeans(lvq, synth, torch, device)
        return
    if args.workload == ENCODE_WORKLOAD:
        line = encode_arm(args, torch, dist, lvq, synth, world, rank, local, device)
    else:
        line = decode_arm(args, torch, dist, lvq, synth, world, rank, local, device)
    if line is not None:
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
