#!/usr/bin/env python
"""Benchmark: decode attention + append-quantize over a quantized KV cache on B200.

Headline workload (default, --workload 5): batched serving under KVarN-style
normalisation -- 64 sequences with ragged contexts of 1k..32k tokens, 32 layers,
32 query / 8 kv heads, head_dim 128, variance normalisation + Hadamard-128 + q4_0
for K and V, a 256-token F16 tail per sequence.  Every step appends a 2048-token
chunk to 8 of the sequences (taken in rotation) and runs one decode query per
sequence, layer by layer.  It is the largest of the five workloads that fits one
GPU (about 41 GB of packed cache).  Synthetic seeded data.

One step = for each layer: kvq_append_quantize + kvq_decode_attention.
  value : device time of one step per sequence (us/token), inputs resident in
          HBM (a CUDA graph of the step's library launches, replayed; the packed
          cache read per step is far larger than L2, so no flush is needed).
  e2e   : the same step through the public API, with the step's new K/V rows and
          queries copied from pinned host memory and the outputs copied back,
          inside the timed region (each layer's copies on their own streams,
          overlapping the other layers' compute).
  roofline : the decode launch (the dominant kernel) against the measured HBM
          copy rate; append_roofline: the chunk append likewise.
  per_workload : the other four workloads (tiny; Llama-8B-shaped 32k; VBR mix with
          a 1024-token tail; per-head rank/bits 128k), each with its step time,
          decode roofline and chunk-append roofline, measured the same way (the
          tiny workload's cache fits in L2, so L2 is flushed before each timed
          call there).
Prints one JSON line (rank 0).  `--impl reference` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_kv_cache_15_b200 import workloads as W  # noqa: E402

W_NAMES = {0: "f16", 1: "q8_0", 2: "q6_0", 3: "q4_0", 4: "q3_0", 5: "q2_0", 6: "q8_1", 7: "q6_1", 8: "q4_1",
           9: "q3_1", 10: "q2_1", 11: "rank", 12: "q5_0", 13: "q5_1"}
METRIC = "decode-attn µs/token & HBM GB/s (% of 8 TB/s); append-quantize tokens/s, 1 B200"
NOMINAL_HBM_GBS = 8000.0
L2_BYTES = 126 * 1024 * 1024
HEADLINE = 5


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (profiling runs only)")
    ap.add_argument("--workload", type=int, default=HEADLINE, choices=[1, 2, 3, 4, 5],
                    help="headline workload (default 5: batch 64, KVarN q4_0, 256-token tail)")
    ap.add_argument("--only", action="store_true", help="measure the headline workload only (no per_workload)")
    return ap.parse_args()


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if args.impl == "kvq" and torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(value: float, world: int, device) -> float:
    """The largest value over all ranks (every rank gets it); identity at world size 1."""
    if world <= 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def measured_peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        return None


# ----------------------------------------------------------------------------- accounting
def row_bytes(codec, r=128, b=0):
    """Bytes of one packed row (codes + scales) in the documented format of
    include/kvq.h: 16 b code bytes and 8 (_0) or 16 (_1) scale bytes per 128 values,
    256 for F16, r b / 8 + 2 ceil(r / 32) for the rank codec."""
    if codec == W.F16:
        return 256
    if codec == W.RANK:
        return r * b // 8 + 2 * ((r + 31) // 32)
    bits = {W.Q8_0: 8, W.Q8_1: 8, W.Q6_0: 6, W.Q6_1: 6, W.Q5_0: 5, W.Q5_1: 5, W.Q4_0: 4, W.Q4_1: 4,
            W.Q3_0: 3, W.Q3_1: 3, W.Q2_0: 2, W.Q2_1: 2}[codec]
    asym = codec in (W.Q8_1, W.Q6_1, W.Q5_1, W.Q4_1, W.Q3_1, W.Q2_1)
    return 16 * bits + (16 if asym else 8)


def token_head_bytes(w, layer):
    """Packed bytes of one cached token of one layer, over all kv heads, K and V."""
    tot = 0
    for h in range(w.n_kv_heads):
        r = w.rank[layer][h] if w.rank else 128
        kb = w.k_bits[layer][h] if w.k_bits else 0
        vb = w.v_bits[layer][h] if w.v_bits else 0
        tot += row_bytes(w.k_codec[layer][h], r, kb) + row_bytes(w.v_codec[layer][h], r, vb)
    return tot


def decode_bytes(w, layer, lengths):
    """Algorithmic bytes of one decode launch: every cached token's packed rows (raw
    rows for the tail), the fp16 queries and the fp32 outputs."""
    tot = 0
    bpt = token_head_bytes(w, layer)
    for n in lengths:
        nq = max(0, n - w.tail)
        tot += nq * bpt + (n - nq) * w.n_kv_heads * 2 * 128 * 2
    return tot + len(lengths) * w.n_q_heads * 128 * (2 + 4)


def decode_macs(w, layer, lengths):
    """Multiply-adds of one decode launch: every visible (token, kv head) costs a score
    and a value product of G query heads over the head's stored width (128, or the
    rank r of a projected head)."""
    width = sum((w.rank[layer][h] if w.rank is not None else 128) for h in range(w.n_kv_heads))
    return sum(lengths) * 2 * w.G * width


def append_bytes(w, layer, len_old, n):
    """Algorithmic bytes of appending n tokens to a sequence of len_old tokens in one
    layer: raw input rows read; rows leaving the tail read from the ring; quantized
    rows written; rows entering the tail written (K and V, every kv head)."""
    raw = w.n_kv_heads * 2 * 128 * 2
    T = w.tail
    if T == 0:
        return n * raw + n * token_head_bytes(w, layer)
    e0, e1 = max(0, len_old - T), min(len_old, len_old + n - T)
    nE = max(0, e1 - e0)
    nP = max(0, len_old + n - T - len_old) if n > T else 0
    nF = min(n, T)
    return n * raw + nE * raw + (nE + nP) * token_head_bytes(w, layer) + nF * raw


def step_cache_bytes(w):
    return sum(decode_bytes(w, l, w.ctx) for l in range(w.n_layers))


def l2_note(w):
    """How the timed steps avoid L2 hits, from the workload alone (same text in both arms)."""
    b = step_cache_bytes(w)
    if b < 4 * L2_BYTES:
        return (f"L2 flushed before every timed call (a 512 MB write): the step reads only {b / 1e6:.2f} MB "
                f"of packed cache")
    return f"no flush: the step reads {b / 1e9:.2f} GB of packed cache, far more than L2 (126 MB)"


DECODE_SOURCES = ("decode.cu", "decode_fast.cuh", "pair_tables.h", "kvq_internal.h", "ptx.cuh", "quant.cuh")


def kernel_source_sha256():
    """sha256 over the decode kernel's source files (in DECODE_SOURCES order)."""
    h = hashlib.sha256()
    for name in DECODE_SOURCES:
        h.update(open(os.path.join(ROOT, "quantized_kv_cache_15_b200", "csrc", name), "rb").read())
    return h.hexdigest()


def traffic_from_profile(workload):
    """DRAM bytes per decode launch recorded under profiles/ for this workload (a
    block "profiled_workload / traffic_bytes_per_launch / kernel_source_sha256"),
    only while the decode kernel's source still matches the one profiled; else None."""
    sha = None
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        text = open(path).read()
        for m in re.finditer(r"profiled_workload:\s*(\S+)\s*\ntraffic_bytes_per_launch:\s*([0-9.eE+]+)\s*\n"
                             r"kernel_source_sha256:\s*([0-9a-f]{64})", text):
            if m.group(1) != workload:
                continue
            sha = sha or kernel_source_sha256()
            if m.group(3) == sha:
                return float(m.group(2))
    return None


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            self.path = f"/tmp/kvq_clocks_{os.getpid()}.csv"
            q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        sm = [r[0] for r in rows]
        mx = max(r[1] for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[2]) if v.lower() == "active"})
        loaded = [s for s in sm if s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- CPU oracle baseline
def _oracle_pair_args(w, h):
    """Oracle inputs for decode pair h of sequence 0: its own packed rows of one
    (layer, kv head) over the full context plus the raw tail rows."""
    import oracle

    def bits16(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    layer, head = (h * 7) % w.n_layers, h % w.n_kv_heads
    n = w.ctx[0]
    nq = max(0, n - w.tail)
    K = bits16(w.rows("K", layer, 0, 0, n)[:, head, :])
    V = bits16(w.rows("V", layer, 0, 0, n)[:, head, :])
    q = bits16(w.queries(layer, 0, 0)[head * w.G:(head + 1) * w.G])
    kc, vc = w.k_codec[layer][head], w.v_codec[layer][head]
    kw = {}
    r, kb, vb = 128, 0, 0
    if w.rot == W.ROT_PROJECTION:
        r, kb, vb = w.rank[layer][head], w.k_bits[layer][head], w.v_bits[layer][head]
        kw["M"] = oracle.fuse_projection(w.proj_basis(layer, head))
    if w.rot == W.ROT_VARNORM_HADAMARD:
        kw["inv_s_k"] = oracle.varnorm_inv_rms(bits16(w.calib_rows("K", layer, 512)[:, head, :]))
        kw["inv_s_v"] = oracle.varnorm_inv_rms(bits16(w.calib_rows("V", layer, 512)[:, head, :]))
    ck = sk = cv = sv = None
    if nq:
        ck, sk = oracle.encode_rows(kc, w.rot, K[:nq], inv_s=kw.get("inv_s_k"), M=kw.get("M"), r=r, b=kb)
        cv, sv = oracle.encode_rows(vc, w.rot, V[:nq], inv_s=kw.get("inv_s_v"), M=kw.get("M"), r=r, b=vb)
    return (ck, sk, cv, sv, K[nq:], V[nq:], q, kc, vc, w.rot), dict(r=r, kb=kb, vb=vb, **kw)


def cpu_oracle_decode_us_per_token(w, seconds, log, max_pairs=None, threads=None):
    """Time the CPU oracle on a bounded sample of the same step: decode attention of
    one (layer, kv head) of sequence 0 over its full context, from the oracle's own
    packed rows (plus the raw tail rows).  `threads` pairs run at once, one per
    host thread (the oracle's C code runs outside the interpreter lock), in rounds
    until `seconds` have passed (at least one round; at most max_pairs pairs); the
    wall time per cached (token, kv head) is scaled to the step (every layer, kv
    head and sequence) and divided by the sequences decoded."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor

    threads = max(1, threads or 1)
    n_pairs = w.n_layers * w.n_kv_heads
    if max_pairs:
        n_pairs = min(n_pairs, max_pairs)
    threads = min(threads, n_pairs)
    done, wall = 0, 0.0
    t_start = time.time()
    with ThreadPoolExecutor(max_workers=threads) as pool:
        while done < n_pairs:
            batch = list(pool.map(lambda h: _oracle_pair_args(w, h), range(done, min(n_pairs, done + threads))))
            t0 = time.perf_counter()
            list(pool.map(lambda a: oracle.decode_packed(*a[0], **a[1]), batch))
            wall += time.perf_counter() - t0
            done += len(batch)
            if time.time() - t_start > seconds:
                break
    sec_per_token_head = wall / (done * w.ctx[0])
    step_s = sec_per_token_head * sum(w.ctx) * w.n_layers * w.n_kv_heads
    us_per_token = step_s * 1e6 / w.batch
    sample = (f"oracle decode of {done} (layer, kv head) pairs of sequence 0 ({w.ctx[0]} tokens, G={w.G}) from the "
              f"oracle's own packed rows, {threads} at a time on {threads} host threads; "
              f"{sec_per_token_head * 1e6:.4f} us wall per cached (token, kv head), scaled to {sum(w.ctx)} tokens x "
              f"{w.n_layers * w.n_kv_heads} (layer, kv head) per step / {w.batch} seq")
    log(f"cpu oracle ({threads} threads): {us_per_token:.3e} us/token")
    return {"value": us_per_token, "unit": "us/token", "cores": threads, "kind": "oracle", "sample": sample}


# ----------------------------------------------------------------------------- reference arm
def workload_config(w, layers, world):
    """The `config` object of both arms' JSON lines for workload w."""
    B = w.batch
    n_app = w.append_tokens if w.append_tokens else 1
    n_app_seqs = w.append_seqs if w.append_seqs else B
    codecs = sorted({W_NAMES[c] for row in w.k_codec for c in row}) + sorted({W_NAMES[c] for row in w.v_codec for c in row})
    return {"workload": w.name, "layers": layers, "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads, "head_dim": 128,
            "batch": B, "context": w.ctx[0] if B == 1 else f"{min(w.ctx)}..{max(w.ctx)} (mean {sum(w.ctx) / B:.0f})",
            "tail": w.tail, "codecs_k_v": codecs,
            "rotation": ["none", "hadamard-128", "varnorm+hadamard-128", "per-head projection"][w.rot],
            "step": f"per layer: append {n_app} token(s) x {n_app_seqs} seq(s) + decode attention for {B} seq(s)",
            "parallelism": f"replicas x{world}", "l2": l2_note(w)}


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    w = W.make_workload(args.workload, "full")
    log = lambda m: print(m, file=sys.stderr, flush=True)  # noqa: E731
    vals = []
    threads = min(os.cpu_count() or 1, 8)
    for i in range(args.warmup + args.steps):
        # one bounded sample per step: `threads` pairs decoded at once
        cb = cpu_oracle_decode_us_per_token(w, 0.0, log, max_pairs=threads, threads=threads)
        if i >= args.warmup:
            vals.append(cb["value"])
    v = statistics.mean(vals)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "us/token", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": v * w.batch / 1000.0,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, w.n_layers, world),
            "cpu_baseline": {"value": v, "unit": "us/token", "cores": threads, "kind": "oracle",
                             "sample": f"each step: oracle decode of {threads} (layer, kv head) pairs of sequence 0 "
                                       f"over its full context on {threads} host threads at once, scaled to every "
                                       f"(layer, kv head, sequence) of the step"},
            "e2e": {"value": v, "unit": "us/token", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- kvq arm
def make_plan(kvq, w, extra, dev):
    """Plan for workload w with `extra` tokens of growth per sequence."""
    kw = {}
    if w.rot == W.ROT_VARNORM_HADAMARD:
        inv = np.zeros((w.n_layers, w.n_kv_heads, 2, 128), np.float32)
        for l in range(w.n_layers):
            for kv, kind in enumerate("KV"):
                x = w.calib_rows(kind, l, 512, device=dev).reshape(512, w.n_kv_heads * 128).contiguous()
                o = torch.empty(w.n_kv_heads * 128, dtype=torch.float32, device=dev)
                kvq.calibrate_varnorm(x, w.n_kv_heads * 128, w.n_kv_heads * 128, o)
                inv[l, :, kv, :] = o.cpu().numpy().reshape(w.n_kv_heads, 128)
        kw["inv_rms"] = inv
    if w.rot == W.ROT_PROJECTION:
        kw.update(rank=np.array(w.rank), k_bits=np.array(w.k_bits), v_bits=np.array(w.v_bits),
                  proj_basis=[w.proj_basis(l, h) for l in range(w.n_layers) for h in range(w.n_kv_heads)])
    pages = sum((c + extra + 63) // 64 for c in w.ctx) + 2 * w.batch
    return kvq.Plan(w.n_layers, w.n_q_heads, w.n_kv_heads, max_seqs=w.batch, max_tokens_per_seq=max(w.ctx) + extra,
                    k_codec=w.k_codec, v_codec=w.v_codec, rot=w.rot, tail_tokens=w.tail, max_pages=pages, **kw)


class L2Flush:
    """Writes a buffer larger than L2 on `stream` (for workloads whose cache fits in L2)."""

    def __init__(self, dev):
        self.buf = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
        self.v = 0

    def __call__(self):
        self.v = (self.v + 1) & 0xFF
        self.buf.fill_(self.v)


def timed_replays(graph, stream, reps, flush=None):
    """Mean ms of one replay of `graph`, timed with events on `stream` (the graph's
    launches run there).  With `flush`, L2 is flushed before each replay and only the
    replay is timed."""
    with torch.cuda.stream(stream):
        if flush is None:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                graph.replay()
            b.record(stream)
            stream.synchronize()
            return a.elapsed_time(b) / reps
        tot = 0.0
        for _ in range(reps):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            graph.replay()
            b.record(stream)
            stream.synchronize()
            tot += a.elapsed_time(b)
        return tot / reps


def measure_workload(kvq, w, dev, K, Wm, world, log, headline):
    """Fill w's cache and measure its step, decode launch and chunk append; the
    headline workload also gets the e2e step, the clocks, a prefill call and a VBR
    regrade.  Frees its device memory before returning."""
    L, Hq, B = w.n_layers, w.n_q_heads, w.batch
    n_app = w.append_tokens if w.append_tokens else 1
    n_app_seqs = w.append_seqs if w.append_seqs else B
    n_groups = max(1, B // n_app_seqs)
    host_steps = Wm + 1 + (K if headline else 0)     # warm-up, captured and e2e steps advance host lengths
    growth = ((host_steps + n_groups - 1) // n_groups) * n_app + 2 * 2048 + 64
    plan = make_plan(kvq, w, growth, dev)
    plan.allocate_cache(dev)
    t0 = time.time()
    chunk = 8192
    for l in range(L):
        for s in range(B):
            for a in range(0, w.ctx[s], chunk):
                b = min(w.ctx[s], a + chunk)
                plan.append(l, [s], [b - a], w.rows("K", l, s, a, b, dev), w.rows("V", l, s, a, b, dev))
    torch.cuda.synchronize()
    plan.check_device_error()
    log(f"[{w.name}] filled {L} layers x {sum(w.ctx)} tokens in {time.time() - t0:.1f} s; "
        f"cache {plan.cache_bytes() / 1e9:.2f} GB")
    flush = L2Flush(dev) if step_cache_bytes(w) < 4 * L2_BYTES else None

    stream = torch.cuda.Stream(dev)
    ws = plan.new_workspace(B, dev)
    seqs = list(range(B))
    knew = torch.stack([torch.cat([w.rows("K", l, s, w.ctx[s], w.ctx[s] + n_app, dev) for s in range(n_app_seqs)])
                        for l in range(L)])
    vnew = torch.stack([torch.cat([w.rows("V", l, s, w.ctx[s], w.ctx[s] + n_app, dev) for s in range(n_app_seqs)])
                        for l in range(L)])
    qall = torch.stack([torch.stack([w.queries(l, s, 0, dev) for s in seqs]) for l in range(L)])  # [L][B][Hq][128]
    out = torch.empty((L, B, Hq, 128), dtype=torch.float32, device=dev)
    step_no = [0]

    def app_group():
        g0 = (step_no[0] % n_groups) * n_app_seqs
        return list(range(g0, g0 + n_app_seqs))

    def step(kd=knew, vd=vnew, qd=qall):
        grp = app_group()
        for l in range(L):
            plan.append(l, grp, [n_app] * len(grp), kd[l], vd[l], stream)
            plan.decode(l, seqs, qd[l], out[l], ws, stream)
        step_no[0] += 1

    with torch.cuda.stream(stream):
        for _ in range(Wm):
            torch.cuda.nvtx.range_push("kvq_step")      # lets a profiler pick the step's launches
            step()
            torch.cuda.nvtx.range_pop()
    stream.synchronize()
    plan.check_device_error(stream)

    # capture one step (fixed positions; every replay does the full step's work)
    lengths = [[plan.seq_length(s, l) for s in seqs] for l in range(L)]
    grp = app_group()
    old_len = [[lengths[l][s] for s in seqs] for l in range(L)]
    for l in range(L):
        for s in grp:
            lengths[l][s] += n_app
    n0 = kvq.launch_count()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step()
    launches_per_step = kvq.launch_count() - n0
    with torch.cuda.stream(stream):
        for _ in range(Wm):
            g.replay()
    stream.synchronize()

    # ---- timed region: device time of K steps
    barrier = (lambda: torch.distributed.barrier()) if world > 1 else (lambda: None)
    clocks = None
    if headline:
        clocks = ClockSampler(dev.index or 0)
        clocks.start()
        time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    step_ms = timed_replays(g, stream, K, flush)
    torch.cuda.synchronize()
    barrier()
    step_ms = max_over_ranks(step_ms, world, dev)
    clk = clocks.stop() if clocks else None
    plan.check_device_error(stream)

    # ---- per-launch decode durations: a CUDA graph of the step's L decode calls
    # (back to back; every layer's cache read once), replayed between two events on
    # the launching stream; duration = elapsed / L
    gd = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gd, stream=stream):
        for l in range(L):
            plan.decode(l, seqs, qall[l], out[l], ws, stream)
    with torch.cuda.stream(stream):
        for _ in range(2):
            gd.replay()
    stream.synchronize()
    dec_ms = max_over_ranks(timed_replays(gd, stream, max(3, K // 4), flush) / L, world, dev)
    plan.check_device_error(stream)
    dec_bytes_all = [decode_bytes(w, l, lengths[l]) for l in range(L)]
    dec_bytes = statistics.mean(dec_bytes_all)
    dec_macs = statistics.mean(decode_macs(w, l, lengths[l]) for l in range(L))

    res = {"workload": w.name, "ms_per_step": step_ms, "us_per_token": step_ms * 1e3 / B,
           "gpu_launches_per_step": launches_per_step, "l2": l2_note(w)}

    # ---- e2e through the public API: host buffers in, host buffers out
    if headline:
        kh, vh, qh = knew.cpu().pin_memory(), vnew.cpu().pin_memory(), qall.cpu().pin_memory()
        oh = torch.empty(out.shape, dtype=torch.float32).pin_memory()
        kd, vd, qd = torch.empty_like(knew), torch.empty_like(vnew), torch.empty_like(qall)
        h2d = (kd.numel() + vd.numel() + qd.numel()) * 2
        d2h = oh.numel() * 4
        # Layer l's rows and queries cross PCIe on their own stream while layer
        # l - 1 computes, and its outputs go back on a third one as soon as its
        # decode is done: the plumbing a serving loop around these calls uses.
        h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(L)]
        ev_out = [torch.cuda.Event() for _ in range(L)]
        e2e_ms = []
        for _ in range(K):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier()
            a.record(stream)
            h2d_s.wait_stream(stream)
            d2h_s.wait_stream(stream)
            with torch.cuda.stream(h2d_s):
                for l in range(L):
                    kd[l].copy_(kh[l], non_blocking=True)
                    vd[l].copy_(vh[l], non_blocking=True)
                    qd[l].copy_(qh[l], non_blocking=True)
                    ev_in[l].record(h2d_s)
            grp = app_group()
            with torch.cuda.stream(stream):
                for l in range(L):
                    stream.wait_event(ev_in[l])
                    plan.append(l, grp, [n_app] * len(grp), kd[l], vd[l], stream)
                    plan.decode(l, seqs, qd[l], out[l], ws, stream)
                    ev_out[l].record(stream)
                    d2h_s.wait_event(ev_out[l])
                    with torch.cuda.stream(d2h_s):
                        oh[l].copy_(out[l], non_blocking=True)
            step_no[0] += 1
            stream.wait_stream(h2d_s)
            stream.wait_stream(d2h_s)
            b.record(stream)
            stream.synchronize()
            e2e_ms.append(a.elapsed_time(b))
        e2e_step = max_over_ranks(statistics.mean(e2e_ms), world, dev)
        plan.check_device_error(stream)
        res["e2e"] = {"value": e2e_step * 1e3 / (B * world), "unit": "us/token", "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": d2h}
        del kd, vd, qd, kh, vh, qh, oh

    # ---- step accounting
    app_step_bytes = sum(append_bytes(w, l, old_len[l][s], n_app) for l in range(L) for s in grp)
    step_bytes = sum(dec_bytes_all) + app_step_bytes
    res["step_gb_s"] = step_bytes / (step_ms / 1e3) / 1e9

    # ---- append-quantize throughput: a 2048-token chunk into every layer of sequence 0
    ck = torch.stack([w.rows("K", l, 0, 0, 2048, dev) for l in range(L)])
    cv = torch.stack([w.rows("V", l, 0, 0, 2048, dev) for l in range(L)])
    with torch.cuda.stream(stream):
        for l in range(L):
            plan.append(l, [0], [2048], ck[l], cv[l], stream)   # warm: allocates the chunk's pages
    stream.synchronize()
    len0 = [plan.seq_length(0, l) for l in range(L)]
    ga = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ga, stream=stream):
        for l in range(L):
            plan.append(l, [0], [2048], ck[l], cv[l], stream)
    with torch.cuda.stream(stream):
        for _ in range(3):
            ga.replay()
    stream.synchronize()
    app_ms = timed_replays(ga, stream, 10)
    plan.check_device_error(stream)
    app_b = sum(append_bytes(w, l, len0[l], 2048) for l in range(L))
    res["append_tokens_per_s"] = 2048 / (app_ms / 1e3)
    res["append_roofline"] = {"bound": "hbm", "kernel": "kvq_append_quantize (2048 tokens, one layer)",
                              "bytes_per_launch": app_b / L, "launch_ms": app_ms / L,
                              "achieved": app_b / (app_ms / 1e3) / 1e9, "unit": "GB/s",
                              "note": "raw rows read (input and ring) + packed rows and ring rows written"}
    res["decode"] = {"bytes_per_launch": dec_bytes, "macs_per_launch": dec_macs, "launch_ms": dec_ms,
                     "achieved": dec_bytes / (dec_ms / 1e3) / 1e9, "kernel": f"decode_kernel<{w.G}>",
                     "traffic": traffic_from_profile(w.name)}
    del ck, cv, ga

    if headline:
        res["clocks"] = clk
        # ---- chunked-prefill attention: the newest (up to) 2048 tokens of the longest
        # sequence in layer 0 attend causally to the cache (one kvq_prefill_attention call)
        ps = max(seqs, key=lambda s: plan.seq_length(s, 0))
        p_len = plan.seq_length(ps, 0)
        n_pq = min(2048, p_len)
        pq = torch.stack([w.queries(0, ps, i, dev) for i in range(n_pq)]).contiguous()
        pout = torch.empty((n_pq, Hq, 128), dtype=torch.float32, device=dev)
        pws = plan.new_workspace(min(n_pq, 256))
        pa, pb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            plan.prefill(0, ps, pq, pout, pws, stream)                      # warm-up
            pa.record(stream)
            for _ in range(2):
                plan.prefill(0, ps, pq, pout, pws, stream)
            pb.record(stream)
        stream.synchronize()
        plan.check_device_error(stream)
        p_ms = pa.elapsed_time(pb) / 2
        res["prefill"] = {"layer": 0, "seq": int(ps), "queries": n_pq, "context": int(p_len), "ms": p_ms,
                          "tokens_per_s": n_pq / (p_ms / 1e3),
                          "note": "causal: query i sees the first len - n_q + i + 1 tokens"}
        del pws, pq, pout
        # ---- VBR regrade of one layer (last, since it changes that layer's codecs)
        res["regrade"] = None
        if w.rot != W.ROT_PROJECTION:
            rl = L // 2
            Hkv = w.n_kv_heads
            nk, nv = [W.Q4_0] * Hkv, [W.Q2_0] * Hkv
            try:
                rbytes = plan.regrade_bytes(rl, nk, nv)
            except kvq.KVQError:
                rbytes = None
            if rbytes:
                rows = sum(max(0, plan.seq_length(s, rl) - w.tail) for s in seqs)
                old_b = rows * token_head_bytes(w, rl)
                scratch = torch.empty(rbytes, dtype=torch.uint8, device=dev)
                ra, rb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(stream):
                    # warm-up on the next layer (same move), so the timed call is not the
                    # kernel's first launch
                    if rl + 1 < L and plan.regrade_bytes(rl + 1, nk, nv) <= rbytes:
                        plan.regrade(rl + 1, nk, nv, scratch, stream)
                    ra.record(stream)
                    plan.regrade(rl, nk, nv, scratch, stream)
                    rb.record(stream)
                stream.synchronize()
                plan.check_device_error(stream)
                new_b = rows * Hkv * (row_bytes(W.Q4_0) + row_bytes(W.Q2_0))
                r_ms = ra.elapsed_time(rb)
                res["regrade"] = {"layer": rl, "ms": r_ms, "rows": rows * Hkv, "to": ["q4_0", "q2_0"],
                                  "gb_s": (old_b + new_b) / (r_ms / 1e3) / 1e9,
                                  "note": "bytes = old rows read + new rows written"}
                del scratch
    del g, gd
    del plan, ws, knew, vnew, qall, out
    if flush is not None:
        del flush
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


# The decode loops' multiply-adds run as dp2a (two per lane per instruction) on the
# fmaheavy pipe: 148 SMs x 4 schedulers x 16 lanes x 2 multiply-adds x 1.965 GHz.
DP2A_PEAK_TMACS = 148 * 4 * 16 * 2 * 1.965e9 / 1e12


def alu_roofline(d):
    """The decode launch against its multiply-add ceiling (the dp2a pipe); the HBM
    roofline above is the metric the workloads name, this one the kernel's own bound
    where its multiply-add floor lies above its HBM floor."""
    achieved = d["macs_per_launch"] / (d["launch_ms"] / 1e3) / 1e12
    return {"bound": "alu", "achieved": achieved, "peak": DP2A_PEAK_TMACS, "unit": "Tmul-add/s",
            "frac": achieved / DP2A_PEAK_TMACS, "kernel": d.get("kernel"), "macs_per_launch": d["macs_per_launch"],
            "peak_source": "unit counts x clock (dp2a on the fmaheavy pipe); tests/test_gpu_ubench.py measures "
                           "about 36 T/s"}


def roofline(d, peak, peaks):
    return {"bound": "hbm", "achieved": d["achieved"], "peak": peak, "unit": "GB/s", "frac": d["achieved"] / peak,
            "traffic": d.get("traffic"), "kernel": d.get("kernel"), "bytes_per_launch": d["bytes_per_launch"],
            "launch_ms": d["launch_ms"],
            "peak_source": "MEASURED_PEAKS.json hbm_gbs (copy, burst), of measured" if peaks
            else "fallback 6650 GB/s"}


def run_kvq(args, world, rank, local):
    from quantized_kv_cache_15_b200 import kvq
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    log = (lambda m: print(m, file=sys.stderr, flush=True)) if rank == 0 else (lambda m: None)

    def load(cfg):
        w = W.make_workload(cfg, "full")
        if args.layers:
            w.n_layers = args.layers
            for f in ("k_codec", "v_codec", "rank", "k_bits", "v_bits"):
                if getattr(w, f) is not None:
                    setattr(w, f, getattr(w, f)[:args.layers])
        return w

    peaks = measured_peaks()
    peak = float(peaks["hbm_gbs"]) if peaks else 6650.0
    w = load(args.workload)
    K, Wm = args.steps, args.warmup
    h = measure_workload(kvq, w, dev, K, Wm, world, log, headline=True)
    step_ms = h["ms_per_step"]
    line = {
        "metric": METRIC, "value": step_ms * 1e3 / (w.batch * world), "unit": "us/token", "n_gpus": world,
        "steps": K, "warmup": Wm, "ms_per_step": step_ms, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(w, w.n_layers, world),
        "us_per_step": step_ms * 1e3,
        "hbm_gbs": h["step_gb_s"], "hbm_frac_of_8tbs": h["step_gb_s"] / NOMINAL_HBM_GBS,
        "hbm_frac_of_measured": h["step_gb_s"] / peak,
        "append_tokens_per_s": h["append_tokens_per_s"],
        "append_roofline": dict(h["append_roofline"], peak=peak, frac=h["append_roofline"]["achieved"] / peak),
        "regrade": h.get("regrade"),
        "prefill": h.get("prefill"),
        "roofline": roofline(h["decode"], peak, peaks),
        "alu_roofline": alu_roofline(h["decode"]),
        "e2e": h["e2e"],
        "gpu_launches": h["gpu_launches_per_step"] * K,
        "clocks": h["clocks"],
    }
    if not args.only:
        per = {}
        for cfg in (1, 2, 3, 4, 5):
            if cfg == args.workload:
                continue
            wc = load(cfg)
            r = measure_workload(kvq, wc, dev, min(K, 10), max(3, min(Wm, 3)), world, log, headline=False)
            per[str(cfg)] = {"workload": r["workload"], "ms_per_step": r["ms_per_step"],
                             "us_per_token": r["us_per_token"], "step_gb_s": r["step_gb_s"], "l2": r["l2"],
                             "roofline": roofline(r["decode"], peak, peaks),
                             "append_tokens_per_s": r["append_tokens_per_s"],
                             "append_roofline": dict(r["append_roofline"], peak=peak,
                                                     frac=r["append_roofline"]["achieved"] / peak)}
        line["per_workload"] = per
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ncpu = os.cpu_count() or 1
        line["cpu_baseline"] = cpu_oracle_decode_us_per_token(w, args.cpu_seconds, log, max_pairs=ncpu, threads=ncpu)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            rc = run_reference(args, world, rank)
        else:
            rc = run_kvq(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
