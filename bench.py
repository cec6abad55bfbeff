#!/usr/bin/env python
"""Benchmark: decode attention + append-quantize over a quantized KV cache on B200.

Workload (default): Llama-3.1-8B-shaped decode over an asymmetric cache -- 32
layers, 32 query / 8 kv heads, head_dim 128, batch 1, context 32768, K q8_0 and
V q4_0 after the Hadamard rotation; every step appends one token per layer and
then runs decode attention for that layer.  Synthetic seeded data.

One step = for each layer: kvq_append_quantize (1 token) + kvq_decode_attention.
  value : device time of one step, inputs resident in HBM (a CUDA graph of the
          step's library launches, replayed; the packed cache read per step,
          1.74 GB, is far larger than L2, so no flush is needed).
  e2e   : the same step through the public API, with the step's new K/V rows and
          queries copied from pinned host memory and the outputs copied back,
          inside the timed region.
Prints one JSON line (rank 0).  `--impl reference` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
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

METRIC = "decode-attn µs/token & HBM GB/s (% of 8 TB/s); append-quantize tokens/s, 1 B200"
NOMINAL_HBM_GBS = 8000.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (profiling runs only)")
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


def measured_peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        return None


# ----------------------------------------------------------------------------- accounting
def bytes_per_token_head(plan, layer, n_kv):
    tot = 0
    for h in range(n_kv):
        for kv in (0, 1):
            cb, sb = plan.row_bytes(layer, h, kv)
            tot += cb + sb
    return tot


def decode_algorithmic_bytes(plan, w, layer, length):
    """Bytes one decode launch must move: the packed cache (codes + scales of every
    cached token of every kv head), the fp16 queries and the fp32 outputs."""
    cache = bytes_per_token_head(plan, layer, w.n_kv_heads) * length
    return cache + w.n_q_heads * 128 * 2 + w.n_q_heads * 128 * 4


def traffic_from_profile(kernel_file):
    """dram bytes per launch recorded in profiles/decode_attention_llama8b.md, if the
    kernel source still matches the one profiled (else None)."""
    path = os.path.join(ROOT, "profiles", "decode_attention_llama8b.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    h = re.search(r"kernel_source_sha256:\s*([0-9a-f]{64})", text)
    if not m or not h:
        return None
    src = open(kernel_file, "rb").read()
    if hashlib.sha256(src).hexdigest() != h.group(1):
        return None
    return float(m.group(1))


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
def cpu_oracle_decode_us_per_token(w, seconds, log):
    """Time the CPU oracle on a bounded sample of the same step: decode attention of
    one (layer, kv head) over the full context from the oracle's own packed rows, for
    as many kv heads as fit in `seconds`; extrapolated to the step (all layers and kv
    heads).  Single-threaded C."""
    import oracle
    T = w.ctx[0]
    times = []
    t_start = time.time()
    h = 0
    while True:
        layer, head = h // w.n_kv_heads, h % w.n_kv_heads
        K = w.rows("K", layer, 0, 0, T)[:, head, :].contiguous().view(torch.int16).numpy().view(np.uint16)
        V = w.rows("V", layer, 0, 0, T)[:, head, :].contiguous().view(torch.int16).numpy().view(np.uint16)
        q = w.queries(layer, 0, 0)[head * w.G:(head + 1) * w.G].contiguous().view(torch.int16).numpy().view(np.uint16)
        kc, vc = w.k_codec[layer][head], w.v_codec[layer][head]
        ck, sk = oracle.encode_rows(kc, w.rot, K)
        cv, sv = oracle.encode_rows(vc, w.rot, V)
        t0 = time.perf_counter()
        oracle.decode_packed(ck, sk, cv, sv, None, None, q, kc, vc, w.rot)
        times.append(time.perf_counter() - t0)
        h += 1
        if (time.time() - t_start > seconds and h >= 2) or h >= w.n_layers * w.n_kv_heads:
            break
    per_head = statistics.mean(times)
    us_per_token = per_head * w.n_layers * w.n_kv_heads * 1e6
    sample = (f"oracle decode of {len(times)} (layer, kv head) pairs x {T} tokens x G={w.G}, from the oracle's own "
              f"packed rows; mean {per_head:.3f} s per pair, scaled by {w.n_layers * w.n_kv_heads} pairs per step")
    log(f"cpu oracle: {per_head:.3f} s per (layer, head) -> {us_per_token:.3e} us/token")
    return {"value": us_per_token, "unit": "us/token", "cores": 1, "kind": "oracle", "sample": sample}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, world, rank):
    if rank != 0:
        return 0
    w = W.make_workload(2, "full")
    log = lambda m: print(m, file=sys.stderr, flush=True)  # noqa: E731
    vals = []
    for i in range(args.warmup + args.steps):
        cb = cpu_oracle_decode_us_per_token(w, 0.0, log)     # one bounded sample (2 kv heads) per step
        if i >= args.warmup:
            vals.append(cb["value"])
    v = statistics.mean(vals)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "us/token", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": v / 1000.0, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "layers": w.n_layers, "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads,
                       "context": w.ctx[0], "batch": 1},
            "cpu_baseline": {"value": v, "unit": "us/token", "cores": 1, "kind": "oracle",
                             "sample": "each step: oracle decode of 2 (layer, kv head) pairs over the full context, "
                                       "scaled to all 256 pairs of the step"},
            "e2e": {"value": v, "unit": "us/token", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- kvq arm
def run_kvq(args, world, rank, local):
    from quantized_kv_cache_15_b200 import kvq
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    log = (lambda m: print(m, file=sys.stderr, flush=True)) if rank == 0 else (lambda m: None)
    w = W.make_workload(2, "full")
    if args.layers:
        w.n_layers = args.layers
        w.k_codec, w.v_codec = w.k_codec[:args.layers], w.v_codec[:args.layers]
    L, Hq, Hkv, T = w.n_layers, w.n_q_heads, w.n_kv_heads, w.ctx[0]
    K, Wm = args.steps, args.warmup
    extra = 2 * Wm + K + 8 + 2048
    plan = kvq.Plan(L, Hq, Hkv, max_seqs=1, max_tokens_per_seq=T + extra, k_codec=w.k_codec, v_codec=w.v_codec,
                    rot=w.rot)
    plan.allocate_cache(dev)
    t0 = time.time()
    chunk = 4096
    for l in range(L):
        for a in range(0, T, chunk):
            b = min(T, a + chunk)
            plan.append(l, [0], [b - a], w.rows("K", l, 0, a, b, dev), w.rows("V", l, 0, a, b, dev))
    torch.cuda.synchronize()
    plan.check_device_error()
    log(f"filled {L} layers x {T} tokens in {time.time() - t0:.1f} s; cache {plan.cache_bytes() / 1e9:.2f} GB")

    stream = torch.cuda.Stream(dev)
    ws = plan.new_workspace(1, dev)
    n_tok_steps = Wm + 1 + K + Wm + 2
    knew = torch.stack([w.rows("K", l, 0, T, T + n_tok_steps, dev) for l in range(L)])  # [L][n][Hkv][128]
    vnew = torch.stack([w.rows("V", l, 0, T, T + n_tok_steps, dev) for l in range(L)])
    qall = torch.stack([torch.stack([w.queries(l, 0, s, dev) for l in range(L)]) for s in range(n_tok_steps)])
    out = torch.empty((L, 1, Hq, 128), dtype=torch.float32, device=dev)
    tok = [0]

    def step(events=None):
        i = tok[0]
        for l in range(L):
            plan.append(l, [0], [1], knew[l, i], vnew[l, i], stream)
            if events is not None:
                events[l][0].record(stream)
            plan.decode(l, [0], qall[i, l].unsqueeze(0), out[l], ws, stream)
            if events is not None:
                events[l][1].record(stream)
        tok[0] += 1

    with torch.cuda.stream(stream):
        for _ in range(Wm):
            step()
    stream.synchronize()
    plan.check_device_error(stream)

    # capture one step (fixed positions; every replay does the full step's work)
    length_at_capture = plan.seq_length(0, 0) + 1
    n0 = kvq.launch_count()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step()
    launches_per_step = kvq.launch_count() - n0
    for _ in range(Wm):
        g.replay()
    stream.synchronize()
    for _ in range(Wm):
        g.replay()
    stream.synchronize()

    # ---- timed region: device time of K steps
    barrier = (lambda: torch.distributed.barrier()) if world > 1 else (lambda: None)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(K):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = e0.elapsed_time(e1)
    clk = clocks.stop()
    if world > 1:
        t = torch.tensor([ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    step_ms = ms / K
    plan.check_device_error(stream)

    # ---- per-launch decode durations: the step's 32 decode launches, each between two
    # events, enqueued behind a GPU sleep so they run back to back (no host gaps)
    dec = []
    ev_pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(L)]
    i_last = tok[0] - 1
    with torch.cuda.stream(stream):
        for _ in range(K):
            torch.cuda._sleep(4_000_000)
            for l in range(L):
                ev_pairs[l][0].record(stream)
                plan.decode(l, [0], qall[i_last, l].unsqueeze(0), out[l], ws, stream)
                ev_pairs[l][1].record(stream)
            stream.synchronize()
            dec.extend(a.elapsed_time(b) for a, b in ev_pairs)
    dec_ms = statistics.mean(dec)

    # ---- e2e through the public API: host buffers in, host buffers out
    kh = knew.cpu().pin_memory()
    vh = vnew.cpu().pin_memory()
    qh = qall.cpu().pin_memory()
    oh = torch.empty((L, 1, Hq, 128), dtype=torch.float32).pin_memory()
    kd = torch.empty_like(knew[:, 0]); vd = torch.empty_like(vnew[:, 0]); qd = torch.empty_like(qall[0])
    h2d = kd.numel() * 2 + vd.numel() * 2 + qd.numel() * 2
    d2h = oh.numel() * 4
    tok[0] = 0
    e2e_ms = []
    base = plan.seq_length(0, 0)
    for s in range(K):
        i = s % n_tok_steps
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        a.record(stream)
        with torch.cuda.stream(stream):
            kd.copy_(kh[:, i], non_blocking=True)
            vd.copy_(vh[:, i], non_blocking=True)
            qd.copy_(qh[i], non_blocking=True)
            for l in range(L):
                plan.append(l, [0], [1], kd[l], vd[l], stream)
                plan.decode(l, [0], qd[l].unsqueeze(0), out[l], ws, stream)
            oh.copy_(out, non_blocking=True)
        b.record(stream)
        stream.synchronize()
        e2e_ms.append(a.elapsed_time(b))
    e2e_step = statistics.mean(e2e_ms)
    if world > 1:
        t = torch.tensor([e2e_step], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        e2e_step = float(t.item())
    plan.check_device_error(stream)

    # ---- append-quantize throughput: a 2048-token chunk into every layer (graph replay)
    ck = torch.stack([w.rows("K", l, 0, 0, 2048, dev) for l in range(L)])
    cv = torch.stack([w.rows("V", l, 0, 0, 2048, dev) for l in range(L)])
    ga = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        for l in range(L):
            plan.append(l, [0], [2048], ck[l], cv[l], stream)   # warm: allocates the chunk's pages
    stream.synchronize()
    with torch.cuda.graph(ga, stream=stream):
        for l in range(L):
            plan.append(l, [0], [2048], ck[l], cv[l], stream)
    for _ in range(3):
        ga.replay()
    stream.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 10
    a.record(stream)
    for _ in range(reps):
        ga.replay()
    b.record(stream)
    stream.synchronize()
    app_ms = a.elapsed_time(b) / reps
    append_tps = 2048 / (app_ms / 1e3)
    app_bytes = L * 2048 * (Hkv * 2 * 128 * 2 + bytes_per_token_head(plan, 0, Hkv))
    plan.check_device_error(stream)

    # ---- accounting
    dec_bytes = decode_algorithmic_bytes(plan, w, 0, length_at_capture)
    step_bytes = L * dec_bytes + L * (Hkv * 2 * 128 * 2 + bytes_per_token_head(plan, 0, Hkv))
    peaks = measured_peaks()
    peak = float(peaks["hbm_gbs"]) if peaks else 6650.0
    achieved = dec_bytes / (dec_ms / 1e3) / 1e9
    traffic = traffic_from_profile(os.path.join(ROOT, "quantized_kv_cache_15_b200", "csrc", "decode.cu"))
    hbm_gbs = step_bytes / (step_ms / 1e3) / 1e9
    us_per_token = step_ms * 1e3 / world
    line = {
        "metric": METRIC, "value": us_per_token, "unit": "us/token", "n_gpus": world, "steps": K, "warmup": Wm,
        "ms_per_step": step_ms, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "layers": L, "q_heads": Hq, "kv_heads": Hkv, "head_dim": 128,
                   "context": T, "batch": 1, "k_codec": "q8_0", "v_codec": "q4_0", "rotation": "hadamard-128",
                   "step": "per layer: append 1 token + decode attention", "parallelism": f"replicas x{world}",
                   "l2": "no flush: packed cache read per step (%.2f GB) >> L2 (126 MB)" % (L * dec_bytes / 1e9)},
        "hbm_gbs": hbm_gbs, "hbm_frac_of_8tbs": hbm_gbs / NOMINAL_HBM_GBS,
        "hbm_frac_of_measured": hbm_gbs / peak,
        "append_tokens_per_s": append_tps,
        "append_note": f"2048-token chunk appended to all {L} layers (K and V quantized): {app_ms:.3f} ms, "
                       f"{app_bytes / (app_ms / 1e3) / 1e9:.0f} GB/s algorithmic",
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "kernel": "decode_kernel<4>",
                     "bytes_per_launch": dec_bytes, "launch_ms": dec_ms,
                     "peak_source": "MEASURED_PEAKS.json hbm_gbs (copy, burst)" if peaks else "fallback 6650 GB/s"},
        "e2e": {"value": e2e_step * 1e3 / world, "unit": "us/token", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * K,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_decode_us_per_token(w, args.cpu_seconds, log)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g, ga
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
