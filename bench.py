#!/usr/bin/env python
"""Benchmark of one Ulysses attention layer step on B200.

A step is the whole hot path over one batch: seq->head permute (Q, K, V),
causal GQA flash attention forward, head->seq permute (O), seq->head permute
(dO), attention backward, head->seq permute (dQ, dK, dV). Default workload:
packed varlen, N = 65536 tokens, P = 4 virtual ranks, H = 32, H_kv = 8, d = 128
("Ulysses layer tokens/s & attn TFLOP/s at 64K tokens; permute HBM GB/s").

Prints one JSON line (rank 0). Multi-GPU (torchrun): every rank runs its own
independent layer (replicas; the path has no cross-GPU step on one GPU's
emulated ranks), value = total tokens of all ranks / max-over-ranks time.

--workload million times the rank-sequential forward (P = 8 virtual ranks one
after another, N = 1,048,576); --all-workloads adds, under the key
"workloads", one summary per other workload of the pages' 8K-1M range
(tokens/s, attention TFLOP/s with roofline fractions, permute GB/s).

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload instead (rank 0 only).
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

MEASURED_PEAKS = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    try:
        with open(MEASURED_PEAKS) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(files):
    """sha256 over the named kernel sources (name + bytes), to tell whether
    stored ncu counters still describe the kernels being run."""
    import hashlib
    csrc = os.path.join(ROOT, "ulysses_sequence_parallelism_b200", "csrc")
    h = hashlib.sha256()
    for f in files:
        h.update(f.encode())
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "roofline_traffic.json")


def stored_traffic(workload, stage, path=None):
    """DRAM bytes per call of `stage` from profiles/roofline_traffic.json, or
    None when they were taken on other kernel sources or another workload."""
    try:
        with open(path or TRAFFIC_FILE) as f:
            t = json.load(f)
        st = t[stage]
        if t.get("workload") != workload or st["source_sha256"] != kernel_source_hash(st["sources"]):
            return None
        return st["bytes"]
    except Exception:
        return None


def flops(w, cu):
    pairs = workloads.causal_pairs(w.N, cu)
    return 4.0 * w.d * w.H * pairs, 10.0 * w.d * w.H * pairs, pairs


def permute_bytes(w):
    """Algorithmic bytes of each permute launch (read + write once)."""
    q = w.N * w.H * w.d * 2
    kv = w.N * w.H_kv * w.d * 2
    return {"qkv_s2h": 2 * (q + 2 * kv), "o_h2s": 2 * q, "do_s2h": 2 * q, "dqkv_h2s": 2 * (q + 2 * kv)}


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def aggregate_over_ranks(local_ms: float, tokens_per_rank: int, world: int, reduce_max=None):
    """Whole-job throughput for `world` ranks that each ran `tokens_per_rank`
    tokens per step: the slowest rank's ms per step sets the job time. With a
    process group, `reduce_max` is an all-reduce(max) over ranks."""
    ms = reduce_max(local_ms) if (world > 1 and reduce_max is not None) else local_ms
    return ms, world * tokens_per_rank / (ms / 1e3)


def device_inputs(w, dev, seed=0):
    """Seeded synthetic inputs drawn on the device (fast at any size): the
    workload's document lengths from its numpy recipe, then Q, K, V, dO as
    N(0,1) x scale rounded to bf16 by a CUDA generator seeded with `seed`.
    Used for timing only; parity tests draw with workloads.generate."""
    import torch
    cu = None
    if w.varlen is not None:
        rng = np.random.Generator(np.random.PCG64(seed))
        cu = workloads.cu_seqlens_from_lengths(workloads.draw_doc_lengths(rng, w.N, *w.varlen))
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    n = w.N // w.P
    mk = lambda hx, sc: [(torch.randn(n, hx, w.d, device=dev, generator=g) * sc).to(torch.bfloat16)
                         for _ in range(w.P)]
    out = {"cu_seqlens": cu, "q": mk(w.H, w.scale), "k": mk(w.H_kv, w.scale), "v": mk(w.H_kv, w.scale)}
    if w.backward:
        out["do"] = mk(w.H, 1.0)
    return out


def time_layer(U, w, dev, q, k, v, do, cu_np, steps, warmup, deterministic=False, barrier=None):
    """Time `steps` layer steps of workload `w` (after `warmup` untimed ones)
    stage by stage with CUDA events on the launching stream. All ranks at once,
    or one rank after another for rank-sequential workloads (the stage times
    are then summed over ranks). Returns the layer, the total ms, per-stage
    mean ms lists and the kernel launch count per step."""
    import torch
    N, P, H, H_kv, d = w.N, w.P, w.H, w.H_kv, w.d
    cu = None if cu_np is None else torch.tensor(cu_np, dtype=torch.int32, device=dev)
    layer = U.UlyssesLayer(N, P, H, H_kv, d, device=dev, cu_seqlens=cu, backward=w.backward,
                           rank_sequential=w.rank_sequential, deterministic=deterministic)
    o = [torch.empty_like(x) for x in q]
    if w.backward:
        dq = [torch.empty_like(x) for x in q]
        dk = [torch.empty_like(x) for x in k]
        dv = [torch.empty_like(x) for x in v]
    stream = torch.cuda.current_stream()
    stages = ["qkv_s2h", "attn_fwd", "o_h2s"] + (["do_s2h", "attn_bwd", "dqkv_h2s"] if w.backward else [])
    ranges = [(r, r + 1) for r in range(P)] if w.rank_sequential else [(0, P)]
    L = layer

    def bufs(b, lo, hi):
        # all-ranks layers hold P head buffers; rank-sequential ones reuse one
        return b if not w.rank_sequential else [b[0] if i == lo else None for i in range(P)]

    def step(ev=None):
        for ri, (lo, hi) in enumerate(ranges):
            rec = (lambda i: ev[ri][i].record(stream)) if ev else (lambda i: None)
            rec(0)
            U.ulysses_a2a_seq_to_head(q, k, v, bufs(L.q_h, lo, hi), bufs(L.k_h, lo, hi), bufs(L.v_h, lo, hi), N, P,
                                      H, H_kv, d, cu, rank_lo=lo, rank_hi=hi)
            rec(1)
            U.ulysses_attn_fwd(bufs(L.q_h, lo, hi), bufs(L.k_h, lo, hi), bufs(L.v_h, lo, hi), bufs(L.o_h, lo, hi),
                               L.lse, N, P, H, H_kv, d, cu, rank_lo=lo, rank_hi=hi)
            rec(2)
            U.ulysses_a2a_head_to_seq(bufs(L.o_h, lo, hi), None, None, o, None, None, N, P, H, H_kv, d, cu,
                                      rank_lo=lo, rank_hi=hi)
            rec(3)
            if w.backward:
                U.ulysses_a2a_seq_to_head(do, None, None, L.do_h, None, None, N, P, H, H_kv, d, cu)
                rec(4)
                U.ulysses_attn_bwd(L.q_h, L.k_h, L.v_h, L.o_h, L.lse, L.do_h, L.dq_h, L.dk_h, L.dv_h, N, P, H, H_kv,
                                   d, L.workspace, cu, deterministic=deterministic)
                rec(5)
                U.ulysses_a2a_head_to_seq(L.dq_h, L.dk_h, L.dv_h, dq, dk, dv, N, P, H, H_kv, d, cu)
                rec(6)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    code, word = U.ulysses_get_device_status()
    if code != 0:
        raise SystemExit(f"{w.name}: device status {code} word {word:#x} after warm-up")
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] for _ in ranges]
           for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if barrier is not None:
        barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for s_ in range(steps):
        step(evs[s_])
    t1.record(stream)
    torch.cuda.synchronize()
    if barrier is not None:
        barrier()
    code, word = U.ulysses_get_device_status()
    if code != 0:
        raise SystemExit(f"{w.name}: device status {code} word {word:#x} after the timed steps")
    stage_ms = {st: [sum(evs[s_][ri][i].elapsed_time(evs[s_][ri][i + 1]) for ri in range(len(ranges)))
                     for s_ in range(steps)] for i, st in enumerate(stages)}
    launches = len(ranges) * 3 + ((1 + 3 + 1) if w.backward else 0)
    outs = {"o": o}
    if w.backward:
        outs.update(dq=dq, dk=dk, dv=dv)
    return layer, t0.elapsed_time(t1), stage_ms, launches, outs


def summarize(w, cu_np, total_ms, stage_ms, steps, peaks):
    """Tokens/s, attention TFLOP/s and permute GB/s of one timed workload."""
    f_fwd, f_bwd, pairs = flops(w, cu_np)
    pb = permute_bytes(w)
    mean = {st: sum(v_) / len(v_) for st, v_ in stage_ms.items()}
    ms = total_ms / steps
    out = {"workload": w.name, "N": w.N, "P": w.P, "pass": "fwd+bwd" if w.backward else "fwd",
           "rank_sequential": w.rank_sequential, "docs": None if cu_np is None else int(len(cu_np) - 1),
           "steps": steps, "ms_per_step": ms, "tokens_per_s": w.N / (ms / 1e3), "stage_ms_mean": mean,
           "pairs": pairs, "attn_fwd_tflops": f_fwd / (mean["attn_fwd"] / 1e3) / 1e12,
           "permute_gbs": {st: pb[st] / (mean[st] / 1e3) / 1e9 for st in pb if st in mean}}
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    sus = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    out["attn_fwd_frac_of_burst"] = out["attn_fwd_tflops"] / burst
    out["attn_fwd_frac_of_sustained"] = out["attn_fwd_tflops"] / sus
    if w.backward:
        out["attn_bwd_tflops"] = f_bwd / (mean["attn_bwd"] / 1e3) / 1e12
        out["attn_bwd_frac_of_sustained"] = out["attn_bwd_tflops"] / sus
    hp = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    out["permute_frac_of_hbm"] = {st: g / hp for st, g in out["permute_gbs"].items()}
    return out


def cpu_oracle_sample(w, inp, budget_s=20.0):
    """Time the fp64 oracle on a bounded sample of the workload and extrapolate
    the layer time linearly in (i, j) pairs x heads. Sample: forward + backward
    of the first document (or the first 2048 tokens), one kv head group
    (H/H_kv query heads), plus the three permutes of that slice."""
    import oracle
    cu = inp["cu_seqlens"]
    L = int(cu[1]) if cu is not None else min(w.N, 2048)
    L = min(L, 4096)
    group = w.H // w.H_kv
    widen = oracle.widen_bf16
    q = widen(inp["q"][:L, :group])
    k = widen(inp["k"][:L, :1])
    v = widen(inp["v"][:L, :1])
    do = widen(inp["do"][:L, :group]) if "do" in inp else None
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.attention_forward(q, k, v)
        if do is not None:
            oracle.attention_backward(q, k, v, do)
        reps += 1
        if time.perf_counter() - t0 > budget_s / 2 or reps >= 50:
            break
    t_attn = (time.perf_counter() - t0) / reps
    sample_pairs = L * (L + 1) // 2 * group
    full_pairs = workloads.causal_pairs(w.N, cu) * w.H
    t_attn_full = t_attn * full_pairs / sample_pairs
    # permutes: time the oracle's seq->head on a token slice and scale by bytes
    sl = min(w.N, 8192)
    xs = workloads.seq_shards(inp["q"][:sl], w.P)
    t1 = time.perf_counter()
    preps = 0
    while time.perf_counter() - t1 < min(2.0, budget_s / 4):
        oracle.head_to_seq(oracle.seq_to_head(xs))
        preps += 1
    t_perm = (time.perf_counter() - t1) / preps / 2       # one permute of the Q slice
    q_bytes = sl * w.H * w.d * 2
    perm_bytes_step = sum(permute_bytes(w).values()) / 2  # tensor bytes moved (each read+write counted once)
    t_perm_full = t_perm * perm_bytes_step / q_bytes
    t_layer = t_attn_full + t_perm_full
    cores = len(os.sched_getaffinity(0))
    return {
        "value": w.N / t_layer, "unit": "tokens/s", "cores": cores, "kind": "oracle",
        "sample": (f"fp64 numpy oracle fwd{'+bwd' if do is not None else ''} on the first {L} tokens x "
                   f"{group} query heads (1 kv head), {reps} reps, {t_attn:.3f} s each, plus seq<->head "
                   f"permutes of {sl} tokens; extrapolated linearly by (i,j)-pairs x heads and by bytes"),
        "t_layer_s": t_layer, "t_sample_s": t_attn,
    }


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    inp = workloads.generate(w, N=min(w.N, 16384) if w.varlen is None else None)
    budget = 10.0
    vals = []
    t_all = time.perf_counter()
    for s in range(args.warmup + args.steps):
        cb = cpu_oracle_sample(w, inp, budget_s=budget)
        if s >= args.warmup:
            vals.append(cb)
    v = statistics.median([c["value"] for c in vals])
    cb = vals[-1]
    line = {
        "impl": "reference", "metric": "Ulysses layer tokens/s (fwd+bwd)" if w.backward else "Ulysses layer tokens/s (fwd)",
        "value": v, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * w.N / v, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "N": w.N, "P": w.P, "H": w.H, "H_kv": w.H_kv, "d": w.d},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cb["cores"], "kind": "oracle",
                         "sample": cb["sample"]},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": time.perf_counter() - t_all,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_exchange(args, w):
    """The real multi-process exchange: P = the number of processes, each
    holding N/P tokens of the workload's sequence (the whole job processes N
    tokens per step, so more GPUs means fewer tokens each: strong scaling).
    A step is UlyssesDistLayer forward (+ backward): pack, NCCL all-to-all,
    attention on the received head chunk, all-to-all back, unpack."""
    import datetime
    import torch
    import torch.distributed as dist
    import ulysses_sequence_parallelism_b200 as U
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    if world == 1:
        import socket
        with socket.socket() as s_:
            s_.bind(("127.0.0.1", 0))
            os.environ.setdefault("MASTER_PORT", str(s_.getsockname()[1]))
        os.environ.setdefault("RANK", "0")
        os.environ.setdefault("WORLD_SIZE", "1")
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    N, H, H_kv, d = w.N, w.H, w.H_kv, w.d
    if N % world or H % world or H_kv % world:
        raise SystemExit(f"--exchange needs N, H, H_kv divisible by the {world} processes")
    cu_np = None
    if w.varlen is not None:
        rng = np.random.Generator(np.random.PCG64(0))
        cu_np = workloads.cu_seqlens_from_lengths(workloads.draw_doc_lengths(rng, N, *w.varlen))
    cu = None if cu_np is None else torch.tensor(cu_np, dtype=torch.int32, device=dev)
    n = N // world
    g = torch.Generator(device=dev)
    g.manual_seed(1000 + rank)
    mk = lambda hx, sc: (torch.randn(n, hx, d, device=dev, generator=g) * sc).to(torch.bfloat16)
    q, k, v = mk(H, w.scale), mk(H_kv, w.scale), mk(H_kv, w.scale)
    do = mk(H, 1.0) if w.backward else None
    layer = U.UlyssesDistLayer(N, H, H_kv, d, device=dev, cu_seqlens=cu, backward=w.backward)
    o = torch.empty_like(q)
    if w.backward:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    stream = torch.cuda.current_stream()

    def step():
        layer.forward(q, k, v, o)
        if w.backward:
            layer.backward(do, dq, dk, dv)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    clk = clocks.stop()
    code, word = U.ulysses_get_device_status()
    if code != 0:
        raise SystemExit(f"device status {code} word {word:#x}")
    t = torch.tensor([e0.elapsed_time(e1) / args.steps], device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item())
    f_fwd, f_bwd, pairs = flops(w, cu_np)
    shard = lambda hx: n * hx * d * 2
    per_pass = 2 * shard(H) + 2 * shard(H_kv)                 # Q, K, V in + O out (forward)
    sent = (world - 1) / world * (per_pass + (2 * shard(H) + 2 * shard(H_kv) if w.backward else 0))
    line = {
        "metric": "Ulysses layer tokens/s (fwd+bwd)" if w.backward else "Ulysses layer tokens/s (fwd)",
        "value": N / (ms / 1e3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "N": N, "P": world, "H": H, "H_kv": H_kv, "d": d,
                   "docs": None if cu_np is None else int(len(cu_np) - 1),
                   "pass": "fwd+bwd" if w.backward else "fwd",
                   "parallelism": f"Ulysses over {world} processes (NCCL all-to-all, "
                                  f"{len(layer.plan.chunks)} head chunks)",
                   "inputs": "seeded N(0,1) drawn on each rank's device"},
        "exchange": {"bytes_sent_per_rank_per_step": sent, "chunks": len(layer.plan.chunks),
                     "attn_tflops_whole_job": (f_fwd + (f_bwd if w.backward else 0)) / (ms / 1e3) / 1e12},
        "clocks": clk,
        # per chunk: pack, attention, unpack (+ backward: pack dO, three backward kernels, unpack)
        "gpu_launches": len(layer.plan.chunks) * (3 + (5 if w.backward else 0)) * args.steps,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del layer
    dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="varlen64k", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--layer-only", action="store_true",
                    help="time only the layer step (no fused / fragment / projection / e2e / CPU extras); "
                         "for profiler captures")
    ap.add_argument("--deterministic", action="store_true",
                    help="time the two-pass backward (bit-reproducible dQ) instead of the one-pass one")
    ap.add_argument("--exchange", choices=["none", "nccl"], default="none",
                    help="nccl: run the real multi-process exchange (P = number of processes) instead of "
                         "independent replicas")
    ap.add_argument("--all-workloads", action="store_true",
                    help="also time llama8k, single64k, long96k and the million-token workload (key 'workloads')")
    ap.add_argument("--tokens", type=int, default=None,
                    help="draw the workload's recipe at a smaller total N (profiling captures)")
    args = ap.parse_args()
    w = workloads.get(args.workload)
    if args.tokens is not None:
        import dataclasses
        w = dataclasses.replace(w, N=args.tokens)
    if args.impl == "reference":
        return run_reference(args, w)
    if args.exchange == "nccl":
        return run_exchange(args, w)

    import torch
    import torch.distributed as dist
    import ulysses_sequence_parallelism_b200 as U

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    inp = workloads.generate(w, seed=0) if not w.rank_sequential else None
    P, H, H_kv, d, N = w.P, w.H, w.H_kv, w.d, w.N

    def shards(x):
        n = N // P
        return [torch.from_numpy(x[p * n:(p + 1) * n].view(np.int16)).view(torch.bfloat16).to(dev) for p in range(P)]

    if inp is not None:
        cu_np = inp["cu_seqlens"]
        q, k, v = shards(inp["q"]), shards(inp["k"]), shards(inp["v"])
        do = shards(inp["do"]) if w.backward else None
    else:
        # rank-sequential (million-token) workload: seeded inputs drawn on the device
        di = device_inputs(w, dev)
        cu_np, q, k, v, do = di["cu_seqlens"], di["q"], di["k"], di["v"], di.get("do")
    cu = None if cu_np is None else torch.tensor(cu_np, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()
    f_fwd, f_bwd, pairs = flops(w, cu_np)
    pb = permute_bytes(w)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    layer, total_ms, stage_ms, launches_per_step, outs = time_layer(
        U, w, dev, q, k, v, do, cu_np, args.steps, args.warmup, deterministic=args.deterministic, barrier=barrier)
    clk = clocks.stop()
    o = outs["o"]
    if w.backward:
        dq, dk, dv = outs["dq"], outs["dk"], outs["dv"]

    def reduce_max(x):
        t = torch.tensor([x], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    ms_per_step, value = aggregate_over_ranks(total_ms / args.steps, N, world, reduce_max)

    med = {st: statistics.median(v_) for st, v_ in stage_ms.items()}
    mean = {st: sum(v_) / len(v_) for st, v_ in stage_ms.items()}
    peaks, peak_src = load_peaks()
    fwd_tflops = f_fwd / (mean["attn_fwd"] / 1e3) / 1e12
    perm_gbs = {st: pb[st] / (mean[st] / 1e3) / 1e9 for st in pb if st in mean}
    detail = {"attn_fwd_tflops": fwd_tflops, "permute_gbs": perm_gbs,
              "stage_ms_mean": mean, "stage_ms_median": med, "pairs": pairs, "attn_fwd_flops": f_fwd}
    if w.rank_sequential:
        detail["note"] = (f"{P} virtual ranks one after another (seq->head, attention, head->seq per rank); "
                          "stage times summed over ranks")
    if w.backward:
        detail["attn_bwd_tflops"] = f_bwd / (mean["attn_bwd"] / 1e3) / 1e12
        detail["attn_bwd_flops"] = f_bwd
        detail["attn_bwd_mode"] = "two-pass (deterministic)" if args.deterministic else "one-pass (fp32 dQ reductions)"
    if w.backward and not args.layer_only:
        # the other backward mode on the same buffers, for comparison (not part of the step)
        other = not args.deterministic
        L = layer
        ws_other = torch.empty(U.ulysses_attn_bwd_workspace_size(N, P, H, H_kv, d, other), dtype=torch.uint8,
                               device=dev)
        run_other = lambda: U.ulysses_attn_bwd(L.q_h, L.k_h, L.v_h, L.o_h, L.lse, L.do_h, L.dq_h, L.dk_h, L.dv_h, N,
                                               P, H, H_kv, d, ws_other, cu, deterministic=other)
        for _ in range(2):
            run_other()
        oe = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        oe[0].record(stream)
        for _ in range(3):
            run_other()
        oe[1].record(stream)
        torch.cuda.synchronize()
        other_ms = oe[0].elapsed_time(oe[1]) / 3
        detail["attn_bwd_other_mode"] = {"mode": "two-pass (deterministic)" if other else "one-pass",
                                         "ms": other_ms, "tflops": f_bwd / (other_ms / 1e3) / 1e12}
        del ws_other
    # dominant kernel by measured time
    dom = max(mean, key=mean.get)
    tensor_peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    if dom in ("attn_fwd", "attn_bwd"):
        achieved = (f_fwd if dom == "attn_fwd" else f_bwd) / (mean[dom] / 1e3) / 1e12
        roof = {"kernel": dom, "bound": "tensor", "achieved": achieved, "peak": tensor_peak, "unit": "TFLOP/s",
                "frac": achieved / tensor_peak, "traffic": stored_traffic(w.name if args.tokens is None else None, dom),
                "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a long step)",
                "traffic_source": "ncu DRAM bytes per call, profiles/roofline_traffic.json (null if the kernels changed)"}
    else:
        achieved = pb[dom] / (mean[dom] / 1e3) / 1e9
        hp = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        roof = {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": hp, "unit": "GB/s",
                "frac": achieved / hp, "traffic": None, "peak_source": f"{peak_src} hbm_gbs"}

    # ---------------------------------------------------------------- fused layer (all-to-alls in the kernels)
    if args.layer_only:
        args.no_e2e = args.no_cpu_baseline = True
    fused = None
    if w.backward and (N // P) % 128 == 0 and not args.layer_only:
        lf = U.UlyssesLayer(N, P, H, H_kv, d, device=dev, cu_seqlens=cu, fused=True,
                            deterministic=args.deterministic)

        def fused_step(ev=None):
            if ev: ev[0].record(stream)
            U.ulysses_attn_fwd_seq(q, k, v, o, lf.lse, N, P, H, H_kv, d, cu)
            if ev: ev[1].record(stream)
            U.ulysses_attn_bwd_seq(q, k, v, o, lf.lse, do, dq, dk, dv, N, P, H, H_kv, d, lf.workspace, cu,
                                   deterministic=args.deterministic)
            if ev: ev[2].record(stream)

        for _ in range(args.warmup):
            fused_step()
        torch.cuda.synchronize()
        fev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
        barrier()
        torch.cuda.synchronize()
        for s_ in range(args.steps):
            fused_step(fev[s_])
        torch.cuda.synchronize()
        f_fwd_ms = sum(e[0].elapsed_time(e[1]) for e in fev) / args.steps
        f_bwd_ms = sum(e[1].elapsed_time(e[2]) for e in fev) / args.steps
        f_ms, f_val = aggregate_over_ranks(f_fwd_ms + f_bwd_ms, N, world, reduce_max)
        staged = (not args.deterministic) and d == 128   # one-pass: Q and dO staged in head shards
        fused = {"value": f_val, "unit": "tokens/s", "ms_per_step": f_ms, "attn_fwd_seq_ms": f_fwd_ms,
                 "attn_bwd_seq_ms": f_bwd_ms, "gpu_launches_per_step": 1 + 3 + (2 if staged else 0),
                 "note": "all-to-alls folded into the attention kernels' addressing; the one-pass backward "
                         "first copies Q and dO into head shards in its workspace (2 permute launches), "
                         "O, dQ, dK, dV go straight to the sequence shards"}
        del lf

    # ---------------------------------------------------------------- head fragmentation (NEXT-3)
    # each rank processes its heads one GQA group at a time: same results, a
    # fraction of the full-sequence activation buffers
    frag = None
    if w.backward and not args.layer_only:
        g = H // H_kv
        lfr = U.UlyssesLayer(N, P, H, H_kv, d, device=dev, cu_seqlens=cu, head_fragment=g,
                             deterministic=args.deterministic)

        def frag_step():
            lfr.forward(q, k, v, o)
            lfr.backward(do, dq, dk, dv)

        for _ in range(max(1, min(args.warmup, 2))):
            frag_step()
        torch.cuda.synchronize()
        barrier()
        fa, fb_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_fr = max(1, min(args.steps, 5))
        fa.record(stream)
        for _ in range(n_fr):
            frag_step()
        fb_.record(stream)
        torch.cuda.synchronize()
        fr_ms, fr_val = aggregate_over_ranks(fa.elapsed_time(fb_) / n_fr, N, world, reduce_max)
        nbytes = lambda ts: sum(t.numel() * t.element_size() for t in ts)
        frag_bytes = nbytes([lfr.q_f, lfr.k_f, lfr.v_f, lfr.o_f, lfr.do_f, lfr.dq_f, lfr.dk_f, lfr.dv_f,
                             lfr.workspace])
        full_bytes = nbytes(layer.q_h + layer.k_h + layer.v_h + layer.o_h + layer.do_h + layer.dq_h + layer.dk_h +
                            layer.dv_h + [layer.workspace])
        frag = {"value": fr_val, "unit": "tokens/s", "ms_per_step": fr_ms, "steps": n_fr, "head_fragment": g,
                "fragments_per_step": P * (H // P) // g, "head_side_bytes": frag_bytes,
                "head_side_bytes_unfragmented": full_bytes}
        del lfr

    # ---------------------------------------------------------------- projections (NEXT-4)
    # QKV projection storing straight into the head shards and output projection
    # reading straight from them (hidden = H d, synthetic seeded weights)
    proj = None
    if not w.rank_sequential and (N // P) % 128 == 0 and not args.layer_only:
        hidden = H * d
        xb, wqb, wob = workloads.projection_inputs(N, H, H_kv, d, hidden, seed=1)
        tdev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        x_seq = [tdev(a) for a in workloads.seq_shards(xb, P)]
        w_qkv, w_o = tdev(wqb), tdev(wob)
        y_seq = [torch.empty_like(t) for t in x_seq]
        del xb, wqb, wob
        L = layer

        def timed(fn, reps=5):
            for _ in range(2):
                fn()
            ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ea.record(stream)
            for _ in range(reps):
                fn()
            eb.record(stream)
            torch.cuda.synchronize()
            return ea.elapsed_time(eb) / reps

        qkv_ms = timed(lambda: U.ulysses_qkv_proj_seq_to_head(x_seq, w_qkv, L.q_h, L.k_h, L.v_h, N, P, H, H_kv, d,
                                                               hidden))
        out_ms = timed(lambda: U.ulysses_out_proj_head_to_seq(L.o_h, w_o, y_seq, N, P, H, H_kv, d, hidden))
        blk_ms = timed(lambda: L.forward_projected(x_seq, w_qkv, w_o, y_seq), reps=3)
        f_qkv = 2.0 * N * hidden * (H + 2 * H_kv) * d
        f_out = 2.0 * N * H * d * hidden
        proj = {"hidden": hidden, "qkv_proj_ms": qkv_ms, "qkv_proj_tflops": f_qkv / (qkv_ms / 1e3) / 1e12,
                "out_proj_ms": out_ms, "out_proj_tflops": f_out / (out_ms / 1e3) / 1e12,
                "block_fwd_ms": blk_ms, "block_fwd_tokens_per_s": N / (blk_ms / 1e3),
                "note": "block_fwd = QKV projection into head shards + attention + output projection from head "
                        "shards (forward only); block_fwd_bwd adds the gradients of all three; no permute launches"}
        if w.backward:
            dy_seq = [torch.randn_like(t, dtype=torch.float32).to(torch.bfloat16) for t in y_seq]
            dw_o = torch.empty(w_o.shape, dtype=torch.float32, device=dev)
            dw_qkv = torch.empty(w_qkv.shape, dtype=torch.float32, device=dev)
            dx_seq = [torch.empty_like(t) for t in x_seq]
            obwd_ms = timed(lambda: U.ulysses_out_proj_bwd(L.o_h, w_o, dy_seq, L.do_h, dw_o, N, P, H, H_kv, d,
                                                           hidden))
            qbwd_ms = timed(lambda: U.ulysses_qkv_proj_bwd(x_seq, w_qkv, L.dq_h, L.dk_h, L.dv_h, dx_seq, dw_qkv, N,
                                                           P, H, H_kv, d, hidden))

            def block_step():
                L.forward_projected(x_seq, w_qkv, w_o, y_seq)
                L.backward_projected(dy_seq, x_seq, w_qkv, w_o)

            full_ms = timed(block_step, reps=3)
            proj.update({"out_proj_bwd_ms": obwd_ms, "out_proj_bwd_tflops": 2 * f_out / (obwd_ms / 1e3) / 1e12,
                         "qkv_proj_bwd_ms": qbwd_ms, "qkv_proj_bwd_tflops": 2 * f_qkv / (qbwd_ms / 1e3) / 1e12,
                         "block_fwd_bwd_ms": full_ms, "block_fwd_bwd_tokens_per_s": N / (full_ms / 1e3)})
            del dy_seq, dw_o, dw_qkv, dx_seq
        del x_seq, y_seq, w_qkv, w_o

    # ---------------------------------------------------------------- end to end through the public API
    # ulysses_host_pipeline_* (C-ABI, host buffers): every step copies its
    # inputs from pinned host memory and reads its results back; copies of
    # neighbouring steps overlap the kernels.
    e2e = None
    if not args.no_e2e and inp is not None:
        pin = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
        n = N // P
        rows = lambda a: [pin(a[p * n:(p + 1) * n]) for p in range(P)]
        host_in = {"q": rows(inp["q"]), "k": rows(inp["k"]), "v": rows(inp["v"])}
        if w.backward:
            host_in["do"] = rows(inp["do"])
        empty_like_pinned = lambda xs: [torch.empty_like(x).pin_memory() for x in xs]
        host_out = []
        for _ in range(2):
            ho = {"o": empty_like_pinned(host_in["q"])}
            if w.backward:
                ho.update(dq=empty_like_pinned(host_in["q"]), dk=empty_like_pinned(host_in["k"]),
                          dv=empty_like_pinned(host_in["v"]))
            host_out.append(ho)
        h2d = sum(x.numel() * 2 for xs in host_in.values() for x in xs)
        d2h = sum(x.numel() * 2 for xs in host_out[0].values() for x in xs)
        hp = U.HostPipeline(layer, device=dev)
        for i in range(max(1, args.warmup)):
            hp.submit(host_in, host_out[i & 1])
        hp.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for i in range(args.steps):
            hp.submit(host_in, host_out[i & 1], before=a if i == 0 else None,
                      after=b if i == args.steps - 1 else None)
        hp.synchronize()
        e_ms, e_val = aggregate_over_ranks(a.elapsed_time(b) / args.steps, N, world, reduce_max)
        e2e = {"value": e_val, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
               "api": "C-ABI ulysses_host_pipeline_submit with host buffers (one cudaMemcpyAsync per shard; "
                      "copies of neighbouring steps overlap the kernels on the library's three streams)"}
        hp.close()
        del hp

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_oracle_sample(w, inp if inp is not None else workloads.generate(w, N=16384), budget_s=20.0)
        cpu = {k_: cb[k_] for k_ in ("value", "unit", "cores", "kind", "sample")}

    if rank == 0:
        line = {
            "metric": "Ulysses layer tokens/s (fwd+bwd)" if w.backward else "Ulysses layer tokens/s (fwd)",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "N": N, "P": P, "H": H, "H_kv": H_kv, "d": d,
                       "docs": None if cu_np is None else int(len(cu_np) - 1),
                       "pass": "fwd+bwd" if w.backward else "fwd",
                       "l2": "inputs larger than L2 (per-tensor working sets 0.27-1.3 GB > 126 MB); no flush",
                       "parallelism": f"{P} virtual ranks per GPU; {world} independent replica(s)"},
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk, "detail": detail, "fused": fused, "head_fragment": frag, "projections": proj,
        }
        if inp is None:
            line["config"]["inputs"] = "seeded N(0,1) drawn on the device (torch CUDA generator, seed 0)"
    # ---------------------------------------------------------------- the other workloads (opt-in)
    # the pages' range, 8K to 1M tokens: one summary per workload, not the headline
    if args.all_workloads:
        extra = {}
        del o, layer, outs
        if w.backward:
            del dq, dk, dv
        torch.cuda.empty_cache()
        for name in ("llama8k", "varlen64k", "single64k", "long96k", "million"):
            if name == w.name:
                continue
            wx = workloads.get(name)
            di = device_inputs(wx, dev)
            steps_x = 1 if wx.rank_sequential else max(3, min(args.steps, 10))
            warm_x = 1 if wx.rank_sequential else 3
            _, tot, st_ms, _, _ = time_layer(U, wx, dev, di["q"], di["k"], di["v"], di.get("do"), di["cu_seqlens"],
                                             steps_x, warm_x, deterministic=args.deterministic, barrier=barrier)
            tot, _ = aggregate_over_ranks(tot, wx.N, world, reduce_max)
            extra[name] = summarize(wx, di["cu_seqlens"], tot, st_ms, steps_x, peaks)
            extra[name]["inputs"] = "seeded N(0,1) x scale drawn on the device (torch CUDA generator, seed 0)"
            del di
            torch.cuda.empty_cache()
        if rank == 0:
            line["workloads"] = extra
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
