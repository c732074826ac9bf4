#!/usr/bin/env python
"""Benchmark of the RRAttention prefill operator (search + block-sparse attention).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole hot path over one attention layer's synthetic
inputs: the round-robin sampled-score search, Top-tau selection and the
block-sparse attention, through the C ABI.  Default workload: the 128K
LLaMA-3.1-8B-shaped GQA layer (H=32, Hkv=8, d=128, L=131072, B=128, S=16,
tau=0.95, planted sinks + local band).

One JSON line (rank 0).  `value` is TFLOP/s over the visited blocks
(4*B*B*d flops per visited block, diagonal blocks counted in full), summed over
ranks and divided by the slowest rank's device time.  Under torchrun every rank
runs its own independent layer (weak scaling, no collective on the data path).

`--impl reference` times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (rank 0 only) and prints the same line with
"impl": "reference".
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import gen  # noqa: E402

METRIC = "sparse prefill attn ms & TFLOP/s at 128K (search+attn); speedup vs dense"
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "bsfa_llama128k_traffic.txt")


def workload_config(cfg: gen.Config, tau: float) -> dict:
    return {"workload": f"{cfg.name}: GQA attention layer H={cfg.H}/Hkv={cfg.Hkv}, d={cfg.d}, L={cfg.L}, "
                        f"B={cfg.B}, S={cfg.S}, tau={tau}, batch 1",
            "structure": {0: "iid", 1: "planted sinks", 2: "planted sinks + local band", 3: "video frames"}[
                cfg.structure],
            "L": cfg.L, "H": cfg.H, "Hkv": cfg.Hkv, "d": cfg.d, "B": cfg.B, "S": cfg.S, "tau": tau,
            "l2": ("inputs exceed L2: q alone is %.2f GB > 126 MB, no flush needed" % (cfg.L * cfg.H * cfg.d * 2 / 1e9)
                   if cfg.L * cfg.H * cfg.d * 2 > 126e6 else "inputs fit in L2 (not flushed)"),
            "seed": cfg.seed}


def block_flops(cfg: gen.Config, visited_blocks: int) -> float:
    return 4.0 * cfg.B * cfg.B * cfg.d * visited_blocks


def search_bytes(cfg: gen.Config, visited_blocks: int) -> dict:
    """Algorithmic HBM bytes of one search stage (sampled keys): every sampled
    query row and sampled key read once, the lower-triangle block masses
    written by the score kernel and read by Top-tau, count and idx written."""
    Ns, Nb = cfg.L // cfg.S, cfg.L // cfg.B
    rows = Ns * cfg.H * cfg.d * 2
    tri = cfg.H * Nb * (Nb + 1) // 2 * 4
    parts = {"q_sampled": rows, "k_sampled": rows, "mass_write": tri, "mass_read": tri,
             "count_write": cfg.H * Nb * 4, "idx_write": visited_blocks * 4}
    parts["total"] = sum(parts.values())
    return parts


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"bf16_tflops": d["bf16_tflops"], "bf16_tflops_sustained": d.get("bf16_tflops_sustained"),
                "hbm_gbs": d["hbm_gbs"], "source": "measured"}
    return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


def kernel_traffic_bytes():
    """DRAM bytes per attention launch from the committed ncu summary, if it was
    taken on the current kernel source (else None)."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    src = os.path.join(ROOT, "dynamic_block_sparse_rr_b200", "csrc", "bsfa.cu")
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    vals = {}
    for line in open(PROFILE_TRAFFIC):
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("bsfa_cu_sha256_16") != digest:
        return None
    try:
        return float(vals["traffic_bytes_per_launch_full"])
    except (KeyError, ValueError):
        return None


def single_thread_tiny_s() -> float:
    """The oracle (search + attention) on the tiny config with one BLAS thread."""
    import oracle
    from threadpoolctl import threadpool_limits
    cfg = gen.CONFIGS["tiny"]
    q, k, v = gen.make_config(cfg)
    Q, K, V = (gen.bf16_bits_to_f32(x) for x in (q, k, v))
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        c, i, _ = oracle.rr_search(Q, K, cfg.B, cfg.S, cfg.tau)
        oracle.sparse_attention(Q, K, V, c, i, cfg.B)
        return time.perf_counter() - t0


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# ---------------------------------------------------------------- CPU oracle
def oracle_sample(cfg: gen.Config, tau: float, q, k, v, heads=1, rows_per_head=12, seed=0):
    """Time the oracle on a bounded sample and extrapolate to one full step.

    Sample: the full search for `heads` heads (every sampled row of the head) and
    the sparse attention of `rows_per_head` query-block rows of each of those
    heads, over the oracle's own mask.  Full-step time = search time x H/heads +
    attention time / (visited blocks of the sampled rows) x (visited blocks of
    the whole layer, estimated from the sampled heads' masks x H/heads).
    """
    import oracle
    Nb = cfg.L // cfg.B
    g = cfg.H // cfg.Hkv
    rng = np.random.default_rng(seed)
    t_search = t_attn = 0.0
    blocks_sampled = blocks_head_total = 0
    for hs in range(heads):
        h = (hs * 7) % cfg.H
        kv = h // g
        Qh = gen.bf16_bits_to_f32(q[:, h:h + 1, :])
        Kh = gen.bf16_bits_to_f32(k[:, kv:kv + 1, :])
        Vh = gen.bf16_bits_to_f32(v[:, kv:kv + 1, :])
        t0 = time.perf_counter()
        count, idx, _ = oracle.rr_search(Qh, Kh, cfg.B, cfg.S, tau)
        t_search += time.perf_counter() - t0
        blocks_head_total += int(count.sum())
        rows = sorted(set([Nb - 1] + [int(x) for x in rng.integers(0, Nb, rows_per_head - 1)]))
        t0 = time.perf_counter()
        for I in rows:
            oracle.sparse_attention_block(Qh, Kh, Vh, 0, I, idx[0, I, :count[0, I]], cfg.B)
        t_attn += time.perf_counter() - t0
        blocks_sampled += int(sum(count[0, I] for I in rows))
    scale_heads = cfg.H / heads
    total_blocks = blocks_head_total * scale_heads
    step_s = t_search * scale_heads + t_attn / max(blocks_sampled, 1) * total_blocks
    flops = block_flops(cfg, total_blocks)
    return {
        "value": flops / step_s / 1e12,
        "unit": "TFLOP/s",
        "cores": blas_threads(),
        "kind": "oracle",
        "sample": (f"fp64 numpy oracle: full search of {heads} head(s) + attention of "
                   f"{rows_per_head} query-block rows per sampled head ({blocks_sampled} visited blocks), "
                   f"extrapolated to all {cfg.H} heads / {int(total_blocks)} visited blocks; "
                   f"measured {t_search + t_attn:.1f} s, extrapolated step {step_s:.1f} s"),
        "step_s": step_s,
        "measured_s": t_search + t_attn,
    }


def run_reference(args, cfg, tau, world):
    q, k, v = gen.make_config(cfg)
    measured, extrapolated, rates = [], [], []
    res = None
    for it in range(args.warmup + args.steps):
        res = oracle_sample(cfg, tau, q, k, v, heads=args.ref_heads, rows_per_head=args.ref_rows, seed=it)
        if it >= args.warmup:
            measured.append(res["measured_s"])
            extrapolated.append(res["step_s"])
            rates.append(res["value"])
    # a reference step is one bounded sample of the workload: ms_per_step is the
    # time such a step took; the rate (TFLOP/s over visited blocks) is the
    # sample's, extrapolated to the layer's work, and the time a whole layer
    # would take at that rate is reported beside it, not as a step
    value = statistics.mean(rates)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(measured) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(cfg, tau),
        "extrapolated_full_layer_ms": statistics.mean(extrapolated) * 1e3,
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": res["cores"], "nproc": os.cpu_count(),
                         "kind": "oracle",
                         "sample": res["sample"] + "; each step is one such sample (ms_per_step is its measured "
                                                   "time; the whole layer is not run)"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- ranks
def aggregate(total_ms: float, e2e_ms: float, flops: float, world: int, device) -> tuple:
    """Max over ranks of the timed regions, sum over ranks of the work.

    Every rank calls this exactly once, after its own timing, so all ranks take
    the same collective steps in the same order."""
    import torch
    t = torch.tensor([total_ms, e2e_ms], dtype=torch.float64, device=device)
    w = torch.tensor([flops], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(w, op=dist.ReduceOp.SUM)
    return float(t[0]), float(t[1]), float(w[0])


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"rr_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        load = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- GPU arm
def run_ours(args, cfg, tau, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import dynamic_block_sparse_rr_b200 as rr

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    q, k, v = gen.make_config(cfg, seed=cfg.seed + rank)
    to_pinned = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()
    qh, kh, vh = to_pinned(q), to_pinned(k), to_pinned(v)
    qd, kd, vd = qh.to(dev), kh.to(dev), vh.to(dev)
    L, H, Hkv, d, B, S = cfg.L, cfg.H, cfg.Hkv, cfg.d, cfg.B, cfg.S
    Nb = L // B
    ws = rr.workspace(L, H, Hkv, d, B, S, dev)
    count, idx = rr.empty_mask(H, Nb, dev)
    o = torch.empty_like(qd)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        rr.search(qd, kd, B, S, tau, count=count, idx=idx, ws=ws)
        if ev is not None:
            ev[1].record(stream)
        rr.sparse_attn(qd, kd, vd, count, idx, B, out=o, ws=ws)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if rr.check_status(ws) != rr.RR_OK:
        raise RuntimeError("device-side status after warm-up: %d" % rr.check_status(ws))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local_rank)
    clocks.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    status = rr.check_status(ws)
    if status != rr.RR_OK:
        raise RuntimeError("device-side status %d" % status)
    total_ms = t_start.elapsed_time(t_end)
    search_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    attn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    visited = int(count.sum().item())
    flops = block_flops(cfg, visited)
    # search, top-tau (one launch per row-length class: rows up to 256, 512 and
    # 1024 blocks, and longer), attention
    nb = cfg.L // cfg.B
    gpu_launches = (2 + 1 + (nb > 256) + (nb > 512) + (nb > 1024)) * args.steps

    # dense baseline: the same attention kernel with every causal block on.  The
    # sparse and dense launches alternate, so that both see the same clocks (the
    # power-capped clock drifts over a run); the speedup compares those two.
    dense_ms = None
    speedup = None
    alt_reading = None
    if not args.no_dense:
        cd, idd = rr.empty_mask(H, Nb, dev)
        rr.search(qd, kd, B, S, 1.0, count=cd, idx=idd, ws=ws)
        rr.sparse_attn(qd, kd, vd, cd, idd, B, out=o, ws=ws)
        torch.cuda.synchronize(dev)

        def one(c, i):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            rr.sparse_attn(qd, kd, vd, c, i, B, out=o, ws=ws)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            return e0.elapsed_time(e1)

        # the alternative reading of the key side (stride-mean keys): its mask,
        # search time and attention time, in the same interleaving
        ws_mk = rr.workspace(L, H, Hkv, d, B, S, dev, flags=rr.VAR_MEAN_KEYS)
        cm, im = rr.empty_mask(H, Nb, dev)
        rr.search_variant(qd, kd, B, S, tau, rr.VAR_MEAN_KEYS, cm, im, ws=ws_mk)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(3):
            rr.search_variant(qd, kd, B, S, tau, rr.VAR_MEAN_KEYS, cm, im, ws=ws_mk)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        mk_search_ms = e0.elapsed_time(e1) / 3
        if rr.check_status(ws_mk) != rr.RR_OK:
            raise RuntimeError("device-side status of the stride-mean search")

        sp, de, mk = [], [], []
        for _ in range(2):
            sp.append(one(count, idx))
            de.append(one(cd, idd))
            mk.append(one(cm, im))
        dense_ms = statistics.mean(de)
        speedup = dense_ms / (search_ms + statistics.mean(sp))
        dense_blocks = H * Nb * (Nb + 1) // 2
        dense_tflops = block_flops(cfg, dense_blocks) / (dense_ms / 1e3) / 1e12
        mk_visited = int(cm.sum().item())
        alt_reading = {"mean_keys": {
            "what": "key side of a stride = mean of its S keys (rr_search_variant RR_VAR_MEAN_KEYS)",
            "search_ms": mk_search_ms, "attn_ms": statistics.mean(mk),
            "visited_fraction": mk_visited / dense_blocks,
            "speedup_vs_dense": dense_ms / (mk_search_ms + statistics.mean(mk))},
            "sampled_keys_default": {"search_ms": search_ms, "attn_ms_interleaved": statistics.mean(sp),
                                     "visited_fraction": visited / dense_blocks, "speedup_vs_dense": speedup}}
        del cd, idd, cm, im, ws_mk

    decode = None if args.no_decode else measure_decode(args, rr, cfg, tau, qd, kd, vd, dev, stream)

    # end to end through the public API with host buffers: rr_attention_host
    # copies q, k, v in and o out (page-locked host memory) inside the call,
    # pipelined against the kernels item by item
    oh = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(1, min(args.steps, 2))
    ws_host = torch.empty(rr.workspace_size_host(L, H, Hkv, d, B, S), dtype=torch.uint8, device=dev)
    copy_stream = torch.cuda.Stream(device=dev)
    rr.attention_host(qh, kh, vh, B, S, tau, out=oh, count=count, idx=idx, ws=ws_host, stream=stream,
                      copy_stream=copy_stream)   # warm-up (first-call setup outside the timed region)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        rr.attention_host(qh, kh, vh, B, S, tau, out=oh, count=count, idx=idx, ws=ws_host, stream=stream,
                          copy_stream=copy_stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if rr.check_status(ws_host) != rr.RR_OK:
        raise RuntimeError("device-side status after the end-to-end run")
    del ws_host
    total_ms_max, e2e_ms_max, flops_all = aggregate(total_ms, e2e_ms, flops, world, dev)
    ms_per_step = total_ms_max / args.steps
    value = flops_all / (ms_per_step / 1e3) / 1e12
    e2e_value = flops_all / (e2e_ms_max / 1e3) / 1e12
    h2d = (qh.numel() + kh.numel() + vh.numel()) * 2
    d2h = oh.numel() * 2

    peaks = measured_peaks()
    peak = peaks["bf16_tflops_sustained"] or peaks["bf16_tflops"]
    achieved = flops / (attn_ms / 1e3) / 1e12
    sb = search_bytes(cfg, visited)
    search_hbm = {"bytes": sb["total"], "gbs": sb["total"] / (search_ms / 1e3) / 1e9,
                  "frac_of_hbm": sb["total"] / (search_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                  "peak_gbs": peaks["hbm_gbs"], "parts": sb,
                  "note": "algorithmic bytes of the whole search stage (sampled q rows and keys read once, "
                          "block-mass write and read, count/idx write) over its CUDA-event time; the stage "
                          "is bound by tensor and exp work, not by HBM"}
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": kernel_traffic_bytes(), "kernel": "bsfa_kernel<128,128>",
                "peak_kind": f"bf16 dense, sustained ({peaks['source']})"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res = oracle_sample(cfg, tau, q, k, v, heads=args.ref_heads, rows_per_head=args.ref_rows)
        cpu = {k2: res[k2] for k2 in ("value", "unit", "cores", "kind", "sample")}
        cpu.update({"nproc": os.cpu_count(), "cores_are": "BLAS threads the oracle ran with",
                    "single_thread_tiny_s": single_thread_tiny_s(),
                    "measured_sample_s": res["measured_s"]})

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded generator, planted structure)",
            "config": workload_config(cfg, tau),
            "search_ms": search_ms, "attn_ms": attn_ms, "search_share": search_ms / (search_ms + attn_ms),
            "search_hbm": search_hbm, "alternative_reading": alt_reading, "decode": decode,
            "dense_attn_ms": dense_ms, "dense_attn_tflops": dense_tflops if dense_ms else None,
            "speedup_vs_dense": speedup,
            "visited_blocks": visited, "visited_fraction": visited / (H * Nb * (Nb + 1) / 2),
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "ms_per_step": e2e_ms_max,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "path": "rr_attention_host: pinned host q/k/v/o, copies pipelined per item "
                            "(a kv head; a single query head for the first and last item)"},
            "gpu_launches": gpu_launches, "clocks": clk, "roofline": roofline, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


def decode_bytes(cfg: gen.Config, lens, count, idx) -> dict:
    """Algorithmic HBM bytes of one decode step: each head's sampled keys up to
    its query, the union over a kv group's heads of the kept K and V blocks (the
    attention kernel loads a kept block once per group), q and o."""
    H, Hkv, d, B, S = cfg.H, cfg.Hkv, cfg.d, cfg.B, cfg.S
    g = H // Hkv
    row = d * 2
    keys = kv = 0
    for n, ln in enumerate(lens):
        t = ln - 1
        for h in range(H):
            off = h % S
            keys += ((t - off) // S + 1 if t >= off else 0) * row
        for c in range(Hkv):
            union = set()
            for h in range(c * g, (c + 1) * g):
                union.update(idx[n, h, :count[n, h]].tolist())
            for J in union:
                kv += 2 * (min(B, t + 1 - J * B)) * row
    qo = 2 * len(lens) * H * row
    return {"sampled_keys": keys, "kv_blocks": kv, "q_o": qo, "total": keys + kv + qo}


def measure_decode(args, rr, cfg, tau, qd, kd, vd, dev, stream):
    """Decode step of the layer for a batch of sequences: caches are copies of
    the resident layer's k and v, sequence n holds L - 1000 n keys and its query
    is the layer's query at its last position.  Times rr_decode (CUDA events)
    at tau and at tau = 1 (every block kept), interleaved."""
    import torch
    Nd = args.decode_batch
    L, H, Hkv, d, B, S = cfg.L, cfg.H, cfg.Hkv, cfg.d, cfg.B, cfg.S
    lens = [L - 1000 * n for n in range(Nd)]
    kc = kd.unsqueeze(0).expand(Nd, -1, -1, -1).contiguous()
    vc = vd.unsqueeze(0).expand(Nd, -1, -1, -1).contiguous()
    qq = torch.stack([qd[ln - 1] for ln in lens]).contiguous()
    ld = torch.tensor(lens, dtype=torch.int32, device=dev)
    ws = torch.empty(rr.decode_workspace_size(Nd, L, H, Hkv, d, B, S), dtype=torch.uint8, device=dev)
    out = torch.empty_like(qq)
    cnt = torch.empty((Nd, H), dtype=torch.int32, device=dev)
    idx = torch.empty((Nd, H, L // B), dtype=torch.int32, device=dev)
    cnt1, idx1 = torch.empty_like(cnt), torch.empty_like(idx)

    def timed(t_, c_, i_, reps=10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            rr.decode(qq, kc, vc, ld, B, S, t_, out=out, count=c_, idx=i_, ws=ws, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / reps

    cnt_g, idx_g = torch.empty_like(cnt), torch.empty_like(idx)

    def timed_g(c_, i_, reps=10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            rr.decode(qq, kc, vc, ld, B, S, tau, out=out, count=c_, idx=i_, ws=ws, stream=stream,
                      flags=rr.VAR_GQA_MASK)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / reps

    for _ in range(3):
        timed(tau, cnt, idx, 1)
        timed(1.0, cnt1, idx1, 1)
        timed_g(cnt_g, idx_g, 1)
    sp, de, gp = [], [], []
    for _ in range(3):
        sp.append(timed(tau, cnt, idx))
        de.append(timed(1.0, cnt1, idx1))
        gp.append(timed_g(cnt_g, idx_g))
    if rr.check_status(ws) != rr.RR_OK:
        raise RuntimeError("device-side status of the decode step")
    ms, dense_ms, g_ms = statistics.median(sp), statistics.median(de), statistics.median(gp)
    peak = measured_peaks()["hbm_gbs"]
    causal = sum(H * ((ln - 1) // B + 1) for ln in lens)

    def summary(c_t, i_t, t_ms):
        c_h, i_h = c_t.cpu().numpy(), i_t.cpu().numpy()
        byts = decode_bytes(cfg, lens, c_h, i_h)
        gbs = byts["total"] / (t_ms / 1e3) / 1e9
        return {"us_per_step": t_ms * 1e3, "speedup_vs_dense": dense_ms / t_ms,
                "visited_fraction": float(c_h.sum()) / causal,
                "hbm": {"bytes": byts["total"], "gbs": gbs, "frac_of_hbm": gbs / peak, "peak_gbs": peak,
                        "parts": byts}}

    # the step captured once in a CUDA graph and replayed, as a serving loop would;
    # and the latency of one step with the host waiting for it, eager and replayed
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for _ in range(2):
            rr.decode(qq, kc, vc, ld, B, S, tau, out=out, count=cnt, idx=idx, ws=ws)
    stream.wait_stream(side)
    with torch.cuda.graph(graph):
        rr.decode(qq, kc, vc, ld, B, S, tau, out=out, count=cnt, idx=idx, ws=ws)

    def timed_graph(reps=10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / reps

    def latency(fn, n=30):
        ts = []
        for _ in range(n):
            torch.cuda.synchronize(dev)
            t0 = time.perf_counter()
            fn()
            torch.cuda.synchronize(dev)
            ts.append(time.perf_counter() - t0)
        return statistics.median(ts) * 1e3

    timed_graph(3)
    graph_ms = statistics.median([timed_graph() for _ in range(3)])
    lat_eager = latency(lambda: rr.decode(qq, kc, vc, ld, B, S, tau, out=out, count=cnt, idx=idx, ws=ws,
                                          stream=stream))
    lat_graph = latency(graph.replay)
    if rr.check_status(ws) != rr.RR_OK:
        raise RuntimeError("device-side status of the replayed decode step")
    del graph

    res = {"what": "rr_decode: one new token per sequence over its KV cache (search, block-sparse attention "
                   "with the partials merged); caches are copies of this layer, sequence n holds L - 1000 n keys",
           "batch": Nd, "dense_us_per_step": dense_ms * 1e3}
    res.update(summary(cnt, idx, ms))
    res["gqa_mask"] = summary(cnt_g, idx_g, g_ms)
    res["cuda_graph"] = {"us_per_step": graph_ms * 1e3,
                         "latency_us": {"eager": lat_eager * 1e3, "graph": lat_graph * 1e3},
                         "note": "one step captured in a CUDA graph and replayed back to back; latency is the "
                                 "host-clock median of one step with a synchronize on each side"}
    del kc, vc, ws
    torch.cuda.empty_cache()
    return res


def run_decode_only(args, cfg, tau):
    import torch
    import dynamic_block_sparse_rr_b200 as rr
    dev = torch.device("cuda", 0)
    q, k, v = gen.make_config(cfg)
    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    del q, k, v
    res = measure_decode(args, rr, cfg, tau, qd, kd, vd, dev, torch.cuda.current_stream(dev))
    print(json.dumps({"diagnostic": "decode step", "config": workload_config(cfg, tau), "decode": res}), flush=True)


def run_recall(args, cfg, taus, variants=(0,)):
    """Mask diagnostics: per tau, the RR mask's visited fraction and its recall of
    the exact attention mass, next to the exact Top-tau selection (the search at
    stride 1).  Prints one JSON line."""
    import torch
    import dynamic_block_sparse_rr_b200 as rr
    q, k, _ = gen.make_config(cfg)
    dev = torch.device("cuda", 0)
    qd = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).to(dev)
    kd = torch.from_numpy(k.view(np.int16)).view(torch.bfloat16).to(dev)
    Nb = cfg.L // cfg.B
    causal = cfg.H * Nb * (Nb + 1) / 2
    m_exact = rr.exact_block_mass(qd, kd, cfg.B)
    rows = []
    for tau in taus:
        c_ex, i_ex = rr.search(qd, kd, cfg.B, 1, tau)
        rec_ex = rr.mask_recall(m_exact, c_ex, i_ex)[:, :-1]
        row = {"tau": tau, "visited_exact": c_ex.sum().item() / causal, "recall_exact_mean": rec_ex.mean().item()}
        for flags in variants:
            c_rr, i_rr = rr.search_variant(qd, kd, cfg.B, cfg.S, tau, flags)
            rec_rr = rr.mask_recall(m_exact, c_rr, i_rr)[:, :-1]
            tag = variant_name(flags)
            row.update({f"visited_{tag}": c_rr.sum().item() / causal, f"recall_{tag}_mean": rec_rr.mean().item(),
                         f"recall_{tag}_min": rec_rr.min().item()})
        rows.append(row)
    # search time per variant (device events; one warm call first)
    search_ms = {}
    for flags in variants:
        ws = rr.workspace(cfg.L, cfg.H, cfg.Hkv, cfg.d, cfg.B, cfg.S, dev, flags=flags)
        count, idx = rr.empty_mask(cfg.H, Nb, dev)
        rr.search_variant(qd, kd, cfg.B, cfg.S, taus[0], flags, count, idx, ws=ws)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(5):
            rr.search_variant(qd, kd, cfg.B, cfg.S, taus[0], flags, count, idx, ws=ws)
        e1.record()
        torch.cuda.synchronize()
        search_ms[variant_name(flags)] = e0.elapsed_time(e1) / 5
        if rr.check_status(ws) != rr.RR_OK:
            raise RuntimeError("device-side wait timed out")
    torch.cuda.synchronize()
    print(json.dumps({"diagnostic": "mask recall of exact attention mass (last query block excluded)",
                      "config": workload_config(cfg, taus[0]), "rows": rows, "search_ms": search_ms}), flush=True)


def run_sweep(args):
    """Per-config table (diagnostic, not the contract line): for every config
    and tau, search and attention ms (mean of `steps` after `warmup`), attention
    TFLOP/s over visited blocks and its share of the measured sustained peak,
    the visited fraction, and the speedup over the same kernel on every causal
    block.  One JSON line per (config, tau, sampling variant); `--variants`
    picks the variants (0: the plain search)."""
    import torch
    import dynamic_block_sparse_rr_b200 as rr
    dev = torch.device("cuda", 0)
    peaks = measured_peaks()
    peak = peaks["bf16_tflops_sustained"] or peaks["bf16_tflops"]
    variants = [int(f) for f in args.variants.split(",")]
    for name in ("llama16k", "llama32k", "video64k", "llama128k"):
        cfg = gen.CONFIGS[name]
        q, k, v = gen.make_config(cfg)
        to_dev = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
        qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
        del q, k, v
        L, H, Hkv, d, B, S = cfg.L, cfg.H, cfg.Hkv, cfg.d, cfg.B, cfg.S
        Nb = L // B
        # room for every variant asked for and for the plain search (the sizes differ either way)
        ws_bytes = max(rr.workspace_size_variant(L, H, Hkv, d, B, S, f) for f in set(variants) | {0})
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        count, idx = rr.empty_mask(H, Nb, dev)
        o = torch.empty_like(qd)
        stream = torch.cuda.current_stream(dev)

        def timed(fn, reps):
            for _ in range(args.warmup):
                fn()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                fn()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            return e0.elapsed_time(e1) / reps

        cd, idd = rr.empty_mask(H, Nb, dev)
        rr.search(qd, kd, B, S, 1.0, count=cd, idx=idd, ws=ws)
        for tau, flags in [(t, f) for t in cfg.taus for f in variants]:
            search_ms = timed(lambda: rr.search_variant(qd, kd, B, S, tau, flags, count, idx, ws=ws), args.steps)
            # sparse and dense attention alternate, round by round, so that both
            # see the same clocks (the power-capped clock drifts over a run)
            a_ms, d_ms = [], []
            for _ in range(3):
                a_ms.append(timed(lambda: rr.sparse_attn(qd, kd, vd, count, idx, B, out=o, ws=ws), args.steps))
                d_ms.append(timed(lambda: rr.sparse_attn(qd, kd, vd, cd, idd, B, out=o, ws=ws), args.steps))
            attn_ms, dense_ms = statistics.mean(a_ms), statistics.mean(d_ms)
            if rr.check_status(ws) != rr.RR_OK:
                raise RuntimeError("device-side status %d" % rr.check_status(ws))
            visited = int(count.sum().item())
            tf = block_flops(cfg, visited) / (attn_ms / 1e3) / 1e12
            print(json.dumps({"sweep": name, "tau": tau, "variant": variant_name(flags), "search_ms": search_ms, "attn_ms": attn_ms,
                              "step_ms": search_ms + attn_ms, "attn_tflops": tf, "attn_frac_of_sustained": tf / peak,
                              "visited_fraction": visited / (H * Nb * (Nb + 1) / 2), "dense_attn_ms": dense_ms,
                              "speedup_vs_dense": dense_ms / (search_ms + attn_ms),
                              "search_share": search_ms / (search_ms + attn_ms)}), flush=True)
        del qd, kd, vd, ws, count, idx, o, cd, idd
        torch.cuda.empty_cache()


def variant_name(flags: int) -> str:
    """rr: the plain search (sampled keys); rot / mk / gqa: the sampling variants of
    rr_search_variant (rotation, stride-mean keys, one mask per GQA group)."""
    parts = [n for bit, n in ((1, "rot"), (2, "mk"), (4, "gqa")) if flags & bit]
    return "+".join(parts) if parts else "rr"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="llama128k", choices=sorted(gen.CONFIGS))
    ap.add_argument("--tau", type=float, default=None)
    ap.add_argument("--ref-heads", type=int, default=2, help="oracle sample: heads searched in full")
    ap.add_argument("--ref-rows", type=int, default=16, help="oracle sample: attention rows per head")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode-step measurement")
    ap.add_argument("--decode-batch", type=int, default=8, help="sequences per decode step")
    ap.add_argument("--decode", action="store_true",
                    help="decode-step measurement only (one JSON line), on the chosen config's layer")
    ap.add_argument("--recall", action="store_true",
                    help="mask diagnostics instead of timing: recall of exact attention mass per tau")
    ap.add_argument("--sweep", action="store_true",
                    help="per-config table instead of the contract line: every config and tau")
    ap.add_argument("--variants", default="0",
                    help="with --recall or --sweep: comma-separated sampling-variant flags (1 rotate, "
                         "2 stride-mean keys, 4 GQA mask; 0 the plain search)")
    args = ap.parse_args()
    if args.warmup < 3:
        print("note: fewer than 3 warm-up steps requested", file=sys.stderr)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = gen.CONFIGS[args.config]
    tau = args.tau if args.tau is not None else cfg.tau

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, cfg, tau, world)
        return
    if args.sweep:
        if rank == 0:
            run_sweep(args)
        return
    if args.decode:
        if rank == 0:
            run_decode_only(args, cfg, tau)
        return
    if args.recall:
        if rank == 0:
            run_recall(args, cfg, list(cfg.taus) if args.tau is None else [tau],
                       [int(x) for x in args.variants.split(",")])
        return

    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, cfg, tau, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
