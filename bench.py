#!/usr/bin/env python
"""Throughput of the fused LongFlow decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

One step = one call of lf_decode_step: attention + score + eviction for a
whole batch, one kernel launch.  Default workload (the throughput point):
batch 64, 32 query / 8 KV heads, head_dim 128, bf16 cache, budget 4096,
sink 4, window 128, full cache.  Every step's new token is distinct (drawn
on the device); the queries cycle through 256 seeded sets.  The 1 GiB KV
cache read per step is far larger than L2, so no L2 flush is needed between
steps.  At least 3 warm-up steps run, whatever --warmup says.

Rank 0 prints ONE JSON line.  Under torchrun each rank runs its own batch
(weak scaling, no collective on the data path); time is the max over ranks.
`--impl reference` times the CPU oracle (the reference arm of this build)
on bounded samples of the same workload.
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

for _v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
    os.environ.setdefault(_v, "1")  # the CPU oracle runs single-threaded

import numpy as np  # noqa: E402

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused decode steps/s per layer and achieved HBM GB/s vs B200 peak"
UNIT = "steps/s"
FALLBACK_HBM_GBS = 6650.0
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "fused_decode_throughput_b64_n4096.md")


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--config", default="throughput")
    ap.add_argument("--split", type=int, default=0, help="CTAs per row (0 = automatic)")
    ap.add_argument("--kv", default="bf16", choices=["bf16", "fp8"],
                    help="KV cache storage: bf16, or E4M3 codes with one scale per tensor")
    ap.add_argument("--k-scale", type=float, default=1.0)
    ap.add_argument("--v-scale", type=float, default=1.0)
    ap.add_argument("--attention-only", action="store_true",
                    help="time the no-eviction control: the same kernel with scoring and "
                         "eviction compiled out (lf_decode_attention*)")
    ap.add_argument("--score", default="mean_prob", choices=["mean_prob", "alpha_l1v"],
                    help="eviction score: head-averaged probability (default) or the "
                         "page's attention weight times the value L1 norm")
    ap.add_argument("--batch", type=int, default=0, help="override the batch (profiling cases)")
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="replay a captured CUDA graph of the timed steps; its kernel nodes "
                         "hold fixed inputs, so new tokens repeat every graph length")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every step from Python (the default)")
    return ap.parse_args()


# ------------------------------------------------------------------ bytes

def algorithmic_bytes(cfg, filled, kv_bytes: int = 2) -> dict:
    """Bytes one step must move: the K and V of every filled slot once, plus
    every write (fp32 output, the new token's K/V row, its position, the
    evicted index).  q, k_new, v_new and the position table are read too;
    they are listed apart (under 1%).  filled: slots per row, or per
    sequence ([B], ragged batches).  kv_bytes: bytes per cached element
    (2 for bf16, 1 for E4M3)."""
    rows = cfg.batch * cfg.hkv
    kv_read = int(np.sum(np.broadcast_to(np.asarray(filled, np.int64), (cfg.batch,)))) \
        * cfg.hkv * cfg.head_dim * kv_bytes * 2
    writes = (cfg.batch * cfg.hq * cfg.head_dim * 4 + rows * cfg.head_dim * kv_bytes * 2 + rows * 4
              + rows * 4)
    other_reads = (cfg.batch * cfg.hq * cfg.head_dim * 2 + rows * cfg.head_dim * 2 * 2
                   + rows * cfg.budget * 4)
    return {"kv_read": kv_read, "writes": writes, "algorithmic": kv_read + writes,
            "other_reads": other_reads}


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy burst)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s, earlier measurement on this pool)"


def kernel_hash() -> str:
    """Hash of every kernel source file (the library's csrc directory)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "attention_lf_decode_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(csrc, name), "rb") as fh:
                h.update(name.encode() + b"\0" + fh.read())
    return h.hexdigest()[:16]


def ncu_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source (else None)."""
    try:
        txt = open(PROFILE_SUMMARY).read()
    except OSError:
        return None
    m = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", txt)
    t = re.search(r"traffic_bytes_per_launch:\s*([0-9.e+]+)", txt)
    if not m or not t or m.group(1) != kernel_hash():
        return None
    return float(t.group(1))


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, enabled: bool = True):
        self.proc = None
        self.idx = gpu_index
        if enabled:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------------ oracle

def oracle_rate(cfg, gen, kpre_bits, vpre_bits, seconds: float, batch_sel, max_steps: int,
                score: str = "mean_prob", seq_budget=None, fp8_scales=None):
    """Time the CPU oracle, as it stands, on sampled batch entries; returns
    (full steps/s extrapolated from rows/s, sample description, steps run)."""
    import oracle
    from attention_lf_decode_b200 import synth
    kc, vc, pos = synth.prefill_layout(kpre_bits[batch_sel], vpre_bits[batch_sel], cfg.budget)
    K, V = synth.bf16_bits_to_f64(kc), synth.bf16_bits_to_f64(vc)
    if fp8_scales is not None:  # an E4M3 cache: the oracle steps on the codes
        K, V = oracle.quantize(K, fp8_scales[0]), oracle.quantize(V, fp8_scales[1])
    P = pos.astype(np.int64)
    del kc, vc
    rows = len(batch_sel) * cfg.hkv
    t_total, n = 0.0, 0
    while n < max_steps and (t_total < seconds or n == 0):
        qb, knb, vnb = gen.step_inputs(n)
        q = synth.bf16_bits_to_f64(qb[batch_sel])
        kn = synth.bf16_bits_to_f64(knb[batch_sel])
        vn = synth.bf16_bits_to_f64(vnb[batch_sel])
        t0 = time.perf_counter()
        nb = None if seq_budget is None else seq_budget[batch_sel]
        if fp8_scales is None:
            res = oracle.decode_step(K, V, P, q, kn, vn, cfg.sink, cfg.window, score=score,
                                     seq_budget=nb)
        else:
            res = oracle.decode_step_fp8(K, V, P, q, kn, vn, cfg.sink, cfg.window, *fp8_scales,
                                         score=score, seq_budget=nb)
        t_total += time.perf_counter() - t0
        K, V, P = res.kcache, res.vcache, res.pos
        n += 1
    per_row = t_total / (n * rows)
    full_rows = cfg.batch * cfg.hkv
    rate = 1.0 / (per_row * full_rows)
    sample = (f"{n} step(s) on {len(batch_sel)} of {cfg.batch} batch entries "
              f"({rows} of {full_rows} rows), {t_total:.1f} s; steps/s scaled to all rows")
    return rate, sample, n


def threads_used():
    v = os.environ.get("OMP_NUM_THREADS") or os.environ.get("OPENBLAS_NUM_THREADS")
    return int(v) if v and v.isdigit() else os.cpu_count()


# ------------------------------------------------------------------ main

def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    from attention_lf_decode_b200 import synth
    cfg = synth.CONFIGS[args.config]
    if args.batch:
        cfg = cfg.with_(batch=args.batch)
    workload = (f"{cfg.name}: batch {cfg.batch}, {cfg.hq} query / {cfg.hkv} KV heads, "
                f"head_dim {cfg.head_dim}, bf16 KV cache, budget {cfg.budget}, sink {cfg.sink}, "
                f"window {cfg.window}, prefill {cfg.prefill}")

    if args.impl == "reference":
        return reference_arm(args, cfg, workload, world, rank)

    import torch
    import torch.distributed as dist
    from attention_lf_decode_b200 import binding, scaling

    torch.cuda.set_device(local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))

    # per-rank synthetic data: the same recipe, a different seed per rank
    rcfg = scaling.rank_config(cfg, rank)
    gen = synth.SynthDecode(rcfg)
    t0 = time.time()
    kpre, vpre = gen.prefill()
    log(f"[rank {rank}] prefill drawn in {time.time() - t0:.1f} s")
    n_inputs = min(cfg.steps, 256)
    inputs = [gen.step_inputs(s) for s in range(n_inputs)]

    stream = torch.cuda.current_stream()
    h = binding.lf_init(cfg.batch, cfg.hq, cfg.hkv, cfg.head_dim, cfg.budget, stream)
    if args.split:
        binding.lf_set_split(h, args.split)
    score_code = {"mean_prob": binding.LF_SCORE_MEAN_PROB,
                  "alpha_l1v": binding.LF_SCORE_ALPHA_L1V}[args.score]
    binding.lf_set_score(h, score_code)
    split = binding.lf_get_split(h, cfg.budget)
    dev = "cuda"
    fp8 = args.kv == "fp8"
    kv_bytes = 1 if fp8 else 2
    kcache = torch.empty((cfg.batch, cfg.hkv, cfg.budget, cfg.head_dim),
                         dtype=torch.uint8 if fp8 else torch.bfloat16, device=dev)
    vcache = torch.empty_like(kcache)
    pos = torch.empty((cfg.batch, cfg.hkv, cfg.budget), dtype=torch.int32, device=dev)
    if fp8:
        binding.lf_prefill_cache_fp8(h, binding.bf16_from_bits(kpre), binding.bf16_from_bits(vpre),
                                     cfg.prefill, kcache, vcache, pos, cfg.budget,
                                     args.k_scale, args.v_scale)
    else:
        binding.lf_prefill_cache(h, binding.bf16_from_bits(kpre), binding.bf16_from_bits(vpre),
                                 cfg.prefill, kcache, vcache, pos, cfg.budget)
    q_all = torch.stack([binding.bf16_from_bits(x[0]) for x in inputs])
    kn_all = torch.stack([binding.bf16_from_bits(x[1]) for x in inputs])
    vn_all = torch.stack([binding.bf16_from_bits(x[2]) for x in inputs])
    out = torch.empty((cfg.batch, cfg.hq, cfg.head_dim), dtype=torch.float32, device=dev)
    ev = torch.empty((cfg.batch, cfg.hkv), dtype=torch.int32, device=dev)
    # ragged batch: a budget per sequence (the prefill fills every slot; the
    # slots beyond a sequence's budget are never read)
    nb_host = gen.seq_budgets()
    nb_dev = None if nb_host is None else torch.from_numpy(nb_host).to(dev)

    def run(q, kn, vn, out=out, ev=ev):
        if args.attention_only:
            if fp8:
                binding.lf_decode_attention_fp8(h, q, kn, vn, kcache, vcache, pos, cfg.budget,
                                                args.k_scale, args.v_scale, out, nb_dev)
            elif nb_dev is None:
                binding.lf_decode_attention(h, q, kn, vn, kcache, vcache, pos, cfg.budget, out)
            else:
                binding.lf_decode_attention_ragged(h, q, kn, vn, kcache, vcache, pos, cfg.budget,
                                                   nb_dev, out)
        elif fp8:
            binding.lf_decode_step_fp8(h, q, kn, vn, kcache, vcache, pos, cfg.budget, cfg.sink,
                                       cfg.window, args.k_scale, args.v_scale, out, ev, nb_dev)
        elif nb_dev is None:
            binding.lf_decode_step(h, q, kn, vn, kcache, vcache, pos, cfg.budget, cfg.sink,
                                   cfg.window, out, ev)
        else:
            binding.lf_decode_step_ragged(h, q, kn, vn, kcache, vcache, pos, cfg.budget, nb_dev,
                                          cfg.sink, cfg.window, out, ev)

    # Every step's new token is distinct: re-inserting a token already cached
    # would tie its score exactly with its copy's and send that row through
    # the fp64 rescoring, which real decoding does not do.  The new K/V of the
    # steps are drawn on the device with the synthetic recipe (N(0, 1); key
    # outliers along u when the config has them); the queries cycle through
    # the seeded sets.
    u_dev = torch.from_numpy(gen.u).to(dev)

    def draw_new_kv(n, seed):
        g = torch.Generator(device=dev)
        g.manual_seed(seed)
        shape = (n, cfg.batch, cfg.hkv, cfg.head_dim)
        kn = torch.empty(shape, dtype=torch.bfloat16, device=dev)
        vn = torch.empty_like(kn)
        for c0 in range(0, n, 1024):  # bounded fp32 scratch
            c1 = min(n, c0 + 1024)
            k = torch.randn((c1 - c0,) + shape[1:], generator=g, device=dev)
            if cfg.new_key_outliers:
                m = torch.rand((c1 - c0,) + shape[1:3] + (1,), generator=g, device=dev)
                k += (m < cfg.key_outlier_frac).float() * (cfg.key_outlier_mag * u_dev)
            kn[c0:c1] = k.to(torch.bfloat16)
            vn[c0:c1] = torch.randn((c1 - c0,) + shape[1:], generator=g, device=dev).to(torch.bfloat16)
        return kn, vn

    warmup = max(args.warmup, 3)  # at least 3 untimed warm-up steps
    n_fresh = warmup + args.steps
    kn_u, vn_u = draw_new_kv(n_fresh, 1000003 * cfg.seed + rank)

    def step(i):
        run(q_all[i % n_inputs], kn_u[i % n_fresh], vn_u[i % n_fresh])

    # warm-up
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    if binding.lf_get_status(h) != binding.LF_OK:
        raise RuntimeError(f"device status bits {binding.lf_status_bits(h)} after warm-up")

    # By default every timed step is launched from Python (the host runs
    # ahead of the ~0.2 ms kernels, so launches are not on the critical path);
    # --graph replays a captured CUDA graph instead.
    graph, glen = None, 0
    if args.graph and not args.no_graph:
        glen = max(d for d in range(1, min(args.steps, n_inputs) + 1) if args.steps % d == 0)
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        binding.lf_set_stream(h, cap)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            for i in range(glen):
                step(warmup + i)
        binding.lf_set_stream(h, stream)
        graph.replay()  # one untimed replay
        torch.cuda.synchronize()

    # timed region: K back-to-back steps, CUDA events on the launching stream
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank, enabled=not args.no_clocks)
    time.sleep(0.3 if not args.no_clocks else 0.0)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    if graph is not None:
        for _ in range(args.steps // glen):
            graph.replay()
    else:
        for i in range(args.steps):
            step(warmup + i)
    e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    if binding.lf_get_status(h) != binding.LF_OK:
        raise RuntimeError(f"device status bits {binding.lf_status_bits(h)} in the timed region")
    ms_max = scaling.max_over_ranks(ms, dev)
    ms_per_step = ms_max / args.steps
    value = scaling.whole_job_rate(world, args.steps, ms_max)

    # End to end, through the public call: every step copies its inputs from
    # pinned host memory to the device, runs lf_decode_step, copies out and
    # evicted_idx back to pinned host memory, and the host reads that result.
    # The steps are pipelined two deep into double-buffered device and host
    # buffers.  Host-to-device copies run on one copy stream and
    # device-to-host copies on another, so step i + 1's inputs arrive while
    # step i computes, and step i's results return while step i + 1
    # computes.  The host reads step i's result before it enqueues step
    # i + 2, which reuses step i's buffers (that read also orders the reuse).
    e2e = None
    if not args.no_e2e:
        hq = torch.from_numpy(np.stack([x[0] for x in inputs]).view(np.int16)).view(torch.bfloat16).pin_memory()
        ek, evv = draw_new_kv(args.e2e_steps + 3, 1000003 * cfg.seed + 7919 + rank)
        hk = ek.cpu().pin_memory()
        hv = evv.cpu().pin_memory()
        del ek, evv
        NBUF = 2
        cs_in = torch.cuda.Stream()   # host-to-device copies
        cs_out = torch.cuda.Stream()  # device-to-host copies
        d_in = [(torch.empty_like(q_all[0]), torch.empty_like(kn_all[0]), torch.empty_like(vn_all[0]))
                for _ in range(NBUF)]
        d_out = [out] + [torch.empty_like(out) for _ in range(NBUF - 1)]
        d_ev = [ev] + [torch.empty_like(ev) for _ in range(NBUF - 1)]
        h_out = [torch.empty(out.shape, dtype=torch.float32).pin_memory() for _ in range(NBUF)]
        h_ev = [torch.empty(ev.shape, dtype=torch.int32).pin_memory() for _ in range(NBUF)]
        ev_h2d = [torch.cuda.Event() for _ in range(NBUF)]
        ev_k = [torch.cuda.Event() for _ in range(NBUF)]
        ev_d2h = [torch.cuda.Event() for _ in range(NBUF)]
        pending = []  # buffers whose step's result the host has not read yet
        results = []
        n_e2e = args.e2e_steps

        def consume():
            b = pending.pop(0)
            ev_d2h[b].synchronize()
            results.append(float(h_out[b][0, 0, 0]))  # the host reads the step's result

        def e2e_step(i):
            b = i % NBUF
            j = i % n_inputs  # the query set
            jn = i % hk.shape[0]  # the step's own new token
            if len(pending) == NBUF:  # buffer b is free once its last step's result is read
                consume()
            with torch.cuda.stream(cs_in):
                for dst, src in zip(d_in[b], (hq[j], hk[jn], hv[jn])):
                    dst.copy_(src, non_blocking=True)
                ev_h2d[b].record(cs_in)
            stream.wait_event(ev_h2d[b])
            run(*d_in[b], out=d_out[b], ev=d_ev[b])
            ev_k[b].record(stream)
            with torch.cuda.stream(cs_out):
                cs_out.wait_event(ev_k[b])
                h_out[b].copy_(d_out[b], non_blocking=True)
                h_ev[b].copy_(d_ev[b], non_blocking=True)
                ev_d2h[b].record(cs_out)
            pending.append(b)

        for i in range(3):
            e2e_step(i)
        while pending:
            consume()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(cs_in)  # before the first step's input copies
        for i in range(n_e2e):
            e2e_step(3 + i)  # after the 3 warm-up steps' tokens
        a1.record(cs_out)  # after the last step's result copies
        while pending:
            consume()
        a1.synchronize()
        ems = scaling.max_over_ranks(a0.elapsed_time(a1), dev)
        h2d = sum(t.numel() for t in d_in[0]) * 2
        d2h = h_out[0].numel() * 4 + h_ev[0].numel() * 4
        e2e = {"value": scaling.whole_job_rate(world, n_e2e, ems), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": n_e2e,
               "ms_per_step": ems / n_e2e,
               "note": "per step: pinned H2D of q/k_new/v_new, lf_decode_step, D2H of out and "
                       "evicted_idx, host read of the result; pipelined two steps deep "
                       "(H2D and D2H on two copy streams, double-buffered inputs and "
                       "outputs); the KV cache stays resident"}
        if binding.lf_get_status(h) != binding.LF_OK:
            raise RuntimeError("device status after e2e")

    filled = min(cfg.budget, cfg.prefill) if nb_host is None else np.minimum(nb_host, cfg.prefill)
    by = algorithmic_bytes(cfg, filled, kv_bytes)
    if args.attention_only:  # the control writes nothing but out
        by["writes"] = cfg.batch * cfg.hq * cfg.head_dim * 4
        by["algorithmic"] = by["kv_read"] + by["writes"]
    kern_s = ms_per_step / 1e3  # one launch per step
    achieved = by["algorithmic"] / kern_s / 1e9
    peak, peak_src = measured_peak()
    traffic = ncu_traffic()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        rate, sample, _ = oracle_rate(cfg, gen, kpre, vpre, args.cpu_seconds, list(range(4)), 64,
                                      score=args.score, seq_budget=nb_host,
                                      fp8_scales=(args.k_scale, args.v_scale) if fp8 else None)
        cpu = {"value": rate, "unit": UNIT, "cores": threads_used(), "kind": "oracle",
               "sample": sample}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    binding.lf_destroy(h)
    if rank != 0:
        return 0

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {
            "workload": workload, "batch": cfg.batch, "hq": cfg.hq, "hkv": cfg.hkv,
            "head_dim": cfg.head_dim, "budget": cfg.budget, "sink": cfg.sink,
            "window": cfg.window,
            "kv_dtype": (f"e4m3 (k_scale {args.k_scale}, v_scale {args.v_scale})" if fp8 else "bf16"),
            "accumulate": "f32",
            "parallelism": f"dp{world} (batch per rank, no collective)",
            "split_ctas_per_row": split,
            "seq_budgets": (None if nb_host is None else
                            {"min": int(nb_host.min()), "max": int(nb_host.max()),
                             "mean": float(nb_host.mean()),
                             "schedule": "dynamic (rows taken from a device counter)"}),
            "score": None if args.attention_only else args.score,
            "step": ("attention only (no scoring or eviction)" if args.attention_only
                     else "fused attention + score + eviction"),
            "l2": "inputs larger than L2: each step reads the 1 GiB K/V cache (L2 is 126 MB)",
            "tokens_per_s": value * cfg.batch,
            "us_per_step_per_layer": ms_per_step * 1e3,
            "inputs": (f"new K/V drawn per step on the device ({n_fresh} distinct), queries "
                       f"cycling {n_inputs} seeded sets" if not glen else
                       f"graph of {glen} steps: its new tokens repeat every {glen} steps"),
            "launch": (f"CUDA graph of {glen} steps replayed" if glen else "one launch per step from Python"),
        },
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": peak_src,
                     "bytes_per_launch": by["algorithmic"],
                     "kernel": (f"lf::fused_decode_kernel<{cfg.head_dim},{cfg.group},"
                                f"{0 if args.attention_only else 1 + score_code},{kv_bytes}>")},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


def reference_arm(args, cfg, workload, world, rank):
    """The CPU oracle as the reference arm: each of the W + K steps is a
    bounded sample (a few rows of the batch), the value is scaled to full
    steps/s.  Only rank 0 works under torchrun."""
    if rank != 0:
        return 0
    from attention_lf_decode_b200 import synth
    import oracle
    gen = synth.SynthDecode(cfg)
    sel = [0]  # one batch entry = hkv rows per sample
    kb, vb = gen.prefill(sel)
    kc, vc, pos = synth.prefill_layout(kb, vb, cfg.budget)
    K, V, P = synth.bf16_bits_to_f64(kc), synth.bf16_bits_to_f64(vc), pos.astype(np.int64)
    fp8 = args.kv == "fp8"
    if fp8:  # an E4M3 cache: the oracle steps on the codes
        K, V = oracle.quantize(K, args.k_scale), oracle.quantize(V, args.v_scale)

    def ostep(K, V, P, q, kn, vn, nb):
        if fp8:
            return oracle.decode_step_fp8(K, V, P, q, kn, vn, cfg.sink, cfg.window, args.k_scale,
                                          args.v_scale, score=args.score, seq_budget=nb)
        return oracle.decode_step(K, V, P, q, kn, vn, cfg.sink, cfg.window, score=args.score,
                                  seq_budget=nb)
    budget_s = 150.0
    rows_full = cfg.batch * cfg.hkv
    nb = gen.seq_budgets()  # ragged batch: the sample's budget and every sequence's
    nb0 = None if nb is None else nb[:1]
    # full-step work relative to the sampled rows' (rows of unequal budget)
    work_ratio = 1.0 if nb is None else float(nb.sum()) / (float(nb[0]) * cfg.batch)
    # calibrate: one row-step
    qb, knb, vnb = gen.step_inputs(0)
    t0 = time.perf_counter()
    ostep(K[:, :1], V[:, :1], P[:, :1], synth.bf16_bits_to_f64(qb[:1, :cfg.group]),
          synth.bf16_bits_to_f64(knb[:1, :1]), synth.bf16_bits_to_f64(vnb[:1, :1]), nb0)
    t_row = time.perf_counter() - t0
    nsteps = args.warmup + args.steps
    rows_per_step = int(max(1, min(cfg.hkv, budget_s / max(nsteps, 1) / max(t_row, 1e-6))))
    heads = rows_per_step
    # the sampled rows' inputs of 256 steps, drawn once (drawing a whole
    # batch every step would take longer than the timed oracle itself)
    sets = []
    for s in range(min(nsteps, 256)):
        qb, knb, vnb = gen.step_inputs(s)
        sets.append((synth.bf16_bits_to_f64(qb[:1, :heads * cfg.group]),
                     synth.bf16_bits_to_f64(knb[:1, :heads]),
                     synth.bf16_bits_to_f64(vnb[:1, :heads])))
    t_total = 0.0
    for s in range(nsteps):
        q, kn, vn = sets[s % len(sets)]
        t0 = time.perf_counter()
        res = ostep(K[:, :heads], V[:, :heads], P[:, :heads], q, kn, vn, nb0)
        dt = time.perf_counter() - t0
        K[:, :heads], V[:, :heads], P[:, :heads] = res.kcache, res.vcache, res.pos
        if s >= args.warmup:
            t_total += dt
    per_row = t_total / (args.steps * heads)
    value = 1.0 / (per_row * rows_full * work_ratio)
    sample = (f"each step: oracle on {heads} of {rows_full} rows (batch entry 0), "
              f"{args.steps} timed steps after {args.warmup} warm-up; steps/s scaled to all rows"
              + ("" if nb is None else " in proportion to their budgets"))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": workload, "batch": cfg.batch, "budget": cfg.budget,
                   "score": args.score, "kv_dtype": "e4m3" if fp8 else "bf16"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads_used(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
