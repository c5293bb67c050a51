#!/usr/bin/env python
"""Decode benchmark: tok/s/user and TPOT at batch 1 on the 8B-shape decoder, plus
achieved HBM bandwidth against the bytes-per-token roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]

One bench step = one greedy decode of the workload's 256 tokens per sequence
from the same prompt state (one persistent-kernel launch).  Prints ONE JSON
line on rank 0.  Under torchrun (N > 1) every rank runs an independent replica
on its own GPU (the path does not shard: no collective on the data path);
the timed region is bracketed by barriers and the max over ranks is taken.

--impl reference times the oracle (plain fp32 CPU decode) on this machine's
host cores on a bounded sample of the same workload, as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode tok/s/user (TPOT) at batch 1; achieved HBM GB/s vs roofline, 1 B200"
UNIT = "tok/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="xlpk", choices=["xlpk", "reference"])
    ap.add_argument("--workload", default="llama8b")
    ap.add_argument("--decode-steps", type=int, default=0, help="override tokens per call (profiling)")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (sequences per call)")
    ap.add_argument("--kv", default="bf16", choices=["bf16", "fp8"],
                    help="KV cache entries: bf16, or e4m3 codes with a power-of-two scale per tensor")
    ap.add_argument("--no-baselines", action="store_true", help="skip the unfused and CPU legs")
    ap.add_argument("--serve", action="store_true",
                    help="also time one-step requests through the resident loop against one launch per request")
    return ap.parse_args()


def dist_env():
    from persistent_decode_b200.replicas import dist_env as _env
    return _env()


# ----------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.proc = None
        self.path = os.path.join("/tmp", f"xlpk_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.uuid}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
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
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------- helpers

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


TILE_SECTION = b"\n// ---- tensor-core tile entry point"


def kernel_source_hash() -> str:
    """Hash of the sources the persistent decode kernel and its host planning
    come from (the tensor-core tile entry point appended to xlpk.cu is not
    among them)."""
    h = hashlib.sha256()
    for f in ("engine.cuh", "xlpk.cu", "params.h", "kernels.cu", "kernels.h"):
        data = open(os.path.join(ROOT, "persistent_decode_b200", "csrc", f), "rb").read()
        if f == "xlpk.cu" and TILE_SECTION in data:
            data = data[:data.index(TILE_SECTION)]
        h.update(data)
    return h.hexdigest()[:16]


def ncu_traffic(workload: str):
    """DRAM bytes per decode step from the committed ncu summary, if it was
    taken on the current kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(workload)
    if not e or e.get("kernel_hash") != kernel_source_hash():
        return None
    return e


def build_cpu_sample(cfg, dev):
    """Host copies of a bounded sample of the workload for the oracle: the
    first two layers (with their synthetic KV), the embedding and the LM head."""
    import torch

    import synth
    from oracle import OracleDecoder
    nl = min(2, cfg.n_layers)
    sub = cfg.with_(n_layers=nl)
    w = synth.make_weights(sub, device=dev)
    w = {k: v.cpu() for k, v in w.items()}
    o = OracleDecoder(sub, w, cfg.batch, max_seq=cfg.kv_len + 8)
    for l in range(nl):
        kl, vl = synth.make_synthetic_kv(cfg, l, device=dev)
        o.load_kv(l, kl.cpu(), vl.cpu())
    o.pos = [cfg.kv_len] * cfg.batch
    head = OracleDecoder(cfg.with_(n_layers=0), w, cfg.batch, max_seq=8)
    del torch
    return o, head, nl


def time_cpu_sample(cfg, o, head, nl, start_tok):
    """Seconds per token of the full model, from one oracle step of the sample."""
    t0 = time.perf_counter()
    head.step(start_tok)
    t_head = time.perf_counter() - t0
    t0 = time.perf_counter()
    o.step(start_tok)
    t_sample = time.perf_counter() - t0
    # both samples go back to their start position, so any number of calls
    # stays inside their caches
    o.pos = [cfg.kv_len] * cfg.batch
    head.pos = [0] * cfg.batch
    per_layer = max(t_sample - t_head, 0.0) / nl
    return t_head + per_layer * cfg.n_layers, t_sample + t_head


def cpu_sample_desc(cfg, nl):
    return (f"one oracle decode step of layers 0-{nl - 1} (KV {cfg.kv_len}) plus the embedding/final-norm/"
            f"LM-head pass of the {cfg.name} model, scaled to {cfg.n_layers} layers")


# ----------------------------------------------------------------- reference arm

def bench_config(args):
    """The workload's config with the command line's overrides."""
    import synth
    cfg = synth.get_config(args.workload)
    if getattr(args, "decode_steps", 0):
        cfg = cfg.with_(steps=args.decode_steps)
    if getattr(args, "batch", 0):
        cfg = cfg.with_(batch=args.batch)
    if getattr(args, "kv", "bf16") == "fp8":
        cfg = synth.fp8_kv(cfg)
    return cfg


def run_reference(args):
    import torch

    import synth
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    cfg = bench_config(args)
    dev = "cuda:0" if torch.cuda.is_available() else "cpu"
    o, head, nl = build_cpu_sample(cfg, dev)
    start = synth.make_start_tokens(cfg).tolist()
    for _ in range(args.warmup):
        time_cpu_sample(cfg, o, head, nl, start)
    per_tok = []
    for _ in range(args.steps):
        per_tok.append(time_cpu_sample(cfg, o, head, nl, start)[0])
    tpot = statistics.mean(per_tok)
    value = cfg.batch / tpot
    cores = torch.get_num_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tpot * 1e3 * cfg.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": workload_config(cfg, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": cpu_sample_desc(cfg, nl)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def dtype_label(cfg) -> str:
    """The arithmetic the decode runs in: weights as stored, fp32 accumulation."""
    if cfg.weight_dtype == "fp8_e4m3":
        w = "fp8_e4m3 weights (fp32 scale per 128x128 block)"
    elif cfg.weight_dtype == "nvfp4":
        w = "nvfp4 weights (e2m1, e4m3 scale per 16 elements, fp32 scale per matrix)"
    else:
        w = "bf16 weights"
    act = "fp32 activations"
    if cfg.batch == 8 and not cfg.is_moe:
        act = "activations as bf16 high + low parts into tcgen05 MMAs, fp32 accumulation"
    kv = "e4m3 KV (power-of-two scale per tensor)" if cfg.kv_dtype == "fp8_e4m3" else "bf16 KV"
    return f"{w}, {kv}, {act}"


def workload_config(cfg, n):
    return {"workload": f"{cfg.name}: {cfg.n_layers} layers, hidden {cfg.hidden}, {cfg.n_q_heads}q/"
                        f"{cfg.n_kv_heads}kv heads x {cfg.head_dim}, ffn {cfg.ffn}, vocab {cfg.vocab}, "
                        f"{cfg.weight_dtype} weights, KV {cfg.kv_len}"
                        f"{' (e4m3 cache)' if cfg.kv_dtype == 'fp8_e4m3' else ''}, {cfg.steps} greedy steps, "
                        f"batch {cfg.batch}",
            "global_batch": cfg.batch * n, "seq_len": cfg.kv_len, "decode_steps": cfg.steps,
            "parallelism": "replicas" if n > 1 else "single-gpu",
            "l2": "inputs larger than L2 (all weights streamed every token)"}


def serve_latency(dev, requests: int = 200):
    """Round trip of one-step requests on the tiny decoder (latency-bound): one
    decode launch per request (launch, token copy to the host, synchronise)
    against the device-resident loop (post a request word, wait for its
    token in host-mapped memory).  Both decode consecutive steps."""
    import torch

    import synth
    from persistent_decode_b200 import workload
    cfg = synth.get_config("tiny")
    m = workload.build(cfg, device=dev, max_seq=cfg.kv_len + 2 * requests + 16)
    tok = torch.empty(1, cfg.batch, dtype=torch.int32, device=dev)
    out = torch.empty(1, cfg.batch, dtype=torch.int32).pin_memory()

    def per_launch(n):
        workload.reset_state(m)
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        for _ in range(n):
            m.engine.decode(1, tok)
            out.copy_(tok)            # synchronous copy: the token is on the host
        return (time.perf_counter() - t0) / n

    def resident(n):
        workload.reset_state(m)
        torch.cuda.synchronize(dev)
        m.engine.serve_start(idle_limit_us=2_000_000)
        try:
            t0 = time.perf_counter()
            for _ in range(n):
                m.engine.serve_wait(m.engine.serve_post(1), 1)
            dt = (time.perf_counter() - t0) / n
        finally:
            m.engine.serve_stop()
        return dt

    per_launch(16)
    resident(16)
    a = per_launch(requests)
    b = resident(requests)
    m.engine.check()
    return {"workload": "tiny, batch 1, one greedy step per request", "requests": requests,
            "launch_per_request_us": round(a * 1e6, 2), "resident_loop_us": round(b * 1e6, 2),
            "speedup": round(a / b, 3)}


# ----------------------------------------------------------------- main arm

def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    import torch
    import torch.distributed as dist

    import synth
    from persistent_decode_b200 import roofline, workload

    from persistent_decode_b200 import replicas
    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        replicas.init("nccl", device=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    cfg = bench_config(args)
    n = cfg.steps
    B = cfg.batch

    m = workload.build(cfg, device=dev)
    m.weights.clear()                      # the engine holds its own packed copy
    torch.cuda.empty_cache()
    stream = torch.cuda.current_stream(dev)
    tok = torch.empty(n, B, dtype=torch.int32, device=dev)

    def one_call():
        workload.reset_state(m)
        m.engine.decode(n, tok)

    for _ in range(args.warmup):
        one_call()
    m.engine.check()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(uuid) as clk:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            workload.reset_state(m)
            ev[i][0].record(stream)
            m.engine.decode(n, tok)
            ev[i][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    status = m.engine.status()
    if world > 1:
        dist.barrier()
    total_ms = replicas.max_over_ranks(t_start.elapsed_time(t_end), dev)
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    value = replicas.job_rate(args.steps * n * B, total_ms / 1e3, world)
    tpot_ms = total_ms / (args.steps * n)

    # roofline of the persistent kernel (one launch = one bench step)
    bytes_launch = roofline.call_bytes(cfg, cfg.kv_len, n)
    avg_launch_s = statistics.mean(launch_ms) / 1e3
    achieved = bytes_launch / avg_launch_s / 1e9
    peak, peak_kind = measured_peaks()
    tr = ncu_traffic(cfg.name)
    traffic = None
    if tr is not None:
        traffic = tr["dram_bytes_per_step"] * n
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": traffic, "peak_kind": peak_kind,
            "algorithmic_bytes_per_launch": bytes_launch,
            "kernel": "engine_persistent (whole decode, one launch)"}

    # end to end through the C ABI with host buffers (H2D state, D2H tokens)
    out_host = torch.empty(n, B, dtype=torch.int32).pin_memory()
    m.engine.generate(m.start_tokens.tolist(), [cfg.kv_len] * B, n, out_host)
    e2e_t = []
    for _ in range(max(2, args.steps)):
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        m.engine.generate(m.start_tokens.tolist(), [cfg.kv_len] * B, n, out_host)
        e2e_t.append(time.perf_counter() - t0)
    e2e_s = replicas.max_over_ranks(statistics.mean(e2e_t), dev)
    e2e = {"value": replicas.job_rate(n * B, e2e_s, world), "unit": UNIT, "h2d_bytes_per_step": 4 * B,
           "d2h_bytes_per_step": 4 * B * n}

    extra = {}
    if not args.no_baselines:
        # kernel-per-op baseline, same tiles, one launch per stage
        un_steps = min(n, 16)
        workload.reset_state(m)
        m.engine.decode(un_steps, tok, unfused=True)
        torch.cuda.synchronize(dev)
        workload.reset_state(m)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        m.engine.decode(un_steps, tok, unfused=True)
        b.record(stream)
        torch.cuda.synchronize(dev)
        un_tpot = a.elapsed_time(b) / un_steps
        # the same launches recorded once into a CUDA graph and replayed: the
        # kernel-per-op baseline without host launch overhead
        workload.reset_state(m)
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.graph(g, stream=cap):
            m.engine.decode(un_steps, tok, unfused=True)
        stream.wait_stream(cap)
        g.replay()
        torch.cuda.synchronize(dev)
        gt = []
        for _ in range(3):
            a.record(stream)
            g.replay()
            b.record(stream)
            torch.cuda.synchronize(dev)
            gt.append(a.elapsed_time(b) / un_steps)
        del g
        m.engine.check()
        un_graph = statistics.median(gt)
        info = m.engine.info()
        extra["unfused"] = {"tpot_ms": round(un_tpot, 4), "tok_s_per_user": round(1e3 / un_tpot, 2),
                            "graph_tpot_ms": round(un_graph, 4),
                            "steps_timed": un_steps, "launches_per_token": info.kernels_per_step_unfused,
                            "persistent_speedup": round(un_tpot / tpot_ms, 3),
                            "persistent_speedup_vs_graph": round(un_graph / tpot_ms, 3)}
    if args.serve:
        extra["serve_loop"] = serve_latency(dev)
    cpu = None
    if rank == 0 and world == 1 and not args.no_baselines:
        o, head, nl = build_cpu_sample(cfg, dev)
        per_tok, _ = time_cpu_sample(cfg, o, head, nl, m.start_tokens.tolist())
        cpu = {"value": round(B / per_tok, 4), "unit": UNIT, "cores": torch.get_num_threads(), "kind": "oracle",
               "sample": cpu_sample_desc(cfg, nl)}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": dtype_label(cfg), "data": "synthetic",
            "config": workload_config(cfg, world),
            "tpot_ms": round(tpot_ms, 4), "tok_s_per_user": round(1e3 / tpot_ms, 2),
            "roofline": roof,
            "roofline_spec_8tbs_frac": round(achieved / 8000.0, 4),
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps, "clocks": clk.summary(),
            "status": status, **extra,
        }
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0 if status == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
