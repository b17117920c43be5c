#!/usr/bin/env python
"""Benchmark of the sparse MoE FFN block forward on B200.

One step = one moe_block_forward over one batch: router, top-k, permutation,
routed experts, shared expert and combine. The default workload is the
Klear-shaped bf16 block (hidden 2048, 256 experts, top-8, intermediate 768,
sigmoid routing with a select-only bias, shared expert blended) at 4096 tokens,
with seeded synthetic inputs resident in HBM. Rank 0 prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun): every rank runs its own independent batch (the block has
no cross-token exchange); the throughput is the total over ranks, the time the
max over ranks ("scaling": "weak").
--impl reference times the fp64 CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_moe_ffn_gemv_b200 import inputs  # noqa: E402
from sparse_moe_ffn_gemv_b200 import moe as M  # noqa: E402

METRIC = "MoE block tokens/sec on 1 B200; % HBM roofline (decode) / % TC peak (prefill)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="klear_bf16", choices=sorted(inputs.WORKLOADS))
    p.add_argument("--tokens", type=int, default=4096)
    p.add_argument("--decode-tokens", default="1,8,64", help="extra decode-sized token counts ('' = none)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ bytes and flops
def expert_bytes(spec) -> int:
    """Bytes of one routed expert's weights (gate, up, down, biases / 4-bit companions)."""
    I, K = spec.intermediate, spec.expert_in
    if spec.weight_format == "q4":  # packed codes + bf16 scale and bias per group
        g = spec.group_size
        b = 3 * I * K // 2 + (2 * I * (K // g) + K * (I // g)) * 2 * 2
    elif spec.weight_format == "mxfp4":  # packed E2M1 codes + one E8M0 byte per 32
        b = 3 * I * K // 2 + (2 * I * (K // 32) + K * (I // 32))
    else:
        b = 3 * I * K * (4 if spec.weight_format == "f32" else 2)
    if spec.has_expert_bias:
        b += (2 * I + K) * (4 if spec.act_dtype == "f32" else 2)
    return b


def dense_bytes(spec) -> int:
    """Non-routed weights read once per step: router, coefficient head, shared, latent."""
    ab = 4 if spec.act_dtype == "f32" else 2
    H, E = spec.hidden, spec.num_experts
    b = E * H * ab + (E * 4 if spec.has_selection_bias else 0)
    if spec.shared_mode == "blend":
        b += 2 * H * ab
    if spec.shared_mode != "none":
        b += 3 * spec.shared_intermediate * H * ab
    if spec.latent_dim:
        b += 2 * spec.latent_dim * H * ab + spec.latent_dim * ab
    return b


def block_flops(spec, T) -> float:
    H, E, k, I, K = spec.hidden, spec.num_experts, spec.top_k, spec.intermediate, spec.expert_in
    f = 2.0 * T * E * H + 2.0 * T * k * 3 * I * K
    if spec.shared_mode != "none":
        f += 2.0 * T * 3 * spec.shared_intermediate * H
    if spec.latent_dim:
        f += 2.0 * T * 2 * spec.latent_dim * H
    return f


# ------------------------------------------------------------------ clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            self.path = f"/tmp/moe_clocks_{os.getpid()}.csv"
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ launches
def kernels_per_step(block, x, y) -> int:
    """Kernel nodes in a CUDA graph of one step (the library's own launches)."""
    try:
        from cuda.bindings import runtime as rt
        g = torch.cuda.CUDAGraph(keep_graph=True)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            g.capture_begin()
            block.forward(x, y, stream=s)
            g.capture_end()
        torch.cuda.current_stream().wait_stream(s)
        graph = g.raw_cuda_graph()
        err, _, n = rt.cudaGraphGetNodes(graph)          # first call: the count only
        err, nodes, n = rt.cudaGraphGetNodes(graph, n)
        count = 0
        for node in nodes:
            e2, t = rt.cudaGraphNodeGetType(node)
            if t == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                count += 1
        del g
        return count
    except Exception as exc:  # introspection unavailable: report unknown
        print(f"[bench] launch count unavailable: {exc}", file=sys.stderr)
        return -1


def source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_moe_ffn_gemv_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, T: int):
    """DRAM bytes per launch of the dominant stage from a committed ncu summary,
    only if it was taken on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path))
    e = d.get(f"{workload}/T{T}")
    if not e or e.get("source_hash") != source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ CPU oracle
def cpu_baseline(spec, w_cpu, x_cpu, target_s: float = 10.0):
    import oracle
    wnp = {k: inputs.to_numpy_storage(v) for k, v in w_cpu.items()}
    xnp = inputs.to_numpy_storage(x_cpu)
    threads = oracle.max_threads()
    n = min(8, xnp.shape[0])
    t0 = time.perf_counter()
    oracle.forward(spec, wnp, xnp, tokens=np.arange(n), threads=threads)
    dt = time.perf_counter() - t0
    n2 = int(min(xnp.shape[0], max(n, n * target_s / max(dt, 1e-6))))
    t0 = time.perf_counter()
    oracle.forward(spec, wnp, xnp, tokens=np.arange(n2), threads=threads)
    dt2 = time.perf_counter() - t0
    return {"value": n2 / dt2, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"first {n2} of the {xnp.shape[0]} tokens of the same batch "
                      f"({dt2:.1f} s, fp64, OpenMP over tokens)"}


L2_BYTES = 126 * 2**20  # B200 L2 cache


def needs_l2_flush(spec, T) -> bool:
    """True when the step's weights could stay in L2 between timed steps: the largest
    possible activated set (min(E, T k) experts plus the dense weights) is under twice the
    L2 size. Those steps are timed one by one with L2 flushed in between."""
    most = min(spec.num_experts, T * spec.top_k) * expert_bytes(spec) + dense_bytes(spec)
    return most < 2 * L2_BYTES


def workload_config(spec, T, world):
    """The `config` object of both arms' JSON lines."""
    l2 = ("L2 flushed between timed steps (activated weights could fit in L2)" if needs_l2_flush(spec, T)
          else "activated weights larger than L2 (no flush needed)")
    return {"workload": f"{spec.name} (hidden {spec.hidden}, {spec.num_experts} experts, "
                        f"top-{spec.top_k}, intermediate {spec.intermediate})",
            "tokens_per_gpu": T, "parallelism": f"replicas x{world}",
            "l2": l2 + "; decode rows flush L2"}


def max_over_ranks(v: float, dist, device) -> float:
    """The largest of every rank's value (a step time): the whole job is as slow as its
    slowest replica. Identity on one rank."""
    if dist is None:
        return float(v)
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reference_arm(args, rank, world):
    if rank != 0:
        return
    spec = inputs.WORKLOADS[args.workload]
    T = args.tokens
    w_cpu = inputs.make_weights(spec)
    x_cpu = inputs.make_x(spec, T)
    import oracle
    wnp = {k: inputs.to_numpy_storage(v) for k, v in w_cpu.items()}
    xnp = inputs.to_numpy_storage(x_cpu)
    threads = oracle.max_threads()
    # each step: a bounded sample of the batch, sized so the whole run stays within minutes
    t0 = time.perf_counter()
    oracle.forward(spec, wnp, xnp, tokens=np.arange(4), threads=threads)
    per_tok = (time.perf_counter() - t0) / 4
    n = int(max(1, min(T, 6.0 / max(per_tok, 1e-9) / max(1, args.steps + args.warmup) * 4)))
    for _ in range(args.warmup):
        oracle.forward(spec, wnp, xnp, tokens=np.arange(n), threads=threads)
    times = []
    for s in range(args.steps):
        toks = (np.arange(n) + s * n) % T
        t0 = time.perf_counter()
        oracle.forward(spec, wnp, xnp, tokens=toks, threads=threads)
        times.append(time.perf_counter() - t0)
    tot = sum(times)
    value = n * args.steps / tot
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded; no checkpoint)",
            "config": workload_config(spec, T, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": f"{n} tokens of the {T}-token batch per step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ main arm
def l2_flush_buffer(dev):
    return torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)


def time_steps(fn, steps, warmup, flush=None):
    """Per-step CUDA-event times (ms) on the current stream; optional L2 flush between steps."""
    for _ in range(warmup):
        fn()
    ts = []
    for _ in range(steps):
        if flush is not None:
            flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        ts.append((e0, e1))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ts]


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference":
            reference_arm(args, rank, world)
            return
        run(args, rank, world, local, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


def run(args, rank, world, local, dist):
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    spec = inputs.WORKLOADS[args.workload]
    T = args.tokens
    w_cpu = inputs.make_weights(spec)
    x_cpu = inputs.make_x(spec, T)
    block = M.MoeBlock(spec, w_cpu, max_tokens=max(T, 64), device=str(dev))
    x = x_cpu.to(dev)
    act_dt = block.act_dtype
    y = torch.empty((T, spec.hidden), dtype=act_dt, device=dev)
    block.forward(x, y)
    torch.cuda.synchronize()
    if block.device_status() != 0:
        raise SystemExit("device status set after the first forward")

    # routing of this batch -> distinct activated experts (algorithmic bytes)
    idx = torch.empty((T, spec.top_k), dtype=torch.int32, device=dev)
    wts = torch.empty((T, spec.top_k), dtype=torch.float32, device=dev)
    coef = torch.empty((T, 2), dtype=torch.float32, device=dev)
    M.moe_route(block.cfg, block.w, x, T, idx, wts, coef, block.ws)
    n_distinct = int(torch.unique(idx).numel())
    ab = 4 if spec.act_dtype == "f32" else 2
    K = spec.expert_in
    ffn_bytes = n_distinct * expert_bytes(spec) + T * K * ab + T * K * 4
    blk_bytes = n_distinct * expert_bytes(spec) + dense_bytes(spec) + 2 * T * spec.hidden * ab

    launches = kernels_per_step(block, x, y)

    # ---- timed region: K whole steps (one by one with L2 flushed in between when the
    # activated weights could stay in L2)
    l2_flush = l2_flush_buffer(dev) if needs_l2_flush(spec, T) else None
    sampler = ClockSampler(local)
    for _ in range(args.warmup):
        block.forward(x, y)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    if l2_flush is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            block.forward(x, y)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
    else:
        ms = statistics.mean(time_steps(lambda: block.forward(x, y), args.steps, 0, flush=l2_flush))
    if dist is not None:
        dist.barrier()
    # dominant stage (routed experts: gate/up + down kernels), same inputs, CUDA events
    off = torch.empty(spec.num_experts + 1, dtype=torch.int32, device=dev)
    ss = torch.empty(T * spec.top_k, dtype=torch.int32, device=dev)
    sp = torch.empty(T * spec.top_k, dtype=torch.int32, device=dev)
    u = x
    if spec.latent_dim:
        u = torch.empty((T, spec.latent_dim), dtype=act_dt, device=dev)
        M.moe_latent_down(block.cfg, block.w, x, T, u, block.ws)
    M.moe_permute(block.cfg, idx, T, off, ss, sp, block.ws)
    y_acc = torch.empty((T, K), dtype=torch.float32, device=dev)
    ffn_ms = time_steps(lambda: M.moe_grouped_ffn(block.cfg, block.w, u, T, off, ss, wts, y_acc, block.ws),
                        args.steps, args.warmup, flush=l2_flush)
    clocks = sampler.stop()
    if block.device_status() != 0:
        raise SystemExit("device status set during the timed region")

    ms_max = max_over_ranks(ms, dist, dev)
    value = world * T / (ms_max / 1000.0)

    pk, pk_src = peaks()
    ffn_avg = statistics.mean(ffn_ms)
    achieved = ffn_bytes / (ffn_avg / 1000.0) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "traffic": recorded_traffic(spec.name, T),
                "kernel": "routed experts: gate/up + down (moe_grouped_ffn)",
                "algorithmic_bytes_per_launch": ffn_bytes, "ms_per_launch": ffn_avg,
                "peak_source": f"{pk_src} (MEASURED_PEAKS.json hbm_gbs)" if pk_src == "measured" else "fallback"}

    # ---- end to end: pinned host x -> device, forward, device y -> pinned host, every step
    e2e = None
    if not args.no_e2e:
        x_host = x_cpu.pin_memory()
        y_host = torch.empty((T, spec.hidden), dtype=act_dt).pin_memory()
        x_dev = torch.empty_like(x)

        def e2e_step():
            x_dev.copy_(x_host, non_blocking=True)
            block.forward(x_dev, y)
            y_host.copy_(y, non_blocking=True)

        e2e_ms = time_steps(e2e_step, args.steps, args.warmup, flush=l2_flush)
        e_max = max_over_ranks(statistics.mean(e2e_ms), dist, dev)
        e2e = {"value": world * T / (e_max / 1000.0), "unit": "tokens/s",
               "h2d_bytes_per_step": T * spec.hidden * ab, "d2h_bytes_per_step": T * spec.hidden * ab}

    # ---- decode-sized batches (L2 flushed between iterations; graphs remove launch gaps)
    decode = []
    dec_tokens = [int(t) for t in args.decode_tokens.split(",") if t.strip()]
    flush = l2_flush_buffer(dev) if dec_tokens else None
    for Td in dec_tokens:
        xd = inputs.make_x(spec, Td).to(dev)
        yd = torch.empty((Td, spec.hidden), dtype=act_dt, device=dev)
        idd = torch.empty((Td, spec.top_k), dtype=torch.int32, device=dev)
        M.moe_route(block.cfg, block.w, xd, Td, idd, torch.empty((Td, spec.top_k), device=dev),
                    torch.empty((Td, 2), device=dev), block.ws)
        nd = int(torch.unique(idd).numel())
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            block.forward(xd, yd, stream=s)
            g.capture_begin()
            block.forward(xd, yd, stream=s)
            g.capture_end()
        torch.cuda.current_stream().wait_stream(s)
        d_ms = time_steps(g.replay, max(args.steps, 20), args.warmup, flush=flush)
        med = statistics.median(d_ms)
        db = nd * expert_bytes(spec) + dense_bytes(spec) + 2 * Td * spec.hidden * ab
        decode.append({"tokens": Td, "tokens_per_s": Td / (med / 1000.0), "us_per_step": med * 1000.0,
                       "distinct_experts": nd, "algorithmic_bytes": db,
                       "gbs": db / (med / 1000.0) / 1e9, "hbm_frac": db / (med / 1000.0) / 1e9 / pk["hbm_gbs"]})
        del g
    torch.cuda.synchronize()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(spec, w_cpu, x_cpu)

    if rank == 0:
        flops = block_flops(spec, T)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": spec.act_dtype if spec.weight_format in ("bf16", "f32") else "bf16+" + spec.weight_format,
            "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights; no checkpoint)",
            "config": workload_config(spec, T, world),
            "roofline": roofline,
            "block": {"algorithmic_bytes": blk_bytes, "gbs": blk_bytes / (ms_max / 1000) / 1e9,
                      "hbm_frac": blk_bytes / (ms_max / 1000) / 1e9 / pk["hbm_gbs"],
                      "tflops": flops / (ms_max / 1000) / 1e12,
                      "tc_frac": flops / (ms_max / 1000) / 1e12 / pk["bf16_tflops"],
                      "distinct_experts": n_distinct},
            "decode": decode,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches * args.steps if launches >= 0 else None,
            "gpu_launches_per_step": launches,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
