#!/usr/bin/env python
"""Benchmark of the sparse MoE FFN block forward on B200.

One step = one moe_block_forward over one batch: router, top-k, permutation,
routed experts, shared expert and combine (and, for the latent block, the
latent down projection, RMSNorm and up projection). The headline workload is
the largest single-GPU configuration: the Kimi-shaped latent block (hidden
7168 -> latent 3584, 384 experts, top-8, expert intermediate 2048, shared
expert 2048 added) at 8192 tokens, with seeded synthetic inputs resident in
HBM. The same JSON line carries a prefill row and decode rows for every
workload (Klear bf16, Klear 4-bit, clamped bf16, latent bf16, clamped MXFP4),
each with its HBM and tensor-core fractions and a sampled oracle baseline.
Rank 0 prints one JSON line.

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
import re
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

HEADLINE = ("latent_bf16", 8192)
# Per-workload rows: the prefill-sized batch (graded on tensor-core peak) and the
# decode-sized batches (graded on HBM bandwidth over the activated bytes).
PREFILL = {"klear_bf16": 4096, "klear_q4": 2048, "clamped_bf16": 8192, "latent_bf16": 8192,
           "clamped_mxfp4": 8192, "klear_q4_dense": 2048}
DECODE = {"klear_bf16": (1, 8, 64), "klear_q4": (1, 32), "clamped_bf16": (1,), "latent_bf16": (1, 128),
          "clamped_mxfp4": (1, 8), "klear_q4_dense": (1, 32)}
ROW_ORDER = ("latent_bf16", "klear_bf16", "klear_q4", "clamped_bf16", "clamped_mxfp4", "klear_q4_dense")


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=HEADLINE[0], choices=sorted(inputs.WORKLOADS))
    p.add_argument("--tokens", type=int, default=HEADLINE[1])
    p.add_argument("--rows", default="all",
                   help="workloads that get prefill/decode rows: 'all', 'none' or a comma list")
    p.add_argument("--decode-tokens", default=None,
                   help="decode token counts of the headline workload (default: its table entry; '' = none)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-kernel-table", action="store_true")
    p.add_argument("--experts", type=int, default=0,
                   help="keep only the first E routed experts of the workload (a smaller copy for ncu captures)")
    return p.parse_args(argv)


def workload_spec(args):
    spec = inputs.WORKLOADS[args.workload]
    if args.experts:
        if not spec.top_k <= args.experts <= spec.num_experts:
            raise SystemExit("--experts must lie between top_k and the workload's expert count")
        spec = spec.replace(num_experts=args.experts, name=f"{spec.name}_e{args.experts}")
    return spec


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        out = dict(FALLBACK_PEAKS)
        out.update({k: float(v) for k, v in d.items() if k in FALLBACK_PEAKS and v})
        return out, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ bytes and flops
def plane_bytes(spec, rows: int, cols: int, fmt: str = None) -> int:
    """Bytes of one [rows, cols] weight plane in a format (default: the routed format)."""
    fmt = fmt or spec.weight_format
    if fmt == "q4":  # packed codes + bf16 scale and bias per group
        return rows * cols // 2 + rows * (cols // spec.group_size) * 4
    if fmt == "mxfp4":  # packed E2M1 codes + one E8M0 byte per 32
        return rows * cols // 2 + rows * (cols // 32)
    return rows * cols * (4 if fmt == "f32" else 2)


def expert_bytes(spec) -> int:
    """Bytes of one routed expert's weights (gate, up, down, biases / 4-bit companions)."""
    I, K = spec.intermediate, spec.expert_in
    b = 2 * plane_bytes(spec, I, K) + plane_bytes(spec, K, I)
    if spec.has_expert_bias:
        b += (2 * I + K) * (4 if spec.act_dtype == "f32" else 2)
    return b


def dense_plane_bytes(spec, rows: int, cols: int) -> int:
    """Bytes of a router / shared / latent plane: the activation dtype, or 4-bit affine words
    with a bf16 scale and bias per dense_group_size columns."""
    if getattr(spec, "dense_format", "act") == "q4":
        return rows * cols // 2 + rows * (cols // spec.dense_group_size) * 4
    return rows * cols * (4 if spec.act_dtype == "f32" else 2)


def dense_bytes(spec) -> int:
    """Non-routed weights read once per step: router, coefficient head, shared, latent."""
    ab = 4 if spec.act_dtype == "f32" else 2
    H, E = spec.hidden, spec.num_experts
    b = dense_plane_bytes(spec, E, H) + (E * 4 if spec.has_selection_bias else 0)
    if spec.shared_mode == "blend":
        b += 2 * H * ab
    if spec.shared_mode != "none":
        b += 3 * dense_plane_bytes(spec, spec.shared_intermediate, H)
    if spec.latent_dim:
        b += 2 * dense_plane_bytes(spec, spec.latent_dim, H) + spec.latent_dim * ab
    return b


def block_bytes(spec, T: int, n_distinct: int) -> int:
    """Algorithmic bytes of one step: the distinct activated experts' weights, every
    non-routed weight, x in and y out (intermediates excluded)."""
    ab = 4 if spec.act_dtype == "f32" else 2
    return n_distinct * expert_bytes(spec) + dense_bytes(spec) + 2 * T * spec.hidden * ab


def block_flops(spec, T) -> float:
    H, E, k, I, K = spec.hidden, spec.num_experts, spec.top_k, spec.intermediate, spec.expert_in
    f = 2.0 * T * E * H + 2.0 * T * k * 3 * I * K
    if spec.shared_mode != "none":
        f += 2.0 * T * 3 * spec.shared_intermediate * H
    if spec.latent_dim:
        f += 2.0 * T * 2 * spec.latent_dim * H
    return f


def kernel_roles(spec, T: int, n_distinct: int) -> dict:
    """Algorithmic bytes and flops of the two expert launches of the tensor-core engine
    (one launch each carries the routed experts and the shared expert): the weights
    they read (distinct activated experts' planes, the shared planes), their token
    input read once and their output written once."""
    H, k, I, K, Is = spec.hidden, spec.top_k, spec.intermediate, spec.expert_in, spec.shared_intermediate
    ab = 4 if spec.act_dtype == "f32" else 2
    sh = spec.shared_mode != "none"
    gu_w = n_distinct * 2 * plane_bytes(spec, I, K) + (2 * dense_plane_bytes(spec, Is, H) if sh else 0)
    dn_w = n_distinct * plane_bytes(spec, K, I) + (dense_plane_bytes(spec, H, Is) if sh else 0)
    if spec.has_expert_bias:
        gu_w += n_distinct * 2 * I * ab
        dn_w += n_distinct * K * ab
    gu = {"bytes": gu_w + T * K * ab + (T * H * ab if sh else 0) + T * k * I * ab + (T * Is * ab if sh else 0),
          "flops": 2.0 * T * k * 2 * I * K + (2.0 * T * 2 * Is * H if sh else 0.0)}
    dn = {"bytes": dn_w + T * k * I * ab + (T * Is * ab if sh else 0) + T * K * 4 + (T * H * 4 if sh else 0),
          "flops": 2.0 * T * k * I * K + (2.0 * T * H * Is if sh else 0.0)}
    return {"gate/up": gu, "down": dn}


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


# ------------------------------------------------------------------ kernels of one step
def short_kernel_name(mangled: str) -> str:
    """'_ZN3moe12_GLOBAL__N_114tc_gemm_kernelILb1ELi128ELi4ELb0EEEv..' ->
    'tc_gemm_kernel<1,128,4,0>' (the first length-prefixed identifier ending in
    'kernel', with its integer template arguments)."""
    pos = 0
    digits = re.compile(r"\d+")
    while True:
        m = digits.search(mangled, pos)
        if not m:
            return mangled
        n, start = int(m.group(0)), m.end()
        ident = mangled[start:start + n]
        if len(ident) == n and re.fullmatch(r"[A-Za-z_][A-Za-z0-9_]*", ident):
            if ident.endswith("kernel"):
                rest = mangled[start + n:]
                if rest.startswith("I"):
                    args = re.findall(r"L[a-z]+(-?\d+)E", rest.split("EE")[0] + "E")
                    return ident + ("<" + ",".join(args) + ">" if args else "<..>")
                return ident
            pos = start + n
        else:
            pos = start


def _capture(fn):
    g = torch.cuda.CUDAGraph(keep_graph=True)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        g.capture_begin()
        fn(s)
        g.capture_end()
    torch.cuda.current_stream().wait_stream(s)
    return g


def _kernel_nodes(g):
    from cuda.bindings import driver as drv
    graph = drv.CUgraph(int(g.raw_cuda_graph()))
    err, _, n = drv.cuGraphGetNodes(graph)
    err, nodes, n = drv.cuGraphGetNodes(graph, n)
    out = []
    for node in nodes:
        err, t = drv.cuGraphNodeGetType(node)
        if t != drv.CUgraphNodeType.CU_GRAPH_NODE_TYPE_KERNEL:
            continue
        name = "?"
        try:
            err, prm = drv.cuGraphKernelNodeGetParams(node)
            err, nm = drv.cuFuncGetName(prm.func)
            if err == drv.CUresult.CUDA_SUCCESS and nm:
                name = nm.decode() if isinstance(nm, bytes) else str(nm)
        except Exception:
            pass
        out.append((node, name))
    return graph, out


def kernels_per_step(fn) -> int:
    """Kernel nodes in a CUDA graph of one step (the library's own launches)."""
    try:
        g = _capture(fn)
        _, nodes = _kernel_nodes(g)
        del g
        return len(nodes)
    except Exception as exc:  # introspection unavailable: report unknown
        print(f"[bench] launch count unavailable: {exc}", file=sys.stderr)
        return -1


def kernel_table(fn, reps: int, flush=None):
    """CUDA-event time of every kernel launch of one step, each replayed alone.

    The step is captured once into a CUDA graph; for every kernel node a clone of the
    graph keeps that node only (same function, grid and arguments, the buffers holding
    the step's data), is instantiated and launched `reps` times on the current stream,
    bracketed by CUDA events (L2 flushed before each launch when `flush` is given).
    Returns [(short name, mean ms)] in launch order, or None if the graph API is missing.
    """
    try:
        from cuda.bindings import driver as drv
        g = _capture(fn)
        graph, nodes = _kernel_nodes(g)
        stream = drv.CUstream(torch.cuda.current_stream().cuda_stream)
        rows = []
        for node, name in nodes:
            err, clone = drv.cuGraphClone(graph)
            for other, _ in nodes:
                err, c = drv.cuGraphNodeFindInClone(other, clone)
                if int(other) != int(node):
                    drv.cuGraphDestroyNode(c)
            err, exe = drv.cuGraphInstantiate(clone, 0)
            if err != drv.CUresult.CUDA_SUCCESS:
                raise RuntimeError(f"instantiate: {err}")
            drv.cuGraphLaunch(exe, stream)  # warm-up
            ts = []
            for _ in range(reps):
                if flush is not None:
                    flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                drv.cuGraphLaunch(exe, stream)
                e1.record()
                ts.append((e0, e1))
            torch.cuda.synchronize()
            rows.append((short_kernel_name(name), statistics.mean(a.elapsed_time(b) for a, b in ts)))
            drv.cuGraphExecDestroy(exe)
            drv.cuGraphDestroy(clone)
        del g
        return rows
    except Exception as exc:
        print(f"[bench] per-kernel timing unavailable: {exc}", file=sys.stderr)
        return None


def label_expert_launches(table):
    """Indices of the expert gate/up launch and the down launch that follows it."""
    gu = next((i for i, (n, _) in enumerate(table) if n.startswith("tc_gemm_kernel<1,")), None)
    dn = None
    if gu is not None:
        dn = next((i for i in range(gu + 1, len(table)) if table[i][0].startswith("tc_gemm_kernel<0,")), None)
    return gu, dn


# the sources a kernel is compiled from (its own file and the headers it includes)
KERNEL_SOURCES = {
    "tc_gemm_kernel": ("umma.cu", "ptx.cuh", "common.cuh", "internal.h"),
    "decode_kernel": ("decode.cu", "gemv_dev.cuh", "topk_dev.cuh", "ptx.cuh", "common.cuh", "internal.h"),
}


def code_of(text: str) -> str:
    """C++ source without comments and blank-line or indentation differences."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.strip() for line in text.splitlines() if line.strip())


def source_hash(kernel: str = "") -> str:
    """Hash of the code (comments aside) of `kernel`'s sources, or of every CUDA source."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_moe_ffn_gemv_b200", "csrc")
    files = KERNEL_SOURCES.get(kernel.split("<")[0], None) or sorted(os.listdir(csrc))
    for f in files:
        h.update(code_of(open(os.path.join(csrc, f)).read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, T: int, kernel: str):
    """DRAM bytes per launch of a kernel from a committed ncu summary, only if it was
    taken on the kernel's current sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path))
    e = d.get(f"{workload}/T{T}/{kernel}")
    if not e or e.get("source_hash") != source_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ CPU oracle
def cpu_baseline(spec, w_cpu, x_cpu, target_s: float = 10.0):
    """The fp64 oracle, as it stands, on a bounded sample of the batch's tokens."""
    import oracle
    wnp = {k: inputs.to_numpy_storage(v) for k, v in w_cpu.items()}
    xnp = inputs.to_numpy_storage(x_cpu)
    threads = oracle.max_threads()
    n = min(max(4, threads), xnp.shape[0])
    t0 = time.perf_counter()
    oracle.forward(spec, wnp, xnp, tokens=np.arange(n), threads=threads)
    dt = time.perf_counter() - t0
    n2 = int(min(xnp.shape[0], max(n, n * target_s / max(dt, 1e-6))))
    t0 = time.perf_counter()
    oracle.forward(spec, wnp, xnp, tokens=np.arange(n2), threads=threads)
    dt2 = time.perf_counter() - t0
    return {"value": n2 / dt2, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"first {n2} of the {xnp.shape[0]} tokens of the same batch "
                      f"({dt2:.1f} s, fp64, OpenMP over tokens)",
            "sampled": n2 < xnp.shape[0]}


L2_BYTES = 126 * 2**20  # B200 L2 cache


def needs_l2_flush(spec, T) -> bool:
    """True when the step's weights could stay in L2 between timed steps: the largest
    possible activated set (min(E, T k) experts plus the dense weights) is under twice the
    L2 size. Those steps are timed one by one with L2 flushed in between."""
    most = min(spec.num_experts, T * spec.top_k) * expert_bytes(spec) + dense_bytes(spec)
    return most < 2 * L2_BYTES


def workload_name(spec) -> str:
    return (f"{spec.name} (hidden {spec.hidden}, {spec.num_experts} experts, top-{spec.top_k}, "
            f"intermediate {spec.intermediate}" + (f", latent {spec.latent_dim}" if spec.latent_dim else "") + ")")


def workload_config(spec, T, world):
    """The `config` object of both arms' JSON lines."""
    l2 = ("L2 flushed between timed steps (activated weights could fit in L2)" if needs_l2_flush(spec, T)
          else "activated weights larger than L2 (no flush needed)")
    return {"workload": workload_name(spec), "tokens_per_gpu": T, "parallelism": f"replicas x{world}",
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
    spec = workload_spec(args)
    T = args.tokens
    w_cpu = inputs.make_weights(spec)
    x_cpu = inputs.make_x(spec, T)
    import oracle
    wnp = {k: inputs.to_numpy_storage(v) for k, v in w_cpu.items()}
    xnp = inputs.to_numpy_storage(x_cpu)
    threads = oracle.max_threads()
    # each step: a bounded sample of the batch, sized so the whole run stays within minutes
    n0 = min(T, max(4, threads))
    t0 = time.perf_counter()
    oracle.forward(spec, wnp, xnp, tokens=np.arange(n0), threads=threads)
    per_tok = (time.perf_counter() - t0) / n0
    n = int(max(1, min(T, 30.0 / max(per_tok, 1e-9) / max(1, args.steps + args.warmup))))
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


# ------------------------------------------------------------------ timing helpers
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


def time_block(block, x, y, steps, warmup, flush):
    """Mean ms of one whole step: K back-to-back steps between two events, or (when the
    activated weights could stay in L2) one by one with L2 flushed in between."""
    for _ in range(warmup):
        block.forward(x, y)
    torch.cuda.synchronize()
    if flush is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            block.forward(x, y)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps
    return statistics.mean(time_steps(lambda: block.forward(x, y), steps, 0, flush=flush))


def e2e_pipelined(block, x_cpu, T, H, act_dt, steps, warmup, dev):
    """Mean ms per step through the public API with host buffers: every step copies its
    input from pinned host memory and its output back. Two buffer sets alternate, so the
    input copy of step i (one copy stream) and the output copy of step i-1 (another)
    overlap the compute of neighbouring steps; all K steps' copies are inside the timed
    region, which ends when the last output has reached the host."""
    xh = [x_cpu.pin_memory(), x_cpu.clone().pin_memory()]
    yh = [torch.empty((T, H), dtype=act_dt).pin_memory() for _ in range(2)]
    xd = [torch.empty((T, H), dtype=act_dt, device=dev) for _ in range(2)]
    yd = [torch.empty((T, H), dtype=act_dt, device=dev) for _ in range(2)]
    sc = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(n, start=None):
        if start is not None:
            s_in.wait_event(start)
        for i in range(n):
            b = i & 1
            if i >= 2:
                s_in.wait_event(ev_comp[b])      # step i-2 has finished reading xd[b]
            with torch.cuda.stream(s_in):
                xd[b].copy_(xh[b], non_blocking=True)
            ev_in[b].record(s_in)
            sc.wait_event(ev_in[b])
            if i >= 2:
                sc.wait_event(ev_out[b])         # yd[b] of step i-2 has reached the host
            block.forward(xd[b], yd[b], stream=sc)
            ev_comp[b].record(sc)
            s_out.wait_event(ev_comp[b])
            with torch.cuda.stream(s_out):
                yh[b].copy_(yd[b], non_blocking=True)
            ev_out[b].record(s_out)
        sc.wait_event(ev_out[(n - 1) & 1])
        if n >= 2:
            sc.wait_event(ev_out[n & 1])

    run(warmup)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(sc)
    run(steps, start=e0)
    e1.record(sc)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def distinct_experts(block, spec, x, T, dev) -> int:
    idx = torch.empty((T, spec.top_k), dtype=torch.int32, device=dev)
    wts = torch.empty((T, spec.top_k), dtype=torch.float32, device=dev)
    coef = torch.empty((T, 2), dtype=torch.float32, device=dev)
    M.moe_route(block.cfg, block.w, x, T, idx, wts, coef, block.ws)
    return int(torch.unique(idx).numel()), idx, wts


def fractions(spec, T, nd, ms, pk):
    b = block_bytes(spec, T, nd)
    f = block_flops(spec, T)
    s = ms / 1000.0
    return {"algorithmic_bytes": b, "gbs": b / s / 1e9, "hbm_frac": b / s / 1e9 / pk["hbm_gbs"],
            "tflops": f / s / 1e12, "tc_frac": f / s / 1e12 / pk["bf16_tflops"],
            "tc_frac_sustained": f / s / 1e12 / pk["bf16_tflops_sustained"]}


def decode_rows(block, spec, Ts, pk, steps, warmup, dev, dist):
    """Decode-sized batches: a CUDA graph of one step replayed with L2 flushed before each."""
    rows = []
    flush = l2_flush_buffer(dev) if Ts else None
    act_dt = block.act_dtype
    for Td in Ts:
        xd = inputs.make_x(spec, Td).to(dev)
        yd = torch.empty((Td, spec.hidden), dtype=act_dt, device=dev)
        nd, _, _ = distinct_experts(block, spec, xd, Td, dev)
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            block.forward(xd, yd, stream=s)
            g.capture_begin()
            block.forward(xd, yd, stream=s)
            g.capture_end()
        torch.cuda.current_stream().wait_stream(s)
        d_ms = time_steps(g.replay, max(steps, 20), warmup, flush=flush)
        med = max_over_ranks(statistics.median(d_ms), dist, dev)
        row = {"workload": spec.name, "tokens": Td, "tokens_per_s": Td / (med / 1000.0),
               "us_per_step": med * 1000.0, "distinct_experts": nd, "graded_on": "hbm"}
        row.update(fractions(spec, Td, nd, med, pk))
        rows.append(row)
        del g
    torch.cuda.synchronize()
    return rows


# ------------------------------------------------------------------ main arm
def main(argv=None):
    args = parse(argv)
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


def row_workloads(args):
    if args.rows == "none":
        return []
    if args.rows == "all":
        return list(ROW_ORDER)
    return [w.strip() for w in args.rows.split(",") if w.strip()]


def run(args, rank, world, local, dist):
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pk, pk_src = peaks()
    cpu_ok = rank == 0 and world == 1 and not args.no_cpu_baseline
    spec = workload_spec(args)
    T = args.tokens
    w_cpu = inputs.make_weights(spec)
    x_cpu = inputs.make_x(spec, T)
    block = M.MoeBlock(spec, w_cpu, max_tokens=max(T, 128), device=str(dev))
    x = x_cpu.to(dev)
    act_dt = block.act_dtype
    ab = 4 if spec.act_dtype == "f32" else 2
    y = torch.empty((T, spec.hidden), dtype=act_dt, device=dev)
    block.forward(x, y)
    torch.cuda.synchronize()
    if block.device_status() != 0:
        raise SystemExit("device status set after the first forward")
    n_distinct, idx, wts = distinct_experts(block, spec, x, T, dev)
    launches = kernels_per_step(lambda s: block.forward(x, y, stream=s))

    # ---- timed region: K whole steps
    l2_flush = l2_flush_buffer(dev) if needs_l2_flush(spec, T) else None
    sampler = ClockSampler(local)
    for _ in range(args.warmup):
        block.forward(x, y)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    ms = time_block(block, x, y, args.steps, 0, l2_flush)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()

    # ---- every kernel of the step, each timed alone with CUDA events (same arguments)
    table = None
    if not args.no_kernel_table:
        table = kernel_table(lambda s: block.forward(x, y, stream=s), max(5, args.steps // 2), flush=l2_flush)

    # ---- the routed-expert stage through the stepwise API (moe_grouped_ffn)
    K = spec.expert_in
    off = torch.empty(spec.num_experts + 1, dtype=torch.int32, device=dev)
    ss = torch.empty(T * spec.top_k, dtype=torch.int32, device=dev)
    sp = torch.empty(T * spec.top_k, dtype=torch.int32, device=dev)
    u = x
    if spec.latent_dim:
        u = torch.empty((T, spec.latent_dim), dtype=act_dt, device=dev)
        M.moe_latent_down(block.cfg, block.w, x, T, u, block.ws)
    M.moe_permute(block.cfg, idx, T, off, ss, sp, block.ws)
    y_acc = torch.empty((T, K), dtype=torch.float32, device=dev)
    ffn_ms = statistics.mean(time_steps(
        lambda: M.moe_grouped_ffn(block.cfg, block.w, u, T, off, ss, wts, y_acc, block.ws),
        args.steps, args.warmup, flush=l2_flush))
    clocks = sampler.stop()
    if block.device_status() != 0:
        raise SystemExit("device status set during the timed region")

    ms_max = max_over_ranks(ms, dist, dev)
    value = world * T / (ms_max / 1000.0)
    routed_bytes = n_distinct * expert_bytes(spec) + T * K * ab  # weights + expert inputs
    routed_flops = 2.0 * T * spec.top_k * 3 * spec.intermediate * K
    ffn_max = max_over_ranks(ffn_ms, dist, dev)
    routed_stage = {"ms_per_call": ffn_max, "algorithmic_bytes": routed_bytes,
                    "hbm_frac": routed_bytes / (ffn_max / 1000) / 1e9 / pk["hbm_gbs"],
                    "tc_frac": routed_flops / (ffn_max / 1000) / 1e12 / pk["bf16_tflops"]}

    # ---- roofline of the dominant kernel (the longest launch of the step)
    roofline = None
    per_kernel = None
    if table:
        tot = sum(t for _, t in table)
        per_kernel = [{"kernel": n, "us": round(t * 1000, 2), "share": round(t / tot, 4)} for n, t in table]
        gu, dn = label_expert_launches(table)
        roles = kernel_roles(spec, T, n_distinct)
        dom = max(range(len(table)), key=lambda i: table[i][1])
        role = "gate/up" if dom == gu else "down" if dom == dn else None
        if role is not None:
            r = roles[role]
            t_ms = max_over_ranks(table[dom][1], dist, dev)
            t_bw = r["bytes"] / (pk["hbm_gbs"] * 1e9)
            t_tc = r["flops"] / (pk["bf16_tflops"] * 1e12)
            bound = "hbm" if t_bw >= t_tc else "tensor"
            if bound == "hbm":
                ach, peak, unit, alg = r["bytes"] / (t_ms / 1000) / 1e9, pk["hbm_gbs"], "GB/s", r["bytes"]
            else:
                ach, peak, unit, alg = r["flops"] / (t_ms / 1000) / 1e12, pk["bf16_tflops"], "TFLOP/s", r["flops"]
            roofline = {"bound": bound, "achieved": ach, "peak": peak, "unit": unit, "frac": ach / peak,
                        "traffic": recorded_traffic(spec.name, T, table[dom][0]),
                        "kernel": f"{table[dom][0]} (expert {role}: routed + shared experts, one launch)",
                        "algorithmic_per_launch": alg, "ms_per_launch": t_ms,
                        "hbm_frac": r["bytes"] / (t_ms / 1000) / 1e9 / pk["hbm_gbs"],
                        "tc_frac": r["flops"] / (t_ms / 1000) / 1e12 / pk["bf16_tflops"],
                        "peak_source": f"{pk_src} (MEASURED_PEAKS.json)" if pk_src == "measured" else "fallback"}
    if roofline is None:  # no per-kernel table: the routed-expert stage instead
        ach = routed_bytes / (ffn_max / 1000) / 1e9
        roofline = {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": ach / pk["hbm_gbs"], "traffic": None,
                    "kernel": "routed experts stage (moe_grouped_ffn)",
                    "algorithmic_per_launch": routed_bytes, "ms_per_launch": ffn_max,
                    "peak_source": f"{pk_src} (MEASURED_PEAKS.json)" if pk_src == "measured" else "fallback"}

    # ---- end to end through the public API with host buffers (copies overlapped)
    e2e = None
    if not args.no_e2e:
        e_ms = e2e_pipelined(block, x_cpu, T, spec.hidden, act_dt, args.steps, args.warmup, dev)
        e_max = max_over_ranks(e_ms, dist, dev)
        e2e = {"value": world * T / (e_max / 1000.0), "unit": "tokens/s", "ms_per_step": e_max,
               "h2d_bytes_per_step": T * spec.hidden * ab, "d2h_bytes_per_step": T * spec.hidden * ab,
               "copies": "pinned host -> device and back every step, on two copy streams overlapping "
                         "the neighbouring steps' compute"}

    # ---- per-workload rows: prefill (the headline's own numbers for its workload) + decode
    prefill_rows, dec_rows = [], []
    head_row = {"workload": spec.name, "tokens": T, "tokens_per_s": T / (ms_max / 1000.0),
                "us_per_step": ms_max * 1000.0, "distinct_experts": n_distinct, "graded_on": "tc"}
    head_row.update(fractions(spec, T, n_distinct, ms_max, pk))
    cpu = None
    if cpu_ok:
        cpu = cpu_baseline(spec, w_cpu, x_cpu, target_s=12.0)
        head_row["cpu_baseline"] = cpu
    prefill_rows.append(head_row)
    dts = DECODE.get(spec.name, ()) if args.decode_tokens is None else \
        tuple(int(t) for t in args.decode_tokens.split(",") if t.strip())
    dec_rows += decode_rows(block, spec, dts, pk, args.steps, args.warmup, dev, dist)
    del block, w_cpu, x, y, u, y_acc
    torch.cuda.empty_cache()
    for wl in row_workloads(args):
        if wl == spec.name or wl not in PREFILL:
            continue
        rs = inputs.WORKLOADS[wl]
        Tp = PREFILL[wl]
        wc = inputs.make_weights(rs)
        xc = inputs.make_x(rs, Tp)
        blk = M.MoeBlock(rs, wc, max_tokens=max(Tp, 128), device=str(dev))
        xr = xc.to(dev)
        yr = torch.empty((Tp, rs.hidden), dtype=blk.act_dtype, device=dev)
        blk.forward(xr, yr)
        nd, _, _ = distinct_experts(blk, rs, xr, Tp, dev)
        fl = l2_flush_buffer(dev) if needs_l2_flush(rs, Tp) else None
        if dist is not None:
            dist.barrier()
        pm = max_over_ranks(time_block(blk, xr, yr, args.steps, args.warmup, fl), dist, dev)
        row = {"workload": rs.name, "tokens": Tp, "tokens_per_s": Tp / (pm / 1000.0), "us_per_step": pm * 1000.0,
               "distinct_experts": nd, "graded_on": "tc"}
        row.update(fractions(rs, Tp, nd, pm, pk))
        if cpu_ok:
            row["cpu_baseline"] = cpu_baseline(rs, wc, xc, target_s=4.0)
        prefill_rows.append(row)
        dec_rows += decode_rows(blk, rs, DECODE.get(wl, ()), pk, args.steps, args.warmup, dev, dist)
        if blk.device_status() != 0:
            raise SystemExit(f"device status set in the {wl} rows")
        del blk, wc, xr, yr
        torch.cuda.empty_cache()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": spec.act_dtype if spec.weight_format in ("bf16", "f32") else "bf16+" + spec.weight_format,
            "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights; no checkpoint)",
            "config": workload_config(spec, T, world),
            "roofline": roofline,
            "block": head_row,
            "routed_stage": routed_stage,
            "per_kernel": per_kernel,
            "prefill": prefill_rows,
            "decode": dec_rows,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches * args.steps if launches >= 0 else None,
            "gpu_launches_per_step": launches,
            "clocks": clocks,
            "peaks": {**pk, "source": pk_src},
        }
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
