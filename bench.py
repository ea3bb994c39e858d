#!/usr/bin/env python3
"""Benchmark of the W4A8 MXFP4 MoE decode step on B200.

Workload: the Ling-shaped MoE layer at M=1 token (H=2560, I=768, E=256
experts, top-8; MXFP4 expert weights, FP8 E4M3 activations; softmax router
with the 8th/9th logit gap forced >= 1e-3). Inputs are synthetic and seeded.

The timed unit is one layer-step: the whole hot path (quantise, route, top-k,
union, gate/up + SwiGLU, down, combine). To keep the 126 MB L2 from serving
the weights, each layer-step reads a different layer of a 32-layer pool
(32 x 256 experts = 25.7 GB of MXFP4 weights), with the same x. One bench
"step" is one pass over the pool: 32 layer-steps, captured in one CUDA graph
and replayed.

Output: one JSON line from rank 0. `value` is tokens per second summed over
all ranks, where a token-step is M tokens through one layer-step. The line
also reports us/layer-step, expert-weight GB/s, the roofline of the kernel,
the CPU oracle baseline, an end-to-end number through the public API with
host buffers, and the SM clocks sampled during the timed region.

--impl reference times the CPU oracle (test infrastructure) on a bounded
sample of the same workload and prints the same metric.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MXFP4 MoE decode µs/layer-step, tokens/s; HBM GB/s as % of B200 peak"
H, I, E, K = 2560, 768, 256, 8
POOL_LAYERS = 32
SEED = 0


def expert_bytes(h=H, i=I):
    return 2 * i * h // 2 + 2 * i * h // 32 + h * i // 2 + h * i // 32


def algorithmic_bytes(M, U, h=H, i=I, e=E):
    """Bytes a layer-step must move: active expert weights, router, x, y."""
    return U * expert_bytes(h, i) + e * h * 4 + 2 * M * h * 2


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


KERNEL_SOURCES = {
    # the device code each kernel is compiled from
    "k_fused": ("moe_fused.cuh", "moe_device.cuh"),
    "k_tc": ("moe_tc.cuh", "moe_fused.cuh", "moe_device.cuh"),
    "k_lm_head": ("moe_lmhead.cu", "moe_device.cuh"),
}


def kernel_source_hash(kernel: str = "k_fused"):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mxfp4_weight_streaming_fp8_b200", "csrc")
    for fn in KERNEL_SOURCES.get(kernel, ()):
        h.update(open(os.path.join(csrc, fn), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path))[kernel][workload]
    except Exception:
        return None
    if rec.get("source_hash") != kernel_source_hash(kernel):
        return None
    return rec.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ distributed
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, ws: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity at world size 1)."""
    if ws == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, ws: int, device=None) -> float:
    if ws == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------------ workload
def build_pool(device, M, mode, layers=POOL_LAYERS, seed=SEED, flags=0, stack=False, shared=False, repack=False):
    """One context per layer of the pool. With stack=True, layers after the
    first normalise their input (RMSNorm) and take the previous output. With
    shared=True every layer has one more expert (index E), the shared one."""
    import torch
    from mxfp4_weight_streaming_fp8_b200 import moe, synth
    x = synth.gen_x(seed, M, H)
    ctxs, weights = [], []
    for l in range(layers):
        # routing forced against the shared input (a stacked layer's input is
        # the previous output, so its routing stays natural)
        wr = synth.gen_router(seed, l, E, H)
        if not (stack and l > 0):
            wr = synth.force_router(x, wr, K, mode, seed=seed, layer=l)
        ex = synth.layer_experts_torch(seed, l, E + int(shared), H, I, device)
        wr_d = torch.from_numpy(wr).to(device)
        lflags = flags | (moe.MOE_FLAG_PRE_RMSNORM if (stack and l > 0) else 0)
        lflags |= moe.MOE_FLAG_SHARED_EXPERT if shared else 0
        ctx = moe.MoELayer(H, I, E, K, M, flags=lflags, device=device.index)
        ctx.load_experts(wr_d, *ex, validate=False, repack=repack)
        ctxs.append(ctx)
        weights.append((wr_d, ex))
    return x, ctxs, weights


def run_ours(args):
    import torch
    ws, rank, local = dist_env()
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local if ws > 1 else 0)
    torch.cuda.set_device(device)
    from mxfp4_weight_streaming_fp8_b200 import moe
    M = args.tokens
    L = args.layers
    flags = {"split": moe.MOE_FLAG_SPLIT_KERNELS, "cuda": moe.MOE_FLAG_CUDA_CORES,
             "tc": moe.MOE_FLAG_TENSOR_CORES}.get(args.variant, 0)
    flags |= moe.MOE_FLAG_FP8_INTERMEDIATE if args.fp8_intermediate else 0
    flags |= moe.MOE_FLAG_SPLITK_DOWN if args.splitk_down else 0
    flags |= {"mma": moe.MOE_FLAG_TC_DOWN_MMA, "cuda": moe.MOE_FLAG_TC_DOWN_CUDA}.get(args.tc_down, 0)
    x, ctxs, _weights = build_pool(device, M, args.routing, layers=L, flags=flags, stack=args.stack,
                                   shared=args.shared_expert, repack=args.repack)
    n_shared = int(args.shared_expert)
    info = ctxs[0].query()
    x_d = x.to(device)
    ys = [torch.empty_like(x_d) for _ in range(L)]
    # layer l reads x (independent layer-steps) or, stacked, the previous output
    inputs = [x_d if (l == 0 or not args.stack) else ys[l - 1] for l in range(L)]

    # union size of each layer (from the kernel's own routing outputs)
    Us = []
    for l in range(L):
        out = ctxs[l].decode(inputs[l], y=ys[l], routing=True)
        Us.append(len(set(out[1].cpu().numpy().ravel().tolist())))
    torch.cuda.synchronize()
    for c in ctxs:
        st = c.sync_status()
        if st != moe.MOE_OK:
            raise RuntimeError(f"kernel status {moe.status_string(st)}")

    # one bench step = L layer-steps, captured once
    stream = torch.cuda.Stream(device)
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        for l in range(L):
            assert ctxs[l].decode_raw(inputs[l], M, ys[l], stream=stream) == moe.MOE_OK
    torch.cuda.current_stream().wait_stream(stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for l in range(L):
            st = ctxs[l].decode_raw(inputs[l], M, ys[l], stream=stream)
            assert st == moe.MOE_OK, moe.status_string(st)

    # the same pool as a dependent chain: layer l+1 takes RMSNorm(y_l), so no
    # layer-step can overlap the previous one (timed after the headline graph)
    chain = None if args.stack else build_chain(device, ctxs, _weights, x_d, M, flags, args.shared_expert,
                                                args.repack)

    cur = torch.cuda.current_stream()
    for _ in range(args.warmup):
        graph.replay()
        if chain:
            chain["graph"].replay()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev2, ev3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(device.index) as clk:
        ev0.record(cur)
        for _ in range(args.steps):
            graph.replay()
        ev1.record(cur)
        ev1.synchronize()
        if chain:
            ev2.record(cur)
            for _ in range(args.steps):
                chain["graph"].replay()
            ev3.record(cur)
            ev3.synchronize()
    torch.cuda.synchronize()
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
    ms_local = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms_local, ws, device)
    for c in ctxs:
        st = c.sync_status()
        if st != moe.MOE_OK:
            raise RuntimeError(f"kernel status {moe.status_string(st)}")

    layer_steps = args.steps * L
    us_per_layer = ms * 1e3 / layer_steps
    U_mean = sum(Us) / len(Us)
    tokens_total = ws * M * layer_steps
    value = tokens_total / (ms / 1e3)
    alg = algorithmic_bytes(M, U_mean + n_shared)
    exp_b = (U_mean + n_shared) * expert_bytes()
    peak, peak_kind = load_peaks()
    achieved = alg / (us_per_layer * 1e-6) / 1e9
    workload = (f"ling_stack{L}_rmsnorm_M{M}" if args.stack else f"ling_layer_M{M}_{args.routing}")
    workload += "_shared1" if n_shared else ""
    workload += "_a8" if args.fp8_intermediate else ""
    traffic = recorded_traffic({"fused": "k_fused", "tc": "k_tc"}.get(info["variant"], "split"), workload)

    # ---- end to end through the public API with host buffers
    e2e = run_e2e(args, ctxs, x, device, M, L, stack=args.stack)

    # ---- CPU oracle baseline (rank 0 only)
    cpu = (run_cpu_baseline(args, M, shared=args.shared_expert, a8=args.fp8_intermediate)
           if rank == 0 and not args.no_cpu else None)

    launches = layer_steps * (3 if info["variant"] == "split" else 1)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp8e4m3 x mxfp4 (f16/fp32 accumulate)",
        "data": "synthetic (seeded SplitMix64; random MXFP4 weights, N(0,1) bf16 activations)",
        "config": {"workload": workload, "hidden": H, "inter": I, "num_experts": E, "top_k": K, "tokens": M,
                   "routing": args.routing, "shared_experts": n_shared,
                   "fp8_intermediate": bool(args.fp8_intermediate), "layers_in_pool": L,
                   "pool_weight_bytes": L * (E + n_shared) * expert_bytes(),
                   "l2": "inputs larger than L2: each layer-step reads a different layer of the pool",
                   "step": (f"{L}-layer stack (RMSNorm between layers) in one CUDA graph" if args.stack
                            else f"{L} layer-steps in one CUDA graph"), "parallelism": f"replicas x{ws}",
                   "variant": info["variant"], **({"down": info["down"]} if "down" in info else {}),
                   **({"splitk_down": True} if args.splitk_down else {})},
        "us_per_layer_step": round(us_per_layer, 3),
        "union_experts": U_mean,
        "expert_gbs": round(exp_b / (us_per_layer * 1e-6) / 1e9, 1),
        "expert_frac_of_8tbs": round(exp_b / (us_per_layer * 1e-6) / 8e12, 4),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                     "traffic": traffic,
                     "kernel": {"fused": "k_fused", "tc": "k_tc"}.get(info["variant"], "k_gateup+k_down"),
                     "algorithmic_bytes_per_launch": alg},
        "gpu_launches": launches,
        "clocks": clk.summary(),
        "e2e": e2e,
    }
    if args.stack:
        line["stack_tokens_per_s"] = round(ws * M * args.steps / (ms / 1e3), 1)
        line["us_per_stack_step"] = round(ms * 1e3 / args.steps, 2)
    if chain:
        ms_chain = max_over_ranks(ev2.elapsed_time(ev3), ws, device)
        for c in chain["ctxs"]:
            st = c.sync_status()
            if st != moe.MOE_OK:
                raise RuntimeError(f"kernel status {moe.status_string(st)}")
        us_chain = ms_chain * 1e3 / (args.steps * L)
        line["dependent_chain"] = {
            "us_per_layer_step": round(us_chain, 3),
            "tokens_per_s": round(ws * M * args.steps / (ms_chain / 1e3), 1),
            "frac_of_peak": round(alg / (us_chain * 1e-6) / 1e9 / peak, 4),
            "how": (f"the same {L} layers as a stack in one CUDA graph: layer l+1 takes RMSNorm(y_l) "
                    f"(unit weight), so each layer-step starts after the previous one ends; "
                    f"{args.steps} replays timed with CUDA events after the headline graph")}
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph
    if chain:
        del chain["graph"]
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def run_split(args):
    """--parts G: the intra-expert split of every pool layer (part g holds
    gate/up rows [g*I/G, (g+1)*I/G) of each expert and the same down
    columns). Under torchrun with N = G ranks, rank g holds part g and a
    layer-step is moe_decode of the part (fp32 sums), one NCCL all-reduce of
    the M x H sums and the bf16 round (moe.decode_split); the whole layer's
    work is fixed, so scaling is strong and each token counts once. In one
    process with G > 1 it times part 0 of G alone in one CUDA graph, as the
    default bench times whole layers: the per-GPU kernel time of a G-way
    split, without the exchange."""
    import torch
    ws, rank, local = dist_env()
    G = args.parts
    if ws > 1 and ws != G:
        raise SystemExit("--parts must equal the number of ranks")
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local if ws > 1 else 0)
    torch.cuda.set_device(device)
    from mxfp4_weight_streaming_fp8_b200 import moe, synth
    M, L, g = args.tokens, args.layers, (rank if ws > 1 else 0)
    x = synth.gen_x(SEED, M, H)
    ctxs = []
    for l in range(L):
        wr = synth.force_router(x, synth.gen_router(SEED, l, E, H), K, args.routing, seed=SEED, layer=l)
        ex = synth.layer_experts_torch(SEED, l, E, H, I, device)
        ctx = moe.MoELayer(H, I, E, K, M, device=device.index, shard=(g, G))
        ctx.load_experts(torch.from_numpy(wr).to(device), *ex, validate=False)  # keeps a copy of part g
        del ex
        ctxs.append(ctx)
    info = ctxs[0].query()
    x_d = x.to(device)
    y32 = [torch.empty((M, H), dtype=torch.float32, device=device) for _ in range(L)]
    ys = [torch.empty_like(x_d) for _ in range(L)]
    Us = []
    for l in range(L):
        out = ctxs[l].decode(x_d, y=y32[l], routing=True)
        Us.append(len(set(out[1].cpu().numpy().ravel().tolist())))
    torch.cuda.synchronize()
    cur = torch.cuda.current_stream()
    graph = None
    if ws == 1:
        stream = torch.cuda.Stream(device)
        stream.wait_stream(cur)
        with torch.cuda.stream(stream):
            for l in range(L):
                assert ctxs[l].decode_raw(x_d, M, y32[l], stream=stream) == moe.MOE_OK
        cur.wait_stream(stream)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for l in range(L):
                assert ctxs[l].decode_raw(x_d, M, y32[l], stream=stream) == moe.MOE_OK

    def step():
        if graph is not None:
            graph.replay()
        else:
            for l in range(L):
                moe.decode_split(ctxs[l], x_d, y32=y32[l], y=ys[l])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(device.index) as clk:
        ev0.record(cur)
        for _ in range(args.steps):
            step()
        ev1.record(cur)
        ev1.synchronize()
    torch.cuda.synchronize()
    ms = max_over_ranks(ev0.elapsed_time(ev1), ws, device)
    for c in ctxs:
        st = c.sync_status()
        if st != moe.MOE_OK:
            raise RuntimeError(f"kernel status {moe.status_string(st)}")
    us = ms * 1e3 / (args.steps * L)
    U_mean = sum(Us) / len(Us)
    # a part reads 1/G of each active expert, the whole router, x, and writes fp32 sums
    alg = U_mean * expert_bytes(H, I // G) + E * H * 4 + M * H * 2 + M * H * 4
    peak, peak_kind = load_peaks()
    achieved = alg / (us * 1e-6) / 1e9
    alone = ws == 1
    line = {
        "metric": METRIC, "value": round(M * args.steps * L / (ms / 1e3), 1), "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak" if alone else "strong", "vs_baseline": None,
        "dtype": "fp8e4m3 x mxfp4 (f16/fp32 accumulate)",
        "data": "synthetic (seeded SplitMix64; random MXFP4 weights, N(0,1) bf16 activations)",
        "config": {"workload": f"ling_layer_M{M}_{args.routing}_split{G}" + ("_part0_alone" if alone else ""),
                   "hidden": H, "inter": I, "inter_per_part": I // G, "num_experts": E, "top_k": K,
                   "tokens": M, "routing": args.routing, "layers_in_pool": L,
                   "l2": "inputs larger than L2: each layer-step reads a different layer of the pool",
                   "step": (f"part 0 of {G} of {L} layers in one CUDA graph (no exchange)" if alone else
                            f"{L} layers, each: part of rank g, NCCL all-reduce of fp32 sums, bf16 round"),
                   "parallelism": f"intra-expert split x{G}", "variant": info["variant"]},
        "us_per_layer_step": round(us, 3),
        "union_experts": U_mean,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": peak_kind, "traffic": None,
                     "kernel": {"fused": "k_fused", "tc": "k_tc"}.get(info["variant"], "k_gateup+k_down"),
                     "algorithmic_bytes_per_launch": alg},
        "gpu_launches": args.steps * L * (1 if alone else 2),
        "clocks": clk.summary(),
        "e2e": None,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def build_chain(device, ctxs, weights, x_d, M, flags, shared, repack=False):
    """Contexts over the pool's own weights chained as a stack (layers after
    the first normalise their input), captured in one CUDA graph."""
    import torch
    from mxfp4_weight_streaming_fp8_b200 import moe
    L = len(ctxs)
    chain = []
    for l, (wr_d, ex) in enumerate(weights):
        lflags = flags | (moe.MOE_FLAG_PRE_RMSNORM if l > 0 else 0)
        lflags |= moe.MOE_FLAG_SHARED_EXPERT if shared else 0
        c = moe.MoELayer(H, I, E, K, M, flags=lflags, device=device.index)
        c.load_experts(wr_d, *ex, validate=False, repack=repack)
        chain.append(c)
    ys = [torch.empty_like(x_d) for _ in range(L)]
    stream = torch.cuda.Stream(device)
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        for l in range(L):
            assert chain[l].decode_raw(x_d if l == 0 else ys[l - 1], M, ys[l], stream=stream) == moe.MOE_OK
    torch.cuda.current_stream().wait_stream(stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for l in range(L):
            assert chain[l].decode_raw(x_d if l == 0 else ys[l - 1], M, ys[l], stream=stream) == moe.MOE_OK
    return {"ctxs": chain, "graph": g, "ys": ys}


def run_e2e(args, ctxs, x_cpu, device, M, L, stack=False):
    """Per step: pinned-host x -> device, L moe_decode calls through the
    Python/C-ABI API, final y -> pinned host; timed with events."""
    import torch
    from mxfp4_weight_streaming_fp8_b200 import moe
    xh = x_cpu.pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    xd = torch.empty_like(xh, device=device)
    ys = [torch.empty_like(xd) for _ in range(L)]
    cur = torch.cuda.current_stream()

    def step():
        xd.copy_(xh, non_blocking=True)
        for l in range(L):
            ctxs[l].decode_raw(ys[l - 1] if (stack and l > 0) else xd, M, ys[l], stream=cur)
        yh.copy_(ys[-1], non_blocking=True)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    for _ in range(args.steps):
        step()
    e1.record(cur)
    e1.synchronize()
    ms = e0.elapsed_time(e1)
    ws, _, _ = dist_env()
    ms = max_over_ranks(ms, ws, device)
    tokens = ws * M * L * args.steps
    return {"value": round(tokens / (ms / 1e3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": xh.numel() * 2, "d2h_bytes_per_step": yh.numel() * 2,
            "how": f"per step: H2D x, {L} moe_decode calls (direct launches), D2H y"}


def cpu_sample_steps(M, n_layers, seed=SEED, shared=False):
    """Inputs of a bounded oracle sample: n_layers layer-steps of the pool
    (with the shared expert's arrays when shared=True)."""
    import numpy as np
    import oracle
    from mxfp4_weight_streaming_fp8_b200 import synth
    x = synth.gen_x(seed, M, H)
    xb = x.view(__import__("torch").int16).numpy().view(np.uint16)
    steps = []
    for l in range(n_layers):
        wr = synth.force_router(x, synth.gen_router(seed, l, E, H), K, "gap", seed=seed, layer=l)
        ids, _ = oracle.topk(oracle.router_logits(xb, wr), K)
        per = [[None] * E for _ in range(4)]
        for e in sorted(set(ids.ravel().tolist())):
            parts = synth.expert_np(seed, l, e, H, I)
            for t in range(4):
                per[t][e] = parts[t]
        steps.append((wr, per, synth.expert_np(seed, l, E, H, I) if shared else None))
    return xb, steps


def oracle_step(xb, step, a8=False):
    import oracle
    wr, per, sh = step
    if a8:
        return oracle.moe_decode_a8(xb, wr, *per, H, I, E, K, shared=sh)
    if sh is None:
        return oracle.moe_decode(xb, wr, *per, H, I, E, K)
    return oracle.moe_decode_shared(xb, wr, *per, sh, H, I, E, K)


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def time_oracle_steps(xb, steps, n_steps, threads, a8=False):
    """Wall time of n_steps oracle layer-steps (cycling over `steps`) run by
    `threads` host threads, each step whole on one thread. The oracle is a
    C library called through ctypes, which releases the GIL, so the threads
    run on separate cores; the oracle itself is unchanged."""
    from concurrent.futures import ThreadPoolExecutor
    t0 = time.perf_counter()
    if threads == 1:
        for i in range(n_steps):
            oracle_step(xb, steps[i % len(steps)], a8)
    else:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(lambda i: oracle_step(xb, steps[i % len(steps)], a8), range(n_steps)))
    return time.perf_counter() - t0


def run_cpu_baseline(args, M, n_layers=None, shared=False, a8=False):
    """The oracle on the host cores: one thread, then every core the process
    may use (independent layer-steps in parallel). The all-core leg is the
    reported value."""
    n_layers = n_layers or args.cpu_layers
    xb, steps = cpu_sample_steps(M, n_layers, shared=shared)
    dt1 = time_oracle_steps(xb, steps, n_layers, 1, a8)
    cores = host_cores()
    n_all = max(n_layers, 2 * cores)
    dtn = time_oracle_steps(xb, steps, n_all, cores, a8)
    return {"value": round(M * n_all / dtn, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"{n_all} layer-steps of the same workload (M={M}, cycling over {n_layers} distinct pool "
                      f"layers) on {cores} host threads, one layer-step per thread at a time; fp64 C++ oracle, "
                      f"{dtn:.2f} s",
            "single_thread": {"value": round(M * n_layers / dt1, 3), "unit": "tokens/s", "cores": 1,
                              "sample": f"{n_layers} layer-steps on one thread, {dt1:.2f} s"}}


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    M = args.tokens
    n = max(1, args.ref_layers)
    xb, steps = cpu_sample_steps(M, n, shared=args.shared_expert)
    for _ in range(min(args.warmup, 1)):
        oracle_step(xb, steps[0], args.fp8_intermediate)
    cores = host_cores()
    # each bench step is one layer-step per host thread, all threads at once
    dt = time_oracle_steps(xb, steps, args.steps * cores, cores, args.fp8_intermediate)
    value = M * args.steps * cores / dt
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt * 1e3 / args.steps, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"ling_layer_M{M}_{args.routing}" + ("_shared1" if args.shared_expert else "")
                       + ("_a8" if args.fp8_intermediate else ""),
                       "hidden": H, "inter": I, "num_experts": E, "top_k": K, "tokens": M,
                       "shared_experts": int(args.shared_expert),
                       "step": f"{cores} layer-steps of the CPU oracle at once, one per host thread"},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "cpu_model": cpu_model(),
                             "sample": f"{args.steps * cores} layer-steps cycling over {n} pool layers on "
                                       f"{cores} threads, {dt:.2f} s"},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


LM_V, LM_H = 157184, 2560
LM_METRIC = "FP8 LM head GEMV (157,184 x 2,560) µs/call, tokens/s; HBM GB/s as % of B200 peak"


def run_lm_head(args):
    """The FP8 LM head on one GPU: each step is one call for M tokens; the
    402 MB FP8 matrix is far larger than L2, so every call streams it."""
    import numpy as np
    import torch
    from mxfp4_weight_streaming_fp8_b200 import moe
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    M = args.tokens
    g = torch.Generator(device=device).manual_seed(SEED)
    lm = moe.LMHead(LM_V, LM_H, max_tokens=M)
    w = (torch.randn(LM_V, LM_H, generator=g, device=device) * 0.02).to(torch.bfloat16)
    lm.load(w)
    w_cpu_rows = w[:65536].cpu()  # CPU baseline sample (~1-2 s of oracle work)
    del w
    x = torch.randn(M, LM_H, generator=g, device=device).to(torch.bfloat16)
    logits = torch.empty((M, LM_V), dtype=torch.float32, device=device)
    calls = 8  # calls per graph replay
    stream = torch.cuda.Stream(device)
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        assert lm.head_raw(x, M, logits, stream=stream) == moe.MOE_OK
    torch.cuda.current_stream().wait_stream(stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for _ in range(calls):
            assert lm.head_raw(x, M, logits, stream=stream) == moe.MOE_OK
    cur = torch.cuda.current_stream()
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index) as clk:
        ev0.record(cur)
        for _ in range(args.steps):
            graph.replay()
        ev1.record(cur)
        ev1.synchronize()
    ms = ev0.elapsed_time(ev1)
    st = lm.sync_status()
    if st != moe.MOE_OK:
        raise RuntimeError(f"kernel status {moe.status_string(st)}")
    n_calls = args.steps * calls
    us_call = ms * 1e3 / n_calls
    alg = LM_V * LM_H + 4 * LM_V + 2 * M * LM_H + 4 * M * LM_V
    peak, peak_kind = load_peaks()
    achieved = alg / (us_call * 1e-6) / 1e9
    workload = f"lm_head_fp8_V{LM_V}_H{LM_H}_M{M}"
    # end to end: pinned x in, one call, logits out
    xh = x.cpu().pin_memory()
    lh = torch.empty((M, LM_V), dtype=torch.float32).pin_memory()
    xd = torch.empty_like(x)
    for _ in range(args.warmup):
        xd.copy_(xh, non_blocking=True)
        lm.head_raw(xd, M, logits, stream=cur)
        lh.copy_(logits, non_blocking=True)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    for _ in range(args.steps):
        xd.copy_(xh, non_blocking=True)
        lm.head_raw(xd, M, logits, stream=cur)
        lh.copy_(logits, non_blocking=True)
    e1.record(cur)
    e1.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    line = {
        "metric": LM_METRIC, "value": round(M * n_calls / (ms / 1e3), 1), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8e4m3 x bf16 (f16 MMA, fp32 accumulate)", "data": "synthetic (seeded N(0,0.02) bf16 weights)",
        "config": {"workload": workload, "vocab": LM_V, "hidden": LM_H, "tokens": M,
                   "l2": "inputs larger than L2: every call streams the 402 MB FP8 matrix",
                   "step": f"{calls} calls in one CUDA graph"},
        "us_per_call": round(us_call, 3),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                     "traffic": recorded_traffic("k_lm_head", workload), "kernel": "k_lm_head",
                     "algorithmic_bytes_per_launch": alg},
        "gpu_launches": n_calls, "clocks": clk.summary(),
        "e2e": {"value": round(M * args.steps / (e2e_ms / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": M * LM_H * 2, "d2h_bytes_per_step": M * LM_V * 4,
                "how": "per step: H2D x, one moe_lm_head call, D2H logits"},
    }
    if not args.no_cpu:
        import oracle
        rows = w_cpu_rows.shape[0]
        codes, scales = oracle.lm_quantize(w_cpu_rows.view(torch.int16).numpy().view(np.uint16))
        xb = x.cpu().view(torch.int16).numpy().view(np.uint16)
        t0 = time.perf_counter()
        oracle.lm_head(codes, scales, xb)
        dt = time.perf_counter() - t0
        per_call = dt * LM_V / rows
        line["cpu_baseline"] = {"value": round(M / per_call, 4), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "sample": f"{rows} of {LM_V} rows for M={M} ({dt:.2f} s), scaled to the full "
                                          "matrix; single-threaded fp64 C++ oracle"}
    print(json.dumps(line), flush=True)
    del graph
    lm.close()


def run_reference_lm_head(args):
    """Reference arm of --op lm_head: the CPU oracle's FP8 LM head on a
    bounded sample of rows, each step one call for M tokens, scaled to the
    full vocabulary. The FP8 copy is made once, outside the timed steps, as
    the library does at load."""
    import numpy as np
    import torch
    import oracle
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    M = args.tokens
    rows = max(1, min(LM_V, args.ref_rows))
    g = torch.Generator().manual_seed(SEED)
    w = (torch.randn(rows, LM_H, generator=g) * 0.02).to(torch.bfloat16)
    x = torch.randn(M, LM_H, generator=g).to(torch.bfloat16)
    codes, scales = oracle.lm_quantize(w.view(torch.int16).numpy().view(np.uint16))
    xb = x.view(torch.int16).numpy().view(np.uint16)
    for _ in range(min(args.warmup, 1)):
        oracle.lm_head(codes, scales, xb)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.lm_head(codes, scales, xb)
    dt = time.perf_counter() - t0
    per_call = dt / args.steps * LM_V / rows
    value = M / per_call
    line = {"impl": "reference", "metric": LM_METRIC, "value": round(value, 4), "unit": "tokens/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(per_call * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"lm_head_fp8_V{LM_V}_H{LM_H}_M{M}", "vocab": LM_V, "hidden": LM_H,
                       "tokens": M, "step": "one LM head call of the CPU oracle on host cores"},
            "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": f"{rows} of {LM_V} rows per call ({args.steps} calls, {dt:.2f} s), "
                                       "scaled to the full matrix"},
            "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--tokens", type=int, default=1)
    ap.add_argument("--routing", default="gap", choices=["gap", "zipf", "distinct", "shared", "natural"])
    ap.add_argument("--layers", type=int, default=POOL_LAYERS)
    ap.add_argument("--cpu-layers", type=int, default=16)
    ap.add_argument("--ref-layers", type=int, default=4)
    ap.add_argument("--ref-rows", type=int, default=32768,
                    help="LM head rows per reference (CPU oracle) call, scaled to the vocabulary")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--variant", choices=["auto", "cuda", "tc", "split"], default="auto",
                    help="auto: the library's choice for the shape; cuda: the CUDA-core persistent kernel; "
                         "tc: the tensor-core persistent kernel; split: the three-kernel path")
    ap.add_argument("--repack", action="store_true",
                    help="load the layers with MOE_LOAD_COPY_REPACK (context-owned, kernel-private weight layout)")
    ap.add_argument("--shared-expert", action="store_true",
                    help="one always-active shared expert per layer besides the top-8 routed ones")
    ap.add_argument("--tc-down", choices=["auto", "mma", "cuda"], default="auto",
                    help="tensor-core kernel's down projection: auto (the library's choice), mma (tcgen05), "
                         "cuda (CUDA cores)")
    ap.add_argument("--splitk-down", action="store_true",
                    help="down projection split over K with CTA-local h (max 4 tokens)")
    ap.add_argument("--fp8-intermediate", action="store_true",
                    help="quantise the SwiGLU output to E4M3 per (token, expert) before the down projection")
    ap.add_argument("--stack", action="store_true",
                    help="chain the pool as a stack: layer l+1 takes RMSNorm(y_l)")
    ap.add_argument("--parts", type=int, default=1,
                    help="intra-expert split into this many parts: one per rank under torchrun; in one "
                         "process, part 0 alone (its per-GPU kernel time)")
    ap.add_argument("--op", choices=["moe", "lm_head"], default="moe",
                    help="moe: the MoE layer step (default); lm_head: the FP8 LM head GEMV")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference" and args.op == "lm_head":
        run_reference_lm_head(args)
    elif args.impl == "reference":
        run_reference(args)
    elif args.op == "lm_head":
        run_lm_head(args)
    elif args.parts > 1:
        run_split(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
