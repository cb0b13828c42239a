#!/usr/bin/env python
"""Benchmark of the quantized top-10 MoE layer on B200.

Headline (one JSON line on rank 0): MoE-layer tokens/s for a decode window of
T = 5 tokens (1 token + 4 speculative drafts) on a layer of E = 512 experts,
k = 10, H = 2048, I = 512, 4-bit block-32 weights.  Objects in the same line
report the other workloads, each with its own roofline:
  decode_T1      the same layer shape, T = 1;
  prefill        one 8,192-token chunk, 4-bit, Gaussian router;
  decode_stack   48 layers x 256 experts, 2/2/4-bit, Zipf router, T = 5, chained;
  prefill_stack  48 layers x 512 experts, 2/2/4-bit, Zipf router, T = 8,192, chained,
                 with the per-expert roofline sum_e max(flops_e / TC, bytes_e / HBM).
A step is one full layer call (router, grouping, expert FFN, combine,
histogram), or one pass through the 48-layer stack for the stacks.

Weights never come from L2: single-layer workloads rotate through several
layer arenas (8 x 906 MB for decode, 2 for prefill) with a fresh input per
layer; a stack step streams 48 layers' experts (GBs) before it repeats.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs an independent replica on its own seeds (the
layer has no cross-token exchange); value = tokens of all ranks / max time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s (decode T=5, prefill T=8192); % HBM / tensor-pipe roofline"
DECODE_LAYERS = 8
PREFILL_LAYERS = 2
DECODE_WORKLOAD = "decode window: 1 layer, E=512, top_k=10, H=2048, I=512, T=5, 4-bit block-32"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-prefill", action="store_true")
    p.add_argument("--no-decode", action="store_true", help="profiling runs: no decode sections")
    p.add_argument("--no-stacks", action="store_true", help="skip the two 48-layer stacks")
    p.add_argument("--no-midt", action="store_true", help="skip the mid-T (T = 16, 64, 256) prefill lines")
    p.add_argument("--no-cpu-baseline", action="store_true", help="profiling runs: skip the oracle timing")
    p.add_argument("--decode-layers", type=int, default=DECODE_LAYERS,
                   help="rotating decode layer arenas (profiling runs use 1)")
    p.add_argument("--prefill-steps", type=int, default=None)
    p.add_argument("--stack-steps", type=int, default=None)
    return p.parse_args()


def profiled_traffic(summary: str, sources) -> int | None:
    """DRAM bytes per launch from a committed ncu summary under profiles/, or None
    when the kernel's sources changed since that capture."""
    import hashlib
    try:
        text = open(os.path.join(ROOT, "profiles", summary)).read()
        m = hashlib.sha256()
        for f in sources:
            m.update(open(os.path.join(ROOT, "quantized_expert_ffn_top10_b200", "csrc", f), "rb").read())
        fields = dict(l.split(": ", 1) for l in text.splitlines() if l.startswith(("traffic_", "kernel_sources")))
        if fields.get("kernel_sources_sha256", "").strip() != m.hexdigest():
            return None
        return int(fields["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return m["hbm_gbs"], m["bf16_tflops"], m["bf16_tflops_sustained"], "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ----------------------------------------------------------------------------- clocks

class Clocks:
    """nvidia-smi samples every 200 ms while the timed region runs."""

    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, dev: int):
        self.dev, self.rows, self.proc = dev, [], None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([v.strip() for v in line.split(",")])

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=2)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[0]) for r in self.rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if len(r) > 3 + i and r[3 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


# ----------------------------------------------------------------------------- workloads

class Inputs:
    """NL seeded layers of one shape on the device (arena, slot table, router,
    bias, one input per layer).  Uses moe_synth and torch only."""

    def __init__(self, cfg, NL: int, rank: int):
        import numpy as np
        import torch
        import moe_synth as S
        self.cfg = S.config(cfg.name, L=NL, T=cfg.T, seed=replica_seed(cfg.seed, rank))
        c = self.cfg
        self.NL = NL
        self.desc = c.desc()
        self.arena = S.gen_arena_device(c)
        self.table = torch.from_numpy(S.gen_slot_table(c)).cuda()
        self.W = [torch.from_numpy(S.gen_router(c, l)).cuda() for l in range(NL)]
        self.b = [None if S.gen_bias(c, l) is None else torch.from_numpy(S.gen_bias(c, l)).cuda() for l in range(NL)]
        self.x_host = [S.gen_x(c, c.T, stream_offset=l) for l in range(NL)]
        self.x = [torch.from_numpy(h.view(np.int16)).cuda() for h in self.x_host]


class Layers(Inputs):
    """Inputs plus what a call through the library needs: workspace, outputs,
    the histogram and per-layer expert offsets."""

    def __init__(self, cfg, NL: int, rank: int):
        import torch
        import quantized_expert_ffn_top10_b200 as M
        super().__init__(cfg, NL, rank)
        c = self.cfg
        self.out = [torch.empty_like(v) for v in self.x]
        self.ws = torch.empty(M.moe_workspace_bytes(c.T, c.E, c.top_k, c.H, c.I), dtype=torch.uint8, device="cuda")
        self.hist = torch.zeros((NL, c.E), dtype=torch.int32, device="cuda")
        self.offsets = [torch.zeros(c.E + 1, dtype=torch.int32, device="cuda") for _ in range(NL)]
        self.fn = M.moe_forward_prefill if c.T > M.MOE_DECODE_MAX_T else M.moe_forward_decode

    def call(self, l: int, x=None, out=None):
        c = self.cfg
        self.fn(self.desc, self.arena, self.table, self.NL, l, self.x[l] if x is None else x, self.W[l], self.b[l],
                c.top_k, True, self.out[l] if out is None else out, hist=self.hist,
                route_out={"expert_offsets": self.offsets[l]}, ws=self.ws)

    def call_stack(self, a, b):
        """Layers 0..NL-1 chained: layer l reads one buffer and writes the other."""
        bufs = (a, b)
        for l in range(self.NL):
            self.call(l, x=bufs[l % 2], out=bufs[(l + 1) % 2])

    def distinct(self):
        return [int((o[1:] - o[:-1] > 0).sum().item()) for o in self.offsets]

    def loads(self):
        return [(o[1:] - o[:-1]).cpu().numpy() for o in self.offsets]


def time_graphs(layers: Layers, steps: int, warmup: int, dev: int, dist):
    """Capture one graph per layer, replay K times round-robin; device time
    with CUDA events, max over ranks.  The headline graphs hold the layer call
    alone; a second set, replayed in a second timed pass of K steps, also
    records the stage events (an event record inside a graph costs a few
    microseconds, which must not land in the headline)."""
    import torch
    import quantized_expert_ffn_top10_b200 as M
    NL = layers.NL
    n0 = M.moe_launch_count()
    layers.call(0)  # eager call: one-time init, launches per call
    torch.cuda.synchronize()
    per_call = M.moe_launch_count() - n0
    fused = per_call == 1
    plain, staged, evs = [], [], []
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for l in range(NL):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                layers.call(l)
            plain.append(g)
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
            M.moe_set_stage_events(ev)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                layers.call(l)
            M.moe_set_stage_events([])
            staged.append(g)
            evs.append(ev)
    torch.cuda.current_stream().wait_stream(s)
    ms, clk = replay(plain, steps, warmup, dev, dist)
    replay(staged, steps, warmup, dev, dist)
    # stage durations of each graph's last replay (all inside the second pass when steps >= NL);
    # a fused call records only the kernel's start and end
    try:
        if fused:
            stages = [[ev[0].elapsed_time(ev[1]), 0.0, 0.0, 0.0] for ev in evs]
        else:
            stages = [[ev[j].elapsed_time(ev[j + 1]) for j in range(4)] for ev in evs]
    except Exception as ex:  # keep the headline even if the stage hook fails
        print(f"stage events unavailable: {ex}", file=sys.stderr)
        stages = [[float("nan")] * 4 for _ in evs]
    distinct = layers.distinct()
    del plain, staged
    return ms, stages, distinct, per_call, clk


def replay(graphs, steps: int, warmup: int, dev: int, dist):
    """Warm-up replays, then `steps` timed replays round-robin between a
    barrier and a synchronize on each side; CUDA events, max over ranks."""
    import torch
    n = len(graphs)
    for i in range(warmup):
        graphs[i % n].replay()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(dev) as clk:
        e0.record()
        for i in range(steps):
            graphs[(warmup + i) % n].replay()
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if dist:
        dist.barrier()
    return max_over_ranks(dist, ms), clk.summary()


def time_stack(layers: Layers, steps: int, warmup: int, dev: int, dist):
    """One graph holding the whole chained stack, replayed `steps` times.  Each
    replay first copies the stack's input x0 into the first buffer, so every
    step runs the same 48 layers on the same input (a replay that went on from
    the previous step's output would chain 96, 144, ... layers)."""
    import torch
    import quantized_expert_ffn_top10_b200 as M
    x0 = layers.x[0]
    a = torch.empty_like(x0)
    b = torch.empty_like(x0)
    a.copy_(x0)
    n0 = M.moe_launch_count()
    layers.call_stack(a, b)  # eager pass: one-time init, launches per step
    torch.cuda.synchronize()
    per_step = M.moe_launch_count() - n0
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            a.copy_(x0)
            layers.call_stack(a, b)
    torch.cuda.current_stream().wait_stream(s)
    ms, clk = replay([g], steps, warmup, dev, dist)
    del g
    return ms, per_step, clk


def time_e2e(layers: Layers, steps: int, warmup: int, dist):
    """Through the C ABI with host buffers: each step copies x from pinned host
    memory, runs the layer and copies the output back, all on one stream."""
    import torch
    NL = layers.NL
    xh = [torch.from_numpy(h.view("int16")).pin_memory() for h in layers.x_host]
    oh = [torch.empty_like(v).pin_memory() for v in xh]
    xd = torch.empty_like(layers.x[0])
    od = torch.empty_like(xd)

    def step(i):
        l = i % NL
        xd.copy_(xh[l], non_blocking=True)
        layers.call(l, x=xd, out=od)
        oh[l].copy_(od, non_blocking=True)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        step(warmup + i)
    e1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(dist, e0.elapsed_time(e1))
    nbytes = xh[0].numel() * 2
    return ms, nbytes, nbytes


# ----------------------------------------------------------------------------- oracle (CPU baseline / reference arm)

def oracle_sample(inp, l: int, n_tokens: int, host_slots: bool = False):
    """Run the CPU oracle on the first n_tokens of layer l's input (router over
    every expert, then the selected experts' FFNs and the combine); returns
    (seconds, tokens).  Slots come from the arena in HBM, or (host_slots) are
    regenerated on the host from the workload's seeded streams."""
    import numpy as np
    import moe_synth as S
    import oracle as O
    c = inp.cfg
    x = inp.x_host[l][:n_tokens]
    W = inp.W[l] if isinstance(inp.W[l], np.ndarray) else inp.W[l].cpu().numpy()
    b = inp.b[l]
    if b is not None and not isinstance(b, np.ndarray):
        b = b.cpu().numpy()
    table = inp.table if isinstance(inp.table, np.ndarray) else inp.table.cpu().numpy()
    sb = inp.desc.slot_bytes
    lg = O.router_logits(x, W, b)  # untimed: only to know which slots to gather
    idx, _ = O.topk(lg, c.top_k)
    ex = sorted(set(idx.reshape(-1).tolist()))
    mini = np.zeros(len(ex) * sb, np.uint8)
    mt = np.full(c.L * c.E, -1, np.int32)
    for i, e in enumerate(ex):
        s = int(table[l * c.E + e])
        mini[i * sb:(i + 1) * sb] = S.gen_slot_host(c, s) if host_slots else inp.arena[s * sb:(s + 1) * sb].cpu().numpy()
        mt[l * c.E + e] = i
    d = S.make_desc(c.H, c.I, c.bits, n_slots=len(ex))
    t1 = time.perf_counter()
    O.moe_layer(d, mini, mt, c.L, l, x, W, b, c.top_k)  # routes again, then the FFNs
    return time.perf_counter() - t1, n_tokens


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(inp, l: int, n_tokens: int, sample: str, host_slots: bool = False) -> dict:
    """The oracle as it stands on this host: all cores (its OpenMP loops over
    tokens and pairs) and one thread, on the same bounded sample."""
    import oracle as O
    allc = O.max_threads()
    secs, n = oracle_sample(inp, l, n_tokens, host_slots)
    O.set_threads(1)
    try:
        secs1, _ = oracle_sample(inp, l, n_tokens, host_slots)
    finally:
        O.set_threads(allc)
    return {"value": round(n / secs, 3), "unit": "tokens/s", "cores": allc, "kind": "oracle", "sample": sample,
            "single_thread": {"value": round(n / secs1, 3), "unit": "tokens/s", "cores": 1},
            "cpu_model": cpu_model(), "host_cpus": cores()}


# ----------------------------------------------------------------------------- main

def rank_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), ws


def max_over_ranks(dist, ms: float) -> float:
    """The slowest rank's time (every rank gets it); the value itself when
    running alone.  NCCL reduces a device tensor, gloo a host one."""
    if not dist:
        return ms
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, world: int, ms: float) -> float:
    """Units of all ranks per second, timed by the slowest rank (weak scaling:
    every rank processes the same amount of independent work)."""
    return units_per_rank * world / (ms / 1e3)


def replica_seed(base_seed: int, rank: int) -> int:
    """Each rank's replica draws its own inputs and weights."""
    return base_seed + 1000 * rank


def decode_bytes(c, distinct: int):
    """Algorithmic bytes of one decode layer: each selected expert once, the
    router, the window's input and output."""
    return distinct * c.desc().slot_bytes + c.E * c.H * 4 + 2 * c.T * c.H * 2


def gateup_bytes(c, distinct: int):
    per = 0
    for m in (0, 1):
        per += c.I * c.H * c.bits[m] // 8 + c.I * (c.H // 32) * 2
    return distinct * per + c.T * c.H * 2 + c.T * c.top_k * c.I * 4


def prefill_min_ms(c, loads, hbm_gbs: float, tc_tflops: float) -> float:
    """Per-expert roofline of one prefill layer: sum over experts with pairs of
    max(flops_e / tensor peak, bytes_e / HBM peak), plus the router's
    max(flops / tensor peak, (router weights + x in + out) / HBM peak), in ms."""
    sb = c.desc().slot_bytes
    t = 0.0
    for n in loads:
        if n > 0:
            t = t + max(6.0 * n * c.H * c.I / (tc_tflops * 1e9), sb / (hbm_gbs * 1e6))
    t += max(2.0 * c.T * c.E * c.H / (tc_tflops * 1e9), (c.E * c.H * 4 + 4 * c.T * c.H) / (hbm_gbs * 1e6))
    return t


def run_ours(args):
    import torch
    rank, local, world = rank_env()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        dist = tdist
    pk = peaks()
    K, W = args.steps, max(3, args.warmup)
    base = rank == 0 and world == 1 and not args.no_cpu_baseline
    line = {"metric": METRIC}
    if not args.no_decode:
        line = decode_section(args, rank, local, world, dist, pk, K, W, base)
        line["decode_T1"] = decode_t1_section(args, rank, local, world, dist, pk, K, W, base)
    if not args.no_prefill:
        prefill_section(args, line, rank, local, world, dist, pk, K, W, base)
        if not args.no_midt:
            line["prefill_midT"] = midt_section(args, rank, local, world, dist, pk, K, W)
    if not args.no_stacks:
        if not args.no_decode:
            line["decode_stack"] = decode_stack_section(args, rank, local, world, dist, pk, W, base)
        if not args.no_prefill:
            line["prefill_stack"] = prefill_stack_section(args, rank, local, world, dist, pk, W, base)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


DECODE_DTYPE = ("u4/u2 codes; decode: gate/up fp16 x fp16 mma.sync on exact (1024 + code) and power-of-two "
                "scaled x, down bf16 x bf16 mma.sync on exact (128 + code) and h, fp32 accumulation, scales "
                "applied in fp32, h rounded to bf16; router fp64 (tensor-core DMMA); prefill: bf16 tcgen05 MMA "
                "on dequantised weights, fp32 accumulation in TMEM, h and per-pair outputs in bf16; output bf16")


def decode_section(args, rank, local, world, dist, pk, K, W, base):
    import torch
    import moe_synth as S
    hbm, _, _, src = pk
    NLd = max(1, args.decode_layers)
    dl = Layers(S.config("decode"), NLd, rank)
    c = dl.cfg
    ms, stages, distinct, per_call, clk = time_graphs(dl, K, W, local, dist)
    value = whole_job_rate(c.T * K, world, ms)
    fused = per_call == 1  # the decode layer is one kernel: its roofline is the layer's
    gu_ms = statistics.mean(s[0] + s[1] + s[2] + s[3] for s in stages) if fused else statistics.mean(s[1] for s in stages)
    gu_bytes = statistics.mean((decode_bytes if fused else gateup_bytes)(c, d) for d in distinct)
    layer_bytes = statistics.mean(decode_bytes(c, d) for d in distinct)
    e2e_ms, h2d, d2h = time_e2e(dl, K, W, dist)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(ms / K, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": DECODE_DTYPE,
        "data": "synthetic (seeded; random-init weights of the stated shape)",
        "config": {"workload": DECODE_WORKLOAD,
                   "l2": f"{NLd} rotating layer arenas ({NLd * 0.906:.1f} GB) with fresh inputs",
                   "graph": "one CUDA graph per layer call; stage events only in a second timed pass", "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "kernel": "k_decode_fused (whole layer)" if fused else "decode gate/up + SwiGLU",
                     "achieved": round(gu_bytes / (gu_ms * 1e6), 1),
                     "peak": hbm, "unit": "GB/s", "frac": round(gu_bytes / (gu_ms * 1e6) / hbm, 4),
                     "traffic": profiled_traffic("k_decode_fused_decode_T5.md",
                                                 ("common.cuh", "perm.cuh", "router.cuh", "decode_fused.cuh"))
                     if fused else None,
                     "peak_source": src, "ms": round(gu_ms, 5),
                     "bytes": int(gu_bytes)},
        "layer_roofline": {"bound": "hbm", "achieved": round(layer_bytes / (ms / K * 1e6), 1), "peak": hbm,
                           "unit": "GB/s", "frac": round(layer_bytes / (ms / K * 1e6) / hbm, 4),
                           "frac_of_8tbs": round(layer_bytes / (ms / K * 1e6) / 8000.0, 4),
                           "bytes_per_layer": int(layer_bytes), "distinct_experts": statistics.mean(distinct),
                           "stage_ms": [round(statistics.mean(s[j] for s in stages), 5) for j in range(4)]},
        "e2e": {"value": round(whole_job_rate(c.T * K, world, e2e_ms), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": per_call * K,
        "clocks": clk,
    }
    if base:
        line["cpu_baseline"] = cpu_baseline(dl, 0, 5, "one decode window (T=5) of one layer: router over 512 "
                                                      "experts, the selected experts' FFNs, combine")
    del dl
    torch.cuda.empty_cache()
    return line


def decode_t1_section(args, rank, local, world, dist, pk, K, W, base):
    import torch
    import moe_synth as S
    hbm, _, _, src = pk
    NLd = max(1, args.decode_layers)
    dl = Layers(S.config("decode", T=1), NLd, rank)
    c = dl.cfg
    ms, stages, distinct, per_call, clk = time_graphs(dl, K, W, local, dist)
    kern = statistics.mean(s[0] + s[1] + s[2] + s[3] for s in stages)
    nbytes = statistics.mean(decode_bytes(c, d) for d in distinct)
    sec = {"value": round(whole_job_rate(c.T * K, world, ms), 1), "unit": "tokens/s", "steps": K,
           "ms_per_step": round(ms / K, 5),
           "workload": "decode, 1 token: 1 layer, E=512, top_k=10, H=2048, I=512, T=1, 4-bit block-32",
           "roofline": {"bound": "hbm", "kernel": "k_decode_fused (whole layer)" if per_call == 1 else "decode layer",
                        "achieved": round(nbytes / (kern * 1e6), 1), "peak": hbm, "unit": "GB/s",
                        "frac": round(nbytes / (kern * 1e6) / hbm, 4), "peak_source": src, "ms": round(kern, 5),
                        "bytes": int(nbytes), "distinct_experts": statistics.mean(distinct)},
           "layer_frac": round(nbytes / (ms / K * 1e6) / hbm, 4),
           "gpu_launches": per_call * K, "clocks": clk}
    if base:
        sec["cpu_baseline"] = cpu_baseline(dl, 0, 1, "one decode token (T=1) of one layer")
    del dl
    torch.cuda.empty_cache()
    return sec


def prefill_section(args, line, rank, local, world, dist, pk, K, W, base):
    import torch
    import moe_synth as S
    hbm, tc_burst, tc_sus, src = pk
    pl = Layers(S.config("prefill"), PREFILL_LAYERS, rank)
    cp = pl.cfg
    Kp = args.prefill_steps or max(PREFILL_LAYERS, min(K, 20))
    msp, stp, dsp, pcp, clkp = time_graphs(pl, Kp, W, local, dist)
    P = cp.T * cp.top_k
    g1 = statistics.mean(s[1] for s in stp)
    g2 = statistics.mean(s[2] for s in stp)
    f1 = 4.0 * P * cp.H * cp.I
    f2 = 2.0 * P * cp.H * cp.I
    flops = f1 + f2 + 2.0 * cp.T * cp.E * cp.H
    e2p, h2p, d2p = time_e2e(pl, max(2, Kp // 4), 2, dist)
    step_ms = msp / Kp
    line["prefill"] = {
        "value": round(whole_job_rate(cp.T * Kp, world, msp), 1), "unit": "tokens/s", "steps": Kp,
        "ms_per_step": round(step_ms, 4),
        "workload": "prefill chunk: 1 layer, E=512, top_k=10, H=2048, I=512, T=8192, 4-bit, Gaussian router",
        "roofline": {"bound": "tensor", "kernel": "prefill gate/up grouped GEMM + SwiGLU",
                     "achieved": round(f1 / (g1 * 1e9), 1), "peak": tc_burst, "unit": "TFLOP/s",
                     "frac": round(f1 / (g1 * 1e9) / tc_burst, 4),
                     "traffic": profiled_traffic("k_prefill_gemm_prefill_T8192.md", ("common.cuh", "prefill.cuh")),
                     "peak_source": src + " burst (a ~1 ms step, a timed region of tens of ms)",
                     "ms": round(g1, 4)},
        "gemm2": {"achieved": round(f2 / (g2 * 1e9), 1), "unit": "TFLOP/s", "frac": round(f2 / (g2 * 1e9) / tc_burst, 4),
                  "ms": round(g2, 4)},
        "layer_tc_frac": round(flops / (step_ms * 1e9) / tc_burst, 4),
        "layer_tc_frac_sustained": round(flops / (step_ms * 1e9) / tc_sus, 4),
        "stage_ms": [round(statistics.mean(s[j] for s in stp), 4) for j in range(4)],
        "e2e": {"value": round(whole_job_rate(cp.T * max(2, Kp // 4), world, e2p), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2p, "d2h_bytes_per_step": d2p},
        "gpu_launches": pcp * Kp, "clocks": clkp,
    }
    if base:
        line["prefill"]["cpu_baseline"] = cpu_baseline(pl, 0, 16, "16 tokens of the 8,192-token chunk, full layer")
    del pl
    torch.cuda.empty_cache()


MIDT = (16, 64, 256)


def midt_section(args, rank, local, world, dist, pk, K, W):
    """Mid-T chunks (batched verify windows, short prompts) through the prefill
    entry point at the model's shape.  With 1-14 pairs per expert the layer
    reads each selected expert's weights once for a handful of columns, so the
    roofline is HBM: bytes = the distinct selected experts' slots + the router
    + x in and out, over the layer call's device time."""
    import torch
    import moe_synth as S
    hbm, _, _, src = pk
    NLd = max(1, args.decode_layers)
    sec = {"workload": "prefill entry point, 1 layer, E=512, top_k=10, H=2048, I=512, 4-bit, Gaussian router; "
                       f"{NLd} rotating layer arenas with fresh inputs", "graph": "one CUDA graph per layer call"}
    for T in MIDT:
        dl = Layers(S.config("prefill", T=T), NLd, rank)
        c = dl.cfg
        ms, stages, distinct, per_call, clk = time_graphs(dl, K, W, local, dist)
        nbytes = statistics.mean(decode_bytes(c, d) for d in distinct)
        step_ms = ms / K
        sec[f"T{T}"] = {
            "value": round(whole_job_rate(c.T * K, world, ms), 1), "unit": "tokens/s", "steps": K,
            "ms_per_step": round(step_ms, 5), "distinct_experts": statistics.mean(distinct),
            "roofline": {"bound": "hbm", "achieved": round(nbytes / (step_ms * 1e6), 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(nbytes / (step_ms * 1e6) / hbm, 4), "peak_source": src,
                         "bytes": int(nbytes)},
            "stage_ms": [round(statistics.mean(s[j] for s in stages), 5) for j in range(4)],
            "gpu_launches": per_call * K, "clocks": clk}
        del dl
        torch.cuda.empty_cache()
    return sec


def decode_stack_section(args, rank, local, world, dist, pk, W, base):
    import torch
    import moe_synth as S
    hbm, _, _, src = pk
    st = Layers(S.config("decode_stack"), 48, rank)
    c = st.cfg
    Ks = args.stack_steps or 20
    ms, per_step, clk = time_stack(st, Ks, W, local, dist)
    distinct = st.distinct()  # of the last replay (the same input every step)
    nbytes = sum(decode_bytes(c, d) for d in distinct)
    step_ms = ms / Ks
    sec = {"value": round(whole_job_rate(c.T * c.L * Ks, world, ms), 1), "unit": "token-layers/s",
           "tokens_per_s_through_stack": round(whole_job_rate(c.T * Ks, world, ms), 1), "steps": Ks,
           "ms_per_step": round(step_ms, 4), "ms_per_layer": round(step_ms / c.L, 5),
           "workload": "pruned decode stack: 48 layers x E=256, top_k=10, H=2048, I=512, T=5, gate/up 2-bit, "
                       "down 4-bit, Zipf(1.1) router bias, residual chain",
           "roofline": {"bound": "hbm", "achieved": round(nbytes / (step_ms * 1e6), 1), "peak": hbm, "unit": "GB/s",
                        "frac": round(nbytes / (step_ms * 1e6) / hbm, 4), "peak_source": src,
                        "bytes_per_step": int(nbytes), "distinct_experts_mean": round(statistics.mean(distinct), 2),
                        "distinct_experts_max": max(distinct)},
           "gpu_launches": per_step * Ks, "clocks": clk,
           "l2": "a step streams 48 layers' selected experts from a 15.3 GB arena"}
    if base:
        sec["cpu_baseline"] = cpu_baseline(st, 0, 5, "one T=5 window through layer 0 of the stack")
    del st
    torch.cuda.empty_cache()
    return sec


def prefill_stack_section(args, rank, local, world, dist, pk, W, base):
    import torch
    import moe_synth as S
    hbm, tc_burst, tc_sus, src = pk
    st = Layers(S.config("prefill_stack"), 48, rank)
    c = st.cfg
    Ks = args.stack_steps or 6
    ms, per_step, clk = time_stack(st, Ks, W, local, dist)
    loads = st.loads()
    step_ms = ms / Ks
    flops = c.L * (6.0 * c.T * c.top_k * c.H * c.I + 2.0 * c.T * c.E * c.H)
    tmin_b = sum(prefill_min_ms(c, ld, hbm, tc_burst) for ld in loads)
    tmin_s = sum(prefill_min_ms(c, ld, hbm, tc_sus) for ld in loads)
    nz = [int((ld > 0).sum()) for ld in loads]
    sec = {"value": round(whole_job_rate(c.T * c.L * Ks, world, ms), 1), "unit": "token-layers/s",
           "tokens_per_s_through_stack": round(whole_job_rate(c.T * Ks, world, ms), 1), "steps": Ks,
           "ms_per_step": round(step_ms, 3), "ms_per_layer": round(step_ms / c.L, 4),
           "workload": "prefill stack: 48 layers x E=512, top_k=10, H=2048, I=512, T=8192, gate/up 2-bit, down 4-bit, "
                       "Zipf(1.1) router bias, residual chain; outputs plus the 48 x 512 histogram",
           "roofline": {"bound": "per-expert max(tensor, hbm)", "t_min_ms": round(tmin_b, 3),
                        "frac": round(tmin_b / step_ms, 4), "frac_sustained_tc": round(tmin_s / step_ms, 4),
                        "peak_tc": tc_burst, "peak_hbm": hbm, "peak_source": src + " burst tensor, copy HBM",
                        "dense_tc_frac": round(flops / (step_ms * 1e9) / tc_burst, 4)},
           "loads": {"max_pairs_per_expert": int(max(ld.max() for ld in loads)),
                     "experts_used_min": min(nz), "experts_used_mean": round(statistics.mean(nz), 1)},
           "gpu_launches": per_step * Ks, "clocks": clk}
    if base:
        sec["cpu_baseline"] = cpu_baseline(st, 0, 16, "16 tokens through layer 0 of the stack")
    del st
    torch.cuda.empty_cache()
    return sec


class HostInputs:
    """The reference arm's inputs on the host only (moe_synth; no GPU and no
    part of the library): x, router and bias of each layer, the slot table;
    slots are regenerated from their seeded streams when the oracle needs them."""

    def __init__(self, cfg, NL: int):
        import moe_synth as S
        self.cfg = S.config(cfg.name, L=NL, T=cfg.T, seed=cfg.seed)
        c = self.cfg
        self.NL = NL
        self.desc = c.desc()
        self.table = S.gen_slot_table(c)
        self.W = [S.gen_router(c, l) for l in range(NL)]
        self.b = [S.gen_bias(c, l) for l in range(NL)]
        self.x_host = [S.gen_x(c, c.T, stream_offset=l) for l in range(NL)]


def run_reference(args):
    """The oracle as the reference arm: each step is one decode window (T=5)
    of a seeded layer, on the host cores of rank 0."""
    rank, local, world = rank_env()
    if rank != 0:
        return
    import moe_synth as S
    import oracle as O
    inp = HostInputs(S.config("decode"), 2)
    for i in range(args.warmup):
        oracle_sample(inp, i % 2, 5, host_slots=True)
    tot, n = 0.0, 0
    for i in range(args.steps):
        s, t = oracle_sample(inp, i % 2, 5, host_slots=True)
        tot += s
        n += t
    v = n / tot
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp64 (CPU oracle)",
        "data": "synthetic", "config": {"workload": DECODE_WORKLOAD},
        "cpu_baseline": {"value": round(v, 3), "unit": "tokens/s", "cores": O.max_threads(), "kind": "oracle",
                         "sample": "each step one decode window (T=5) of one layer", "cpu_model": cpu_model()},
        "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


if __name__ == "__main__":
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)
