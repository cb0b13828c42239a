#!/usr/bin/env python
"""Benchmark of the quantized top-10 MoE layer on B200.

Headline (one JSON line on rank 0): MoE-layer tokens/s for a decode window of
T = 5 tokens (1 token + 4 speculative drafts) on a layer of E = 512 experts,
k = 10, H = 2048, I = 512, 4-bit block-32 weights.  A "prefill" object in the
same line reports the 8,192-token chunk on the same layer shape.  A step is
one full layer call (router, grouping, expert FFN, combine, histogram).

Weights never come from L2: decode steps rotate through 8 layer arenas
(8 x 906 MB) with a fresh input per layer, prefill through 2 (each 906 MB of
weights streamed per step, far above the 126 MB L2).

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


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-prefill", action="store_true")
    p.add_argument("--no-decode", action="store_true", help="profiling runs: prefill only")
    p.add_argument("--no-cpu-baseline", action="store_true", help="profiling runs: skip the oracle timing")
    p.add_argument("--decode-layers", type=int, default=DECODE_LAYERS,
                   help="rotating decode layer arenas (profiling runs use 1)")
    p.add_argument("--prefill-steps", type=int, default=None)
    return p.parse_args()


def profiled_traffic(summary: str, sources) -> int | None:
    """DRAM bytes per launch from a committed ncu summary under profiles/, or None
    when the kernel's sources changed since that capture."""
    import hashlib
    root = os.path.dirname(os.path.abspath(__file__))
    try:
        text = open(os.path.join(root, "profiles", summary)).read()
        m = hashlib.sha256()
        for f in sources:
            m.update(open(os.path.join(root, "quantized_expert_ffn_top10_b200", "csrc", f), "rb").read())
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


# ----------------------------------------------------------------------------- our arm

class Layers:
    """NL seeded layers of one shape on the device, each with its own router,
    input and output; arena slots for layer l are slot_table[l]."""

    def __init__(self, cfg, NL: int, rank: int):
        import numpy as np
        import torch
        import moe_synth as S
        import quantized_expert_ffn_top10_b200 as M
        self.cfg = S.config(cfg.name, L=NL, seed=replica_seed(cfg.seed, rank))
        c = self.cfg
        self.NL = NL
        self.desc = c.desc()
        self.arena = S.gen_arena_device(c)
        self.table = torch.from_numpy(S.gen_slot_table(c)).cuda()
        self.W = [torch.from_numpy(S.gen_router(c, l)).cuda() for l in range(NL)]
        self.b = [None if S.gen_bias(c, l) is None else torch.from_numpy(S.gen_bias(c, l)).cuda() for l in range(NL)]
        self.x_host = [S.gen_x(c, c.T, stream_offset=l) for l in range(NL)]
        self.x = [torch.from_numpy(h.view(np.int16)).cuda() for h in self.x_host]
        self.out = [torch.empty_like(v) for v in self.x]
        self.ws = torch.empty(M.moe_workspace_bytes(c.T, c.E, c.top_k, c.H, c.I), dtype=torch.uint8, device="cuda")
        self.hist = torch.zeros((NL, c.E), dtype=torch.int32, device="cuda")
        P = c.T * c.top_k
        self.offsets = [torch.zeros(c.E + 1, dtype=torch.int32, device="cuda") for _ in range(NL)]
        self.fn = M.moe_forward_prefill if c.T > M.MOE_DECODE_MAX_T else M.moe_forward_decode
        self.P = P

    def call(self, l: int, x=None, out=None):
        c = self.cfg
        self.fn(self.desc, self.arena, self.table, self.NL, l, self.x[l] if x is None else x, self.W[l], self.b[l],
                c.top_k, True, self.out[l] if out is None else out, hist=self.hist,
                route_out={"expert_offsets": self.offsets[l]}, ws=self.ws)


def time_graphs(layers: Layers, steps: int, warmup: int, dev: int, dist):
    """Capture one graph per layer (stage events inside), replay K times
    round-robin; device time with CUDA events, max over ranks."""
    import torch
    import quantized_expert_ffn_top10_b200 as M
    NL = layers.NL
    n0 = M.moe_launch_count()
    layers.call(0)  # eager call: one-time init, launches per call
    torch.cuda.synchronize()
    per_call = M.moe_launch_count() - n0
    graphs, evs = [], []
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for l in range(NL):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
            M.moe_set_stage_events(ev)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                layers.call(l)
            graphs.append(g)
            evs.append(ev)
    M.moe_set_stage_events([])
    torch.cuda.current_stream().wait_stream(s)
    for i in range(warmup):
        graphs[i % NL].replay()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(dev) as clk:
        e0.record()
        for i in range(steps):
            graphs[(warmup + i) % NL].replay()
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if dist:
        dist.barrier()
    ms = max_over_ranks(dist, ms)
    # stage durations of each graph's last replay (all inside the timed region when steps >= NL)
    try:
        stages = [[ev[j].elapsed_time(ev[j + 1]) for j in range(4)] for ev in evs]
    except Exception as ex:  # keep the headline even if the stage hook fails
        print(f"stage events unavailable: {ex}", file=sys.stderr)
        stages = [[float("nan")] * 4 for _ in evs]
    distinct = [int((layers.offsets[l][1:] - layers.offsets[l][:-1] > 0).sum().item()) for l in range(NL)]
    del graphs
    return ms, stages, distinct, per_call, clk.summary()


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

def oracle_sample(layers: Layers, l: int, n_tokens: int):
    """Run the CPU oracle on the first n_tokens of layer l's input (router over
    every expert, then the selected experts' FFNs and the combine); returns
    (seconds, tokens).  Slots are read from the generated arena in HBM."""
    import numpy as np
    import moe_synth as S
    import oracle as O
    c = layers.cfg
    x = layers.x_host[l][:n_tokens]
    W = layers.W[l].cpu().numpy()
    b = None if layers.b[l] is None else layers.b[l].cpu().numpy()
    table = layers.table.cpu().numpy()
    sb = layers.desc.slot_bytes
    lg = O.router_logits(x, W, b)  # untimed: only to know which slots to copy to the host
    idx, _ = O.topk(lg, c.top_k)
    ex = sorted(set(idx.reshape(-1).tolist()))
    mini = np.zeros(len(ex) * sb, np.uint8)
    mt = np.full(c.L * c.E, -1, np.int32)
    for i, e in enumerate(ex):
        s = int(table[l * c.E + e])
        mini[i * sb:(i + 1) * sb] = layers.arena[s * sb:(s + 1) * sb].cpu().numpy()
        mt[l * c.E + e] = i
    d = S.make_desc(c.H, c.I, c.bits, n_slots=len(ex))
    t1 = time.perf_counter()
    O.moe_layer(d, mini, mt, c.L, l, x, W, b, c.top_k)  # routes again, then the FFNs
    t_layer = time.perf_counter() - t1
    return t_layer, n_tokens


def cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


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
    d = c.desc()
    per = 0
    for m in (0, 1):
        per += c.I * c.H * c.bits[m] // 8 + c.I * (c.H // 32) * 2
    return distinct * per + c.T * c.H * 2 + c.T * c.top_k * c.I * 4


def run_ours(args):
    import torch
    import moe_synth as S
    rank, local, world = rank_env()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        dist = tdist
    hbm, tc_burst, tc_sus, src = peaks()
    K, W = args.steps, max(3, args.warmup)

    line = {"metric": METRIC}
    if args.no_decode:
        run_prefill_only = True
    else:
        run_prefill_only = False
    # ---- decode (headline)
    if not run_prefill_only:
        line = decode_section(args, rank, local, world, dist, hbm, src, K, W)
    prefill_section(args, line, rank, local, world, dist, tc_burst, tc_sus, src, K, W)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not run_prefill_only:
        dl = Layers(S.config("decode"), 1, rank)
        secs, n = oracle_sample(dl, 0, 5)
        line["cpu_baseline"] = {"value": round(n / secs, 3), "unit": "tokens/s", "cores": cores(), "kind": "oracle",
                                "sample": "one decode window (T=5) of one layer: router over 512 experts, "
                                          "the selected experts' FFNs, combine"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def decode_section(args, rank, local, world, dist, hbm, src, K, W):
    import torch
    import moe_synth as S
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
        "dtype": "u4 codes, fp32 math (decode); bf16 tensor-core MMA, fp32 accumulate (prefill)",
        "data": "synthetic (seeded; random-init weights of the stated shape)",
        "config": {"workload": "decode window: 1 layer, E=512, top_k=10, H=2048, I=512, T=5, 4-bit block-32",
                   "l2": f"{NLd} rotating layer arenas ({NLd * 0.906:.1f} GB) with fresh inputs",
                   "graph": "one CUDA graph per layer call", "parallelism": f"replicas x{world}"},
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
    del dl
    torch.cuda.empty_cache()
    return line


def prefill_section(args, line, rank, local, world, dist, tc_burst, tc_sus, src, K, W):
    import torch
    import moe_synth as S
    if not args.no_prefill:
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
        line["prefill"] = {
            "value": round(whole_job_rate(cp.T * Kp, world, msp), 1), "unit": "tokens/s", "steps": Kp,
            "ms_per_step": round(msp / Kp, 4),
            "workload": "prefill chunk: 1 layer, E=512, top_k=10, H=2048, I=512, T=8192, 4-bit, Gaussian router",
            "roofline": {"bound": "tensor", "kernel": "prefill gate/up grouped GEMM + SwiGLU",
                         "achieved": round(f1 / (g1 * 1e9), 1), "peak": tc_sus, "unit": "TFLOP/s",
                         "frac": round(f1 / (g1 * 1e9) / tc_sus, 4),
                         "traffic": profiled_traffic("k_prefill_gemm_prefill_T8192.md", ("common.cuh", "prefill.cuh")),
                         "peak_source": src + " sustained",
                         "ms": round(g1, 4)},
            "gemm2": {"achieved": round(f2 / (g2 * 1e9), 1), "unit": "TFLOP/s", "frac": round(f2 / (g2 * 1e9) / tc_sus, 4),
                      "ms": round(g2, 4)},
            "layer_tc_frac": round(flops / (msp / Kp * 1e9) / tc_sus, 4),
            "layer_tc_frac_burst": round(flops / (msp / Kp * 1e9) / tc_burst, 4),
            "stage_ms": [round(statistics.mean(s[j] for s in stp), 4) for j in range(4)],
            "e2e": {"value": round(whole_job_rate(cp.T * max(2, Kp // 4), world, e2p), 1), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2p, "d2h_bytes_per_step": d2p},
            "gpu_launches": pcp * Kp, "clocks": clkp,
        }
        line["gpu_launches"] = line.get("gpu_launches", 0) + pcp * Kp
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            secs, n = oracle_sample(pl, 0, 16)
            line["prefill"]["cpu_baseline"] = {"value": round(n / secs, 3), "unit": "tokens/s", "cores": cores(),
                                               "kind": "oracle",
                                               "sample": "16 tokens of the 8,192-token chunk, full layer"}
        del pl
        torch.cuda.empty_cache()


def run_reference(args):
    """The oracle as the reference arm: each step is one decode window (T=5)
    of a seeded layer on the host cores."""
    rank, local, world = rank_env()
    if rank != 0:
        return
    import torch
    import moe_synth as S
    torch.cuda.set_device(local)
    dl = Layers(S.config("decode"), 2, 0)
    for i in range(args.warmup):
        oracle_sample(dl, i % 2, 5)
    tot, n = 0.0, 0
    for i in range(args.steps):
        s, t = oracle_sample(dl, i % 2, 5)
        tot += s
        n += t
    v = n / tot
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp64 (CPU oracle)",
        "data": "synthetic", "config": {"workload": "decode window: 1 layer, E=512, top_k=10, H=2048, I=512, T=5, "
                                                    "4-bit block-32"},
        "cpu_baseline": {"value": round(v, 3), "unit": "tokens/s", "cores": cores(), "kind": "oracle",
                         "sample": "each step one decode window (T=5) of one layer"},
        "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


if __name__ == "__main__":
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)
