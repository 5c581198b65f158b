#!/usr/bin/env python
"""Benchmark: MoE-layer decode tokens/s and achieved HBM GB/s for one
512-expert, hidden-4096, 4-bit MoE layer at decode batch 1 on one B200.

One step = one call of the whole expert forward (router, top-k, gate/up
dequant + SwiGLU, down dequant, combine + shared gate + residual + RMSNorm)
for one fresh token. Inputs are seeded synthetic tensors of the layer's shape
(no model weights exist here); the routed-expert pool is 3.4 GB and each step
uses one of 48 copies of the router, shared expert, gate vector and RMSNorm
weight (~11 MB each, 0.5 GB in all), so no step finds its inputs in the 126 MB L2.

--impl reference times the CPU oracle (plain C, double precision) on the
same workload; it is the deliberately slow baseline arm.

Prints one JSON line (rank 0). Multi-GPU (torchrun): independent replicas,
one per GPU, no data-path collective; time = max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer decode tokens/s and achieved HBM GB/s (% of 8 TB/s), 4-bit experts, 1 B200"
UNIT = "tokens/s"
NOMINAL_HBM = 8000.0  # GB/s


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=120000)
    ap.add_argument("--warmup", type=int, default=480)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="layer_q4",
                    choices=["layer_q4", "layer_q2", "prefill_q4", "stack_q4", "cached_q4", "mxfp4_q4", "mxfp4_gemm"],
                    help="prefill_q4: one step = one 512-token forward of the layer (the prefill path); "
                         "cached_q4: decode of layer_q4 with its routed experts in host memory and an HBM cache")
    ap.add_argument("--cache-slots", type=int, default=64, help="cached_q4: experts the HBM cache holds")
    ap.add_argument("--copies", type=int, default=48)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU-oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20000)
    ap.add_argument("--prof-steps", type=int, default=2000)
    return ap.parse_args()


def dist_info():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


# ------------------------------------------------------------------ clocks sampler
class Clocks:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id, self.proc, self.out = gpu_id, None, None

    def start(self):
        try:
            self.out = open(os.devnull, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            text, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            text, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in text.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0])); smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(smax), "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ end-to-end timing
E2E_REPS = 3


def e2e_ms(step, n, stream, warm=4):
    """Milliseconds for n calls of step(s) (host copies in, the public call, the result back) on
    stream, after warm untimed calls: the median of E2E_REPS timed runs of the same loop."""
    import torch
    with torch.cuda.stream(stream):
        for s in range(warm):
            step(s)
        stream.synchronize()
        runs = []
        for _ in range(E2E_REPS):
            f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            for s in range(n):
                step(s)
            f1.record(stream)
            f1.synchronize()
            runs.append(f0.elapsed_time(f1))
    return sorted(runs)[len(runs) // 2]


# ------------------------------------------------------------------ host buffers
def packed_inputs(x_bits, h, dev):
    """Pinned host rows holding a step's x (bf16 bits) and h (fp32) back to back, and a device twin
    with x and h views: one host->device copy per step carries both inputs (both views 16-byte
    aligned). x_bits: uint16 [N, ...]; h: float32 [N, ...] of the same shape; returns
    (host [N, bytes], device [bytes], x view, h view)."""
    import numpy as np
    import torch

    n = x_bits.shape[0]
    shape = x_bits.shape[1:]
    xb = np.ascontiguousarray(x_bits).view(np.uint8).reshape(n, -1)
    hb = np.ascontiguousarray(h, dtype=np.float32).view(np.uint8).reshape(n, -1)
    host = torch.from_numpy(np.concatenate([xb, hb], axis=1)).pin_memory()
    devbuf = torch.empty(host.shape[1], dtype=torch.uint8, device=dev)
    nx = xb.shape[1]
    xv = devbuf[:nx].view(torch.int16).view(*shape)
    hv = devbuf[nx:].view(torch.float32).view(*shape)
    return host, devbuf, xv, hv


# ------------------------------------------------------------------ workload
def build_workload(cfg, copies, dev):
    import numpy as np
    import torch

    import fixtures.gpu as fxg
    import quantized_expert_decode_moe_b200 as qm
    from fixtures import gen

    base = fxg.device_layer(cfg, 0, device=dev)
    routed = [qm.Expert(*[qm.QMat(base["q"][m][e], base["s"][m][e], base["b"][m][e]) for m in range(3)])
              for e in range(cfg.E)]
    layers, keep = [], [base]
    for c in range(copies):
        t = base if c == 0 else fxg.device_layer(cfg, 100 + c, device=dev, expert_ids=[cfg.E])
        keep.append(t)
        j = cfg.E if c == 0 else 0
        shared = qm.Expert(*[qm.QMat(t["q"][m][j], t["s"][m][j], t["b"][m][j]) for m in range(3)])
        layers.append(qm.Layer(hidden=cfg.H, inter=cfg.I, top_k=cfg.k, bits=cfg.bits, router_w=t["router_w"],
                               experts=routed, rms_gamma=t["gamma"], shared=shared, shared_gate_w=t["gate_w"],
                               router_bias=None, rms_eps=cfg.rms_eps))
    P = copies * 5
    x = np.stack([gen.x_tokens(cfg, s, T=1)[0] for s in range(P)])
    xd = torch.from_numpy(x.view(np.int16)).to(dev)
    h0 = torch.from_numpy(gen.bf16_bits_to_f32(x).astype(np.float32)).to(dev)
    return dict(layers=layers, keep=keep, x=xd, h=h0.clone(), h0=h0, P=P, x_host=x)


def touch_pool(t):
    """Reads every expert tensor of a layer once (untimed): the whole routed pool has been touched
    before timing, as it is in a long-running decode, so the timed steps do not pay first-touch costs."""
    import torch
    acc = torch.zeros((), dtype=torch.int64, device=t["q"][0].device)
    for m in range(3):
        for part in (t["q"][m], t["s"][m], t["b"][m]):
            acc += part.view(-1)[:: 1024].to(torch.int64).sum()   # one element per 2-4 KB: every page of the pool
    return acc


def busy(fn, stream, seconds: float = 0.25):
    """Runs fn repeatedly for about `seconds` of device time (untimed) on `stream`."""
    import torch
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        fn()
        stream.synchronize()


# kernels of each decode path, in launch order
KERNELS = {"fused": ["fused_decode_kernel"],
           "chain": ["route_logits_kernel", "gateup_decode_kernel", "down_decode_kernel", "norm_kernel"],
           "digit": ["route_logits_kernel", "topk_kernel", "mx_gateup_kernel+mx_down_kernel", "norm_cluster_kernel"]}
LAUNCHES = {"fused": 1, "chain": 4, "digit": 5}   # kernels per decode step
DTYPES = {"fused": "u4 codes x s8 activation digits on int8 tensor cores (s32), fp32 scale+accumulate",
          "chain": "u4 codes x s8 activation digits on int8 tensor cores (s32), fp32 scale+accumulate",
          "digit": "u4/u2 codes x s8 digits of 22-bit fixed-point activations by dp4a (s32), fp32 scale+bias"}


def kernel_bytes(cfg, name: str, layers: int = 1) -> int:
    """Algorithmic bytes one launch of a decode kernel moves for one token: every active
    expert's codes, scales and biases it reads (k routed + the shared one), the router rows, and
    the token's vectors (x, h, gamma, the shared gate vector in; x_out, h' out)."""
    mat = lambda R, K: R * K * cfg.bits // 8 + 2 * 2 * R * (K // cfg.G)
    S = cfg.k + 1
    router = (cfg.E + 1) * cfg.H * 2
    gu = S * 2 * mat(cfg.I, cfg.H)
    dn = S * mat(cfg.H, cfg.I)
    vec = cfg.H * (2 + 4 + 2) + cfg.H * (2 + 4)
    per = {"fused_decode_kernel": router + gu + dn + vec,
           "route_logits_kernel": router + 2 * cfg.H,
           "gateup_decode_kernel": gu + 2 * cfg.H,
           "down_decode_kernel": dn + 4 * cfg.H * (S + 2),
           "norm_kernel": 6 * cfg.H * 4,
           "topk_kernel": 12 * (cfg.E + 1),
           "mx_gateup_kernel+mx_down_kernel": gu + dn + 2 * 4 * cfg.H,
           "norm_cluster_kernel": 6 * cfg.H * 4}[name]
    return per * layers


# the files that define each kernel (its translation unit and the headers it includes); recorded
# ncu traffic is tied to their hash
DECODE_SOURCES = ("common.cuh", "kernels.cuh", "decode.cu", "stage.cuh", "sync.cuh", "topk.cuh")   # gate/up, down
ROUTER_SOURCES = ("common.cuh", "kernels.cu", "kernels.cuh", "topk.cuh", "digits.cuh")             # router, norm
FUSED_SOURCES = ("common.cuh", "kernels.cuh", "fused.cu", "stage.cuh", "sync.cuh", "topk.cuh")
PREFILL_SOURCES = ("common.cuh", "kernels.cuh", "prefill.cu")
MX_SOURCES = ("common.cuh", "kernels.cuh", "digits.cuh", "mx.cu")
SOURCES_OF = {"route_logits_kernel": ROUTER_SOURCES, "norm_kernel": ROUTER_SOURCES,
              "fused_decode_kernel": FUSED_SOURCES, "mx_gateup_kernel+mx_down_kernel": MX_SOURCES}
TRAFFIC_KEY = {"mx_gateup_kernel+mx_down_kernel": "mx_experts"}   # name of a stage's record in traffic.txt


def kernel_src_sha(files=DECODE_SOURCES):
    h = hashlib.sha256()
    for f in files:
        p = os.path.join(ROOT, "quantized_expert_decode_moe_b200", "csrc", f)
        if os.path.exists(p):
            h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, config: str, files=DECODE_SOURCES):
    """dram bytes per launch from the committed ncu summary, if it was taken on the current sources."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    sha = kernel_src_sha(files)
    for line in open(p):
        if line.startswith("#") or not line.strip():
            continue
        kv = dict(x.split("=", 1) for x in line.split() if "=" in x)
        if kv.get("kernel") == kernel and kv.get("config") == config and kv.get("src_sha") == sha:
            return float(kv["dram_bytes_per_launch"])
    return None


# ------------------------------------------------------------------ CPU oracle sample
def oracle_sample(cfg, seconds: float, max_tokens: int = 10 ** 9, warmup: int = 3, threads: int = 0):
    """Times the CPU oracle on decode tokens of this workload after `warmup` untimed tokens, on
    `threads` host threads (0: all cores); returns (tokens/s, tokens, threads, seconds)."""
    import numpy as np

    import fixtures
    import oracle
    from fixtures import gen

    threads = oracle.set_threads(threads if threads > 0 else (os.cpu_count() or 1))
    Wr, rb, gs, gamma = fixtures.layer_vectors(cfg, 0)
    cache = {}

    def expert(e):
        if e not in cache:
            cache[e] = fixtures.host_expert(cfg, 0, e)
        return cache[e]

    shared = expert(cfg.E)
    done, elapsed = 0, 0.0
    s = 0
    for _ in range(warmup):   # untimed: the same work on tokens that are not counted
        x = gen.x_tokens(cfg, 10 ** 6 + s, T=1)
        s += 1
        idx, w, sg = oracle.route(x, Wr, cfg.k, bias=rb, gs=gs)
        h = gen.bf16_bits_to_f32(x[0]).astype(np.float64)
        ys = np.stack([oracle.expert(expert(int(e)), h, cfg.H, cfg.I, cfg.G, cfg.bits) for e in idx[0]])
        oracle.combine_norm(ys, w[0], oracle.expert(shared, h, cfg.H, cfg.I, cfg.G, cfg.bits), sg[0], h, gamma,
                            cfg.rms_eps)
    s = 0
    while done < max_tokens and (elapsed < seconds or done < 2):
        x = gen.x_tokens(cfg, s, T=1)
        s += 1
        # routing first (untimed) only to regenerate the touched experts on the host
        idx, _, _ = oracle.route(x, Wr, cfg.k, bias=rb, gs=gs)
        exps = [expert(int(e)) for e in idx[0]]
        h = gen.bf16_bits_to_f32(x[0]).astype(np.float64)
        t0 = time.perf_counter()
        idx, w, sg = oracle.route(x, Wr, cfg.k, bias=rb, gs=gs)
        xd = h
        ys = np.stack([oracle.expert(ex, xd, cfg.H, cfg.I, cfg.G, cfg.bits) for ex in exps])
        ysh = oracle.expert(shared, xd, cfg.H, cfg.I, cfg.G, cfg.bits)
        oracle.combine_norm(ys, w[0], ysh, sg[0], h, gamma, cfg.rms_eps)
        elapsed += time.perf_counter() - t0
        done += 1
        if len(cache) > 48:
            cache.clear()
    return done / elapsed, done, threads, elapsed


def reference_arm(args, cfg):
    ws_, rank, _ = dist_info()
    if rank != 0:
        return
    budget = max(args.cpu_seconds, 5.0)
    steps = max(1, min(args.steps, 10 ** 6))
    warm = max(args.warmup, 3)
    rate, n, threads, el = oracle_sample(cfg, budget, max_tokens=steps, warmup=warm)
    sample = (f"{n} decode tokens of the {cfg.name} workload (one token = one step, capped by a "
              f"{budget:.0f} s budget), experts regenerated on the host before timing")
    line = {
        "impl": "reference", "metric": METRIC, "value": rate, "unit": UNIT, "n_gpus": args.gpus,
        "steps": n, "steps_requested": args.steps, "warmup": warm, "ms_per_step": 1e3 * el / n,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; no model weights)",
        "config": {"workload": cfg.note, "H": cfg.H, "E": cfg.E, "top_k": cfg.k, "I": cfg.I, "bits": cfg.bits,
                   "T": 1},
        "cpu_baseline": {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": rate, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ replicas
def max_over_ranks(value: float, dist, device) -> float:
    """The slowest rank's time: every rank contributes its own, all get the max."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, steps_per_rank: int, ms: float) -> float:
    """Whole-job tokens/s: every rank decodes steps_per_rank tokens in ms (the max over ranks)."""
    return world * steps_per_rank / (ms * 1e-3)


# ------------------------------------------------------------------ our arm
def ours(args, cfg):
    import numpy as np
    import torch

    import quantized_expert_decode_moe_b200 as qm

    world, rank, local = dist_info()
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    qm.lib()
    W = build_workload(cfg, args.copies, dev)
    layers, P = W["layers"], W["P"]
    C = len(layers)
    ws = qm.new_workspace(layers[0], 1)
    xo = torch.empty((P, cfg.H), dtype=torch.int16, device=dev)
    stream = torch.cuda.Stream(device=dev)
    G = P  # steps per graph replay: every (token, copy) pair once

    def step(s):
        i = s % P
        qm.moe_layer_forward(layers[s % C], W["x"][i:i + 1], W["h"][i:i + 1], xo[i:i + 1], ws=ws, stream=stream)

    graphs = {}

    def graph_of(n):
        if n not in graphs:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                for s in range(n):   # eager pass first: lazy kernel attributes are set outside capture
                    step(s)
                stream.synchronize()
                with torch.cuda.graph(g, stream=stream):
                    for s in range(n):
                        step(s)
            graphs[n] = g
        return graphs[n]

    def run(n):
        full, rem = divmod(n, G)
        for _ in range(full):
            graph_of(G).replay()
        if rem:
            graph_of(rem).replay()

    with torch.cuda.stream(stream):
        # every graph the timed region replays is captured and replayed once here, so no graph is
        # uploaded or run for the first time inside the timed region
        for n in sorted({G, args.steps % G, args.warmup % G} - {0}):
            graph_of(n).replay()
        touch_pool(W["keep"][0])
        run(max(args.warmup, 3))
    stream.synchronize()
    assert qm.moe_poll_status(ws, stream) == 0

    gpu_uuid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", "") or "")
    clocks = Clocks(("GPU-" + gpu_uuid) if gpu_uuid and not gpu_uuid.startswith("GPU-") else (gpu_uuid or str(local)))
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        busy(lambda: run(G), stream)   # untimed load right before the timed steps (clock samples, warm clocks)
        e0.record(stream)
        run(args.steps)
        e1.record(stream)
        busy(lambda: run(G), stream)
    e1.synchronize()
    torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    assert qm.moe_poll_status(ws, stream) == 0

    # per-kernel durations (events between the kernels of the path, no overlap)
    path, nev = qm.moe_layer_path(layers[0], 1)
    nk = nev - 1
    names = KERNELS[path]
    prof_n = min(args.prof_steps, args.steps)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(prof_n)]
    with torch.cuda.stream(stream):
        for row in evs:            # torch creates the CUDA event on its first record
            for e in row:
                e.record(stream)
        for s in range(prof_n):
            i = s % P
            qm.moe_layer_forward_timed(layers[s % C], W["x"][i:i + 1], W["h"][i:i + 1], xo[i:i + 1], ws=ws,
                                       events=evs[s], stream=stream)
    stream.synchronize()
    dur = [sum(evs[s][j].elapsed_time(evs[s][j + 1]) for s in range(prof_n)) / prof_n for j in range(nk)]
    chain_ms = sum(evs[s][0].elapsed_time(evs[s][nk]) for s in range(prof_n)) / prof_n

    # end to end through the public API with host buffers
    e2e_n = min(args.e2e_steps, args.steps)
    inh, ind, xdev, hdev = packed_inputs(W["x_host"].reshape(P, 1, cfg.H),
                                         W["h0"].cpu().numpy().reshape(P, 1, cfg.H), dev)
    outh = torch.empty((P, cfg.H), dtype=torch.int16).pin_memory()
    odev = torch.empty((1, cfg.H), dtype=torch.int16, device=dev)
    def e2e_step(s):
        i = s % P
        ind.copy_(inh[i], non_blocking=True)   # x and h of the step, one copy
        qm.moe_layer_forward(layers[s % C], xdev, hdev, odev, ws=ws, stream=stream)
        outh[i:i + 1].copy_(odev, non_blocking=True)

    e2e_step(0)
    stream.synchronize()
    if dist:
        dist.barrier()
    e2e_ms_ = max_over_ranks(e2e_ms(e2e_step, e2e_n, stream, warm=8), dist, dev)

    peaks, peak_kind = measured_peaks()
    active = cfg.active_bytes_per_token                      # expert bytes per token (4 experts)
    router_bytes = cfg.E * cfg.H * 2
    tok_s = job_throughput(world, args.steps, ms)
    per_tok_s = args.steps / (ms * 1e-3)
    gbs = active * per_tok_s / 1e9
    # dominant kernel and its algorithmic bytes per launch
    j_dom = max(range(nk), key=lambda j: dur[j])
    dom_bytes = kernel_bytes(cfg, names[j_dom])
    achieved = dom_bytes / (dur[j_dom] * 1e-3) / 1e9
    traffic = recorded_traffic(TRAFFIC_KEY.get(names[j_dom], names[j_dom]), cfg.name,
                               SOURCES_OF.get(names[j_dom], DECODE_SOURCES))
    line = {
        "metric": METRIC, "value": tok_s, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": DTYPES[path],
        "data": "synthetic (seeded; no model weights)",
        "config": {"workload": cfg.note, "H": cfg.H, "E": cfg.E, "top_k": cfg.k, "shared": 1, "I": cfg.I,
                   "bits": cfg.bits, "group": cfg.G, "T": 1, "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2: 3.4 GB routed-expert pool, {C} rotating router/shared copies"},
        "hbm_gbs": gbs, "pct_of_8tbs": 100.0 * gbs / NOMINAL_HBM,
        "pct_of_measured_copy": 100.0 * gbs / peaks["hbm_gbs"],
        "active_bytes_per_token": active, "router_bytes_per_token": router_bytes,
        "kernel_ms": dict(zip(names, dur)), "chain_ms_serialised": chain_ms,
        "roofline": {"bound": "hbm", "kernel": names[j_dom], "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                     "algorithmic_bytes": dom_bytes, "peak_kind": peak_kind},
        "e2e": {"value": job_throughput(world, e2e_n, e2e_ms_), "unit": UNIT, "steps": e2e_n, "reps": E2E_REPS,
                "h2d_bytes_per_step": cfg.H * 2 + cfg.H * 4, "d2h_bytes_per_step": cfg.H * 2},
        "gpu_launches": LAUNCHES[path] * args.steps, "path": path,
        "clocks": clk,
    }
    if rank == 0 and not args.no_cpu_baseline:
        rate, n, threads, el = oracle_sample(cfg, args.cpu_seconds)
        rate1, n1, _, el1 = oracle_sample(cfg, max(2.0, args.cpu_seconds / 4), threads=1)
        line["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": f"{n} decode tokens of this workload ({el:.1f} s of oracle time)",
                                "single_thread": {"value": rate1, "unit": UNIT, "cores": 1,
                                                  "sample": f"{n1} decode tokens ({el1:.1f} s)"}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    for g in graphs.values():
        del g
    if dist:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------------ prefill arm (--config prefill_q4)
def ours_prefill(args, cfg):
    import numpy as np
    import torch

    import fixtures.gpu as fxg
    import quantized_expert_decode_moe_b200 as qm
    from fixtures import gen

    world, rank, local = dist_info()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    qm.lib()
    t = fxg.device_layer(cfg, 0, dev)
    layer = qm.layer_from_tensors(cfg, t)
    T, NB = cfg.T, 4
    xs_host = [gen.x_tokens(cfg, 100 + b, T=T) for b in range(NB)]
    xs = [torch.from_numpy(x.view(np.int16)).to(dev) for x in xs_host]
    hs = [torch.from_numpy(gen.bf16_bits_to_f32(x).astype(np.float32)).to(dev) for x in xs_host]
    ws = qm.new_workspace(layer, T)
    xo = torch.empty((T, cfg.H), dtype=torch.int16, device=dev)
    idx = torch.empty((NB, T, cfg.k), dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for b in range(NB):   # eager pass (lazy attributes), and the routing of every batch
            qm.moe_layer_forward(layer, xs[b], hs[b].clone(), xo, None, idx[b], None, ws=ws, stream=stream)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for b in range(NB):
                qm.moe_layer_forward(layer, xs[b], hs[b], xo, ws=ws, stream=stream)
    steps = max(NB, (args.steps // NB) * NB)
    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3) // NB + 1):
            g.replay()
    stream.synchronize()
    assert qm.moe_poll_status(ws, stream) == 0
    gpu_uuid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", "") or "")
    clocks = Clocks(("GPU-" + gpu_uuid) if gpu_uuid and not gpu_uuid.startswith("GPU-") else (gpu_uuid or str(local)))
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        busy(g.replay, stream)   # untimed load right before the timed steps (clock samples, warm clocks)
        e0.record(stream)
        for _ in range(steps // NB):
            g.replay()
        e1.record(stream)
        busy(g.replay, stream)
    e1.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    assert qm.moe_poll_status(ws, stream) == 0
    # stages, timed one by one: router, top-k + grouping, gate/up, down, combine + norm
    nst, reps = 5, 8
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)] for _ in range(reps)]
    with torch.cuda.stream(stream):
        for row in evs:
            for e in row:
                e.record(stream)
        for r in range(reps):
            qm.moe_layer_forward_timed(layer, xs[r % NB], hs[r % NB], xo, ws=ws, events=evs[r], stream=stream)
    stream.synchronize()
    names = ["route_logits", "topk+group", "gateup_grouped", "down_grouped", "combine_norm"]
    dur = [sum(evs[r][j].elapsed_time(evs[r][j + 1]) for r in range(reps)) / reps for j in range(nst)]
    # end to end with host buffers: x, h in; x_out back, every step
    inh, ind, xd, hd = packed_inputs(np.stack(xs_host), np.stack([h.cpu().numpy() for h in hs]), dev)
    outh = torch.empty((T, cfg.H), dtype=torch.int16).pin_memory()
    e2e_n = min(steps, 32)
    def e2e_step(i):
        ind.copy_(inh[i % NB], non_blocking=True)   # x and h of the batch, one copy
        qm.moe_layer_forward(layer, xd, hd, xo, ws=ws, stream=stream)
        outh.copy_(xo, non_blocking=True)

    e2e_ms_ = e2e_ms(e2e_step, e2e_n, stream, warm=2)
    peaks, peak_kind = measured_peaks()
    shared_tc = cfg.T >= 64 and os.environ.get("MOE_PREFILL_SHARED", "") != "mma" or \
        os.environ.get("MOE_PREFILL_SHARED", "") == "tc"
    touched = [len(np.unique(idx[b].cpu().numpy())) for b in range(NB)]
    bytes_mat = cfg.I * cfg.H * cfg.bits // 8 + 2 * 2 * cfg.I * (cfg.H // cfg.G)   # one matrix: codes, scales, biases
    gu_bytes = (np.mean(touched) + 1) * 2 * bytes_mat + 2 * T * cfg.H * 2
    flops = 2.0 * (T * cfg.k + T) * 3 * cfg.H * cfg.I
    achieved = gu_bytes / (dur[2] * 1e-3) / 1e9
    line = {
        "metric": "MoE-layer prefill tokens/s (512-token batch), 4-bit experts, 1 B200", "value": T * steps / (ms * 1e-3),
        "unit": "tokens/s", "n_gpus": world, "steps": steps, "warmup": max(args.warmup, 3),
        "ms_per_step": ms / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "routed experts: u4 codes x s8 digits of 16-bit fixed-point activations on int8 tensor cores "
                 "(s32), fp32 scale+accumulate; shared expert: exact fp16 s*(q-8) x fp16 activations on tcgen05 "
                 "(fp32 accumulate in tensor memory); router logits f64" if shared_tc else
                 "u4 codes x s8 digits of 16-bit fixed-point activations on int8 tensor cores (s32), "
                 "fp32 scale+accumulate; router logits f64",
        "data": "synthetic (seeded; no model weights)",
        "config": {"workload": cfg.note, "H": cfg.H, "E": cfg.E, "top_k": cfg.k, "I": cfg.I, "bits": cfg.bits,
                   "T": T, "experts_touched_per_step": float(np.mean(touched)),
                   "l2": "inputs larger than L2: every step streams the ~3.3 GB of touched experts"},
        "stage_ms": dict(zip(names, dur)),
        "tflops": flops / (ms / steps * 1e-3) / 1e12,
        "roofline": {"bound": "hbm", "kernel": "gateup_grouped", "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "traffic": recorded_traffic("prefill_grouped_gateup", cfg.name, PREFILL_SOURCES),
                     "algorithmic_bytes": gu_bytes, "peak_kind": peak_kind},
        "e2e": {"value": T * e2e_n / (e2e_ms_ * 1e-3), "unit": "tokens/s", "steps": e2e_n, "reps": E2E_REPS,
                "h2d_bytes_per_step": T * cfg.H * (2 + 4), "d2h_bytes_per_step": T * cfg.H * 2},
        # router (GEMM, norms, combine), top-k, grouping, digits of x, gate/up, digits of a, down,
        # combine + norm; with the shared expert on tcgen05 also its tables of x, gate/up, tables of a, down
        "gpu_launches": (14 if shared_tc else 10) * steps, "clocks": clk,
    }
    if rank == 0 and not args.no_cpu_baseline:
        rate, n, threads, el = oracle_sample(cfg, args.cpu_seconds)
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                "sample": f"{n} tokens of the batch, one at a time as the oracle has no batching "
                                          f"({el:.1f} s of oracle time)"}
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ 24-layer stack (--config stack_q4)
def ours_stack(args, cfg):
    """One step = moe_stack_forward of one fresh token through all 24 resident layers."""
    import numpy as np
    import torch

    import fixtures.gpu as fxg
    import quantized_expert_decode_moe_b200 as qm
    from fixtures import gen

    world, rank, local = dist_info()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    qm.lib()
    tensors = [fxg.device_layer(cfg, l, dev) for l in range(cfg.layers)]
    layers = [qm.layer_from_tensors(cfg, t) for t in tensors]
    arr = qm.stack_array(layers)
    P, G = 64, 16                                   # distinct tokens; steps per graph
    x_host = np.stack([gen.x_tokens(cfg, s, T=1)[0] for s in range(P)])
    xs = torch.from_numpy(x_host.view(np.int16)).to(dev)
    h0 = torch.from_numpy(gen.bf16_bits_to_f32(x_host).astype(np.float32)).to(dev)
    hs = h0.clone()
    xo = torch.empty((P, cfg.H), dtype=torch.int16, device=dev)
    ws = qm.new_workspace(layers[0], 1)
    stream = torch.cuda.Stream(device=dev)

    def step(s):
        i = s % P
        qm.moe_stack_forward(arr, xs[i], hs[i], xo[i], ws=ws, stream=stream)

    with torch.cuda.stream(stream):
        for s in range(G):   # eager pass (lazy kernel attributes)
            step(s)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for s in range(G):
                step(s)
        for _ in range(max(args.warmup, 3) // G + 1):
            g.replay()
    stream.synchronize()
    assert qm.moe_poll_status(ws, stream) == 0
    steps = max(G, (min(args.steps, 4096) // G) * G)
    gpu_uuid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", "") or "")
    clocks = Clocks(("GPU-" + gpu_uuid) if gpu_uuid and not gpu_uuid.startswith("GPU-") else (gpu_uuid or str(local)))
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        busy(g.replay, stream)   # untimed load right before the timed steps (clock samples, warm clocks)
        e0.record(stream)
        for _ in range(steps // G):
            g.replay()
        e1.record(stream)
        busy(g.replay, stream)
    e1.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    assert qm.moe_poll_status(ws, stream) == 0
    # the dominant kernel: with the fused path one launch runs all the layers, timed around the call
    path, _ = qm.moe_layer_path(layers[0], 1)
    prof_n = 48
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(prof_n)]
    with torch.cuda.stream(stream):
        for s in range(prof_n):
            i = s % P
            evs[s][0].record(stream)
            qm.moe_stack_forward(arr, xs[i], hs[i], xo[i], ws=ws, stream=stream)
            evs[s][1].record(stream)
    stream.synchronize()
    stack_ms = sum(e0_.elapsed_time(e1_) for e0_, e1_ in evs) / prof_n
    kname = "fused_decode_kernel" if path == "fused" else "stack_chain"
    # end to end with host buffers: x, h in; x_out back, every step
    inh, ind, xd, hd = packed_inputs(x_host, h0.cpu().numpy(), dev)
    outh = torch.empty((P, cfg.H), dtype=torch.int16).pin_memory()
    od = torch.empty(cfg.H, dtype=torch.int16, device=dev)
    e2e_n = min(steps, 256)
    def e2e_step(s):
        i = s % P
        ind.copy_(inh[i], non_blocking=True)   # x and h of the step, one copy
        qm.moe_stack_forward(arr, xd, hd, od, ws=ws, stream=stream)
        outh[i].copy_(od, non_blocking=True)

    e2e_ms_ = e2e_ms(e2e_step, e2e_n, stream)
    peaks, peak_kind = measured_peaks()
    active = cfg.active_bytes_per_token               # 24 layers x 4 experts
    tok_s = steps / (ms * 1e-3)
    gbs = active * tok_s / 1e9
    dom_bytes = kernel_bytes(cfg, "fused_decode_kernel", cfg.layers)
    achieved = dom_bytes / (stack_ms * 1e-3) / 1e9
    line = {
        "metric": "24-layer MoE decode tokens/s and achieved HBM GB/s (% of 8 TB/s), 4-bit experts, 1 B200",
        "value": tok_s, "unit": UNIT, "n_gpus": world, "steps": steps, "warmup": max(args.warmup, 3),
        "ms_per_step": ms / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": DTYPES[path],
        "data": "synthetic (seeded; no model weights)",
        "config": {"workload": cfg.note, "H": cfg.H, "E": cfg.E, "top_k": cfg.k, "shared": 1, "I": cfg.I,
                   "bits": cfg.bits, "layers": cfg.layers, "T": 1,
                   "l2": "inputs larger than L2: every step streams 24 layers' experts (679 MB) from an 87 GB stack"},
        "hbm_gbs": gbs, "pct_of_8tbs": 100.0 * gbs / NOMINAL_HBM, "pct_of_measured_copy": 100.0 * gbs / peaks["hbm_gbs"],
        "active_bytes_per_token": active, "us_per_layer": ms / steps / cfg.layers * 1e3,
        "kernel_ms": {kname: stack_ms}, "path": path,
        "roofline": {"bound": "hbm", "kernel": kname, "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                     "algorithmic_bytes": dom_bytes, "peak_kind": peak_kind},
        "e2e": {"value": e2e_n / (e2e_ms_ * 1e-3), "unit": UNIT, "steps": e2e_n, "reps": E2E_REPS,
                "h2d_bytes_per_step": cfg.H * (2 + 4), "d2h_bytes_per_step": cfg.H * 2},
        "gpu_launches": (1 if path == "fused" else LAUNCHES[path] * cfg.layers) * steps, "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g


# ------------------------------------------------------------------ host-resident experts (--config cached_q4)
def ours_cached(args, cfg):
    """Decode of the 4-bit layer with its 512 routed experts in page-locked host memory and an HBM
    cache of --cache-slots experts: each step routes a fresh token, loads the missing experts over
    the host link and runs the layer (moe_layer_forward_cached; the call synchronises the stream
    once, after routing). Timed with CUDA events around the steps; the roofline is the host link:
    bytes copied per second against a page-locked host -> device copy measured in this process."""
    import numpy as np
    import torch

    import fixtures.gpu as fxg
    import quantized_expert_decode_moe_b200 as qm
    from fixtures import gen

    world, rank, local = dist_info()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    qm.lib()
    t = fxg.device_layer(cfg, 0, dev)
    layer = qm.layer_from_tensors(cfg, t)
    E = cfg.E
    host = {a: [t[a][m][:E].cpu().pin_memory() for m in range(3)] for a in ("q", "s", "b")}
    hex_ = [qm.Expert(*[qm.QMat(host["q"][m][e], host["s"][m][e], host["b"][m][e]) for m in range(3)])
            for e in range(E)]
    cache = qm.ExpertCache(layer, hex_, args.cache_slots, device=dev)
    ws = qm.new_workspace(layer, 1, device=dev)
    n = max(args.steps, 1) + max(args.warmup, 3)
    xs = torch.from_numpy(gen.x_tokens(cfg, 300, T=n).view(np.int16)).to(dev)
    hs = torch.from_numpy(gen.bf16_bits_to_f32(gen.x_tokens(cfg, 300, T=n)).astype(np.float32)).to(dev)
    xo = torch.empty((1, cfg.H), dtype=torch.int16, device=dev)
    stream = torch.cuda.Stream(device=dev)
    # the host link, measured: one 256 MB page-locked host -> device copy (best of 3)
    src = torch.empty(256 << 20, dtype=torch.uint8).pin_memory()
    dst = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    link = 0.0
    with torch.cuda.stream(stream):
        for _ in range(3):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            dst.copy_(src, non_blocking=True)
            b.record(stream)
            b.synchronize()
            link = max(link, src.numel() / (a.elapsed_time(b) * 1e-3) / 1e9)
    del src, dst
    W = max(args.warmup, 3)
    with torch.cuda.stream(stream):
        for i in range(W):
            qm.moe_layer_forward_cached(layer, cache, xs[i:i + 1], hs[i:i + 1], xo, ws=ws, stream=stream)
        stream.synchronize()
        h0, m0, b0 = qm.moe_cache_stats(cache)
        gpu_uuid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", "") or "")
        clocks = Clocks(("GPU-" + gpu_uuid) if gpu_uuid and not gpu_uuid.startswith("GPU-") else (gpu_uuid or str(local)))
        clocks.start()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(W, W + args.steps):
            qm.moe_layer_forward_cached(layer, cache, xs[i:i + 1], hs[i:i + 1], xo, ws=ws, stream=stream)
        e1.record(stream)
    e1.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    assert qm.moe_poll_status(ws, stream) == 0
    h1, m1, b1 = qm.moe_cache_stats(cache)
    steps = args.steps
    copied = (b1 - b0) / steps
    achieved = copied * steps / (ms * 1e-3) / 1e9
    line = {
        "metric": "MoE-layer decode tokens/s, 4-bit experts in host memory behind an HBM expert cache, 1 B200",
        "value": steps / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world, "steps": steps, "warmup": W,
        "ms_per_step": ms / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "u4 codes x s8 activation digits on int8 tensor cores (s32), fp32 scale+accumulate",
        "data": "synthetic (seeded; no model weights)",
        "config": {"workload": "one 512-expert hidden-4096 layer, decode batch 1, 4-bit, routed experts in "
                               "page-locked host memory", "H": cfg.H, "E": E, "top_k": cfg.k, "I": cfg.I,
                   "bits": cfg.bits, "cache_slots": args.cache_slots, "T": 1},
        "cache": {"hits": h1 - h0, "misses": m1 - m0, "hit_rate": (h1 - h0) / max(1, (h1 - h0) + (m1 - m0)),
                  "bytes_copied_per_token": copied},
        "roofline": {"bound": "host link", "kernel": "host-to-HBM expert copies", "achieved": achieved,
                     "peak": link, "unit": "GB/s", "frac": achieved / link if link else None, "traffic": None,
                     "peak_kind": "measured in this run (256 MB page-locked copy)"},
        "e2e": {"value": steps / (ms * 1e-3), "unit": "tokens/s", "steps": steps,
                "h2d_bytes_per_step": copied, "d2h_bytes_per_step": 4 * cfg.k},
        "gpu_launches": (2 + LAUNCHES[qm.moe_layer_path(layer, 1)[0]]) * steps, "clocks": clk,   # routing, then the layer
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ MXFP4 experts (--config mxfp4_q4)
MX_METRIC = "MoE-layer decode tokens/s, MXFP4 experts (E2M1 + E8M0 per 32), 1 B200"


def mx_bytes_per_expert(cfg) -> int:
    return 3 * (cfg.I * cfg.H // 2 + cfg.I * cfg.H // 32)


def mx_oracle_sample(cfg, seconds: float, max_tokens: int = 10 ** 9, warmup: int = 1, threads: int = 0):
    """The oracle's MXFP4 layer on decode tokens of this workload (the touched experts regenerated
    on the host before timing); returns (tokens/s, tokens, threads, seconds)."""
    import numpy as np

    import fixtures
    import oracle
    from fixtures import gen

    threads = oracle.set_threads(threads if threads > 0 else (os.cpu_count() or 1))
    Wr, rb, gs, gamma = fixtures.layer_vectors(cfg, 0)
    cache = {}

    def ex(e):
        if e not in cache:
            cache[e] = gen.mx_expert(e, cfg.H, cfg.I)
        return cache[e]

    shared = ex(cfg.E)
    done, elapsed, s = 0, 0.0, 0
    for timed in [False] * warmup + [True] * (10 ** 9):
        if timed and (done >= max_tokens or (elapsed >= seconds and done >= 2)):
            break
        x = gen.x_tokens(cfg, 500 + s, T=1)
        s += 1
        idx, _, _ = oracle.route(x, Wr, cfg.k, bias=rb, gs=gs)
        experts = {int(e): ex(int(e)) for e in idx[0]}
        h0 = gen.bf16_bits_to_f32(x).astype(np.float64)
        table = [experts.get(e) for e in range(cfg.E)]
        t0 = time.perf_counter()
        oracle.mx_layer(x, h0, Wr, gamma, table, shared, k=cfg.k, eps=cfg.rms_eps, router_bias=rb, gs=gs)
        if timed:
            elapsed += time.perf_counter() - t0
            done += 1
        if len(cache) > 48:
            cache = {cfg.E: shared}
    return done / elapsed, done, threads, elapsed


def ours_mx(args, cfg):
    """Decode of one 512-expert hidden-4096 layer whose experts are MXFP4 (moe_layer group 32): router,
    certified top-k, MXFP4 gate/up + SwiGLU and down + combine + residual, RMSNorm. Tokens rotate over
    64 inputs; the 3.4 GB expert pool is larger than L2."""
    import numpy as np
    import torch

    import fixtures
    import quantized_expert_decode_moe_b200 as qm
    from fixtures import gen

    world, rank, local = dist_info()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    qm.lib()
    Wr, rb, gs, gamma = fixtures.layer_vectors(cfg, 0)

    def t16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev)

    experts = []
    for e in range(cfg.E + 1):
        mats = [qm.QMat(torch.from_numpy(q.view(np.int32)).to(dev), torch.from_numpy(sc).to(dev), None)
                for q, sc in gen.mx_expert(e, cfg.H, cfg.I)]
        experts.append(qm.Expert(*mats))
    layer = qm.Layer(hidden=cfg.H, inter=cfg.I, top_k=cfg.k, bits=4, group=32, router_w=t16(Wr),
                     experts=experts[:cfg.E], rms_gamma=t16(gamma), shared=experts[cfg.E], shared_gate_w=t16(gs),
                     router_bias=torch.from_numpy(rb).to(dev) if rb is not None else None, rms_eps=cfg.rms_eps)
    P = 64
    x_host = gen.x_tokens(cfg, 900, T=P)
    xs = torch.from_numpy(x_host.view(np.int16)).to(dev)
    h0 = torch.from_numpy(gen.bf16_bits_to_f32(x_host).astype(np.float32)).to(dev)
    hs = h0.clone()
    xo = torch.empty((P, cfg.H), dtype=torch.int16, device=dev)
    ws = qm.new_workspace(layer, 1)
    stream = torch.cuda.Stream(device=dev)

    def step(i):
        qm.moe_layer_forward(layer, xs[i:i + 1], hs[i:i + 1], xo[i:i + 1], ws=ws, stream=stream)

    with torch.cuda.stream(stream):
        for i in range(P):
            step(i)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(P):
                step(i)
        for _ in range(max(args.warmup, 3) // P + 1):
            g.replay()
    stream.synchronize()
    assert qm.moe_poll_status(ws, stream) == 0
    reps = max(1, args.steps // P)
    steps = reps * P
    gpu_uuid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", "") or "")
    clocks = Clocks(("GPU-" + gpu_uuid) if gpu_uuid and not gpu_uuid.startswith("GPU-") else (gpu_uuid or str(local)))
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        busy(g.replay, stream)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        busy(g.replay, stream)
    e1.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    assert qm.moe_poll_status(ws, stream) == 0
    # stages, timed one by one: router, top-k, MXFP4 experts (gate/up + down), RMSNorm
    path, nev = qm.moe_layer_path(layer, 1)
    nst = nev - 1
    prof_n = min(args.prof_steps, 256)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(prof_n)]
    with torch.cuda.stream(stream):
        for row in evs:
            for e in row:
                e.record(stream)
        for s in range(prof_n):
            i = s % P
            qm.moe_layer_forward_timed(layer, xs[i:i + 1], hs[i:i + 1], xo[i:i + 1], ws=ws, events=evs[s],
                                       stream=stream)
    stream.synchronize()
    names = ["route_logits (+ digit blocks of x)", "topk", "mx_gateup+mx_down", "norm"]
    dur = [sum(evs[s][j].elapsed_time(evs[s][j + 1]) for s in range(prof_n)) / prof_n for j in range(nst)]
    # end to end with host buffers: x and h in, x_out back, every step
    e2e_n = min(args.e2e_steps, steps, 512)
    inh, ind, xdev, hdev = packed_inputs(x_host.reshape(P, 1, cfg.H), h0.cpu().numpy().reshape(P, 1, cfg.H), dev)
    outh = torch.empty((P, cfg.H), dtype=torch.int16).pin_memory()
    odev = torch.empty((1, cfg.H), dtype=torch.int16, device=dev)
    def e2e_step(s):
        i = s % P
        ind.copy_(inh[i], non_blocking=True)
        qm.moe_layer_forward(layer, xdev, hdev, odev, ws=ws, stream=stream)
        outh[i:i + 1].copy_(odev, non_blocking=True)

    e2e_ms_ = e2e_ms(e2e_step, e2e_n, stream, warm=8)
    peaks, peak_kind = measured_peaks()
    per_tok = (cfg.k + 1) * mx_bytes_per_expert(cfg)
    achieved = per_tok / (dur[2] * 1e-3) / 1e9
    line = {
        "metric": MX_METRIC, "value": steps / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world, "steps": steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms / steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "E2M1 codes x fp32 activations, fp32 block sums times E8M0 scales; router logits f64",
        "data": "synthetic (seeded; no model weights)",
        "config": {"workload": "one 512-expert hidden-4096 layer of MXFP4 experts, decode batch 1", "H": cfg.H,
                   "E": cfg.E, "top_k": cfg.k, "shared": 1, "I": cfg.I, "codec": "mxfp4", "T": 1,
                   "l2": "inputs larger than L2: 3.4 GB expert pool, 64 rotating tokens"},
        "hbm_gbs": per_tok * steps / (ms * 1e-3) / 1e9, "active_bytes_per_token": per_tok,
        "stage_ms": dict(zip(names, dur)),
        "roofline": {"bound": "hbm", "kernel": "mx_gateup_kernel + mx_down_kernel",
                     "achieved": achieved,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "traffic": recorded_traffic("mx_experts", "mxfp4_q4", MX_SOURCES),
                     "algorithmic_bytes": per_tok, "peak_kind": peak_kind},
        "e2e": {"value": e2e_n / (e2e_ms_ * 1e-3), "unit": "tokens/s", "steps": e2e_n, "reps": E2E_REPS,
                "h2d_bytes_per_step": cfg.H * 6, "d2h_bytes_per_step": cfg.H * 2},
        "gpu_launches": 5 * steps, "path": path, "clocks": clk,
    }
    if rank == 0 and not args.no_cpu_baseline:
        rate, n, threads, el = mx_oracle_sample(cfg, args.cpu_seconds)
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                "sample": f"{n} decode tokens of this workload ({el:.1f} s of oracle time)"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def ours_mxgemm(args):
    """The many-token MXFP4 product on tcgen05 (kind::mxf4 with block scaling): Y = X W^T for the
    512 tokens of the prefill workload and a 2048 x 4096 MXFP4 matrix (the shared expert's gate and
    up rows); one step = one moe_expert_gemm_mxfp4 call (prep of the activation terms, the
    block-scaled product, the sum of the column splits). 48 rotating weight copies (214 MB, larger
    than L2)."""
    import numpy as np
    import torch

    import oracle
    import quantized_expert_decode_moe_b200 as qm
    from fixtures import gen

    world, rank, local = dist_info()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    qm.lib()
    R, K, T, C = 2048, 4096, 512, 48
    q, e = gen.mx_matrix(5, R, K)
    qd = torch.from_numpy(q.view(np.int32)).to(dev)
    ed = torch.from_numpy(e).to(dev)
    mats = [qm.MxMat(qd.clone(), ed.clone()) for _ in range(C)]
    x_host = gen.mx_tokens(6, T, K)
    xd = torch.from_numpy(x_host.view(np.int16)).to(dev)
    y = torch.empty((T, R), device=dev)
    ws = qm.new_mx_workspace(R, K, T)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for c in range(C):
            qm.moe_expert_gemm_mxfp4(mats[c], xd, y, ws=ws, stream=stream)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for c in range(C):
                qm.moe_expert_gemm_mxfp4(mats[c], xd, y, ws=ws, stream=stream)
        for _ in range(max(1, max(args.warmup, 3) // C + 1)):
            g.replay()
    stream.synchronize()
    assert qm.moe_poll_status(ws, stream) == 0
    reps = max(1, args.steps // C)
    steps = reps * C
    gpu_uuid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", "") or "")
    clocks = Clocks(("GPU-" + gpu_uuid) if gpu_uuid and not gpu_uuid.startswith("GPU-") else (gpu_uuid or str(local)))
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        busy(g.replay, stream)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        busy(g.replay, stream)
    e1.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    assert qm.moe_poll_status(ws, stream) == 0
    # end to end: x in from page-locked host memory, Y back, every step
    xh = torch.from_numpy(x_host.view(np.int16)).pin_memory()
    yh = torch.empty((T, R), dtype=torch.float32).pin_memory()
    e2e_n = min(args.e2e_steps, steps, 96)
    def e2e_step(i):
        xd.copy_(xh, non_blocking=True)
        qm.moe_expert_gemm_mxfp4(mats[i % C], xd, y, ws=ws, stream=stream)
        yh.copy_(y, non_blocking=True)

    e2e_ms_ = e2e_ms(e2e_step, e2e_n, stream, warm=2)
    peaks, peak_kind = measured_peaks()
    fp4_peak = 4.0 * peaks["bf16_tflops"]   # dense fp4 = 4 x dense bf16 (nominal 9 / 2.25 PFLOP/s)
    flops = 2.0 * R * K * T
    per_step_ms = ms / steps
    achieved = flops / (per_step_ms * 1e-3) / 1e12
    line = {
        "metric": "MXFP4 expert product, tokens/s (512-token batch, 2048 x 4096 MXFP4 matrix), tcgen05 kind::mxf4, 1 B200",
        "value": T * steps / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world, "steps": steps,
        "warmup": max(args.warmup, 3), "ms_per_step": per_step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "E2M1 weights x five E2M1 terms of the bf16 activations (E8M0 block scales), fp32 in tensor memory",
        "data": "synthetic (seeded; no model weights)",
        "config": {"workload": "512 tokens x one 2048 x 4096 MXFP4 matrix (the shared expert's gate and up rows)",
                   "R": R, "K": K, "T": T, "copies": C, "l2": "48 rotating weight copies (214 MB), larger than L2"},
        "tflops": achieved,
        "roofline": {"bound": "tensor", "kernel": "moe_expert_gemm_mxfp4 (prep + mx_gemm_kernel + split sum)",
                     "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s", "frac": achieved / fp4_peak,
                     "traffic": None, "algorithmic_flops": flops,
                     "peak_kind": f"{peak_kind} bf16 x 4 (fp4 / bf16 nominal ratio); achieved counts the product once, "
                                  f"the five activation terms issue 5x these fp4 MMA flops"},
        "e2e": {"value": T * e2e_n / (e2e_ms_ * 1e-3), "unit": "tokens/s", "steps": e2e_n, "reps": E2E_REPS,
                "h2d_bytes_per_step": T * K * 2, "d2h_bytes_per_step": T * R * 4},
        "gpu_launches": 3 * steps, "clocks": clk,
    }
    if rank == 0 and not args.no_cpu_baseline:
        n = 16
        t0 = time.perf_counter()
        oracle.mx_gemm(q, e, x_host[:n], K)
        el = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": n / el, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "sample": f"{n} tokens of this workload ({el:.1f} s: dequantisation and one numpy "
                                          f"matrix product in double)"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    import fixtures
    if args.config == "mxfp4_gemm":
        if args.impl == "reference":
            if dist_info()[1] == 0:
                import oracle
                from fixtures import gen
                R, K, n = 2048, 4096, max(1, min(args.steps, 64))
                q, e = gen.mx_matrix(5, R, K)
                x = gen.mx_tokens(6, n, K)
                t0 = time.perf_counter()
                oracle.mx_gemm(q, e, x, K)
                el = time.perf_counter() - t0
                rate = n / el
                print(json.dumps({
                    "impl": "reference", "metric": "MXFP4 expert product, tokens/s (512-token batch, 2048 x 4096 MXFP4 "
                    "matrix), tcgen05 kind::mxf4, 1 B200", "value": rate, "unit": "tokens/s", "n_gpus": args.gpus,
                    "steps": n, "warmup": 0, "ms_per_step": 1e3 * el / n, "higher_is_better": True, "scaling": "weak",
                    "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded; no model weights)",
                    "config": {"workload": "512 tokens x one 2048 x 4096 MXFP4 matrix", "tokens_timed": n},
                    "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                     "sample": f"{n} tokens"},
                    "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
                    flush=True)
        else:
            ours_mxgemm(args)
        return
    if args.config == "mxfp4_q4":
        cfg = fixtures.CONFIGS["layer_q4"]
        if args.impl == "reference":
            rate, n, threads, el = mx_oracle_sample(cfg, max(args.cpu_seconds, 5.0), max_tokens=max(1, args.steps))
            line = {"impl": "reference", "metric": MX_METRIC, "value": rate, "unit": "tokens/s", "n_gpus": args.gpus,
                    "steps": n, "warmup": max(args.warmup, 3), "ms_per_step": 1e3 * el / n,
                    "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                    "data": "synthetic (seeded; no model weights)",
                    "config": {"workload": "one 512-expert hidden-4096 layer of MXFP4 experts, decode batch 1"},
                    "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                     "sample": f"{n} decode tokens"},
                    "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
            if dist_info()[1] == 0:
                print(json.dumps(line), flush=True)
        else:
            ours_mx(args, cfg)
        return
    if args.config == "cached_q4":
        cfg = fixtures.CONFIGS["layer_q4"]
        if args.impl == "reference":
            reference_arm(args, cfg)
        else:
            ours_cached(args, cfg)
        return
    cfg = fixtures.CONFIGS[args.config]
    if args.impl == "reference":
        reference_arm(args, cfg)
    elif cfg.T > 1:
        ours_prefill(args, cfg)
    elif cfg.layers > 1:
        ours_stack(args, cfg)
    else:
        ours(args, cfg)


if __name__ == "__main__":
    main()
