#!/usr/bin/env python3
"""Benchmark of the per-layer cache-append + attention step on B200.

One step = one layer-step of the full-shape workload (40 heads, head_dim 128,
44x68 = 2992 tokens per latent frame, one frame per chunk, window of 8
committed frames, so 9 x 2992 = 26928 keys per query) in steady state with
the ring full: rtv_cache_append (fused RoPE + amax + E4M3 of Q, K, V), then
rtv_attend (FP8 tcgen05 attention over the ring), then rtv_cache_advance
(host bookkeeping, no launch).  Inputs rotate over 6 synthetic chunks
(552 MB, above the 126 MB L2); the K/V key set read per step (276 MB) is
above L2 too.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
    python bench.py --workload seq48 [--steps K] [--warmup W]

On one GPU the same JSON line also carries, under "workloads", the other
full-shape workloads timed on their own: the long-window layer (2 frames per
chunk, W = 16 plus the pinned slot), three denoising passes per chunk, and
the 48-layer step (every layer appended and attended, then one advance) with
the spread of its per-layer times.  --workload seq48 prints only the latter.

"e2e" is the same layer-step through the public API with the inputs copied
from pinned host memory and the output copied back every step, the copies on
their own streams so that they overlap the kernels of neighbouring steps.

N > 1 runs N independent replicas (one per GPU, launched by torchrun); the
path has no data exchange, the process group only carries the barrier and
the max-over-ranks of the timed region.  --impl reference times the CPU
oracle on whole layer-steps of the same workload on the host cores.
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
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "µs per layer-step (append+attn) at full shape; append HBM GB/s; attn FP8 TFLOPS"
CFG_ID = 3
N_INPUT_SETS = 6


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        pk = json.load(open(path))
        return pk["hbm_gbs"], pk["bf16_tflops"], pk.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def workload(cfg):
    T = cfg["grid_h"] * cfg["grid_w"]
    H, D, W, F = cfg["n_heads"], cfg["head_dim"], cfg["window_frames"], cfg["max_frames_per_chunk"]
    M = F * T
    N = (cfg["pinned_frames"] + W + F) * T
    flops = 4.0 * M * N * D * H               # QK^T + PV, algorithmic
    exps = float(M) * N * H                   # one exponential per score
    append_bytes = (3 * 2 * D + 3 * D + 12) * M * H   # bf16 in, codes + 3 fp32 scales out
    return dict(T=T, H=H, D=D, M=M, N=N, flops=flops, exps=exps, append_bytes=append_bytes)


def ncu_traffic(kernel_file: str, summary: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (sha256 recorded in the summary), else None."""
    path = os.path.join(ROOT, "profiles", summary)
    src = os.path.join(ROOT, "kv_cache_serving_append_b200", "csrc", kernel_file)
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    t = re.search(r"dram_bytes_per_full_launch:\s*([0-9.eE+]+)", text)
    if not m or not t:
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    return float(t.group(1)) if sha == m.group(1) else None


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    FIELDS = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, props):
        # nvidia-smi prints the PCI id as DDDDDDDD:BB:DD.F
        self.bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        time.sleep(0.3)

    def stop(self):
        if self.p is None:
            return None
        time.sleep(0.25)
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        rows = []
        for line in open(self.f.name):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10 or not parts[1].lower().endswith(self.bus[-12:]):
                continue
            try:
                rows.append(dict(sm=float(parts[2]), smax=float(parts[3]), power=float(parts[4]),
                                 hw=parts[6], hwt=parts[7], swt=parts[8], swp=parts[9]))
            except ValueError:
                continue
        os.unlink(self.f.name)
        if not rows:
            return None
        load = [r for r in rows if r["power"] > 200.0] or rows
        reasons = set()
        for r in load:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["smax"] for r in load), "reasons": sorted(reasons),
                "samples": len(load), "power_w_max": max(r["power"] for r in load)}


class OracleTimer:
    """The CPU oracle, as it stands, timed on whole layer-steps of the
    full-shape workload: the ring holds W committed frames (their codes are
    synthetic and not timed), and each step times the oracle's append of all
    T token rows of Q, K and V (all heads, the C oracle), its fp64 attention
    of every query row of every head over the full key set (the oracle's
    library-matmul form of the definition) and the ring advance."""

    def __init__(self, cfg):
        import numpy as np
        import oracle
        from kv_cache_serving_append_b200 import synth
        self.np, self.oracle, self.synth, self.cfg = np, oracle, synth, cfg
        self.wl = workload(cfg)
        self.ora = oracle.OracleCache(cfg)
        rng = np.random.default_rng(0)
        L = self.ora.layers[0]
        for _ in range(cfg["window_frames"]):
            s = self.ora.ring.staged_slots(1)[0]
            L["kc"][s] = rng.integers(0, 0x7E, L["kc"][s].shape, dtype=np.uint8)
            L["vc"][s] = rng.integers(0, 0x7E, L["vc"][s].shape, dtype=np.uint8)
            L["sk"][s] = 0.01
            L["sv"][s] = 0.01
            L["staged"] = 1
            self.ora.advance()
        self.inputs = []
        for i in range(2):
            q, k, v = synth.chunk(CFG_ID, cfg, 0, 100 + i, 1)
            self.inputs.append([synth.bf16_bits(t) for t in (q, k, v)])

    def step(self, i: int) -> float:
        """Seconds for one whole layer-step (append, attention, advance)."""
        t0 = time.perf_counter()
        self.ora.append(0, *self.inputs[i % 2], 1)
        out = self.ora.attend(0, matmul=True)
        self.ora.advance()
        dt = time.perf_counter() - t0
        assert out.shape == (self.wl["M"], self.wl["H"], self.wl["D"])
        return dt

    def describe(self) -> str:
        wl = self.wl
        return (f"full layer-step: oracle append of all {wl['T']} token rows of Q, K and V "
                f"({wl['H']} heads, plain C), fp64 attention of all {wl['M']} query rows x "
                f"{wl['H']} heads over {wl['N']} keys (the oracle's library-matmul form: "
                f"PyTorch CPU float64), ring advance; timed, not extrapolated")


def max_over_ranks(value_ms: float, world: int, device) -> float:
    """The slowest rank's time: every rank's timed region is reduced with MAX
    (replicas: one independent cache per GPU, no data-path collective)."""
    if world <= 1:
        return value_ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([value_ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def us_per_layer_step(elapsed_ms: float, steps: int, world: int) -> float:
    """Whole-job figure: the max-over-ranks time over the layer-steps all ranks did."""
    return elapsed_ms * 1e3 / (steps * world)


def run_seq48_timing(dev, steps: int, warmup: int) -> dict:
    """48 layers x (append + attend), then advance, per step, ring full; the
    step time and the spread of the per-layer (append + attend) times."""
    import torch
    from kv_cache_serving_append_b200 import configs, rtv, synth
    cfg = configs.get(4)
    wl = workload(cfg)
    L = cfg["n_layers"]
    cache = rtv.Cache(cfg, dev)
    sets = [synth.chunk(4, cfg, 0, 100 + i, 1, device=dev) for i in range(N_INPUT_SETS)]
    out = torch.empty((wl["T"], wl["H"], wl["D"]), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i, ev=None):
        for layer in range(L):
            q, k, v = sets[(i * L + layer) % N_INPUT_SETS]
            if ev is not None:
                ev[layer][0].record(stream)
            if cache.append(layer, q, k, v, 1, stream) or cache.attend(layer, out, stream):
                raise RuntimeError("append/attend failed")
            if ev is not None:
                ev[layer][1].record(stream)
        if cache.advance():
            raise RuntimeError("advance failed")

    for i in range(cfg["window_frames"] + 1 + warmup):   # fill the ring, warm up
        step(i)
    torch.cuda.synchronize()
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(L)]
           for _ in range(steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        step(i, evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    if cache.poll_error():
        raise RuntimeError("kernel error in the timed region")
    ms = t0.elapsed_time(t1) / steps
    per_layer = [statistics.mean(evs[i][l][0].elapsed_time(evs[i][l][1]) for i in range(steps)) * 1e3
                 for l in range(L)]
    res = {"workload": "48 layers x (append + attend), 40 heads x D128, 2992 tokens/frame, W=8, "
                       "ring full, then one advance", "ms_per_step": ms, "steps": steps,
           "cache_bytes": cache.nbytes,
           "per_layer_us": {"mean": statistics.mean(per_layer), "stdev": statistics.pstdev(per_layer),
                            "min": min(per_layer), "max": max(per_layer)},
           "attend_key_splits": cache.state().last_attend_splits}
    cache.close()
    return res


def run_seq48_graph_timing(dev, steps: int, warmup: int) -> dict:
    """The same 48-layer step replayed from one captured CUDA graph (ring
    state on the device; rtv_step_graph_*): one launch per step."""
    import torch
    from kv_cache_serving_append_b200 import configs, rtv, synth
    cfg = configs.get(4)
    wl = workload(cfg)
    L = cfg["n_layers"]
    cache = rtv.Cache(cfg, dev)
    sets = [synth.chunk(4, cfg, 0, 100 + i, 1, device=dev) for i in range(N_INPUT_SETS)]
    out = torch.empty((wl["T"], wl["H"], wl["D"]), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        for i in range(cfg["window_frames"]):          # direct calls fill the window
            for layer in range(L):
                q, k, v = sets[(i * L + layer) % N_INPUT_SETS]
                if cache.append(layer, q, k, v, 1, stream) or cache.attend(layer, out, stream):
                    raise RuntimeError("append/attend failed")
            if cache.advance():
                raise RuntimeError("advance failed")
        g = rtv.StepGraph(cache, 1, [sets[l % N_INPUT_SETS][0] for l in range(L)],
                          [sets[l % N_INPUT_SETS][1] for l in range(L)],
                          [sets[l % N_INPUT_SETS][2] for l in range(L)], [out] * L, stream)
        for _ in range(warmup):
            if g.launch(stream):
                raise RuntimeError("graph launch failed")
        stream.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        host0 = time.perf_counter()
        for _ in range(steps):
            if g.launch(stream):
                raise RuntimeError("graph launch failed")
        host_us = (time.perf_counter() - host0) * 1e6 / steps
        t1.record(stream)
        stream.synchronize()
    if cache.poll_error():
        raise RuntimeError("kernel error in the timed region")
    res = {"workload": "48 layers x (append + attend) + device ring advance, one CUDA graph "
                       "launch per step, ring full", "ms_per_step": t0.elapsed_time(t1) / steps,
           "host_us_per_launch": host_us, "steps": steps}
    g.close()
    cache.close()
    return res


def run_seq48(args):
    """--workload seq48: the 48-layer step on its own JSON line (one GPU)."""
    import torch
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    r = run_seq48_timing(dev, args.steps, args.warmup)
    line = {"metric": "ms per 48-layer step (append+attn per layer, then advance) at full shape",
            "value": r["ms_per_step"], "unit": "ms/step", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": False, "data": "synthetic",
            "config": {"workload": r["workload"], "cache_bytes": r["cache_bytes"]},
            "per_layer_us": r["per_layer_us"], "attend_key_splits": r["attend_key_splits"]}
    print(json.dumps(line))
    return 0


def run_project(args):
    """--workload project: the fused QKV projection + append on its own JSON
    line (one GPU), beside the unfused library path it replaces."""
    import torch
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    r = time_project(dev, args.steps, args.warmup)
    hbm_gbs, bf16_tf, bf16_tf_sus, peak_src = load_peaks()
    line = {"metric": "us per fused QKV projection + append (2992 x 15360 x 5120 FP8 GEMM)",
            "value": r["fused_us"], "unit": "us/call", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": False, "data": "synthetic",
            "config": {"workload": r["workload"]},
            "roofline": {"bound": "tensor", "achieved": r["fused_tflops"], "peak": 2.0 * bf16_tf,
                         "unit": "TFLOP/s", "frac": r["fused_tflops"] / (2.0 * bf16_tf),
                         "peak_source": f"{peak_src} bf16 burst x 2 (nominal fp8:bf16 ratio)",
                         "traffic": ncu_traffic("project_kernel.cu", "project_full_shape_ncu.md"),
                         "algorithmic_flop_per_launch": r["gemm_flop"]},
            "unfused_us": r.get("unfused_us"), "unfused_path": r.get("unfused_path")}
    print(json.dumps(line))
    return 0


def run_reference(args):
    """--impl reference: the CPU oracle as it stands, on the host cores, one
    whole full-shape layer-step per step (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    import torch
    from kv_cache_serving_append_b200 import configs
    cfg = configs.get(CFG_ID)
    timer = OracleTimer(cfg)
    for i in range(args.warmup):
        timer.step(i)
    t0 = time.perf_counter()
    vals = [timer.step(args.warmup + i) for i in range(args.steps)]
    wall = time.perf_counter() - t0
    v = statistics.mean(vals) * 1e6
    cores = max(oracle.num_threads(), torch.get_num_threads())
    line = {"metric": METRIC, "value": v, "unit": "us/layer-step", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": v / 1000.0, "timed_wall_s": wall, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(cfg),
            "cpu_baseline": {"value": v, "unit": "us/layer-step", "cores": cores,
                             "kind": "oracle", "sample": timer.describe()},
            "e2e": {"value": v, "unit": "us/layer-step", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def config_block(cfg):
    wl = workload(cfg)
    return {"workload": "full-shape single layer-step: append + attend + advance, "
                        "40 heads x D128, 2992 tokens/frame (44x68), 1 frame/chunk, W=8, "
                        "steady state (ring full)",
            "heads": wl["H"], "head_dim": wl["D"], "tokens_per_frame": wl["T"],
            "window_frames": cfg["window_frames"], "keys_per_query": wl["N"],
            "out_dtype": "f32",
            "l2": f"inputs rotate over {N_INPUT_SETS} chunks (552 MB) > L2; "
                  "per-step K/V key set 276 MB > L2",
            "parallelism": "replicas (one independent cache per GPU)"}


def fill_ring(cache, cfg, sets, stream, passes: int = 1):
    """Append + attend + advance until the ring is full (steady state)."""
    F = cfg["max_frames_per_chunk"]
    steps = cfg["window_frames"] // F + 2 + cfg["pinned_frames"]
    out = torch_empty_out(cfg, cache.device)
    for i in range(steps):
        n = 1 if (cfg["pinned_frames"] and i == 0) else F
        q, k, v = sets[i % len(sets)]
        rows = n * cfg["grid_h"] * cfg["grid_w"]
        for _ in range(passes):
            if cache.append(0, q[:rows], k[:rows], v[:rows], n, stream) or \
                    cache.attend(0, out[:rows], stream):
                raise RuntimeError("fill step failed")
        if cache.advance():
            raise RuntimeError("advance failed")


def torch_empty_out(cfg, device):
    import torch
    T = cfg["grid_h"] * cfg["grid_w"]
    return torch.empty((cfg["max_frames_per_chunk"] * T, cfg["n_heads"], cfg["head_dim"]),
                       dtype=torch.float32, device=device)


def time_layer(cfg_id, dev, steps: int, warmup: int, passes: int = 1, events: bool = True,
               barrier=None):
    """Steady-state layer-steps of one workload: per step `passes` x (append +
    attend), then advance.  Returns device times (ms) per step, per append and
    per attend (CUDA events on the launching stream) and the split count."""
    import torch
    from kv_cache_serving_append_b200 import configs, rtv, synth
    cfg = configs.get(cfg_id)
    F = cfg["max_frames_per_chunk"]
    cache = rtv.Cache(cfg, dev)
    sets = [synth.chunk(cfg_id, cfg, 0, 100 + i, F, device=dev) for i in range(N_INPUT_SETS)]
    out = torch_empty_out(cfg, dev)
    stream = torch.cuda.current_stream(dev)
    fill_ring(cache, cfg, sets, stream, passes)

    def step(i, ev=None):
        for p in range(passes):
            q, k, v = sets[(i * passes + p) % N_INPUT_SETS]
            if ev is not None:
                ev[p][0].record(stream)
            if cache.append(0, q, k, v, F, stream):
                raise RuntimeError("append failed")
            if ev is not None:
                ev[p][1].record(stream)
            if cache.attend(0, out, stream):
                raise RuntimeError("attend failed")
            if ev is not None:
                ev[p][2].record(stream)
        if cache.advance():
            raise RuntimeError("advance failed")

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    if cache.poll_error():
        raise RuntimeError("kernel error during warm-up")
    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(passes)]
          for _ in range(steps)] if events else None
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if barrier:
        barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(steps):
        step(i, ev[i] if ev else None)
    t1.record(stream)
    torch.cuda.synchronize()
    if barrier:
        barrier()
    if cache.poll_error():
        raise RuntimeError("kernel error in the timed region")
    res = {"step_ms": t0.elapsed_time(t1) / steps, "splits": cache.state().last_attend_splits,
           "cache": cache, "sets": sets, "out": out, "cfg": cfg, "stream": stream}
    if ev:
        res["append_ms"] = statistics.mean(e[0].elapsed_time(e[1]) for x in ev for e in x)
        res["attend_ms"] = statistics.mean(e[1].elapsed_time(e[2]) for x in ev for e in x)
    return res


def time_e2e(res, steps: int, warmup: int, world: int, dev):
    """End to end through the public API, every step: H2D of the step's Q/K/V
    from pinned host memory, append, attend, D2H of the output.  Copies run on
    their own streams into double-buffered device inputs and outputs, so the
    H2D of step i+1 and the D2H of step i-1 overlap step i's kernels; events
    order every reuse of a buffer.  Timed from the first H2D to the last D2H."""
    import torch
    cache, sets, cfg = res["cache"], res["sets"], res["cfg"]
    stream = res["stream"]
    F = cfg["max_frames_per_chunk"]
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    host_in = [tuple(t.cpu().pin_memory() for t in sets[i]) for i in range(2)]
    dev_in = [tuple(torch.empty_like(t) for t in sets[0]) for _ in range(2)]
    dev_out = [torch.empty_like(res["out"]) for _ in range(2)]
    host_out = [torch.empty(res["out"].shape, dtype=res["out"].dtype).pin_memory() for _ in range(2)]
    ev = lambda: torch.cuda.Event()   # noqa: E731
    in_ready = [ev(), ev()]      # H2D into dev_in[b] done
    in_free = [ev(), ev()]       # append that read dev_in[b] done
    out_ready = [ev(), ev()]     # attend into dev_out[b] done
    out_free = [ev(), ev()]      # D2H out of dev_out[b] done
    for b in range(2):
        in_free[b].record(stream)
        out_free[b].record(d2h_s)

    def h2d(i):
        b = i % 2
        with torch.cuda.stream(h2d_s):
            h2d_s.wait_event(in_free[b])
            for d, h in zip(dev_in[b], host_in[i % 2]):
                d.copy_(h, non_blocking=True)
            in_ready[b].record(h2d_s)

    def compute(i):
        b = i % 2
        stream.wait_event(in_ready[b])
        if cache.append(0, *dev_in[b], F, stream):
            raise RuntimeError("e2e append failed")
        in_free[b].record(stream)
        stream.wait_event(out_free[b])
        if cache.attend(0, dev_out[b], stream) or cache.advance():
            raise RuntimeError("e2e attend failed")
        out_ready[b].record(stream)

    def d2h(i):
        b = i % 2
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(out_ready[b])
            host_out[b].copy_(dev_out[b], non_blocking=True)
            out_free[b].record(d2h_s)

    def run(n):
        h2d(0)
        for i in range(n):
            if i + 1 < n:
                h2d(i + 1)
            compute(i)
            d2h(i)

    run(warmup)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(h2d_s)
    run(steps)
    e1.record(d2h_s)
    torch.cuda.synchronize()
    if cache.poll_error():
        raise RuntimeError("kernel error in the end-to-end region")
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    h2d_bytes = sum(t.numel() * t.element_size() for t in dev_in[0])
    d2h_bytes = host_out[0].numel() * host_out[0].element_size()
    return ms / steps, h2d_bytes, d2h_bytes


def time_project(dev, steps: int, warmup: int) -> dict:
    """The fused QKV projection + append (rtv_cache_append_project) at the
    full layer shape: a 2992 x 15360 x 5120 FP8 GEMM whose epilogue writes
    the cache.  For context, the path it replaces: three library FP8 GEMMs
    (torch._scaled_mm, one per Q/K/V, bf16 out) and then rtv_cache_append."""
    import torch
    from kv_cache_serving_append_b200 import configs, rtv, synth
    cfg = configs.get(CFG_ID)
    hidden = 5120
    H, D = cfg["n_heads"], cfg["head_dim"]
    T = cfg["grid_h"] * cfg["grid_w"]
    HD = H * D
    cache = rtv.Cache(cfg, dev)
    xc, sx, wc, sw = (torch.from_numpy(a).to(dev) for a in synth.projection_inputs(cfg, 0, 0, 1, hidden, False))
    stream = torch.cuda.current_stream(dev)

    def fused():
        if cache.append_project(0, xc, sx, wc, sw, 1, stream):
            raise RuntimeError("append_project failed")

    def timed(fn, n):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    flop = 2.0 * T * 3 * HD * hidden
    res = {"workload": "QKV projection (FP8 GEMM 2992 x 15360 x 5120, per-row / per-feature scales) "
                       "with the append fused into its epilogue, full layer shape",
           "gemm_flop": flop}
    fused_ms = timed(fused, steps)
    res["fused_us"] = fused_ms * 1e3
    res["fused_tflops"] = flop / (fused_ms * 1e-3) / 1e12
    if cache.poll_error():
        raise RuntimeError("kernel error in the fused projection")
    try:
        x8 = xc.view(torch.float8_e4m3fn)
        w8 = [wc[i * HD:(i + 1) * HD].view(torch.float8_e4m3fn) for i in range(3)]
        ws = [sw[i * HD:(i + 1) * HD].view(1, HD) for i in range(3)]
        xs = sx.view(T, 1)
        outs = [torch.empty((T, HD), dtype=torch.bfloat16, device=dev) for _ in range(3)]

        def unfused():
            for i in range(3):
                torch._scaled_mm(x8, w8[i].t(), scale_a=xs, scale_b=ws[i], out_dtype=torch.bfloat16,
                                 out=outs[i])
            if cache.append(0, outs[0].view(T, H, D), outs[1].view(T, H, D), outs[2].view(T, H, D), 1, stream):
                raise RuntimeError("append failed")

        un_ms = timed(unfused, steps)
        res["unfused_us"] = un_ms * 1e3
        res["unfused_path"] = "3 x torch._scaled_mm (rowwise scales, bf16 out) + rtv_cache_append"
    except Exception as e:   # the library GEMM is context only
        res["unfused_us"] = None
        res["unfused_error"] = str(e)[:200]
    cache.close()
    return res


def extra_workloads(dev, steps: int, warmup: int):
    """The other full-shape workloads, each timed on its own (one GPU)."""
    import torch
    out = {}
    k = max(3, min(steps, 10))
    # long window: 2 frames per chunk, W = 16, pinned conditioning slot
    r = time_layer(5, dev, k, 3)
    wl = workload(r["cfg"])
    out["long_window"] = {
        "workload": "1 layer, 40 heads x D128, 2992 tokens/frame, 2 frames/chunk, W=16 + pinned "
                    "slot, steady state", "us_per_layer_step": r["step_ms"] * 1e3,
        "append_us": r["append_ms"] * 1e3, "attn_us": r["attend_ms"] * 1e3,
        "attn_tflops": wl["flops"] / (r["attend_ms"] * 1e-3) / 1e12,
        "append_gbs": wl["append_bytes"] / (r["append_ms"] * 1e-3) / 1e9,
        "keys_per_query": wl["N"], "attend_key_splits": r["splits"], "steps": k}
    r["cache"].close()
    del r
    # several denoising passes per chunk (3 x append + attend, then advance)
    r = time_layer(CFG_ID, dev, k, 3, passes=3)
    out["multipass"] = {
        "workload": "full-shape layer, 3 denoising passes per chunk (append + attend each), "
                    "then one advance", "us_per_chunk": r["step_ms"] * 1e3,
        "us_per_pass": r["step_ms"] * 1e3 / 3, "append_us": r["append_ms"] * 1e3,
        "attn_us": r["attend_ms"] * 1e3, "steps": k}
    r["cache"].close()
    del r
    torch.cuda.empty_cache()
    out["seq48"] = run_seq48_timing(dev, min(steps, 5), 2)
    torch.cuda.empty_cache()
    out["seq48_graph"] = run_seq48_graph_timing(dev, min(steps, 5), 2)
    torch.cuda.empty_cache()
    out["project_append"] = time_project(dev, k, 3)
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the long-window, multi-pass and 48-layer workloads")
    ap.add_argument("--workload", default="layer", choices=["layer", "seq48", "project"])
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "seq48":
        return run_seq48(args)
    if args.workload == "project":
        return run_project(args)

    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=120))

    from kv_cache_serving_append_b200 import configs
    cfg = configs.get(CFG_ID)
    wl = workload(cfg)
    sampler = ClockSampler(torch.cuda.get_device_properties(dev)) if rank == 0 else None
    # time_layer fills the ring and runs the warm-up steps, then times exactly
    # `steps` steps between a barrier + synchronize on each side
    if sampler:
        sampler.start()
    res = time_layer(CFG_ID, dev, args.steps, args.warmup,
                     barrier=dist.barrier if world > 1 else None)
    clocks = sampler.stop() if sampler else None
    elapsed_ms = max_over_ranks(res["step_ms"] * args.steps, world, dev)
    splits = res["splits"]
    launches_per_step = 2 + (1 if splits > 1 else 0)
    append_ms, attend_ms = res["append_ms"], res["attend_ms"]

    e2e_steps = max(20, min(200, args.steps))
    e2e_ms, h2d, d2h = time_e2e(res, e2e_steps, 5, world, dev)
    res["cache"].close()
    del res
    torch.cuda.empty_cache()

    hbm_gbs, bf16_tf, bf16_tf_sus, peak_src = load_peaks()
    fp8_peak = 2.0 * bf16_tf
    props = torch.cuda.get_device_properties(dev)
    sm_count = props.multi_processor_count
    sm_max_ghz = (clocks or {}).get("sm_max_mhz") or 1965.0
    sm_max_ghz = sm_max_ghz / 1e3
    attn_tflops = wl["flops"] / (attend_ms * 1e-3) / 1e12
    append_gbs = wl["append_bytes"] / (append_ms * 1e-3) / 1e9
    us_per_step = us_per_layer_step(elapsed_ms, args.steps, world)
    line = {
        "metric": METRIC, "value": us_per_step, "unit": "us/layer-step", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": elapsed_ms / args.steps, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8e4m3 (QK^T), f16 (PV), f32 accumulate/softmax",
        "data": "synthetic", "config": config_block(cfg),
        "append_gbs": append_gbs, "append_us": append_ms * 1e3,
        "attn_tflops": attn_tflops, "attn_us": attend_ms * 1e3,
        "roofline": {"kernel": "rtv attend (tcgen05 FP8 attention; with a split key range the timed call includes the merge kernel)", "bound": "tensor",
                     "achieved": attn_tflops, "peak": fp8_peak, "unit": "TFLOP/s",
                     "frac": attn_tflops / fp8_peak,
                     "peak_source": f"{peak_src} bf16 burst {bf16_tf} TFLOP/s x 2 (nominal "
                                    "fp8:bf16 dense ratio)",
                     "traffic": ncu_traffic("attend_kernel.cu", "attend_full_shape_ncu.md"),
                     "algorithmic_flop_per_launch": wl["flops"]},
        # context: the same attention call against its exponential throughput
        # (one ex2 per score; 16 per clock per SM, measured by a probe; the
        # SM count and the maximum SM clock of this device)
        "roofline_exp": {"kernel": "rtv attend, softmax exponentials", "bound": "alu",
                         "achieved": wl["exps"] / (attend_ms * 1e-3) / 1e9,
                         "peak": 16 * sm_count * sm_max_ghz, "unit": "Gexp/s",
                         "frac": wl["exps"] / (attend_ms * 1e-3) / 1e9 / (16 * sm_count * sm_max_ghz),
                         "peak_source": "16 ex2/clock/SM x SMs x maximum SM clock"},
        "roofline_append": {"kernel": "rtv append (fused RoPE+amax+E4M3)", "bound": "hbm",
                            "achieved": append_gbs, "peak": hbm_gbs, "unit": "GB/s",
                            "frac": append_gbs / hbm_gbs,
                            "peak_source": f"{peak_src} HBM copy",
                            "traffic": ncu_traffic("append_kernel.cu", "append_full_shape_ncu.md"),
                            "algorithmic_bytes_per_launch": wl["append_bytes"]},
        "e2e": {"value": e2e_ms * 1e3 / world, "unit": "us/layer-step",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "overlap": "H2D of step i+1 and D2H of step i-1 on their own streams beside "
                           "step i's kernels (double-buffered device inputs and outputs)"},
        "gpu_launches": launches_per_step * args.steps,
        "attend_key_splits": splits,
        "clocks": clocks,
    }
    if world == 1 and not args.no_extra:
        line["workloads"] = extra_workloads(dev, args.steps, args.warmup)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        timer = OracleTimer(cfg)
        us = timer.step(0) * 1e6
        line["cpu_baseline"] = {"value": us, "unit": "us/layer-step",
                                "cores": max(oracle.num_threads(), torch.get_num_threads()),
                                "kind": "oracle", "sample": timer.describe()}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
