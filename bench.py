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

--workload seq48 times the 48-layer step at the same shape instead (every
layer appended and attended, then one advance; the ring full), reporting ms
per step and the spread of the per-layer times; it prints a line of its own
and is not the headline metric.

N > 1 runs N independent replicas (one per GPU, launched by torchrun); the
path has no data exchange, the process group only carries the barrier and
the max-over-ranks of the timed region.  --impl reference times the CPU
oracle on a bounded sample of the same workload on the host cores.
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
    N = (W + F) * T
    flops = 4.0 * M * N * D * H               # QK^T + PV, algorithmic
    append_bytes = (3 * 2 * D + 3 * D + 12) * M * H   # bf16 in, codes + 3 fp32 scales out
    return dict(T=T, H=H, D=D, M=M, N=N, flops=flops, append_bytes=append_bytes)


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
    """The CPU oracle, as it stands, timed on bounded samples of one
    full-shape layer-step: the ring holds W committed frames (their codes are
    synthetic and not timed); each sample times the oracle's append of
    `r_app` token rows of Q, K and V (all heads), its fp64 attention for
    `r_att` query rows (all heads) over the full key set, and the ring
    update, and extrapolates each part linearly to the whole step."""

    def __init__(self, cfg):
        import numpy as np
        import oracle
        from kv_cache_serving_append_b200 import synth
        self.np, self.oracle, self.cfg = np, oracle, cfg
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
        q, k, v = synth.chunk(CFG_ID, cfg, 0, 0, 1)
        self.bits = [synth.bf16_bits(t) for t in (q, k, v)]
        self.ora.append(0, *self.bits, 1)
        self.split = (cfg["rope_t"], cfg["rope_h"], cfg["rope_w"])

    def sample(self, r_app: int, r_att: int, h_s: int, offset: int = 0):
        """µs for the whole layer-step, extrapolated from timed pieces.

        Attention is timed on h_s heads for r_att and then 2*r_att query
        rows; the difference is the per-row cost and the rest the per-call
        cost of dequantising the key set, so that
            t_attn = (H / h_s) * (t_call + (M / r_att) * t_rows).
        """
        np, oracle, wl = self.np, self.oracle, self.wl
        T, M, H = wl["T"], wl["M"], wl["H"]
        r0 = (offset * r_app) % (T - r_app + 1)
        t0 = time.perf_counter()
        for i, x in enumerate(self.bits):
            oracle.append_tensor(np.ascontiguousarray(x[r0:r0 + r_app]), r_app,
                                 self.cfg["grid_w"], 8, i < 2, self.split)
        t1 = time.perf_counter()
        L = self.ora.layers[0]
        h0 = (offset * h_s) % (H - h_s + 1)
        hs = slice(h0, h0 + h_s)
        _, kc, sk, vc, sv = self.ora.key_set(0)
        args = (L["qc"][hs], L["sq"][hs], kc[hs], sk[hs], vc[hs], sv[hs])
        times = []
        for r in (r_att, 2 * r_att):
            rows = ((np.arange(r) * 997 + offset * 131) % M).astype(np.int32)
            ta = time.perf_counter()
            oracle.attend(*args, rows=rows)
            times.append(time.perf_counter() - ta)
        t_rows = max(times[1] - times[0], 1e-9)
        t_call = max(times[0] - t_rows, 0.0)
        t2 = time.perf_counter()
        ring = oracle.OracleRing(self.cfg["window_frames"], 1, 0)
        for _ in range(self.cfg["window_frames"] + 1):
            ring.commit(1)
        t3 = time.perf_counter()
        attn_s = (H / h_s) * (t_call + (M / r_att) * t_rows)
        us = ((t1 - t0) * T / r_app + attn_s + (t3 - t2) / (self.cfg["window_frames"] + 1)) * 1e6
        desc = (f"oracle on one full-shape layer-step, sampled: append of {r_app} of {T} token "
                f"rows (Q, K, V, all {H} heads), fp64 attention of {h_s} of {H} heads for "
                f"{r_att} and {2 * r_att} of {M} query rows over {wl['N']} keys (per-row and "
                f"per-call costs separated), each extrapolated linearly to the full step")
        return us, desc


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


def run_seq48(args):
    """48 layers x (append + attend), then advance, per step; one GPU."""
    import torch
    from kv_cache_serving_append_b200 import configs, rtv, synth
    cfg = configs.get(4)
    wl = workload(cfg)
    L = cfg["n_layers"]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cache = rtv.Cache(cfg)
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

    for i in range(cfg["window_frames"] + 1 + args.warmup):   # fill the ring, warm up
        step(i)
    torch.cuda.synchronize()
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(L)]
           for _ in range(args.steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(i, evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    if cache.poll_error():
        raise RuntimeError("kernel error in the timed region")
    ms = t0.elapsed_time(t1) / args.steps
    per_layer = [statistics.mean(evs[i][l][0].elapsed_time(evs[i][l][1]) for i in range(args.steps)) * 1e3
                 for l in range(L)]
    line = {"metric": "ms per 48-layer step (append+attn per layer, then advance) at full shape",
            "value": ms, "unit": "ms/step", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": False, "data": "synthetic",
            "config": {"workload": "48 layers x (append + attend), 40 heads x D128, 2992 tokens/frame, "
                                   "W=8, ring full", "cache_bytes": cache.nbytes},
            "per_layer_us": {"mean": statistics.mean(per_layer), "stdev": statistics.pstdev(per_layer),
                             "min": min(per_layer), "max": max(per_layer)},
            "attend_key_splits": cache.state().last_attend_splits}
    cache.close()
    print(json.dumps(line))
    return 0


def run_reference(args):
    """--impl reference: the CPU oracle as it stands, on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    from kv_cache_serving_append_b200 import configs
    cfg = configs.get(CFG_ID)
    timer = OracleTimer(cfg)
    n = args.warmup + args.steps
    # bound the whole run to a few minutes of CPU work: per step, 8 token rows
    # of the append and 1 head x (n_threads, 2 n_threads) query rows
    r_att = max(1, oracle.num_threads())
    vals = []
    desc = ""
    for i in range(n):
        us, desc = timer.sample(8, r_att, 1, offset=i)
        if i >= args.warmup:
            vals.append(us)
    v = statistics.mean(vals)
    line = {"metric": METRIC, "value": v, "unit": "us/layer-step", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": v / 1000.0, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(cfg),
            "cpu_baseline": {"value": v, "unit": "us/layer-step", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": desc},
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


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default="layer", choices=["layer", "seq48"])
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "seq48":
        return run_seq48(args)

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

    from kv_cache_serving_append_b200 import configs, rtv, synth
    cfg = configs.get(CFG_ID)
    wl = workload(cfg)
    T, H, D = wl["T"], wl["H"], wl["D"]
    cache = rtv.Cache(cfg, dev)
    sets = [synth.chunk(CFG_ID, cfg, 0, 100 + i, 1, device=dev) for i in range(N_INPUT_SETS)]
    # fp32 output: the configuration the parity tests hold to the tolerance
    out = torch.empty((T, H, D), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i):
        q, k, v = sets[i % N_INPUT_SETS]
        st = cache.append(0, q, k, v, 1, stream)
        if st:
            raise rtv.RtvError(st, "append")
        st = cache.attend(0, out, stream)
        if st:
            raise rtv.RtvError(st, "attend")
        st = cache.advance()
        if st:
            raise rtv.RtvError(st, "advance")

    # fill the ring (steady state), then warm up
    for i in range(cfg["window_frames"] + 1 + args.warmup):
        step(i)
    torch.cuda.synchronize()
    if cache.poll_error():
        raise RuntimeError("kernel error during warm-up")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(torch.cuda.get_device_properties(dev)) if rank == 0 else None
    if sampler:
        sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start.record(stream)
    for i in range(args.steps):
        q, k, v = sets[i % N_INPUT_SETS]
        e = ev[i]
        e[0].record(stream)
        if cache.append(0, q, k, v, 1, stream):
            raise RuntimeError("append failed")
        e[1].record(stream)
        if cache.attend(0, out, stream):
            raise RuntimeError("attend failed")
        e[2].record(stream)
        if cache.advance():
            raise RuntimeError("advance failed")
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    if cache.poll_error():
        raise RuntimeError("kernel error in the timed region")
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), world, dev)
    # kernels per step: append, attention, and the split merge when the key range is split
    splits = cache.state().last_attend_splits
    launches_per_step = 2 + (1 if splits > 1 else 0)
    append_ms = statistics.mean(ev[i][0].elapsed_time(ev[i][1]) for i in range(args.steps))
    attend_ms = statistics.mean(ev[i][1].elapsed_time(ev[i][2]) for i in range(args.steps))

    # end to end through the public API: pinned host inputs -> H2D -> append ->
    # attend -> D2H of the output, every step
    host_in = [tuple(t.cpu().pin_memory() for t in sets[i]) for i in range(2)]
    dev_in = tuple(torch.empty_like(t) for t in sets[0])
    host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e2e_steps = max(20, min(200, args.steps // 5))

    def e2e_step(i):
        hq = host_in[i % 2]
        for d, h in zip(dev_in, hq):
            d.copy_(h, non_blocking=True)
        if cache.append(0, *dev_in, 1, stream) or cache.attend(0, out, stream) or cache.advance():
            raise RuntimeError("e2e step failed")
        host_out.copy_(out, non_blocking=True)

    for i in range(5):
        e2e_step(i)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    h2d = sum(t.numel() * t.element_size() for t in dev_in)
    d2h = host_out.numel() * host_out.element_size()

    hbm_gbs, bf16_tf, bf16_tf_sus, peak_src = load_peaks()
    fp8_peak = 2.0 * bf16_tf
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
        "roofline_append": {"kernel": "rtv append (fused RoPE+amax+E4M3)", "bound": "hbm",
                            "achieved": append_gbs, "peak": hbm_gbs, "unit": "GB/s",
                            "frac": append_gbs / hbm_gbs,
                            "traffic": ncu_traffic("append_kernel.cu", "append_full_shape_ncu.md"),
                            "algorithmic_bytes_per_launch": wl["append_bytes"]},
        "e2e": {"value": e2e_ms * 1e3 / (e2e_steps * world), "unit": "us/layer-step",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "attend_key_splits": splits,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        timer = OracleTimer(cfg)
        us, desc = timer.sample(r_app=256, r_att=2 * oracle.num_threads(), h_s=4)
        line["cpu_baseline"] = {"value": us, "unit": "us/layer-step",
                                "cores": oracle.num_threads(), "kind": "oracle", "sample": desc}
    cache.close()
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
