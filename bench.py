"""Benchmark of the quantized MoE expert layer on B200.

Default workload: the Mixtral-8x7B-shaped decode layer (E=8, top-2, d_model
4096, d_ff 14336, SwiGLU, INT3 group-128 asymmetric codes, rank-32
compensators on both blocks) with T=64 tokens per step. One step is one full
forward pass (routing, permute, compensator down-projections, gate/up GEMM +
SwiGLU, down GEMM, combine) through the C ABI.

Prints ONE JSON line (rank 0). Multi-GPU: one process per GPU (torchrun); each
rank runs an independent replica on its own token batch (the layer has no
exchange step on one node in this build), so scaling is weak and the value is
the total tokens/s of all ranks, timed on the device as the max over ranks.

``--impl reference`` times the fp64 CPU oracle (the only reference this method
has) on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {"mixtral_decode": "mixtral8x7b_decode", "mixtral_prefill": "mixtral8x7b_prefill",
             "dsv2lite_decode": "deepseek_v2_lite_decode", "dsv3_bitplane": "deepseek_v3_bitplane", "tiny": "tiny"}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--config", default="mixtral_decode")
    p.add_argument("--tokens", type=int, default=64)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=20.0)
    p.add_argument("--tileq", type=int, default=0,
                   help="rank of 2D-tiled shared compensators on both blocks (replacing the per-expert ones); 0 = off")
    p.add_argument("--tile-m", type=int, default=1024)
    p.add_argument("--redraw-bits", type=int, default=-1,
                   help="bit-plane configs: before timing, re-draw every block's bitwidth from {2,3,4} with this "
                        "seed and commit it with moe_layer_set_bits")
    p.add_argument("--tile-k", type=int, default=1024)
    p.add_argument("--no-extras", action="store_true",
                   help="skip the other workloads that the default single-GPU run also times")
    p.add_argument("--extra-steps", type=int, default=20)
    return p.parse_args()


# the other workloads a default single-GPU run times after the headline one:
# (config, tokens), each on its own layer, reported under "extra_workloads"
EXTRAS = [("mixtral_prefill", 8192), ("dsv3_bitplane", 4096), ("dsv3_bitplane", 128), ("dsv2lite_decode", 256)]


# ---------------------------------------------------------------------------
# algorithmic work
# ---------------------------------------------------------------------------

def block_bytes(cfg, spec, block):
    M, Kin = (2 * cfg.N, cfg.K) if block == 0 else (cfg.K, cfg.N)
    b = spec.bits[block]
    r = spec.rank
    if spec.fmt == 0:
        wb = b * M * Kin / 8 + 4 * M * Kin / spec.group
    elif spec.fmt == 1:
        wb = b * M * Kin / 8 + 2 * (1 << b)
    else:
        wb = 2 * M * Kin
    return wb, 2 * r * M, 2 * r * Kin  # codes+scales, B factor, A factor


def layer_bytes(cfg, counts, T):
    """Weights of touched experts (codes, scales/LUT, both factors) + X, logits, Y."""
    tot = 0.0
    for e, n in enumerate(counts):
        if n > 0:
            for b in (0, 1):
                wb, bb, ab = block_bytes(cfg, cfg.experts[e], b)
                tot += wb + bb + ab
    return tot + 2 * T * cfg.K + 4 * T * cfg.E + 2 * T * cfg.K


def tileq_shape(cfg, block, tq):
    """(M, K_in, P, Q) of a block type under tiled shared compensators tq = (r, tile_m, tile_k)."""
    M, Kin = (2 * cfg.N, cfg.K) if block == 0 else (cfg.K, cfg.N)
    return M, Kin, M // tq[1], Kin // tq[2]


def gemm1_bytes(cfg, counts, tq=None):
    """Algorithmic bytes of one gate/up GEMM launch: codes + scales + B1 of the
    touched experts, the routed activation rows (K + r columns, fp16) and the
    SwiGLU output rows (N columns, fp16). With tiled shared compensators
    (tq = (r, tile_m, tile_k)): the shared U1 once, and P*r compensator
    columns per routed row."""
    tot = 0.0
    if tq:
        M, Kin, P, Q = tileq_shape(cfg, 0, tq)
        tot += 2 * M * tq[0]
    for e, n in enumerate(counts):
        if n > 0:
            wb, bb, _ = block_bytes(cfg, cfg.experts[e], 0)
            r = cfg.experts[e].rank
            if tq:
                tot += wb + 2 * n * (cfg.K + P * tq[0]) + 2 * n * cfg.N
            else:
                tot += wb + bb + 2 * n * (cfg.K + r) + 2 * n * cfg.N
    return tot


def tileq_bytes_flops(cfg, counts, T, tq):
    """Factor bytes (U, V once; the cores of touched experts) and flops of the
    tiled shared compensators of both blocks: z = V x per token (W1) or per
    routed row (W2), u = C z per routed row and row tile, U u per routed row."""
    r = tq[0]
    rows = sum(counts)
    touched = sum(1 for n in counts if n > 0)
    b = f = 0.0
    for block in (0, 1):
        M, Kin, P, Q = tileq_shape(cfg, block, tq)
        b += 2 * (M * r + r * Kin) + touched * 2 * P * Q * r * r
        f += 2.0 * (T if block == 0 else rows) * Kin * r + 2.0 * rows * (P * Q * r * r + M * r)
    return b, f


def gemm1_flops(cfg, counts):
    """Algorithmic flops of one gate/up GEMM launch: 2 * rows * 2N * (K + r)."""
    return sum(2.0 * n * 2 * cfg.N * (cfg.K + cfg.experts[e].rank) for e, n in enumerate(counts))


def layer_flops(cfg, counts):
    """2 * rows * 3NK for the three projections plus the compensator terms
    2 * rows * r * (2K + 3N)."""
    tot = 0.0
    for e, n in enumerate(counts):
        r = cfg.experts[e].rank
        tot += 2.0 * n * 3 * cfg.N * cfg.K + 2.0 * n * r * (2 * cfg.K + 3 * cfg.N)
    return tot


# ---------------------------------------------------------------------------
# clocks sampled during the timed region (NVML reads only)
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index):
        self.samples, self.reasons, self.ok = [], set(), False
        self.stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        while not self.stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self.stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def measured_peaks():
    """(HBM GB/s, dense bf16 TFLOP/s burst, sustained, source)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ---------------------------------------------------------------------------

def cpu_oracle_rate(cfg, blocks_cpu, X, logits, top_k, budget_s):
    """Times the fp64 oracle on the first tokens of the batch, one token at a
    time (each token dequantises its own experts), until ``budget_s`` seconds
    have passed. Returns tokens/s, tokens done, seconds and threads."""
    import numpy as np
    import torch
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from moe_testlib import OracleExperts
    import oracle as orc
    Xn = X.float().cpu().numpy().astype(np.float64)
    Ln = logits.cpu().numpy()
    t0 = time.perf_counter()
    done = 0
    for t in range(Xn.shape[0]):
        orc.moe_forward(Xn, Ln, top_k, OracleExperts(blocks_cpu), cfg.N, rows=[t])
        done += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return done / dt, done, dt, host_threads()


def host_threads():
    """Cores of the host and the threads the oracle's numpy BLAS may use."""
    blas = None
    try:
        from threadpoolctl import threadpool_info
        blas = max((i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"), default=None)
    except Exception:
        pass
    return {"host_cores": os.cpu_count(), "blas_threads": blas}


KERNEL_SOURCES = {
    "decode_gemm_w1_swiglu": ["decode_gemm.cu", "decode_frag.cuh", "tc.cuh", "common.cuh"],
    "prefill_gemm_w1_swiglu": ["prefill_gemm.cu", "decode_frag.cuh", "tc.cuh", "common.cuh"],
}


def kernel_source_digest(kname):
    """sha256 over the sources of a kernel, to tell whether a stored ncu
    capture still describes the code being timed."""
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kname, []):
        with open(os.path.join(ROOT, "bit_quantized_moe_top_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def stored_traffic(kname, workload):
    """DRAM bytes per launch from profiles/traffic.json, or None when absent or
    captured from different kernel sources."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            d = json.load(f)
        e = d[f"{kname}@{workload}"]
        if e["source_sha256"] != kernel_source_digest(kname):
            return None
        return e["dram_bytes_per_launch"]
    except Exception:
        return None


def max_over_ranks(total_ms, world, device):
    """The job's time: the slowest rank's device-timed total (all ranks take
    part in the same collective; a barrier follows)."""
    if world <= 1:
        return total_ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(total_ms)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.barrier()
    return float(t.item())


def weak_scaling_value(world, tokens_per_rank, ms_per_step):
    """Tokens/s of the whole job: every rank runs its own batch of T tokens."""
    return world * tokens_per_rank / (ms_per_step / 1000.0)


def build_layer(bq, cfg, blocks, max_tokens):
    import ctypes
    descs = [bq.ExpertDesc((ctypes.c_int * 2)(*sp.bits), sp.fmt, sp.group, sp.rank) for sp in cfg.experts[:cfg.E]]
    L = bq.MoELayer(cfg.E, cfg.K, cfg.N, max_tokens, cfg.top_k, descs)
    for (e, b), blk in blocks.items():
        L.set_expert_weights(e, b, blk.codes, blk.scales, blk.zeros_or_lut,
                             blk.A if blk.rank else None, blk.B if blk.rank else None)
    return L


# ---------------------------------------------------------------------------

def config_dict(cfg, T, workload, world, tq=None):
    return {"workload": workload, "T": T, "E": cfg.E, "top_k": cfg.top_k, "d_model": cfg.K, "d_ff": cfg.N,
            "bits": sorted(set(b for sp in cfg.experts for b in sp.bits)),
            "format": "bit-plane+LUT" if cfg.experts[0].fmt == 1 else "int asym",
            "group": cfg.experts[0].group, "ranks": sorted(set(sp.rank for sp in cfg.experts)),
            "parallelism": f"replicas x{world}",
            "l2": "flushed between steps (256 MiB write, untimed)",
            **({"compensator": {"kind": "2D-tiled shared factors", "rank": tq[0], "tile_m": tq[1],
                                "tile_k": tq[2]}} if tq else {})}


def make_cfg(ms, name, tq=None):
    cfg = ms.make_config(name)
    if tq:
        # the tiled shared compensators replace every expert's own pair
        cfg.experts = [ms.ExpertSpec(sp.fmt, sp.bits, sp.group, 0) for sp in cfg.experts]
    return cfg


def workload_name(name, T, tq=None, redraw=-1):
    w = f"{WORKLOADS[name]}_T{T}" + (f"_tileq_r{tq[0]}_{tq[1]}x{tq[2]}" if tq else "")
    if redraw >= 0:
        w += f"_bits_redrawn_{redraw}"
    return w


def measure(bq, ms, name, T, dev, steps, warmup, rank=0, world=1, tq=None, redraw=-1, e2e=True):
    """Builds the layer of one workload on ``dev`` and times ``steps`` forward
    passes with CUDA events (L2 flushed between them, untimed). Returns the
    figures of the bench line (without cpu_baseline)."""
    import torch
    cfg = make_cfg(ms, name, tq)
    workload = workload_name(name, T, tq, redraw)
    if redraw >= 0 and any(sp.fmt != ms.FMT_BITPLANE_LUT for sp in cfg.experts):
        raise SystemExit("--redraw-bits needs a bit-plane configuration")
    blocks = {}
    for e in range(cfg.E):
        for b in (0, 1):
            blocks[(e, b)] = ms.make_block(cfg, e, b, device=dev)
    L = build_layer(bq, cfg, blocks, max_tokens=T)
    if redraw >= 0:
        # one set_bits re-draw of every (expert, block): the kernels then read the new number of planes
        import numpy as np
        rng = np.random.default_rng(np.random.SeedSequence([cfg.cid, 3000, redraw]))
        new = rng.integers(2, 5, size=(cfg.E, 2))
        for e in range(cfg.E):
            for b in (0, 1):
                L.set_bits(e, b, int(new[e, b]))
        cfg.experts = [ms.ExpertSpec(sp.fmt, (int(new[e, 0]), int(new[e, 1])), sp.group, sp.rank)
                       for e, sp in enumerate(cfg.experts)]
    if tq:
        for b in (0, 1):
            U, V, C = ms.make_tileq(cfg, b, tq[0], tq[1], tq[2], dev)
            L.set_tileq(b, tq[0], tq[1], tq[2], U, V, C)
    X, logits = ms.make_inputs(cfg, T, dev, key_extra=rank)
    Y = torch.empty_like(X)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def step():
        L.forward(X, logits, cfg.top_k, Y)

    for _ in range(max(3, warmup)):
        step()
    torch.cuda.synchronize()
    st = L.sync_status()
    assert st == 0, f"device status {st} ({bq.moe_status_string(st)})"
    routing = L.routing(T, cfg.top_k)
    counts = routing["counts"].cpu().tolist()
    launches_per_step = L.last_launch_count()

    # timed region: per-step events, L2 flushed (untimed) between steps; the
    # gate/up GEMM alone is bracketed by events (profiling level 2), so the
    # other launches keep their programmatic overlap
    L.set_profiling(2)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    kt = {}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(int(str(dev).split(":")[-1])) as clocks:
        for i in range(steps):
            flush.fill_(i & 0xFF)
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
            if i % 8 == 0 or i == steps - 1:
                # (reading the events synchronises the stream: only now and then)
                for kn, t in L.kernel_times():
                    kt.setdefault(kn, []).append(t)
        torch.cuda.synchronize()
    # the per-kernel breakdown: a few more steps with every launch bracketed
    # (outside the timed region: the events serialise the launches)
    L.set_profiling(True)
    kb = {}
    for i in range(5):
        flush.fill_(i & 0xFF)
        step()
        for kn, t in L.kernel_times():
            kb.setdefault(kn, []).append(t)
    L.set_profiling(False)
    assert L.sync_status() == 0
    step_ms = [a.elapsed_time(b) for a, b in ev]
    pct = {q: statistics.quantiles(step_ms, n=10)[i] if len(step_ms) >= 2 else step_ms[0]
           for q, i in (("p10", 0), ("p50", 4), ("p90", 8))}
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    ms_per_step = total_ms / steps
    value = weak_scaling_value(world, T, ms_per_step)

    # dominant kernel: the gate/up GEMM (2/3 of the weight bytes and flops)
    hbm_peak, tc_peak, tc_sustained, peak_src = measured_peaks()
    kernel_means = {k: statistics.mean(v) for k, v in kb.items()}
    prefill = "prefill_gemm_w1_swiglu" in kt
    kname = "prefill_gemm_w1_swiglu" if prefill else "decode_gemm_w1_swiglu"
    k1 = statistics.mean(kt[kname]) if kname in kt else float("nan")
    layer_b = layer_bytes(cfg, counts, T)
    layer_f = layer_flops(cfg, counts)
    if tq:
        tb, tf = tileq_bytes_flops(cfg, counts, T, tq)
        layer_b += tb
        layer_f += tf
    if prefill:
        # a kernel of a few ms timed inside a step, not a seconds-long loop:
        # the burst peak is its denominator
        f1 = gemm1_flops(cfg, counts)
        achieved = f1 / (k1 * 1e-3) / 1e12
        roofline = {"bound": "tensor", "kernel": kname, "achieved": achieved, "peak": tc_peak,
                    "unit": "TFLOP/s", "frac": achieved / tc_peak,
                    "traffic": stored_traffic(kname, workload),
                    "peak_source": f"{peak_src} bf16 burst (fp16 has the same dense rate)",
                    "frac_of_sustained_peak": achieved / tc_sustained, "algorithmic_flops_per_launch": f1,
                    "launch_ms": k1}
    else:
        b1 = gemm1_bytes(cfg, counts, tq)
        achieved = b1 / (k1 * 1e-3) / 1e9
        roofline = {"bound": "hbm", "kernel": kname, "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                    "frac": achieved / hbm_peak,
                    "traffic": stored_traffic(kname, workload), "peak_source": peak_src,
                    "algorithmic_bytes_per_launch": b1, "launch_ms": k1}
    out = {"value": value, "ms_per_step": ms_per_step, "ms_per_step_percentiles": pct,
           "config": config_dict(cfg, T, workload, world, tq),
           "layer_hbm_gbs": layer_b / (ms_per_step * 1e-3) / 1e9,
           "layer_hbm_frac": layer_b / (ms_per_step * 1e-3) / 1e9 / hbm_peak,
           "layer_tflops": layer_f / (ms_per_step * 1e-3) / 1e12,
           "layer_bytes_per_step": layer_b, "layer_flops_per_step": layer_f,
           "roofline": roofline, "kernels_ms": kernel_means,
           "kernels_ms_note": "every launch bracketed by events in 5 extra steps (serialised); the step time has only the gate/up GEMM bracketed",
           "gpu_launches": launches_per_step * steps, "clocks": clocks.summary(),
           "_cfg": cfg, "_blocks": blocks, "_X": X, "_logits": logits}

    if e2e:
        # end to end: host buffers through moe_layer_forward_host (copies inside the timed region)
        Xh = X.cpu().pin_memory()
        Lh = logits.cpu().pin_memory()
        Yh = torch.empty_like(Xh).pin_memory()
        for _ in range(3):
            L.forward_host(Xh, Lh, cfg.top_k, Yh)
        e2e_steps = max(10, steps // 4)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(e2e_steps):
            L.forward_host(Xh, Lh, cfg.top_k, Yh)
        e2e_s = (time.perf_counter() - t0) / e2e_steps
        out["e2e"] = {"value": world * T / e2e_s, "unit": "tokens/s",
                      "h2d_bytes_per_step": T * cfg.K * 2 + T * cfg.E * 4, "d2h_bytes_per_step": T * cfg.K * 2}
    L.close()
    del flush
    return out


def public(d):
    return {k: v for k, v in d.items() if not k.startswith("_")}


def reference_arm(args, ms):
    """The fp64 CPU oracle timed on the host cores: each step is the oracle on
    a bounded sample of the batch (its first tokens, one at a time)."""
    cfg = make_cfg(ms, args.config)
    T = args.tokens
    blocks = {}
    for e in range(cfg.E):
        for b in (0, 1):
            blocks[(e, b)] = ms.make_block(cfg, e, b, device="cpu")
    X, logits = ms.make_inputs(cfg, T, "cpu")
    budget = max(1.0, args.cpu_seconds / max(1, args.steps + args.warmup))
    rates = []
    for i in range(args.warmup + args.steps):
        r, n, dt, thr = cpu_oracle_rate(cfg, blocks, X, logits, cfg.top_k, budget)
        if i >= args.warmup:
            rates.append((r, n, dt, thr))
    val = statistics.median([r[0] for r in rates])
    thr = rates[0][3]
    cores = thr["blas_threads"] or thr["host_cores"]
    return {"impl": "reference", "metric": "MoE-layer tokens/s", "value": val, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * statistics.mean([r[2] for r in rates]),
            "ms_per_step_note": "measured: one step = the oracle on the bounded sample below",
            "ms_per_step_extrapolated_full_batch": 1000.0 * T / val,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(cfg, T, workload_name(args.config, T), args.gpus),
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": cores, "host_cores": thr["host_cores"],
                             "blas_threads": thr["blas_threads"], "kind": "oracle",
                             "sample": f"first {rates[0][1]} token(s) of the T={T} batch per step, one token "
                                       f"at a time (its experts dequantised in fp64)"},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    import torch
    import torch.distributed as dist
    import moe_synth as ms

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    T = args.tokens
    tq = (args.tileq, args.tile_m, args.tile_k) if args.tileq else None

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(args, ms)), flush=True)
        return

    from bit_quantized_moe_top_b200 import build
    build.build()
    import bit_quantized_moe_top_b200 as bq

    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = f"cuda:{local}"

    head = measure(bq, ms, args.config, T, dev, args.steps, args.warmup, rank, world, tq, args.redraw_bits)
    line = None
    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1 and not tq:
            cfg, blocks = head["_cfg"], head["_blocks"]
            cpu_blocks = {k: ms.BlockWeights(**{**v.__dict__, "codes": v.codes.cpu(),
                                              "scales": None if v.scales is None else v.scales.cpu(),
                                              "zeros_or_lut": None if v.zeros_or_lut is None else v.zeros_or_lut.cpu(),
                                              "A": None if v.A is None else v.A.cpu(),
                                              "B": None if v.B is None else v.B.cpu()})
                          for k, v in blocks.items()}
            r, n, dt, thr = cpu_oracle_rate(cfg, cpu_blocks, head["_X"].cpu(), head["_logits"].cpu(), cfg.top_k,
                                            args.cpu_seconds)
            cpu = {"value": r, "unit": "tokens/s", "cores": thr["blas_threads"] or thr["host_cores"],
                   "host_cores": thr["host_cores"], "blas_threads": thr["blas_threads"], "kind": "oracle",
                   "sample": f"first {n} token(s) of the T={T} batch, one token at a time (its two experts "
                             f"dequantised in fp64), {dt:.1f} s"}
        line = {"metric": "MoE-layer tokens/s", "value": head["value"], "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f16 operands, f32 accumulate", "data": "synthetic"}
        line.update({k: v for k, v in public(head).items() if k not in ("value", "ms_per_step")})
        line["cpu_baseline"] = cpu
    for k in [k for k in head if k.startswith("_")]:
        del head[k]
    torch.cuda.empty_cache()
    # the other workloads, on one GPU only (the scaling runs time the headline workload alone)
    if world == 1 and not args.no_extras and not tq and args.redraw_bits < 0:
        extras = {}
        for name, t in EXTRAS:
            if name == args.config and t == T:
                continue
            r = measure(bq, ms, name, t, dev, args.extra_steps, 3, e2e=False)
            extras[r["config"]["workload"]] = {k: v for k, v in public(r).items() if k != "config"}
            del r
            torch.cuda.empty_cache()
        line["extra_workloads"] = extras
        line["gpu_launches"] += sum(x["gpu_launches"] for x in extras.values())
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
