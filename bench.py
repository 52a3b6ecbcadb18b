#!/usr/bin/env python
"""Benchmark of the dynamic block-sparse attention layer (pool -> select -> attend).

One step = the whole hot path over one layer's synthetic Q/K/V: block means of Q and
K, per-query-block top-k selection, and attention inside the kept blocks.  The default
workload is the long-sequence case: batch 1, 40 heads, d = 128, L = 122,880 tokens
(24 x 64 x 80 latent grid, 960 blocks of 128), keep 10% (96 key blocks per query
block, diagonal included).

Prints ONE JSON line (rank 0).  `value` is effective TFLOP/s over the selected blocks
(4 * Lp * k * block * d * heads per layer, all ranks' layers / max-over-ranks time).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

With N > 1 it runs under torch.distributed (one process per GPU): every rank runs its
own layer (independent problems, weak scaling, no data-path collective).
`--impl reference` times the CPU oracle (the reference arm) on this host instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from video_dit_dynamic_b200 import inputs  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long122880",
                    help="tiny | 480p | 720p | long122880 | sweep<keep%%> e.g. sweep100")
    ap.add_argument("--impl", default="sbsa", choices=["sbsa", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-rope", action="store_true", help="skip timing the fused RoPE + pooling kernel")
    ap.add_argument("--no-fp8", action="store_true", help="skip timing the FP8 path")
    ap.add_argument("--no-nvfp4", action="store_true", help="skip timing the NVFP4 linear layer")
    ap.add_argument("--no-ulysses", action="store_true", help="skip timing the Light-Ulysses kernels")
    return ap.parse_args()


def workload(name: str) -> inputs.Workload:
    if name.startswith("sweep"):
        return inputs.sweep_workload(int(name[5:]) / 100.0)
    return inputs.WORKLOADS[name]


def keep_count(nb: int, keep: float) -> int:
    # the library's own sbsa_keep_blocks is used on the GPU path; this mirrors it for
    # the CPU-only reference arm (round-half-up, clamped to [1, nb])
    return max(1, min(nb, int(math.floor(keep * nb + 0.5))))


def layer_flops(wl: inputs.Workload, k: int) -> float:
    return 4.0 * wl.seq_len_padded * k * wl.block * wl.head_dim * wl.heads * wl.batch


def max_over_ranks(pg, device, timings: dict) -> dict:
    """Each timing (ms) replaced by its maximum over all ranks; one all-reduce for all.

    Every rank calls this with the same keys in the same order.  `pg` is the
    torch.distributed module (or None for a single process)."""
    if pg is None:
        return dict(timings)
    names = sorted(timings)
    t = torch.tensor([float(timings[n]) for n in names], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return {n: float(x) for n, x in zip(names, t.tolist())}


def fp8_summary(fp8: dict, flops: float, pool_select_ms: float, peaks: dict) -> dict:
    """Figures of the FP8 path.  Its attention does the Q.K^T half of the FLOPs in e4m3 and
    the P.V half in bf16, so its tensor roofline is the harmonic mix of the fp8 peak
    (measured bf16 peak x 2, the nominal 4.5 / 2.25 PFLOP/s ratio) and the bf16 peak:
    flops / (flops/2 / fp8 + flops/2 / bf16) = 4/3 of the bf16 peak."""
    bf16 = peaks["bf16_tflops"]
    mixed = flops / (0.5 * flops / (2.0 * bf16) + 0.5 * flops / bf16)
    att_tflops = flops / (fp8["att_ms"] / 1e3) / 1e12
    quant_gbs = fp8["quant_bytes"] / (fp8["quant_ms"] / 1e3) / 1e9
    layer_ms = pool_select_ms + fp8["quant_ms"] + fp8["att_ms"]
    return {"attention": {"ms": fp8["att_ms"], "TFLOP/s": att_tflops, "mixed_peak": mixed,
                          "frac": att_tflops / mixed, "kernel": "attn_kernel<128,128,fp8>"},
            "key_mean_plus_quantize": {"ms": fp8["quant_ms"], "GB/s": quant_gbs,
                                       "hbm_frac": quant_gbs / peaks["hbm_gbs"],
                                       "algorithmic_bytes": fp8["quant_bytes"]},
            "layer_ms": layer_ms, "layer_TFLOP/s": flops / (layer_ms / 1e3) / 1e12,
            "note": "pool + select + key mean + quantize + fp8 attention, timed apart from the step"}


def fp4_summary(fp4: dict, peaks: dict) -> dict:
    """Figures of the NVFP4 linear layer.  Its GEMM is a dense contraction on the
    block-scaled fp4 tensor cores, whose peak is taken as the measured bf16 peak x 4 (the
    nominal 9 / 2.25 PFLOP/s ratio); the quantizer is bandwidth-bound."""
    fp4_peak = 4.0 * peaks["bf16_tflops"]
    tf = fp4["gemm_flop"] / (fp4["gemm_ms"] / 1e3) / 1e12
    qgbs = fp4["quant_bytes"] / (fp4["quant_ms"] / 1e3) / 1e9
    return {"shape": {"m": fp4["m"], "n": fp4["n"], "k": fp4["k"]},
            "gemm": {"ms": fp4["gemm_ms"], "TFLOP/s": tf, "peak": fp4_peak, "frac": tf / fp4_peak,
                     "kernel": "nvfp4_gemm_pair_kernel", "algorithmic_flop": fp4["gemm_flop"],
                     "algorithmic_bytes": fp4["gemm_bytes"],
                     "GB/s": fp4["gemm_bytes"] / (fp4["gemm_ms"] / 1e3) / 1e9},
            "amax_plus_quantize": {"ms": fp4["quant_ms"], "GB/s": qgbs, "hbm_frac": qgbs / peaks["hbm_gbs"],
                                   "algorithmic_bytes": fp4["quant_bytes"]},
            "layer_ms": fp4["quant_ms"] + fp4["gemm_ms"],
            "note": "QKV projection of the same tokens, timed apart from the step"}


def spread(ms_list) -> dict:
    """Median and best of this rank's per-step kernel times (the mean reported beside them is
    the maximum over ranks)."""
    return {"ms_median": statistics.median(ms_list), "ms_best": min(ms_list)}


def job_tflops(flops_per_rank: float, world: int, ms: float) -> float:
    """Whole-job throughput: every rank's layer counted, divided by the slowest rank's time."""
    return flops_per_rank * world / (ms / 1e3) / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons.  Sampling starts before
    the warm-up (nvidia-smi takes a moment to start) every 50 ms; only the samples whose
    timestamps fall inside the timed region (mark_begin .. mark_end) are reported."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.t0 = self.t1 = None
        self.path = os.path.join("/tmp", f"sbsa_clocks_{os.getpid()}.csv")
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.gpu_id = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            self.gpu_id = None

    def start(self):
        if self.gpu_id is None:
            return
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def mark_begin(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    @staticmethod
    def _epoch(stamp: str):
        import datetime
        try:
            return datetime.datetime.strptime(stamp.strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    rows.append((self._epoch(parts[0]), float(parts[1]), float(parts[2]),
                                 [n for n, v in zip(names, parts[4:8]) if v.lower() == "active"]))
                except ValueError:
                    continue
        os.unlink(self.path)
        inside = [r for r in rows if r[0] is not None and self.t0 is not None and self.t1 is not None
                  and self.t0 - 0.05 <= r[0] <= self.t1 + 0.05]
        use = inside if inside else rows[-3:]
        sm = [r[1] for r in use]
        reasons = sorted({n for r in use for n in r[3]})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(r[2] for r in use) if use else None,
                "reasons": reasons, "samples": len(sm),
                "window": "timed region" if inside else "last samples (none inside the timed region)"}


# ------------------------------------------------------------------ traffic record
def recorded_traffic(kernel_src: str, workload_name: str):
    """DRAM bytes per attention launch from a committed ncu capture, valid only while
    the kernel source is unchanged (hash match); else None."""
    path = os.path.join(ROOT, "profiles", "attn_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        with open(kernel_src, "rb") as f:
            h = hashlib.sha256(f.read()).hexdigest()[:16]
        if rec.get("attn_source_sha256_16") != h:
            return None
        return rec.get("dram_bytes_per_launch", {}).get(workload_name)
    except (OSError, ValueError):
        return None


# ------------------------------------------------------------------ CPU oracle sample
CPU_SAMPLE_UNITS = 64  # attention units of the CPU sample


def cpu_sample_inputs(wl: inputs.Workload, q=None, kt=None, v=None):
    """Head 0 of the layer as bf16 bits on the host: from the given tensors (the GPU arm's)
    or freshly generated (the reference arm).  The sample's work does not depend on the
    values, only on the shapes."""
    if q is None:
        one = inputs.Workload(wl.name, 1, 1, wl.grid, wl.head_dim, wl.block, wl.keep, wl.kind)
        q, kt, v = inputs.make_qkv(one, seed=0, device="cpu")
    return tuple(inputs.bf16_bits(t[:, 0:1]) for t in (q, kt, v))


def cpu_oracle_sample(wl: inputs.Workload, k: int, qb, kb, vb, n_units: int = CPU_SAMPLE_UNITS):
    """Time the oracle on one bounded sample of the layer: pool + select of one full head
    and attention of n_units (head 0, query block) units, the same units in every call and
    in both arms; extrapolated to the layer (40 heads x all query blocks).  Returns
    (seconds per layer, description)."""
    import numpy as np
    import oracle
    L, blk, nb = wl.seq_len, wl.block, wl.num_blocks
    t0 = time.perf_counter()
    qm = oracle.pool(qb, L, blk)
    km = oracle.pool(kb, L, blk)
    col = oracle.select(qm, km, k)
    t_ps = time.perf_counter() - t0
    units = sorted(np.random.default_rng(12345).choice(nb, size=min(n_units, nb), replace=False).tolist())
    rp = oracle.uniform_row_ptr(1, 1, nb, k)
    t0 = time.perf_counter()
    oracle.attention(qb, kb, vb, L, blk, rp, col, units=units)
    t_at = time.perf_counter() - t0
    heads = wl.heads * wl.batch
    layer_s = t_ps * heads + t_at / len(units) * (nb * heads)
    desc = (f"pool+select of 1 of {heads} heads ({t_ps:.2f} s) and attention of {len(units)} of "
            f"{nb * heads} (head, query-block) units ({t_at:.2f} s), extrapolated to the layer")
    return layer_s, desc


def cpu_baseline_line(wl: inputs.Workload, k: int, samples_s: list, desc: str, cores: int, extra=None) -> dict:
    """The cpu_baseline object: the mean over the timed samples, with their spread."""
    layer_s = statistics.mean(samples_s)
    out = {"value": layer_flops(wl, k) / layer_s / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
           "sample": f"{desc}; {len(samples_s)} timed samples after one untimed: {layer_s:.1f} s/layer",
           "layer_seconds": layer_s,
           "spread": {"min_TFLOP/s": layer_flops(wl, k) / max(samples_s) / 1e12,
                      "max_TFLOP/s": layer_flops(wl, k) / min(samples_s) / 1e12,
                      "samples": len(samples_s)}}
    if extra:
        out.update(extra)
    return out


def gpu_arm_cpu_baseline(wl: inputs.Workload, k: int, q, kt, v, repeats: int = 3) -> dict:
    """The GPU arm's cpu_baseline: the reference arm's sample (same heads, units and
    oracle), one untimed call, then `repeats` timed ones on all host cores; plus the same
    sample on one core."""
    import oracle
    qb, kb, vb = cpu_sample_inputs(wl, q, kt, v)
    oracle.set_threads(os.cpu_count() or 1)
    cores = oracle.threads_used()
    cpu_oracle_sample(wl, k, qb, kb, vb)
    runs = [cpu_oracle_sample(wl, k, qb, kb, vb) for _ in range(repeats)]
    oracle.set_threads(1)
    try:
        one_s, one_desc = cpu_oracle_sample(wl, k, qb, kb, vb, n_units=4)
    finally:
        oracle.set_threads(os.cpu_count() or 1)
    single = {"value": layer_flops(wl, k) / one_s / 1e12, "unit": "TFLOP/s", "cores": 1,
              "sample": one_desc.replace(f"{CPU_SAMPLE_UNITS} of", "4 of") + " (one core)"}
    return cpu_baseline_line(wl, k, [r[0] for r in runs], runs[0][1], cores, {"single_core": single})


# ------------------------------------------------------------------ reference arm
def run_reference(args, wl):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    nb = wl.num_blocks
    k = keep_count(nb, wl.keep)
    qb, kb, vb = cpu_sample_inputs(wl)
    oracle.set_threads(os.cpu_count() or 1)
    cores = oracle.threads_used()
    # every step is the same bounded sample of the layer (one head's pool + select and
    # 64 attention units), extrapolated; the warm-up steps are not timed
    samples, desc = [], ""
    for i in range(args.warmup + args.steps):
        layer_s, desc = cpu_oracle_sample(wl, k, qb, kb, vb)
        if i >= args.warmup:
            samples.append(layer_s)
    cb = cpu_baseline_line(wl, k, samples, desc, cores)
    value = cb["value"]
    line = {
        "impl": "reference", "metric": "sparse-attn ms/layer & TFLOP/s (selected blocks) at L=122880, 90% sparse",
        "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": cb["layer_seconds"] * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": config_of(wl, k, "oracle on host cores; one bounded sample per step, extrapolated to the layer"),
        "cpu_baseline": {kk: vv for kk, vv in cb.items() if kk != "layer_seconds"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(wl, k, note):
    return {"workload": f"{wl.name}: B={wl.batch} H={wl.heads} d={wl.head_dim} L={wl.seq_len} "
                        f"(Lp={wl.seq_len_padded}, grid {'x'.join(map(str, wl.grid))}) block={wl.block} "
                        f"keep={wl.keep:g} (k={k} of {wl.num_blocks})",
            "batch": wl.batch, "heads": wl.heads, "head_dim": wl.head_dim, "seq_len": wl.seq_len,
            "seq_len_padded": wl.seq_len_padded, "block": wl.block, "keep": wl.keep, "k_blocks": k,
            "num_blocks": wl.num_blocks, "parallelism": "replica per GPU (independent layers)",
            "l2": "inputs larger than L2 (Q+K+V = %.2f GB)" % (3 * wl.batch * wl.heads * wl.seq_len_padded *
                                                                wl.head_dim * 2 / 1e9),
            "note": note}


# ------------------------------------------------------------------ GPU arm
def run_gpu(args, wl):
    from video_dit_dynamic_b200 import sbsa

    ws_n, rank, local = dist_env()
    torch.cuda.set_device(local)
    pg = None
    if ws_n > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        pg = dist
    dev = torch.device("cuda", local)
    sbsa.load()
    nb = wl.num_blocks
    k = sbsa.sbsa_keep_blocks(nb, wl.keep)
    shape = sbsa.make_shape(wl.batch, wl.heads, wl.seq_len, wl.head_dim, wl.block)
    q, kt, v = inputs.make_qkv(wl, seed=rank, device=dev)
    rows = wl.batch * wl.heads * nb
    qm = torch.empty(rows * wl.head_dim, dtype=torch.float32, device=dev)
    km = torch.empty_like(qm)
    rp = torch.empty(rows + 1, dtype=torch.int32, device=dev)
    ci = torch.empty(rows * k, dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)
    flops = layer_flops(wl, k)
    pool_bytes = 2 * q.numel() * 2 + 2 * qm.numel() * 4

    def step(evs=None):
        # sbsa_forward issues exactly these three launches; they are called one by one
        # here so that each kernel's time can be read from events on the same stream
        if evs: evs[0].record(stream)
        sbsa.sbsa_pool_qk(shape, q, kt, qm, km, stream=stream)
        if evs: evs[1].record(stream)
        sbsa.sbsa_select_blocks(shape, qm, km, k, rp, ci, stream=stream)
        if evs: evs[2].record(stream)
        sbsa.sbsa_attention_fwd(shape, q, kt, v, rp, ci, 0.0, o, stream=stream)
        if evs: evs[3].record(stream)

    def barrier():
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize(dev)

    clocks = ClockSampler(local)
    clocks.start()
    for _ in range(args.warmup):
        step()
    sbsa.sbsa_check(stream)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier()
    clocks.mark_begin()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    barrier()
    clocks.mark_end()
    clk = clocks.stop()
    sbsa.sbsa_check(stream)
    elapsed_ms = t_start.elapsed_time(t_end)
    pool_ms = [e[0].elapsed_time(e[1]) for e in evs]
    sel_ms = [e[1].elapsed_time(e[2]) for e in evs]
    att_ms = [e[2].elapsed_time(e[3]) for e in evs]
    # the same step through the fused entry point, for cross-checking
    ws_buf = sbsa.alloc_workspace(shape, k, device=dev)
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    sbsa.sbsa_forward(shape, q, kt, v, k, 0.0, o, None, ws_buf, stream=stream)
    torch.cuda.synchronize(dev)
    f0.record(stream)
    for _ in range(min(args.steps, 5)):
        sbsa.sbsa_forward(shape, q, kt, v, k, 0.0, o, None, ws_buf, stream=stream)
    f1.record(stream)
    torch.cuda.synchronize(dev)
    forward_ms = f0.elapsed_time(f1) / min(args.steps, 5)
    sbsa.sbsa_check(stream)

    # the fused 3D RoPE + pooling kernel (the step before pooling in a DiT layer), timed
    # on its own: it reads Q and K once and writes the rotated tensors and the means
    rope = None
    if not args.no_rope:
        table = torch.empty(sbsa.sbsa_rope_table_floats(wl.head_dim, wl.grid), dtype=torch.float32, device=dev)
        sbsa.sbsa_rope_table_init(wl.head_dim, wl.grid, 10000.0, table, stream=stream)
        qo, ko = torch.empty_like(q), torch.empty_like(kt)
        for _ in range(2):
            sbsa.sbsa_rope_pool_qk(shape, wl.grid, table, q, kt, qo, ko, qm, km, stream=stream)
        r0 = torch.cuda.Event(enable_timing=True)
        r1 = torch.cuda.Event(enable_timing=True)
        n_rope = 5
        r0.record(stream)
        for _ in range(n_rope):
            sbsa.sbsa_rope_pool_qk(shape, wl.grid, table, q, kt, qo, ko, qm, km, stream=stream)
        r1.record(stream)
        torch.cuda.synchronize(dev)
        sbsa.sbsa_check(stream)
        rope_ms = r0.elapsed_time(r1) / n_rope
        rope_bytes = 4 * q.numel() * 2 + 2 * qm.numel() * 4
        rope = {"ms": rope_ms, "algorithmic_bytes": rope_bytes}
        del qo, ko, table

    # the FP8 path (key mean -> per-block e4m3 quantization of Q and smoothed K -> the
    # attention with e4m3 Q.K^T products), timed on its own over the same selection
    fp8 = None
    if not args.no_fp8 and wl.head_dim == 128:
        kbar = torch.empty(wl.batch * wl.heads * wl.head_dim, dtype=torch.float32, device=dev)
        q8 = torch.empty(q.numel(), dtype=torch.uint8, device=dev)
        k8 = torch.empty_like(q8)
        qs = torch.empty(rows, dtype=torch.float32, device=dev)
        ks = torch.empty_like(qs)
        o8 = torch.empty_like(q)

        def fp8_step(fe=None):
            if fe: fe[0].record(stream)
            sbsa.sbsa_key_mean(shape, km, kbar, stream=stream)
            sbsa.sbsa_quantize_qk_fp8(shape, q, kt, kbar, q8, k8, qs, ks, stream=stream)
            if fe: fe[1].record(stream)
            sbsa.sbsa_attention_fwd_fp8(shape, q8, k8, v, qs, ks, rp, ci, 0.0, o8, stream=stream)
            if fe: fe[2].record(stream)

        sbsa.sbsa_pool_qk(shape, q, kt, qm, km, stream=stream)
        sbsa.sbsa_select_blocks(shape, qm, km, k, rp, ci, stream=stream)
        for _ in range(3):
            fp8_step()
        n_fp8 = max(3, min(args.steps, 10))
        fes = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_fp8)]
        for i in range(n_fp8):
            fp8_step(fes[i])
        torch.cuda.synchronize(dev)
        sbsa.sbsa_check(stream)
        fp8 = {"quant_ms": statistics.mean(e[0].elapsed_time(e[1]) for e in fes),
               "att_ms": statistics.mean(e[1].elapsed_time(e[2]) for e in fes),
               # bf16 Q and K read, their codes written, the block means read for the key mean
               "quant_bytes": 2 * q.numel() * 2 + 2 * q.numel() + 2 * rows * 4 + km.numel() * 4}
        del kbar, q8, k8, qs, ks, o8

    # the NVFP4 linear layer that feeds this attention: the fused QKV projection of the
    # same tokens, [L, H*d] x [3*H*d, H*d]^T + bias.  The weights are quantized once; a
    # step quantizes the activations (amax, then codes and scales) and runs the GEMM.
    fp4 = None
    if not args.no_nvfp4 and wl.head_dim * wl.heads % 256 == 0:
        fm, fk = wl.seq_len_padded * wl.batch, wl.heads * wl.head_dim
        fn = 3 * fk
        g4 = torch.Generator(device=dev).manual_seed(100 + rank)
        xa = torch.randn(fm, fk, generator=g4, device=dev).to(torch.bfloat16)
        wb = (torch.randn(fn, fk, generator=g4, device=dev) * 0.02).to(torch.bfloat16)
        bias4 = torch.randn(fn, generator=g4, device=dev)
        a_amax = torch.empty(1, dtype=torch.float32, device=dev)
        b_amax = torch.empty_like(a_amax)
        a_codes = torch.empty(fm * fk // 2, dtype=torch.uint8, device=dev)
        b_codes = torch.empty(fn * fk // 2, dtype=torch.uint8, device=dev)
        a_sf = torch.empty(sbsa.sbsa_nvfp4_scale_bytes(fm, fk), dtype=torch.uint8, device=dev)
        b_sf = torch.empty(sbsa.sbsa_nvfp4_scale_bytes(fn, fk), dtype=torch.uint8, device=dev)
        c4 = torch.empty(fm, fn, dtype=torch.bfloat16, device=dev)
        sbsa.sbsa_nvfp4_amax(wb, b_amax, stream=stream)
        sbsa.sbsa_nvfp4_quantize(wb, b_amax, b_codes, b_sf, stream=stream)

        def fp4_step(fe=None):
            if fe: fe[0].record(stream)
            sbsa.sbsa_nvfp4_amax(xa, a_amax, stream=stream)
            sbsa.sbsa_nvfp4_quantize(xa, a_amax, a_codes, a_sf, stream=stream)
            if fe: fe[1].record(stream)
            sbsa.sbsa_nvfp4_gemm(fm, fn, fk, a_codes, a_sf, a_amax, b_codes, b_sf, b_amax, bias4, c4, stream=stream)
            if fe: fe[2].record(stream)

        for _ in range(3):
            fp4_step()
        n_fp4 = max(3, min(args.steps, 10))
        fes = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_fp4)]
        for i in range(n_fp4):
            fp4_step(fes[i])
        torch.cuda.synchronize(dev)
        sbsa.sbsa_check(stream)
        fp4 = {"quant_ms": statistics.mean(e[0].elapsed_time(e[1]) for e in fes),
               "gemm_ms": statistics.mean(e[1].elapsed_time(e[2]) for e in fes),
               "m": fm, "n": fn, "k": fk,
               # amax pass reads the activations, the quantizer reads them again and
               # writes codes (k/2 bytes per row) and scales (k/16)
               "quant_bytes": 2 * fm * fk * 2 + fm * fk // 2 + fm * fk // 16,
               # the GEMM must read both operands' codes and scales and write C once
               "gemm_bytes": (fm + fn) * (fk // 2 + fk // 16) + fm * fn * 2,
               "gemm_flop": 2.0 * fm * fn * fk}
        del xa, wb, bias4, a_codes, b_codes, a_sf, b_sf, c4

    # Light-Ulysses pre/post-processing of the same layer: the four kernels around the two
    # all-to-alls, over the whole layer (what G ranks do together, 1/G each)
    uly = None
    if not args.no_ulysses and wl.head_dim == 128:
        ushape = sbsa.make_ulysses_shape(1, wl.seq_len, wl.seq_len_padded, wl.heads, wl.head_dim)
        g5 = torch.Generator(device=dev).manual_seed(200 + rank)
        xq = torch.randn(wl.seq_len, 3, wl.heads, wl.head_dim, generator=g5, device=dev).to(torch.bfloat16)
        ub = sbsa.sbsa_ulysses_qkv_bytes(ushape, wl.heads)
        ob = sbsa.sbsa_ulysses_o_bytes(ushape, wl.heads)
        usend = torch.empty(ub, dtype=torch.uint8, device=dev)
        uq, uk, uv = (torch.empty_like(q) for _ in range(3))
        uy = torch.empty(wl.seq_len, wl.heads, wl.head_dim, dtype=torch.bfloat16, device=dev)
        osend = torch.empty(ob, dtype=torch.uint8, device=dev)
        ubase = torch.tensor([usend.data_ptr()], dtype=torch.int64, device=dev)
        obase = torch.tensor([osend.data_ptr()], dtype=torch.int64, device=dev)
        calls = [
            ("pack_qkv", lambda: sbsa.sbsa_ulysses_pack_qkv(ushape, 0, wl.heads, xq, usend, stream=stream),
             xq.numel() * 2 + ub),
            ("unpack_qkv", lambda: sbsa.sbsa_ulysses_unpack_qkv(ushape, 0, wl.heads, usend, uq, uk, uv, stream=stream),
             ub + 3 * uq.numel() * 2),
            ("pack_o", lambda: sbsa.sbsa_ulysses_pack_o(ushape, 0, wl.heads, uq, osend, stream=stream),
             uy.numel() * 2 + ob),
            ("unpack_o", lambda: sbsa.sbsa_ulysses_unpack_o(ushape, 0, wl.heads, osend, uy, stream=stream),
             ob + uy.numel() * 2),
            # the peer-put packs, world 1: the "peer" receive buffer is this GPU's own
            ("put_qkv", lambda: sbsa.sbsa_ulysses_put_qkv(ushape, 0, wl.heads, xq, ubase, 0, 0, stream=stream),
             xq.numel() * 2 + ub),
            ("put_o", lambda: sbsa.sbsa_ulysses_put_o(ushape, 0, wl.heads, uq, obase, 0, 0, stream=stream),
             uy.numel() * 2 + ob),
        ]
        uly = {}
        for uname, ucall, nbytes in calls:
            for _ in range(2):
                ucall()
            u0, u1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            u0.record(stream)
            for _ in range(5):
                ucall()
            u1.record(stream)
            torch.cuda.synchronize(dev)
            uly[uname] = {"ms": u0.elapsed_time(u1) / 5, "algorithmic_bytes": nbytes}
        sbsa.sbsa_check(stream)
        del xq, usend, uq, uk, uv, uy, osend, ubase, obase

    # end to end through the public API from pinned host buffers
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = (t.cpu().pin_memory() for t in (q, kt, v))
        oh = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        bufs = (torch.empty_like(q), torch.empty_like(q), torch.empty_like(q), torch.empty_like(q), ws_buf)
        for _ in range(2):
            sbsa.forward_from_host(shape, qh, kh, vh, k, o_host=oh, device_buffers=bufs, stream=stream)
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        n_e2e = max(3, min(args.steps, 5))
        e0.record(stream)
        for _ in range(n_e2e):
            sbsa.forward_from_host(shape, qh, kh, vh, k, o_host=oh, device_buffers=bufs, stream=stream)
        e1.record(stream)
        barrier()
        sbsa.sbsa_check(stream)
        e2e_ms = e0.elapsed_time(e1) / n_e2e
        e2e = {"ms": e2e_ms, "h2d_bytes_per_step": 3 * q.numel() * 2, "d2h_bytes_per_step": o.numel() * 2}

    t = max_over_ranks(pg, dev, {"elapsed": elapsed_ms, "att": statistics.mean(att_ms),
                                 "pool": statistics.mean(pool_ms), "sel": statistics.mean(sel_ms),
                                 "forward": forward_ms, "e2e": e2e["ms"] if e2e is not None else 0.0,
                                 "rope": rope["ms"] if rope is not None else 0.0,
                                 "fp8_quant": fp8["quant_ms"] if fp8 is not None else 0.0,
                                 "fp8_att": fp8["att_ms"] if fp8 is not None else 0.0,
                                 "fp4_quant": fp4["quant_ms"] if fp4 is not None else 0.0,
                                 "fp4_gemm": fp4["gemm_ms"] if fp4 is not None else 0.0,
                                 **({f"uly_{k}": v["ms"] for k, v in uly.items()} if uly is not None else {})})
    elapsed_ms, att_avg, pool_avg, sel_avg, forward_ms = (t[n] for n in ("elapsed", "att", "pool", "sel", "forward"))
    if e2e is not None:
        e2e["ms"] = t["e2e"]
    if rope is not None:
        rope["ms"] = t["rope"]
    if fp8 is not None:
        fp8["quant_ms"], fp8["att_ms"] = t["fp8_quant"], t["fp8_att"]
    if fp4 is not None:
        fp4["quant_ms"], fp4["gemm_ms"] = t["fp4_quant"], t["fp4_gemm"]
    if uly is not None:
        for uname in uly:
            uly[uname]["ms"] = t[f"uly_{uname}"]
    ms_step = elapsed_ms / args.steps
    value = job_tflops(flops, ws_n, ms_step)

    if rank == 0:
        peaks, peak_src = load_peaks()
        att_tflops = flops / (att_avg / 1e3) / 1e12
        traffic = recorded_traffic(os.path.join(ROOT, "video_dit_dynamic_b200", "csrc", "attn.cuh"), wl.name)
        pool_gbs = pool_bytes / (pool_avg / 1e3) / 1e9
        line = {
            "metric": "sparse-attn ms/layer & TFLOP/s (selected blocks) at L=122880, 90% sparse",
            "value": value, "unit": "TFLOP/s", "n_gpus": ws_n, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": config_of(wl, k, "step = pool + select + attention of one layer; value = selected-block "
                                       "FLOP / step time"),
            "clocks": clk,
            "gpu_launches": 3 * args.steps,
            "roofline": {"bound": "tensor", "achieved": att_tflops, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": att_tflops / peaks["bf16_tflops"], "traffic": traffic,
                         "kernel": f"attn_kernel<{wl.head_dim},{wl.block}>",
                         "peak_source": f"{peak_src} bf16 dense (burst)",
                         "frac_of_sustained": att_tflops / peaks["bf16_tflops_sustained"],
                         "algorithmic_flop_per_launch": flops, "avg_launch_ms": att_avg},
            "kernels": {
                "pool": {"ms": pool_avg, **spread(pool_ms), "GB/s": pool_gbs, "hbm_frac": pool_gbs / peaks["hbm_gbs"],
                         "algorithmic_bytes": pool_bytes},
                "select": {"ms": sel_avg, **spread(sel_ms), "flop": 2.0 * wl.batch * wl.heads * nb * nb * wl.head_dim},
                "pool_plus_select_effective_GB/s": pool_bytes / ((pool_avg + sel_avg) / 1e3) / 1e9,
                "attention": {"ms": att_avg, **spread(att_ms), "TFLOP/s": att_tflops},
                "sbsa_forward_ms": forward_ms,
                **({"rope_pool": {"ms": rope["ms"], "GB/s": rope["algorithmic_bytes"] / (rope["ms"] / 1e3) / 1e9,
                                  "hbm_frac": rope["algorithmic_bytes"] / (rope["ms"] / 1e3) / 1e9 / peaks["hbm_gbs"],
                                  "algorithmic_bytes": rope["algorithmic_bytes"],
                                  "note": "3D RoPE fused with pooling, timed alone (not part of the step)"}}
                   if rope is not None else {}),
                **({"fp8": fp8_summary(fp8, flops, pool_avg + sel_avg, peaks)} if fp8 is not None else {}),
                **({"nvfp4_linear": fp4_summary(fp4, peaks)} if fp4 is not None else {}),
                **({"ulysses": {k: {**v, "GB/s": v["algorithmic_bytes"] / (v["ms"] / 1e3) / 1e9,
                                    "hbm_frac": v["algorithmic_bytes"] / (v["ms"] / 1e3) / 1e9 / peaks["hbm_gbs"]}
                                for k, v in uly.items()}} if uly is not None else {}),
            },
            "peaks": {"source": peak_src, **peaks},
        }
        if e2e is not None:
            line["e2e"] = {"value": job_tflops(flops, ws_n, e2e["ms"]), "unit": "TFLOP/s",
                           "h2d_bytes_per_step": e2e["h2d_bytes_per_step"],
                           "d2h_bytes_per_step": e2e["d2h_bytes_per_step"], "ms_per_step": e2e["ms"]}
        if ws_n == 1 and not args.no_cpu_baseline:
            cb = gpu_arm_cpu_baseline(wl, k, q, kt, v)
            cb.pop("layer_seconds", None)
            line["cpu_baseline"] = cb
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


def main():
    args = parse()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    wl = workload(args.workload)
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_gpu(args, wl)


if __name__ == "__main__":
    main()
