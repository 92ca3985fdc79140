#!/usr/bin/env python
"""Throughput of the KDA hot path on B200: chunkwise prefill tokens/s (with
tensor-core and HBM fractions) and decode-step state GB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kda|reference]

One step = one chunkwise forward (cumulative decay, intra-chunk transform,
state propagation, output) over the batched-prefill workload B=8, H=32,
T=8192, dk=dv=128, bf16 q/k/v/out with fp32 gates and state, seeded synthetic
inputs (3.2 GB per step, larger than L2).  The decode workload (N=256, H=32,
d=128, 1000 chained steps) is timed in the same run and reported under
"decode".  Multi-GPU: one process per GPU under torchrun; every rank runs the
same workload on its own GPU with no collective on the data path (weak
scaling); the timed region is bracketed by barriers and the max over ranks is
reported.  `--impl reference` times the fp64 CPU oracle on a bounded sample of
the same workload instead (rank 0 only).
"""
import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)
import workloads as W  # noqa: E402

METRIC = "KDA fwd tokens/sec (H=32,d=128,bf16) + % TC peak; decode-step state GB/s vs HBM"
CHUNK = 64
BYTES_PER_HEAD_TOKEN = 1540        # q,k,v,out bf16 (4*256) + log_alpha fp32 (512) + beta (4)
FLOP_PER_HEAD_TOKEN = 2 * CHUNK * (3 * 128 + 2 * 128) + 6 * 128 * 128   # 180,224 at C=64, d=128


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.3)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[4:]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        pmax = max(r[2] for r in rows)
        loaded = [r for r in rows if r[2] >= 0.5 * pmax] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3][1:5])
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded),
                "sm_max_mhz": max(r[1] for r in loaded), "power_w_max": pmax,
                "samples": len(loaded), "reasons": reasons}


# ----------------------------------------------------------------------------
# distributed plumbing
# ----------------------------------------------------------------------------
def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, ws):
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------
# oracle timing (CPU baseline / reference arm)
# ----------------------------------------------------------------------------
def oracle_sample(inp_host, cfg, heads, batch=1):
    """Oracle on the first `batch` batch entries and `heads` heads of the workload."""
    import oracle
    sl = lambda x: x[0:batch, :, :heads].contiguous()
    t = time.perf_counter()
    oracle.fwd(sl(inp_host["q"]), sl(inp_host["k"]), sl(inp_host["v"]), sl(inp_host["log_alpha"]),
               sl(inp_host["beta"]), inp_host["scale"], return_state=True)
    dt = time.perf_counter() - t
    head_tokens = cfg.T * heads * batch
    # OpenMP runs over (sequence, head) pairs: no more threads than pairs do work
    return dt, head_tokens, min(oracle.threads(), heads * batch)


def host_sample_inputs(cfg, heads, batch=1):
    """The same seeded workload generated on the host, restricted to `batch`
    batch entries and `heads` heads (the generator the GPU run uses, on CPU)."""
    small = W.PrefillConfig(cfg.name, batch, cfg.T, heads, cfg.dk, cfg.dv, cfg.io_dtype, cfg.seed,
                            cfg.gate_shift, cfg.h0_std)
    return W.make_prefill(small, "cpu")


def run_reference(args, ws, rank):
    cfg = W.BATCHED
    if rank != 0:
        return
    heads = 16
    inp = host_sample_inputs(cfg, heads)
    for _ in range(args.warmup):
        oracle_sample(inp, cfg, heads)
    times = []
    threads = 1
    for _ in range(args.steps):
        dt, ht, threads = oracle_sample(inp, cfg, heads)
        times.append(dt)
    total = sum(times)
    value = cfg.T * heads * args.steps / total / cfg.H     # tokens/s at H=32 equivalent
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(cfg),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"batch entry 0, heads 0..{heads - 1}, all {cfg.T} tokens per "
                                   f"step ({cfg.T * heads} head-tokens); tokens/s = head-tokens/s / {cfg.H}"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(cfg):
    d = {"workload": cfg.name, "B": cfg.B, "T": cfg.T, "H": cfg.H, "dk": cfg.dk, "dv": cfg.dv,
         "chunk": CHUNK, "io": cfg.io_dtype, "gates_state": "fp32",
         "l2": f"inputs larger than L2 ({cfg.tokens * cfg.H * (BYTES_PER_HEAD_TOKEN - 256) / 1e9:.2f} "
               f"GB read per step)",
         "parallelism": "independent replica per GPU (weak scaling, no collective)"}
    if cfg.lengths is not None:
        d["sequence_lengths"] = cfg.lengths
    return d


# ----------------------------------------------------------------------------
# the GPU arm
# ----------------------------------------------------------------------------
def time_region(fn, steps, stream):
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1)


def prefill_config(args):
    cfg = {"batched": W.BATCHED, "single": W.SINGLE}.get(args.workload) or W.varlen_config()
    if args.shape:
        B, T, H = (int(x) for x in args.shape.split(","))
        cfg = W.PrefillConfig(f"prefill_B{B}_H{H}_T{T}_d128_bf16", B, T, H, 128, 128, "bf16",
                              seed=cfg.seed, gate_shift=cfg.gate_shift)
    return cfg


def run_prefill(args, ws, rank, kda, peaks):
    cfg = prefill_config(args)
    inp = W.make_prefill(cfg, "cuda")
    out = torch.empty((cfg.B, cfg.T, cfg.H, cfg.dv), dtype=torch.bfloat16, device="cuda")
    hT = torch.empty((cfg.N, cfg.H, cfg.dk, cfg.dv), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["scale"],
                      h0=inp["h0"], cu_seqlens=inp["cu_seqlens"], out=out, hT=hT,
                      impl=args.prefill_impl)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    kda.profiler_read(reset=True)
    kda.profiler_enable(True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        barrier(ws)
        torch.cuda.synchronize()
        ms = time_region(step, args.steps, stream)
        torch.cuda.synchronize()
        barrier(ws)
    kda.profiler_enable(False)
    stats = kda.profiler_read(reset=True)
    ms_max = max_over_ranks(ms, ws)
    tokens = cfg.B * cfg.T * args.steps * ws
    value = tokens / (ms_max / 1e3)
    head_tokens_per_step = cfg.B * cfg.T * cfg.H
    launches = sum(v[0] for v in stats.values())
    # dominant kernel = largest share of event time
    kern = max(stats.items(), key=lambda kv: kv[1][2])
    kname, (kl, ktimed, kms) = kern
    k_ms_per_step = kms / args.steps
    k_ms_per_launch = kms / max(1, ktimed)
    launches_per_step = ktimed / args.steps
    algo_bytes_step = BYTES_PER_HEAD_TOKEN * head_tokens_per_step
    algo_flop_step = FLOP_PER_HEAD_TOKEN * head_tokens_per_step
    path_gbs = algo_bytes_step / (ms_max / args.steps / 1e3) / 1e9
    path_tflops = algo_flop_step / (ms_max / args.steps / 1e3) / 1e12
    roof = prefill_roofline(kname, cfg, k_ms_per_launch, launches_per_step, peaks)
    roof["share_of_step"] = k_ms_per_step / (ms_max / args.steps)
    res = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(cfg),
        "prefill_impl": args.prefill_impl,
        "tc_frac": path_tflops / (peaks["bf16_tflops"]),
        "hbm_frac": path_gbs / peaks["hbm_gbs"],
        "binding_frac": binding_frac(value / ws, cfg, peaks),
        "path": {"algorithmic_GBps": path_gbs, "algorithmic_TFLOPs": path_tflops,
                 "bytes_per_head_token": BYTES_PER_HEAD_TOKEN,
                 "flop_per_head_token": FLOP_PER_HEAD_TOKEN,
                 "peaks": {"hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": peaks["bf16_tflops"],
                           "source": peaks["source"]}},
        "roofline": roof,
        "kernels": {k: {"launches": v[0], "ms": v[2]} for k, v in stats.items() if v[0]},
        "gpu_launches": launches,
        "clocks": clk.summary(),
    }
    return res, inp, step, (out, hT)


def path_bytes_per_head_token(cfg):
    """The path's minimal I/O per (token, head): q, k, v read and out written in the
    I/O dtype, log_alpha fp32, beta fp32 (1540 B at d = 128 with bf16 I/O)."""
    io = 2 if cfg.io_dtype == "bf16" else 4
    return (2 * cfg.dk + 2 * cfg.dv) * io + cfg.dk * 4 + 4


def path_flop_per_head_token(cfg):
    """Chunk-form flops per (token, head): 2C(3dk + 2dv) + 6 dk dv (180,224 at C = 64, d = 128)."""
    return 2 * CHUNK * (3 * cfg.dk + 2 * cfg.dv) + 6 * cfg.dk * cfg.dv


def prefill_roofline(kname, cfg, ms_per_launch, launches_per_step, peaks):
    """HBM roofline of the dominant prefill kernel.  `achieved` counts only the
    path's minimal bytes: 1540 B (at d = 128, bf16) x the head-tokens one launch
    processes, over that launch's event time, so bytes a kernel moves beyond the
    path minimum (an intermediate image, re-reads) earn nothing; `kernel_io_frac`
    is the kernel's own algorithmic I/O over the same time."""
    ht_launch = cfg.tokens * cfg.H / max(1.0, launches_per_step)
    algo = path_bytes_per_head_token(cfg) * ht_launch
    kbytes = kernel_algorithmic_bytes(kname, cfg) / max(1.0, launches_per_step)
    sec = ms_per_launch / 1e3
    roof = {"kernel": kname, "bound": "hbm", "achieved": algo / sec / 1e9,
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": algo / sec / 1e9 / peaks["hbm_gbs"],
            "traffic": measured_traffic(kname, cfg.name),
            "algorithmic_bytes_per_launch": algo,
            "bytes_per_head_token": path_bytes_per_head_token(cfg),
            "head_tokens_per_launch": ht_launch, "launches_per_step": launches_per_step,
            "ms_per_launch": ms_per_launch,
            "kernel_io_bytes_per_launch": kbytes,
            "kernel_io_frac": kbytes / sec / 1e9 / peaks["hbm_gbs"],
            "peak_source": peaks["source"] + " (burst copy)",
            "traffic_source": "profiles/dram_traffic.json (ncu dram__bytes_read.sum + "
                              "dram__bytes_write.sum per launch)"}
    return roof


def binding_frac(tokens_per_s, cfg, peaks):
    """tokens/s over the lower of the tensor-bound and the HBM-bound tokens/s at the
    path's minimal I/O (HBM binds: 117 flop/B against a ridge near 250)."""
    tc_bound = peaks["bf16_tflops"] * 1e12 / (cfg.H * path_flop_per_head_token(cfg))
    hbm_bound = peaks["hbm_gbs"] * 1e9 / (cfg.H * path_bytes_per_head_token(cfg))
    return tokens_per_s / min(tc_bound, hbm_bound)


_TC_SOURCES = ("kda_chunk_tc.cu", "kda_tc_util.cuh", "kda_umma.cuh", "kda_tma.cuh")
_FUSED_SOURCES = ("kda_fused_tc.cu", "kda_tc_util.cuh", "kda_umma.cuh", "kda_tma.cuh")
_SIMT_SOURCES = ("kda_chunk_simt.cu", "kda_chunk_simt.cuh")
KERNEL_SOURCE = {"chunk_fused_tc": _FUSED_SOURCES,
                 "chunk_prep_tc": _TC_SOURCES, "chunk_state_tc": _TC_SOURCES,
                 "chunk_prep_gdn_tc": _TC_SOURCES,
                 "chunk_prep_simt": _SIMT_SOURCES, "chunk_state_simt": _SIMT_SOURCES,
                 "decode_step": ("kda_decode.cu",)}


def kernel_source_sha(kname):
    """SHA-256 prefix of the source files that define kernel `kname` (concatenated)."""
    import hashlib
    files = KERNEL_SOURCE.get(kname)
    if files is None:
        return None
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, "gated_delta_rule_75_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


TRAFFIC_PATH = os.path.join(ROOT, "profiles", "dram_traffic.json")


def measured_traffic(kname, workload, path=TRAFFIC_PATH):
    """DRAM bytes (read + write) per launch of `kname` on `workload` from the
    committed ncu capture table, or None when no entry matches the kernel's current
    source hash (the kernel changed since the capture).  An entry captured on a
    smaller case of the same kernel carries `scale` = the workload's units per
    launch over the capture's, and its bytes are scaled by it."""
    if not os.path.exists(path):
        return None
    sha = kernel_source_sha(kname)
    for e in json.load(open(path))["entries"]:
        if e["kernel"] == kname and e["workload"] == workload and e["source_sha256"] == sha:
            return (e["dram_read_bytes"] + e["dram_write_bytes"]) / e["launches"] * e.get("scale", 1.0)
    return None


def kernel_algorithmic_bytes(kname, cfg):
    """Minimal bytes the named kernel must move for one step of the workload."""
    ht = cfg.B * cfg.T * cfg.H
    if cfg.lengths is not None:
        chunks = sum(math.ceil(L / CHUNK) for L in cfg.lengths) * cfg.H
    else:
        chunks = cfg.B * math.ceil(cfg.T / CHUNK) * cfg.H
    dk, dv = cfg.dk, cfg.dv
    io = 2 if cfg.io_dtype == "bf16" else 4
    qkvgb = ht * ((2 * dk + dv) * io + dk * 4 + 4)
    if kname == "chunk_prep_simt":       # reads q,k,v,g,beta; writes fp32 W,Ut,Aqk,QG,KG,gamma
        return qkvgb + chunks * 4 * (CHUNK * (3 * dk + dv + CHUNK) + dk)
    if kname == "chunk_state_simt":      # reads the fp32 workspace (Ut once, the rest per dv tile)
        tiles = dv // 32
        per_chunk = 4 * (CHUNK * dv + tiles * (CHUNK * 3 * dk + CHUNK * CHUNK + dk))
        return chunks * per_chunk + ht * dv * io + cfg.N * cfg.H * dk * dv * 4
    if kname == "chunk_prep_tc":         # reads q,k,g,beta; writes the operand image
        return ht * (2 * dk * io + dk * 4 + 4) + chunks * TC_WS_BYTES_PER_CHUNK
    if kname == "chunk_state_tc":        # reads the image and v; writes out and hT
        return chunks * TC_WS_BYTES_PER_CHUNK + ht * 2 * dv * io + cfg.N * cfg.H * dk * dv * 4
    if kname == "chunk_fused_tc":        # reads q,k,v,g,beta (and h0); writes out and hT
        states = cfg.N * cfg.H * dk * dv * 4
        return qkvgb + ht * dv * io + states * (2 if cfg.h0_std > 0 else 1)
    if kname == "chunk_state_seg_tc":    # value walk (image, v) + map walk (image), per step;
        # the per-segment (M, B) matrices they write are not counted
        return 2 * chunks * TC_WS_BYTES_PER_CHUNK + ht * dv * io
    return BYTES_PER_HEAD_TOKEN * ht


TC_WS_BYTES_PER_CHUNK = 66560         # per (chunk, head) operand image of the tensor-core path


def decode_bytes_per_head_step(cfg):
    """Bytes one decode step must move per (sequence, head): the fp32 state read and
    written, q and k (bf16), v (bf16), log_alpha (fp32), beta, and the bf16 output."""
    return 2 * cfg.dk * cfg.dv * 4 + 2 * cfg.dk * 2 + cfg.dv * 2 + cfg.dk * 4 + 4 + cfg.dv * 2


def run_decode(args, ws, rank, kda, peaks):
    cfg = W.DECODE
    if args.decode_steps != cfg.steps:
        cfg = W.DecodeConfig(cfg.name, cfg.N, cfg.H, cfg.dk, cfg.dv, args.decode_steps, cfg.seed)
    gen = W.decode_generator(cfg, "cuda")
    S = W.make_decode_state(cfg, gen, "cuda")
    steps_in = [W.make_decode_step(cfg, gen, "cuda") for _ in range(cfg.steps)]
    out = torch.empty((cfg.N, cfg.H, cfg.dv), dtype=torch.bfloat16, device="cuda")
    scale = 1.0 / math.sqrt(cfg.dk)
    stream = torch.cuda.current_stream()

    def run_all():
        for x in steps_in:
            kda.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S, scale, out=out)

    for x in steps_in[:3]:
        kda.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S, scale, out=out)
    torch.cuda.synchronize()
    kda.profiler_read(reset=True)
    kda.profiler_enable(True)
    barrier(ws)
    torch.cuda.synchronize()
    ms = time_region(run_all, 1, stream)
    barrier(ws)
    kda.profiler_enable(False)
    stats = kda.profiler_read(reset=True)
    ms = max_over_ranks(ms, ws)
    bytes_step = decode_bytes_per_head_step(cfg) * cfg.N * cfg.H
    launches, timed, kms = stats["decode_step"]
    gbs = bytes_step / (kms / max(1, timed) / 1e3) / 1e9
    # the same chained loop captured once as a CUDA graph and replayed (no per-step launch cost)
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        run_all()                                  # warm the side stream before capture
    stream.wait_stream(side)
    with torch.cuda.graph(graph):
        run_all()
    graph.replay()
    torch.cuda.synchronize()
    barrier(ws)
    g_ms = max_over_ranks(time_region(graph.replay, 1, stream), ws)
    del graph
    return {
        "workload": cfg.name, "steps_chained": cfg.steps, "ms_per_step": ms / cfg.steps,
        "tokens_per_s": cfg.N * cfg.steps * ws / (ms / 1e3),
        "state_GBps": bytes_step * cfg.steps * ws / (ms / 1e3) / 1e9,
        "cuda_graph": {"ms_per_step": g_ms / cfg.steps,
                       "state_GBps": bytes_step * cfg.steps * ws / (g_ms / 1e3) / 1e9},
        "roofline": {"kernel": "decode_step", "bound": "hbm", "achieved": gbs,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                     "traffic": measured_traffic("decode_step", cfg.name),
                     "algorithmic_bytes_per_launch": bytes_step,
                     "ms_per_launch": kms / max(1, timed)},
        "gpu_launches": launches,
    }


def bwd_kernel_flops(kname, cfg):
    """fp32 flops the named backward kernel evaluates per step (the chunk
    equations it implements, triangles counted once), per SIMT unit count."""
    C, dk, dv = CHUNK, cfg.dk, cfg.dv
    if cfg.lengths is not None:
        chunks = sum(math.ceil(L / C) for L in cfg.lengths) * cfg.H
    else:
        chunks = cfg.B * math.ceil(cfg.T / C) * cfg.H
    tri = C * (C + 1) / 2
    per = {
        "chunk_prep_simt": tri * dk * 4 + C ** 3 / 3 + tri * (dk + dv) * 2,
        "chunk_state_simt": 4 * C * dk * dv + tri * dv * 2,
        "bwd_state": 6 * C * dk * dv + tri * dv * 2,
        "bwd_dense1": 6 * C * dk * dv + 2 * tri * dv * 2,
        "bwd_dense2": 6 * C * dk * dv + 4 * C * C * dv,
        "bwd_param": 2 * C ** 3 + 4 * C * C * dk,   # dA through the inverse; 4 pairwise sums
    }
    return per.get(kname, 0.0) * chunks


def fp32_alu_peak(clocks):
    """fp32 FMA peak: 148 SMs x 128 fp32 lanes x 2 flop x the SM clock."""
    mhz = (clocks or {}).get("sm_max_mhz") or 1965.0
    return 148 * 128 * 2 * mhz * 1e6 / 1e12


def run_backward(args, ws, kda, peaks):
    """The chunkwise backward (kda_chunk_bwd) on the prefill workload: random
    bf16 output gradients and fp32 final-state gradients, all six gradients
    written every step."""
    cfg = prefill_config(args)
    inp = W.make_prefill(cfg, "cuda")
    gen = torch.Generator(device="cuda").manual_seed(cfg.seed + 77)
    dout = torch.randn((cfg.B, cfg.T, cfg.H, cfg.dv), generator=gen, device="cuda").to(torch.bfloat16)
    dhT = torch.randn((cfg.N, cfg.H, cfg.dk, cfg.dv), generator=gen, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        kda.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["scale"],
                      dout, h0=inp["h0"], dhT=dhT, cu_seqlens=inp["cu_seqlens"])

    steps = max(1, min(args.steps, args.bwd_steps))
    for _ in range(min(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    kda.profiler_read(reset=True)
    kda.profiler_enable(True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        barrier(ws)
        torch.cuda.synchronize()
        ms = time_region(step, steps, stream)
        torch.cuda.synchronize()
        barrier(ws)
    kda.profiler_enable(False)
    stats = kda.profiler_read(reset=True)
    ms = max_over_ranks(ms, ws)
    clocks = clk.summary()
    peak = fp32_alu_peak(clocks)
    kern = max(stats.items(), key=lambda kv: kv[1][2])
    kname, (kl, ktimed, kms) = kern
    kflop = bwd_kernel_flops(kname, cfg) / max(1.0, ktimed / steps)
    k_ms = kms / max(1, ktimed)
    total_flop = sum(bwd_kernel_flops(k, cfg) for k in stats)
    res = {
        "workload": cfg.name.replace("prefill", "backward"), "steps": steps,
        "ms_per_step": ms / steps, "tokens_per_s": cfg.B * cfg.T * steps * ws / (ms / 1e3),
        "dtype": "f32 arithmetic, bf16 I/O",
        "path_TFLOPs": total_flop / (ms / steps / 1e3) / 1e12,
        "roofline": {"kernel": kname, "bound": "alu", "achieved": kflop / (k_ms / 1e3) / 1e12,
                     "peak": peak, "unit": "TFLOP/s",
                     "frac": kflop / (k_ms / 1e3) / 1e12 / peak, "traffic": None,
                     "ms_per_launch": k_ms, "share_of_step": kms / steps / (ms / steps),
                     "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 x max SM clock"},
        "kernels": {k: {"launches": v[0], "ms": v[2]} for k, v in stats.items() if v[0]},
        "gpu_launches": sum(v[0] for v in stats.values()),
        "clocks": clocks,
    }
    del inp, dout, dhT
    torch.cuda.empty_cache()
    return res


def run_variants(args, ws, kda, peaks):
    """The serving and Gated DeltaNet entry points on the benchmark shapes:
    GDN prefill (one gate per token and head) on B=8, H=32, T=8192, and the
    decode step on a pool of 512 state slots addressed through a shuffled slot
    array (N=256 sequences, H=32, d=128)."""
    res = {}
    cfg = prefill_config(args)
    inp = W.make_prefill(cfg, "cuda")
    log_a = W.scalar_gates(cfg.B, cfg.T, cfg.H, seed=cfg.seed, gate_shift=cfg.gate_shift, device="cuda")
    out = torch.empty((cfg.B, cfg.T, cfg.H, cfg.dv), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        kda.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], log_a, inp["beta"], inp["scale"], out=out,
                          output_final_state=False)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(ws)
    ms = max_over_ranks(time_region(step, args.steps, stream), ws)
    res["gdn_prefill"] = {"workload": cfg.name.replace("prefill", "gdn_prefill"),
                          "tokens_per_s": cfg.B * cfg.T * args.steps * ws / (ms / 1e3),
                          "ms_per_step": ms / args.steps}
    del inp, out, log_a
    torch.cuda.empty_cache()

    dcfg = W.DECODE
    P = 2 * dcfg.N
    gen = W.decode_generator(dcfg, "cuda")
    pool = torch.randn((P, dcfg.H, dcfg.dk, dcfg.dv), generator=gen, device="cuda") * dcfg.state_std
    slots = torch.randperm(P, generator=gen, device="cuda")[:dcfg.N].to(torch.int32)
    nsteps = 200
    xs = [W.make_decode_step(dcfg, gen, "cuda") for _ in range(nsteps)]
    o = torch.empty((dcfg.N, dcfg.H, dcfg.dv), dtype=torch.bfloat16, device="cuda")
    scale = 1.0 / math.sqrt(dcfg.dk)

    def run_all():
        for x in xs:
            kda.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool, scale,
                               out=o, slots=slots)

    for x in xs[:3]:
        kda.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool, scale, out=o,
                           slots=slots)
    torch.cuda.synchronize()
    barrier(ws)
    ms = max_over_ranks(time_region(run_all, 1, stream), ws)
    per_head = 2 * dcfg.dk * dcfg.dv * 4 + 2 * dcfg.dk * 2 + dcfg.dv * 2 + dcfg.dk * 4 + 4 + dcfg.dv * 2
    res["slot_decode"] = {"workload": f"slot_decode_N{dcfg.N}_pool{P}_H{dcfg.H}_d128_bf16_x{nsteps}",
                          "ms_per_step": ms / nsteps,
                          "state_GBps": per_head * dcfg.N * dcfg.H * nsteps * ws / (ms / 1e3) / 1e9,
                          "hbm_frac": per_head * dcfg.N * dcfg.H * nsteps / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]}
    return res


L2_FLUSH_BYTES = 256 << 20          # twice the 126 MB L2


def run_workload(kda, cfg, reps, warmup, peaks, ws, flush):
    """One prefill workload through kda_chunk_fwd (AUTO): `warmup` untimed calls, then
    `reps` calls each bracketed by its own CUDA events on the launching stream (with
    `flush`, a 256 MB buffer is written before every rep, outside the events, so a
    workload that fits in L2 is read from HBM); the median rep is reported, max over
    ranks.  The library's per-kernel events are off in those reps (they would sit
    between the call's launches); a second set of `reps` calls with them on gives the
    dominant kernel's roofline and every kernel's time per call."""
    inp = W.make_prefill(cfg, "cuda")
    io = torch.bfloat16 if cfg.io_dtype == "bf16" else torch.float32
    out = torch.empty((cfg.B, cfg.T, cfg.H, cfg.dv), dtype=io, device="cuda")
    hT = torch.empty((cfg.N, cfg.H, cfg.dk, cfg.dv), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    fbuf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda") if flush else None

    def step():
        kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["scale"],
                      h0=inp["h0"], cu_seqlens=inp["cu_seqlens"], out=out, hT=hT)

    def timed_reps():
        t = []
        for _ in range(reps):
            if fbuf is not None:
                fbuf.fill_(1.0)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            step()
            e1.record(stream)
            e1.synchronize()
            t.append(e0.elapsed_time(e1))
        return t

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    barrier(ws)
    times = timed_reps()
    barrier(ws)
    kda.profiler_read(reset=True)
    kda.profiler_enable(True)
    profiled = timed_reps()
    kda.profiler_enable(False)
    stats = kda.profiler_read(reset=True)
    ms = max_over_ranks(statistics.median(times), ws)
    kname, (_, ktimed, kms) = max(stats.items(), key=lambda kv: kv[1][2])
    launches_per_step = ktimed / reps
    roof = prefill_roofline(kname, cfg, kms / max(1, ktimed), launches_per_step, peaks)
    roof["share_of_step"] = kms / reps / statistics.median(profiled)
    res = {"workload": cfg.name, "tokens_per_s": cfg.tokens * ws / (ms / 1e3), "ms": ms,
           "ms_profiled": statistics.median(profiled),
           "reps": reps, "statistic": "median", "io": cfg.io_dtype, "dk": cfg.dk, "H": cfg.H,
           "l2": ("256 MB buffer written before every rep (the inputs fit in L2)" if flush
                  else "inputs larger than L2"),
           "binding_frac": binding_frac(cfg.tokens / (ms / 1e3), cfg, peaks),
           "roofline": roof,
           "kernels": {k: {"launches_per_call": v[0] / reps, "ms_per_call": v[2] / reps}
                       for k, v in stats.items() if v[0]},
           "gpu_launches_per_call": sum(v[0] for v in stats.values()) / reps}
    del inp, out, hT, fbuf
    torch.cuda.empty_cache()
    return res


def run_workloads(args, ws, kda, peaks):
    """The other prefill configurations, each through the default entry point: the
    tiny fp32 case (B=1, H=2, T=256, d=64), one head group (B=1, H=16, T=4096), and
    the long-context packed batch (16 sequences, 2^20 tokens, H=32)."""
    res = {}
    for key, cfg, reps, flush in (("tiny", W.TINY, 10, True), ("single", W.SINGLE, 10, True),
                                  ("varlen", W.varlen_config(), 5, False)):
        res[key] = run_workload(kda, cfg, reps, args.warmup, peaks, ws, flush)
    return res


def run_e2e(args, ws, kda, inp, bufs, steps):
    """Same metric through the public API with host (pinned) buffers: every
    step copies its inputs host->device and its output device->host inside the
    timed region.  Steps are pipelined over two buffer sets: the inputs of step
    i+1 cross PCIe while step i computes and step i-1's output comes back (the
    link is full duplex), so a step costs about max(H2D, D2H) once the pipe is
    full."""
    cfg = prefill_config(args)
    names = ("q", "k", "v", "log_alpha", "beta")
    host = {n: inp[n].to("cpu").pin_memory() for n in names}
    dev = [{n: torch.empty_like(inp[n]) for n in names} for _ in range(2)]
    out0, hT = bufs
    outs = [out0, torch.empty_like(out0)]
    out_h = torch.empty(out0.shape, dtype=out0.dtype).pin_memory()
    main = torch.cuda.current_stream()
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()

    def run(nsteps):
        comp_done, out_done = [None] * nsteps, [None] * nsteps
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(main)
        for st in (s_in, s_comp, s_out):
            st.wait_event(start)
        for i in range(nsteps):
            d, o = dev[i % 2], outs[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(comp_done[i - 2])       # buffer set i % 2 is free again
                for n in names:
                    d[n].copy_(host[n], non_blocking=True)
                in_done = ev()
                in_done.record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(in_done)
                if i >= 2:
                    s_comp.wait_event(out_done[i - 2])      # output buffer i % 2 was read back
                kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], inp["scale"],
                              out=o, hT=hT, impl=args.prefill_impl)
                comp_done[i] = ev()
                comp_done[i].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[i])
                out_h.copy_(o, non_blocking=True)
                out_done[i] = ev()
                out_done[i].record(s_out)
        main.wait_event(out_done[-1])
        end.record(main)
        end.synchronize()
        return start.elapsed_time(end)

    run(2)
    torch.cuda.synchronize()
    barrier(ws)
    ms = run(steps)
    barrier(ws)
    ms = max_over_ranks(ms, ws)
    h2d = sum(host[n].numel() * host[n].element_size() for n in names)
    d2h = out_h.numel() * out_h.element_size()
    del dev, outs
    return {"value": cfg.B * cfg.T * steps * ws / (ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "pipelined": "2 buffer sets; H2D, compute and D2H on separate streams"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["kda", "reference"], default="kda")
    ap.add_argument("--prefill-impl", choices=["auto", "simt", "tensorcore", "tensorcore_chain",
                                               "tensorcore_segmented"], default="auto")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--bwd-steps", type=int, default=3,
                    help="timed steps of the backward leg (at most --steps)")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the tiny, single-head-group and varlen prefill workloads")
    ap.add_argument("--only", choices=["all", "prefill", "decode", "backward"], default="all",
                    help="restrict the run (profiling of one kernel family)")
    ap.add_argument("--decode-steps", type=int, default=W.DECODE.steps)
    ap.add_argument("--workload", choices=["batched", "single", "varlen"], default="batched",
                    help="prefill workload: batched B=8,H=32,T=8192 (the benchmark), single "
                         "B=1,H=16,T=4096, or varlen (16 packed sequences, 2^20 tokens, H=32)")
    ap.add_argument("--shape", default="", help="B,T,H override of the prefill workload "
                    "(profiling of a smaller case; the default is the benchmark workload)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    ws, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, ws, rank)
            return
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA device for the kda arm")
        from gated_delta_rule_75_b200 import build
        if rank == 0:
            build.build()
        barrier(ws)
        import gated_delta_rule_75_b200 as kda
        peaks = load_peaks()
        if args.only == "decode":
            res = {"decode": run_decode(args, ws, rank, kda, peaks)}
            if rank == 0:
                print(json.dumps(res), flush=True)
            return
        if args.only == "backward":
            res = {"backward": run_backward(args, ws, kda, peaks)}
            if rank == 0:
                print(json.dumps(res), flush=True)
            return
        res, inp, step, bufs = run_prefill(args, ws, rank, kda, peaks)
        if not args.no_e2e and args.only == "all":
            res["e2e"] = run_e2e(args, ws, kda, inp, bufs, steps=min(args.steps, 6))
        del inp, bufs
        torch.cuda.empty_cache()
        if not args.no_decode and args.only == "all":
            res["decode"] = run_decode(args, ws, rank, kda, peaks)
            torch.cuda.empty_cache()
            res["variants"] = run_variants(args, ws, kda, peaks)
        if not args.no_backward and args.only == "all":
            torch.cuda.empty_cache()
            res["backward"] = run_backward(args, ws, kda, peaks)
        if not args.no_workloads and args.only == "all":
            torch.cuda.empty_cache()
            res["workloads"] = run_workloads(args, ws, kda, peaks)
        if rank == 0 and not args.no_cpu and args.only == "all":
            cfg = W.BATCHED
            heads, batch = cfg.H, 2
            hinp = host_sample_inputs(cfg, heads, batch)
            dt, ht, thr = oracle_sample(hinp, cfg, heads, batch)
            res["cpu_baseline"] = {"value": ht / dt / cfg.H, "unit": "tokens/s", "cores": thr,
                                   "kind": "oracle",
                                   "sample": f"{batch} of the {cfg.B} sequences, all {heads} heads, "
                                             f"all {cfg.T} tokens ({ht} head-tokens, {dt:.1f} s "
                                             f"wall); tokens/s = head-tokens/s / {cfg.H}"}
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
