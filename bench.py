"""Benchmark of the quantized MoE FFN hot path on B200.

Default workload: 48-layer decode, one token per step (d=2560, 512 experts,
top-10 + 1 shared, SwiGLU intermediate 512, Q4B32 weights, seeded synthetic
inputs).  A step = one token through all 48 layers (router, top-k, dispatch,
expert SwiGLU, down projection, combine, residual + rmsnorm), weights and
inputs resident in HBM.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 (under torchrun): independent replicas, one per GPU, each decoding its
own tokens (the layer does not shard for one token stream); value = tokens
of all ranks / max-over-ranks time.

  python bench.py --sweep [--sweep-workload W] [--sweep-t 1,2,...]

times one layer at each token count on every path that accepts it (single-token
kernel, CUDA-core path, tensor-core path) and ends with the fastest path per
token count next to the one the library's dispatch picks.
"""
from __future__ import annotations

import argparse
import json
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

import synth  # noqa: E402

METRIC = "48-layer MoE decode tok/s & prefill tok/s; % of HBM / MMA roofline"
DEFAULT_WORKLOAD = "decode_48l_q4_t1"


def peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def expert_bytes(cfg) -> int:
    """Packed bytes of one expert (gate + up + down, codes + fp16 scales)."""
    per_block = cfg.block_bytes + 2
    return 3 * cfg.d * cfg.I // 32 * per_block


def router_bytes(cfg) -> int:
    return cfg.E * cfg.d * 4


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch, from one ncu capture of
# the current kernels on one B200:
#   ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum \
#       --clock-control none -k regex:k_decode -s 3 -c 1 \
#       python bench.py --steps 3 --warmup 3 --no-secondary --cpu-layers 1 --layers 4
# (a 4-layer stack: 118,442,240 B read + 2,858,752 B written; traffic grows with the layers a launch
# runs, so a 48-layer launch is scaled by 48/4), and
#   ncu ... -k regex:"k_tc_gemm|k_cache_fill" -s 12 -c 4 python bench.py \
#       --workload prefill_1l_q4_t4096_zipf --steps 2 --warmup 3 --no-secondary --cpu-layers 1
# (the cache fill and the two expert GEMMs of one layer; router excluded).
DECODE_Q4_TRAFFIC_PER_LAYER = (118_442_240 + 2_858_752) / 4
PREFILL_Q4_T4096_TRAFFIC = (61_968_640 + 157_297_920          # k_cache_fill
                            + 500_800_256 + 41_342_720        # k_tc_gemm<gate/up>
                            + 341_344_768 + 61_933_312)       # k_tc_gemm<down>


def max_over_ranks(v: float, dist_on: bool, device) -> float:
    """The largest of every rank's value (a time): the job takes as long as its slowest rank."""
    t = torch.tensor([v], dtype=torch.float64, device=device)
    if dist_on:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, seconds: float) -> float:
    """Units processed by all ranks together per second (weak scaling: fixed units per rank)."""
    return units_per_rank * world / seconds


def decode_traffic(cfg, kernel: str):
    """Measured DRAM bytes per launch of the single-token kernel for the Q4 decode shape."""
    if kernel != "k_decode" or cfg.fmt != "q4" or cfg.T != 1 or (cfg.d, cfg.E, cfg.I, cfg.k) != (2560, 512, 512, 10):
        return None
    return DECODE_Q4_TRAFFIC_PER_LAYER * cfg.L


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class Clocks:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.f = None

    def __enter__(self):
        try:
            self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.f.flush()
        rows = []
        for line in open(self.f.name):
            p = [v.strip() for v in line.split(",")]
            if len(p) >= 9:
                try:
                    rows.append((float(p[1]), float(p[2]), p[5:9]))
                except ValueError:
                    pass
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# CPU oracle timing (the baseline, and the --impl reference arm)
# ---------------------------------------------------------------------------
def oracle_decode_sample(cfg, n_layers: int, token_stream: int, n_tokens: int = 1) -> float:
    """Seconds the oracle (one host core) takes to push `n_tokens` tokens through
    `n_layers` layers; expert generation on the host is excluded from the timing."""
    import oracle
    from tests.parity import ExpertSource
    total = 0.0
    for tk in range(n_tokens):
        x = synth.tokens_bf16(cfg, 1, stream=token_stream + 7919 * tk)[0]
        for l in range(n_layers):
            src = ExpertSource(cfg, l)
            xf = oracle.bf16_to_f64(x)
            ids, _, _ = oracle.route(oracle.router_logits(xf, src.router_w, src.router_b), cfg.k)
            for e in ids:
                src.expert(int(e))          # generate outside the timed region
            src.shared(0)
            t0 = time.perf_counter()
            y, _, _, _ = oracle.moe_token(cfg.fmt, cfg.k, x, src.router_w, src.router_b, src.expert,
                                          src.shared, cfg.n_shared)
            r = oracle.rmsnorm(xf + y)
            total += time.perf_counter() - t0
            x = oracle.round_bf16(r)
    return total


def run_reference(args, cfg) -> dict:
    layers = args.ref_layers
    times = []
    for s in range(args.warmup + args.steps):
        dt = oracle_decode_sample(cfg, layers, token_stream=1000 + s)
        if s >= args.warmup:
            times.append(dt)
    per_token = statistics.mean(times) * cfg.L / layers
    value = 1.0 / per_token
    sample = f"1 token through {layers} of {cfg.L} layers per step, time scaled x{cfg.L / layers:g}"
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_token * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "config": {"workload": cfg.name},
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def timed_stack(sess, cfg, xs, r_out, steps, warmup, stream, dist_on):
    from quantized_expert_ffn_token_b200 import capi
    T = cfg.T
    for s in range(warmup):
        capi.moe_forward_stack(sess.ctx, 0, cfg.L, xs[s % len(xs)], T, r_out, None, stream)
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    capi.moe_timing_read(sess.ctx)                     # reset counters
    capi.moe_timing_enable(sess.ctx, True)
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for s in range(steps):
        capi.moe_forward_stack(sess.ctx, 0, cfg.L, xs[(warmup + s) % len(xs)], T, r_out, None, stream)
    stop.record(stream)
    torch.cuda.synchronize()
    tim = capi.moe_timing_read(sess.ctx)
    capi.moe_timing_enable(sess.ctx, False)
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    return start.elapsed_time(stop), tim


def run_ours(args, cfg, rank, world, local_rank, dist_on) -> dict | None:
    from quantized_expert_ffn_token_b200 import capi, session
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(dev)
    P = peaks()
    sess = session.Session(cfg, device=local_rank, max_tokens=cfg.T)
    with torch.cuda.stream(stream):
        sess.load_synthetic(stream=stream)
    torch.cuda.synchronize()
    n_tok = args.warmup + args.steps
    xs = [torch.from_numpy(synth.tokens_bf16(cfg, cfg.T, stream=rank * 100003 + s).view(np.int16)).to(dev)
          for s in range(n_tok)]
    r_out = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device=dev)

    with Clocks(local_rank) as clk:
        ms, tim = timed_stack(sess, cfg, xs, r_out, args.steps, args.warmup, stream, dist_on)
    clocks = clk.summary()
    ms_max = max_over_ranks(ms, dist_on, dev)
    ms_step = ms_max / args.steps
    value = whole_job_rate(cfg.T, world, ms_step / 1e3)

    # roofline of the dominant (timed) kernel: the bytes it must stream per launch.  The
    # single-token kernel runs one token through the whole stack per launch: k routed + the
    # shared experts and the router rows of every layer; the grouped paths launch once per
    # layer and stream the union of the batch's experts
    union = cfg.k if cfg.T == 1 else measured_union(sess, cfg, xs[0], dev)
    if tim["kernel"] == "k_decode":
        alg_bytes = cfg.L * ((cfg.k + cfg.n_shared) * expert_bytes(cfg) + router_bytes(cfg))
    else:
        alg_bytes = (union + cfg.n_shared) * expert_bytes(cfg)   # experts only
    # the step's algorithmic bytes: every layer's router rows and the union of the experts the
    # batch's tokens chose (a path that streams some of them more than once moves more)
    step_bytes = cfg.L * ((union + cfg.n_shared) * expert_bytes(cfg) + router_bytes(cfg))
    avg_ms = tim["ms"] / max(1, tim["timed_launches"])
    achieved = alg_bytes / (avg_ms / 1e3) / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": P["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / P["hbm_gbs"], "traffic": decode_traffic(cfg, tim["kernel"]), "kernel": tim["kernel"],
            "alg_bytes_per_launch": alg_bytes, "avg_launch_ms": avg_ms,
            "peak_source": P["source"] + " (hbm_gbs, STREAM-style copy)"}

    # end to end through the public host-buffer entry point
    x_host = [torch.from_numpy(synth.tokens_bf16(cfg, cfg.T, stream=rank * 100003 + s).view(np.int16)).pin_memory()
              for s in range(n_tok)]
    r_host = torch.empty((cfg.T, cfg.d), dtype=torch.float32).pin_memory()
    for s in range(args.warmup):
        capi.moe_forward_stack_host(sess.ctx, 0, cfg.L, x_host[s], cfg.T, r_host, stream)
    if dist_on:
        torch.distributed.barrier()
    t0 = time.perf_counter()
    for s in range(args.steps):
        capi.moe_forward_stack_host(sess.ctx, 0, cfg.L, x_host[args.warmup + s], cfg.T, r_host, stream)
    e2e_s = max_over_ranks(time.perf_counter() - t0, dist_on, dev)
    e2e = {"value": whole_job_rate(cfg.T * args.steps, world, e2e_s), "unit": "tok/s",
           "h2d_bytes_per_step": cfg.T * cfg.d * 2, "d2h_bytes_per_step": cfg.T * cfg.d * 4,
           "timer": "host wall clock around synchronous calls"}
    sess.close()
    del xs
    torch.cuda.empty_cache()

    out = {
        "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp32-accumulate over Q4B32/bf16" if cfg.fmt == "q4" else "fp32-accumulate over Q3B32/bf16",
        "data": "synthetic (seeded counter-hash weights, N(0,1) bf16 tokens)",
        "config": {"workload": f"{cfg.name}: d={cfg.d} E={cfg.E} top-{cfg.k}+{cfg.n_shared} shared "
                               f"I={cfg.I} {cfg.fmt.upper()}B32 T={cfg.T} layers={cfg.L}",
                   "global_batch": cfg.T * world, "parallelism": f"replicas x{world}",
                   "l2": f"no flush: each step streams {step_bytes / 1e9:.2f} GB of weights (> 126 MB L2) "
                         "and routes a new token"},
        "roofline": roof,
        "step_roofline": {"alg_bytes_per_step": step_bytes,
                          "achieved_gbs": step_bytes / (ms_step / 1e3) / 1e9,
                          "frac": step_bytes / (ms_step / 1e3) / 1e9 / P["hbm_gbs"]},
        "e2e": e2e,
        "gpu_launches": tim["all_launches"],
        "clocks": clocks,
    }
    return out


def measured_union(sess, cfg, x, dev) -> int:
    """Mean number of distinct routed experts per layer for one step (T > 1)."""
    from quantized_expert_ffn_token_b200 import capi
    L, T, k = cfg.L, cfg.T, cfg.k
    idr = torch.empty((L, T, k), dtype=torch.int32, device=dev)
    rec = capi.make_record(ids=idr)
    r = torch.empty((T, cfg.d), dtype=torch.float32, device=dev)
    capi.moe_forward_stack(sess.ctx, 0, L, x, T, r, rec)
    torch.cuda.synchronize()
    ids = idr.cpu().numpy()
    return int(round(np.mean([len(np.unique(ids[l])) for l in range(L)])))


def secondary_prefill(args, local_rank) -> dict:
    """Single-layer prefill (4096 tokens, Zipf-biased routing): tok/s and the
    expert kernels' throughput against the dense tensor peak."""
    from quantized_expert_ffn_token_b200 import capi, session
    cfg = synth.CONFIGS["prefill_1l_q4_t4096_zipf"]
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(dev)
    sess = session.Session(cfg, device=local_rank, max_tokens=cfg.T)
    sess.load_synthetic(stream=stream)
    x = torch.from_numpy(synth.tokens_bf16(cfg).view(np.int16)).to(dev)
    y = torch.empty((cfg.T, cfg.d), dtype=torch.int16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(2):
        capi.moe_forward(sess.ctx, 0, x, cfg.T, y, None, None, None, stream)
    torch.cuda.synchronize()
    times = []
    capi.moe_timing_read(sess.ctx)
    capi.moe_timing_enable(sess.ctx, True)
    for _ in range(3):
        with torch.cuda.stream(stream):
            flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        capi.moe_forward(sess.ctx, 0, x, cfg.T, y, None, None, None, stream)
        b.record(stream)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    tim = capi.moe_timing_read(sess.ctx)
    sess.close()
    ms = statistics.median(times)
    flops_expert = 2 * cfg.T * (cfg.k + cfg.n_shared) * 3 * cfg.d * cfg.I
    flops = flops_expert + 2 * cfg.T * cfg.E * cfg.d
    P = peaks()
    kms = tim["ms"] / max(1, tim["timed_launches"])
    return {"workload": cfg.name, "tok_per_s": cfg.T / (ms / 1e3), "ms_per_layer": ms,
            "tflops": flops / (ms / 1e3) / 1e12,
            "roofline": {"bound": "tensor", "kernel": tim["kernel"],
                         "achieved": flops_expert / (kms / 1e3) / 1e12,
                         "peak": P["bf16_tflops_sustained"], "unit": "TFLOP/s",
                         "frac": flops_expert / (kms / 1e3) / 1e12 / P["bf16_tflops_sustained"],
                         "traffic": PREFILL_Q4_T4096_TRAFFIC if cfg.name == "prefill_1l_q4_t4096_zipf" else None,
                         "traffic_kernels": "k_cache_fill + k_tc_gemm<gate/up> + k_tc_gemm<down>"},
            "l2": "256 MB flush between timed calls"}


# ---- token-count sweep (python bench.py --sweep): one layer, every path that accepts T ------------

# The library's path selection by T (include/moe.h, moe_forward): the single-token kernel once per
# token up to DISPATCH_DECODE_MAX tokens, the tensor-core path from DISPATCH_TC_MIN tokens, the
# CUDA-core path in between.  The flags below pin a context to one path.
DISPATCH_DECODE_MAX = 8
DISPATCH_TC_MIN = 9
SWEEP_T = (1, 2, 4, 6, 8, 9, 10, 12, 16, 24, 32, 48, 64, 96, 128, 256, 512, 1024, 2048, 4096, 8192)
SWEEP_PATHS = ("single-token kernel", "cuda-core", "tensor-core")


def sweep_flags(path: str) -> int:
    no_decode, no_tensor = 1, 2   # MOE_FLAG_NO_DECODE_KERNEL, MOE_FLAG_NO_TENSOR_PREFILL
    return {"single-token kernel": 0, "cuda-core": no_decode | no_tensor, "tensor-core": no_decode}[path]


def sweep_eligible(path: str, T: int) -> bool:
    """Whether a context pinned to `path` runs T tokens on that path."""
    if path == "single-token kernel":
        return T <= DISPATCH_DECODE_MAX
    if path == "tensor-core":
        return T >= DISPATCH_TC_MIN
    return True


def default_path(T: int) -> str:
    if T <= DISPATCH_DECODE_MAX:
        return "single-token kernel"
    return "tensor-core" if T >= DISPATCH_TC_MIN else "cuda-core"


def sweep_summary(rows: list[dict]) -> list[dict]:
    """Per T: the fastest measured path and whether the default dispatch picks it."""
    out = []
    for T in sorted({r["T"] for r in rows}):
        at = [r for r in rows if r["T"] == T]
        best = min(at, key=lambda r: r["ms"])
        dflt = next((r for r in at if r["path"] == default_path(T)), None)
        out.append({"T": T, "fastest": best["path"], "fastest_ms": best["ms"],
                    "default": default_path(T), "default_ms": dflt["ms"] if dflt else None,
                    "default_is_fastest": dflt is not None and dflt["path"] == best["path"]})
    return out


def sweep(args, local_rank) -> list[dict]:
    """Time one layer of `args.sweep_workload` at every T of the sweep on every path that accepts
    it: a 256 MB L2 flush before each timed call, CUDA events on the call's stream, median of
    args.steps calls after args.warmup untimed ones.  Prints one JSON line per (T, path)."""
    from quantized_expert_ffn_token_b200 import capi, session
    cfg = synth.CONFIGS[args.sweep_workload]
    Ts = [int(t) for t in args.sweep_t.split(",")] if args.sweep_t else list(SWEEP_T)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    x_all = torch.from_numpy(synth.tokens_bf16(cfg, T=max(Ts)).view(np.int16)).to(dev)
    rows = []
    for path in SWEEP_PATHS:
        ts = [T for T in Ts if sweep_eligible(path, T)]
        if not ts:
            continue
        sess = session.Session(cfg, device=local_rank, max_tokens=max(ts), n_layers=1, flags=sweep_flags(path))
        sess.load_synthetic(stream=stream)
        torch.cuda.synchronize()
        for T in ts:
            x = x_all[:T]
            y = torch.empty((T, cfg.d), dtype=torch.int16, device=dev)
            ids = torch.empty((T, cfg.k), dtype=torch.int32, device=dev)
            for _ in range(args.warmup):
                capi.moe_forward(sess.ctx, 0, x, T, y, None, ids, None, stream)
            torch.cuda.synchronize()
            times = []
            for _ in range(args.steps):
                with torch.cuda.stream(stream):
                    flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                capi.moe_forward(sess.ctx, 0, x, T, y, None, ids, None, stream)
                b.record(stream)
                torch.cuda.synchronize()
                times.append(a.elapsed_time(b))
            ms = statistics.median(times)
            union = int(torch.unique(ids).numel())
            nbytes = (union + cfg.n_shared) * expert_bytes(cfg) + router_bytes(cfg)
            flops = 2 * T * (cfg.k + cfg.n_shared) * 3 * cfg.d * cfg.I + 2 * T * cfg.E * cfg.d
            row = {"sweep": cfg.name, "T": T, "path": path, "ms": ms, "tok_per_s": T / (ms / 1e3),
                   "experts_touched": union + cfg.n_shared,
                   "alg_gbs": nbytes / (ms / 1e3) / 1e9, "tflops": flops / (ms / 1e3) / 1e12}
            print(json.dumps(row), flush=True)
            rows.append(row)
        sess.close()
        torch.cuda.synchronize()
    return rows


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.CONFIGS))
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--cpu-layers", type=int, default=12, help="oracle sample: layers per token")
    ap.add_argument("--ref-layers", type=int, default=2, help="reference arm: layers per step")
    ap.add_argument("--layers", type=int, default=None,
                    help="stack depth override (small cases for profiler captures)")
    ap.add_argument("--sweep", action="store_true",
                    help="token-count sweep of one layer over every path (one JSON line per T and path)")
    ap.add_argument("--sweep-workload", default="prefill_1l_q4_t4096_zipf", choices=sorted(synth.CONFIGS),
                    help="layer shape and routing of the sweep (layer 0 of this workload)")
    ap.add_argument("--sweep-t", default=None, help="comma-separated token counts (default: 1 ... 8192)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    cfg = synth.CONFIGS[args.workload]
    if args.layers is not None:
        import dataclasses
        cfg = dataclasses.replace(cfg, L=args.layers)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    dist_on = world > 1

    if args.sweep:
        if rank != 0:
            return 0
        rows = sweep(args, local_rank)
        print(json.dumps({"sweep_summary": sweep_summary(rows), "l2": "256 MB flush between timed calls",
                          "steps": args.steps, "warmup": args.warmup}))
        return 0

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, cfg)))
        return 0

    if dist_on:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                             device_id=torch.device("cuda", local_rank))
    out = run_ours(args, cfg, rank, world, local_rank, dist_on)
    if rank == 0:
        if not args.no_secondary and world == 1:
            out["secondary"] = {"prefill": secondary_prefill(args, local_rank)}
        if world == 1:
            nt = min(cfg.T, 4)
            layers = min(args.cpu_layers, cfg.L)
            sec = oracle_decode_sample(cfg, layers, token_stream=7, n_tokens=nt)
            v = nt / (sec * cfg.L / layers)
            out["cpu_baseline"] = {"value": v, "unit": "tok/s", "cores": 1, "kind": "oracle",
                                   "sample": f"{nt} token(s) through {layers} of {cfg.L} layers, "
                                             f"time scaled x{cfg.L / layers:g}; the oracle's cost is "
                                             "per token, so tokens/s does not depend on the batch"}
        print(json.dumps(out))
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
