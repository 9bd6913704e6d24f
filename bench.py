"""Benchmark of the quantized MoE FFN hot path on B200.

A step is one pass of the whole path over one batch of seeded synthetic input,
weights and inputs resident in HBM: router, top-k, dispatch, expert SwiGLU,
down projection, shared expert, combine and, in the 48-layer stacks, residual
add and rmsnorm between layers.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

The headline is 48-layer single-token decode (d=2560, 512 experts, top-10 + 1
shared, intermediate 512, Q4B32): one token through all 48 layers per step.
The same line carries, under "secondary", the other measured workloads, each
with its own roofline, CPU baseline and end-to-end figure: 48-layer verify
(4 tokens, Q3B32, Zipf-biased routing), single-layer prefill (4096 tokens,
Q4B32, Zipf-biased) and 48-layer long prefill (32768 tokens, Q3B32).

N > 1 (under torchrun): independent replicas of the headline, one per GPU,
each decoding its own tokens (one token stream does not shard); value = tokens
of all ranks / max-over-ranks time.

  python bench.py --sweep [--sweep-workload W] [--sweep-t 1,2,...]

times one layer at each token count on every path that accepts it and ends
with the fastest path per token count next to the one the dispatch picks.
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "48-layer MoE decode tok/s & prefill tok/s; % of HBM / MMA roofline"
DEFAULT_WORKLOAD = "decode_48l_q4_t1"
SECONDARY = ("verify_48l_q3_t4_zipf", "prefill_1l_q4_t4096_zipf", "prefill_48l_q3_t32768")
FLUSH_BYTES = 256 << 20   # L2 flush between timed steps of workloads whose step streams less than ~1 GB


L2_MODES = {"stream": 0, "keep": 1}   # MOE_L2_STREAM, MOE_L2_KEEP_SHARED


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


def expert_flops(cfg, T: int) -> int:
    """Multiply-adds x 2 of the experts of one layer on T tokens (k routed + shared per token)."""
    return 2 * T * (cfg.k + cfg.n_shared) * 3 * cfg.d * cfg.I


def router_flops(cfg, T: int) -> int:
    return 2 * T * cfg.E * cfg.d


# DRAM traffic (ncu dram__bytes_read.sum + dram__bytes_write.sum) of the dominant kernels, per layer,
# each with the SHA-256 of the kernel sources it was measured on (their code: comments and blank lines
# are left out of the hash, so that a documentation edit does not void a measurement): a figure is
# reported only while that code is unchanged (a changed kernel reports null until it is measured
# again).  The decode
# figures come from 4-layer captures (the 48-layer launch is reported as 48 x the per-layer mean:
# the traffic grows with the layers, each streaming its own union of experts); the commands that
# produced them are in the profiles/ summaries named beside each entry.
MEASURED_TRAFFIC = [
    {"kernel": "k_decode", "workload": "decode_48l_q4_t1", "src": ['decode.cu', 'decode_common.cuh', 'moe_internal.cuh'],
     "sha256": "a2d18ae6d699d604e7ad84838a17d28788706e6860a2c0391a24a9ac304f0a62", "bytes_per_layer": 30_823_552,
     "profile": "profiles/k_decode_decode_48l_q4_t1.md"},
    {"kernel": "k_decode_multi", "workload": "verify_48l_q3_t4_zipf", "src": ['decode_multi.cu', 'decode_common.cuh', 'moe_internal.cuh'],
     "sha256": "d4ad631ed59af87bb945793e0acc84987a5dd194c9dff1a3f562204901de8e06", "bytes_per_layer": 42_253_376,
     "profile": "profiles/k_decode_multi_verify_48l_q3_t4_zipf.md"},
    {"kernel": "k_cache_fill+k_tc_gemm<gate/up>+k_tc_gemm<down>+k_small_expert", "workload": "prefill_1l_q4_t4096_zipf",
     "src": ['prefill_tc.cu', 'moe_internal.cuh'], "sha256": "63b61a15554d6c56edb185a70e7e87ad6f2c547418375d632bde9c5b0c49a7ee", "bytes_per_layer": 897_861_120,
     "profile": "profiles/k_tc_gemm_prefill_1l_q4_t4096_zipf.md"},
]


def _code_only(text: str) -> str:
    """C/CUDA source without its comments, trailing blanks and empty lines."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*$", "", ln).rstrip() for ln in text.split("\n"))
    return "\n".join(ln for ln in lines if ln)


def _src_sha(rels) -> str:
    h = hashlib.sha256()
    for rel in ([rels] if isinstance(rels, str) else rels):
        with open(os.path.join(ROOT, "quantized_expert_ffn_token_b200", "csrc", rel), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()


def measured_traffic(kernel: str, workload: str, layers: int):
    """DRAM bytes per launch of `kernel` on `workload` from a capture of the current source, else None."""
    for m in MEASURED_TRAFFIC:
        if m["kernel"] == kernel and m["workload"] == workload and _src_sha(m["src"]) == m["sha256"]:
            return m["bytes_per_layer"] * layers
    return None


def max_over_ranks(v: float, dist_on: bool, device) -> float:
    """The largest of every rank's value (a time): the job takes as long as its slowest rank."""
    t = torch.tensor([v], dtype=torch.float64, device=device)
    if dist_on:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, seconds: float) -> float:
    """Units processed by all ranks together per second (weak scaling: fixed units per rank)."""
    return units_per_rank * world / seconds


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


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
# CPU oracle timing (each entry's cpu_baseline, and the --impl reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(cfg, n_tokens: int, threads: int, token_stream: int) -> dict:
    """Time the oracle (plain C, fp64) on `n_tokens` independent tokens through one layer (layer 0),
    `threads` tokens at a time on the host cores (its C calls release the GIL).  The experts the
    tokens need are generated before the timed region.  The oracle's cost is the same for every
    token and layer of a workload, so the rate of the whole workload follows by scaling."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    from tests.parity import ExpertSource

    src = ExpertSource(cfg, 0)
    x = synth.tokens_bf16(cfg, n_tokens, stream=token_stream)
    xf = oracle.bf16_to_f64(x)
    need = set()
    for t in range(n_tokens):
        ids, _, _ = oracle.route(oracle.router_logits(xf[t], src.router_w, src.router_b), cfg.k)
        need.update(int(e) for e in ids)
    cache = {e: src.expert(e) for e in sorted(need)}       # generated outside the timed region
    shared = {s: src.shared(s) for s in range(cfg.n_shared)}

    def one(t):
        oracle.moe_token(cfg.fmt, cfg.k, x[t], src.router_w, src.router_b, cache.__getitem__,
                         shared.__getitem__, cfg.n_shared)

    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(one, range(min(threads, n_tokens))))    # warm the threads and the code
        t0 = time.perf_counter()
        list(ex.map(one, range(n_tokens)))
        dt = time.perf_counter() - t0
    return {"seconds": dt, "token_layers": n_tokens, "threads": threads}


def cpu_baseline(cfg, budget_s: float = 12.0) -> dict:
    """The oracle's rate on this workload (tok/s over all of its layers), on all host cores, from
    a bounded sample of about `budget_s` seconds."""
    cores = host_cores()
    threads = max(1, min(cores, 64))
    probe = oracle_sample(cfg, threads, threads, token_stream=7)
    per_tl = probe["seconds"] / probe["token_layers"]          # seconds per token-layer, all threads busy
    n = max(threads, min(4096, int(budget_s / max(per_tl, 1e-6)) // threads * threads))
    s = oracle_sample(cfg, n, threads, token_stream=11)
    rate_tl = s["token_layers"] / s["seconds"]
    return {"value": rate_tl / cfg.L, "unit": "tok/s", "cores": threads, "host_cores": cores,
            "kind": "oracle",
            "sample": f"{n} tokens through one layer of {cfg.name} ({threads} at a time, one per host "
                      f"thread), {s['seconds']:.1f} s; tok/s over the workload's {cfg.L} layer(s) = "
                      f"token-layers per second / {cfg.L} (the oracle's cost is the same for every "
                      "token and layer)"}


def run_reference(args, cfg) -> dict:
    """The reference arm: the oracle as it stands, on the host cores; each step is a bounded sample
    (one token per host thread through one layer), timed as a whole."""
    cores = host_cores()
    threads = max(1, min(cores, 64))
    times = []
    for s in range(args.warmup + args.steps):
        r = oracle_sample(cfg, threads, threads, token_stream=1000 + 97 * s)
        if s >= args.warmup:
            times.append(r["seconds"])
    step_s = statistics.mean(times)
    value = threads / (step_s * cfg.L)
    sample = (f"each step: {threads} tokens through one layer of {cfg.name}, one per host thread; "
              f"tok/s = tokens / (step time x {cfg.L} layers)")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "config": {"workload": cfg.name},
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": threads, "host_cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def _step(capi, sess, cfg, x, out, stream):
    if cfg.L > 1:
        capi.moe_forward_stack(sess.ctx, 0, cfg.L, x, cfg.T, out, None, stream)
    else:
        capi.moe_forward(sess.ctx, 0, x, cfg.T, out, None, None, None, stream)


def timed_steps(capi, sess, cfg, xs, out, steps, warmup, stream, dist_on, flush=None):
    """W untimed steps, then K timed ones between a barrier and a device sync on both sides; CUDA
    events on the launching stream around each step (an L2 flush, when given, runs before each
    step outside its events).  Returns (ms of the K steps, the library's timing record)."""
    for s in range(warmup):
        _step(capi, sess, cfg, xs[s % len(xs)], out, stream)
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    capi.moe_timing_read(sess.ctx)                     # reset counters
    capi.moe_timing_enable(sess.ctx, True)
    evs = []
    for s in range(steps):
        if flush is not None:
            with torch.cuda.stream(stream):
                flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        _step(capi, sess, cfg, xs[(warmup + s) % len(xs)], out, stream)
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    tim = capi.moe_timing_read(sess.ctx)
    capi.moe_timing_enable(sess.ctx, False)
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs), tim


def layer_unions(capi, sess, cfg, x, dev) -> list[int]:
    """Distinct routed experts per layer of one step (the bytes a pass must stream)."""
    L, T, k = cfg.L, cfg.T, cfg.k
    if T == 1:
        return [k] * L
    idr = torch.empty((L, T, k), dtype=torch.int32, device=dev)
    if L > 1:
        r = torch.empty((T, cfg.d), dtype=torch.float32, device=dev)
        capi.moe_forward_stack(sess.ctx, 0, L, x, T, r, capi.make_record(ids=idr))
    else:
        y = torch.empty((T, cfg.d), dtype=torch.int16, device=dev)
        capi.moe_forward(sess.ctx, 0, x, T, y, None, idr[0], None)
    torch.cuda.synchronize()
    ids = idr.cpu().numpy()
    return [len(np.unique(ids[l])) for l in range(L)]


def measure(args, cfg, rank, world, local_rank, dist_on, with_cpu: bool) -> dict:
    """One workload: value (tok/s, device-timed), roofline of the dominant kernel, end-to-end rate
    through the host-buffer entry point, clocks, launches, and (rank 0) the oracle's rate."""
    from quantized_expert_ffn_token_b200 import capi, session
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(dev)
    P = peaks()
    sess = session.Session(cfg, device=local_rank, max_tokens=cfg.T)
    capi.moe_set_l2_policy(sess.ctx, L2_MODES[args.l2_policy])
    with torch.cuda.stream(stream):
        sess.load_synthetic(stream=stream)
    torch.cuda.synchronize()
    n_in = min(args.warmup + args.steps, 8)
    xs = [torch.from_numpy(synth.tokens_bf16(cfg, cfg.T, stream=rank * 100003 + s).view(np.int16)).to(dev)
          for s in range(n_in)]
    if cfg.L > 1:
        out = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device=dev)
    else:
        out = torch.empty((cfg.T, cfg.d), dtype=torch.int16, device=dev)
    unions = layer_unions(capi, sess, cfg, xs[0], dev)
    step_bytes = sum((u + cfg.n_shared) * expert_bytes(cfg) + router_bytes(cfg) for u in unions)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if step_bytes < (1 << 30) else None

    with Clocks(local_rank) as clk:
        ms, tim = timed_steps(capi, sess, cfg, xs, out, args.steps, args.warmup, stream, dist_on, flush)
    clocks = clk.summary()
    ms_step = max_over_ranks(ms, dist_on, dev) / args.steps
    value = whole_job_rate(cfg.T, world, ms_step / 1e3)
    kernel = tim["kernel"]
    launches = max(1, tim["timed_launches"])
    avg_ms = tim["ms"] / launches
    tensor_bound = cfg.T >= 9 and kernel.startswith("k_cache_fill")
    if tensor_bound:
        # the expert GEMMs (decoded-weight cache fill + gate/up + down) of one layer per timed region
        flops = expert_flops(cfg, cfg.T)
        burst = cfg.L == 1            # one ~1 ms call timed alone: burst peak; a long step: sustained
        peak = P["bf16_tflops"] if burst else P["bf16_tflops_sustained"]
        achieved = flops / (avg_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": measured_traffic(kernel, cfg.name, 1),
                "kernel": kernel, "alg_flops_per_launch": flops, "avg_launch_ms": avg_ms,
                "peak_source": f"{P['source']} ({'bf16_tflops, burst' if burst else 'bf16_tflops_sustained'}); "
                               "fp16 dense MMA rate = bf16's"}
        step_flops = cfg.L * (expert_flops(cfg, cfg.T) + router_flops(cfg, cfg.T))
        step_roof = {"alg_flops_per_step": step_flops,
                     "achieved_tflops": step_flops / (ms_step / 1e3) / 1e12,
                     "frac": step_flops / (ms_step / 1e3) / 1e12 / peak}
    else:
        # the decode kernels run every layer of the stack in one launch (the few-token kernel: one
        # launch per eight tokens); the timed region is one call, streaming each layer's router rows
        # and the union of the experts its tokens chose: the step's algorithmic bytes
        alg = step_bytes
        achieved = alg / (avg_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": P["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / P["hbm_gbs"], "traffic": measured_traffic(kernel, cfg.name, cfg.L),
                "kernel": kernel, "alg_bytes_per_launch": alg, "avg_launch_ms": avg_ms,
                "timed_regions_per_step": launches / args.steps,
                "peak_source": P["source"] + " (hbm_gbs, STREAM-style copy)"}
        step_roof = {"alg_bytes_per_step": step_bytes, "experts_streamed_per_layer": statistics.mean(unions),
                     "achieved_gbs": step_bytes / (ms_step / 1e3) / 1e9,
                     "frac": step_bytes / (ms_step / 1e3) / 1e9 / P["hbm_gbs"]}
    l2_ab = None
    if not tensor_bound:
        # L2 residency: the same steps once more in the other L2 mode (keep the shared experts of every
        # layer in L2 across steps: evict_last for them, evict_first for the rest; or plain copies)
        other = capi.MOE_L2_KEEP_SHARED if L2_MODES[args.l2_policy] == capi.MOE_L2_STREAM else capi.MOE_L2_STREAM
        capi.moe_set_l2_policy(sess.ctx, other)
        ms_other, _ = timed_steps(capi, sess, cfg, xs, out, args.steps, args.warmup, stream, dist_on, flush)
        capi.moe_set_l2_policy(sess.ctx, L2_MODES[args.l2_policy])
        ms_other = max_over_ranks(ms_other, dist_on, dev) / args.steps
        kept = cfg.L * cfg.n_shared * expert_bytes(cfg)
        v_other = whole_job_rate(cfg.T, world, ms_other / 1e3)
        keep_first = other == capi.MOE_L2_STREAM
        l2_ab = {"mode_of_value": args.l2_policy,
                 "keep_shared": "shared experts copied evict_last, routed experts and router rows evict_first",
                 "kept_bytes": kept, "kept_fraction_of_step_bytes": kept / step_bytes,
                 "value_keep_shared": value if keep_first else v_other,
                 "value_stream": v_other if keep_first else value,
                 "keep_shared_speedup": (ms_other / ms_step) if keep_first else (ms_step / ms_other)}

    # end to end through the public host-buffer entry point (copies inside the timed region)
    x_host = [torch.from_numpy(synth.tokens_bf16(cfg, cfg.T, stream=rank * 100003 + s).view(np.int16)).pin_memory()
              for s in range(min(n_in, 4))]
    r_host = torch.empty((cfg.T, cfg.d), dtype=torch.float32).pin_memory()
    for s in range(max(1, args.warmup)):
        capi.moe_forward_stack_host(sess.ctx, 0, cfg.L, x_host[s % len(x_host)], cfg.T, r_host, stream)
    if dist_on:
        torch.distributed.barrier()
    t0 = time.perf_counter()
    for s in range(args.steps):
        capi.moe_forward_stack_host(sess.ctx, 0, cfg.L, x_host[s % len(x_host)], cfg.T, r_host, stream)
    e2e_s = max_over_ranks(time.perf_counter() - t0, dist_on, dev)
    e2e = {"value": whole_job_rate(cfg.T * args.steps, world, e2e_s), "unit": "tok/s",
           "h2d_bytes_per_step": cfg.T * cfg.d * 2, "d2h_bytes_per_step": cfg.T * cfg.d * 4,
           "entry_point": "moe_forward_stack_host" + (" (one layer: rmsnorm + layer + residual)" if cfg.L == 1 else ""),
           "timer": "host wall clock around synchronous calls"}
    sess.close()
    l2 = (f"{FLUSH_BYTES >> 20} MB flush before each timed step" if flush is not None else
          f"no flush: each step streams {step_bytes / 1e9:.2f} GB (> 126 MB L2)")
    del xs, out, flush
    torch.cuda.empty_cache()

    fmt = cfg.fmt.upper() + "B32"
    entry = {
        "workload": cfg.name, "value": value, "unit": "tok/s", "ms_per_step": ms_step,
        "config": {"workload": f"{cfg.name}: d={cfg.d} E={cfg.E} top-{cfg.k}+{cfg.n_shared} shared "
                               f"I={cfg.I} {fmt} T={cfg.T} layers={cfg.L}",
                   "global_batch": cfg.T * world, "parallelism": f"replicas x{world}",
                   "l2": l2},
        "dtype": ("fp16 tensor-core MMA, fp32 accumulate, over " if tensor_bound else
                  "exact code operands, fp32 accumulate, over ") + fmt + " weights / bf16 activations",
        "roofline": roof, "step_roofline": step_roof, "e2e": e2e,
        **({"l2_residency": l2_ab} if l2_ab else {}),
        "gpu_launches": tim["all_launches"], "clocks": clocks,
    }
    if with_cpu:
        entry["cpu_baseline"] = cpu_baseline(cfg)
    return entry


# ---- token-count sweep (python bench.py --sweep): one layer, every path that accepts T ------------

# The library's path selection by T (include/moe.h, moe_forward): the single-token kernel for one
# token, the few-token kernel for 2 to DISPATCH_FEW_MAX tokens, the tensor-core path above; the
# CUDA-core path only where none fits.  The flags below pin a context to one path.
DISPATCH_FEW_MAX = 32
DISPATCH_SINGLE_MAX = 8      # the single-token kernel, once per token, when pinned to it
DISPATCH_TC_MIN = 9          # the tensor-core path's floor when the decode kernels are off
SWEEP_T = (1, 2, 4, 6, 8, 9, 10, 12, 16, 17, 24, 32, 33, 40, 48, 64, 96, 128, 256, 512, 1024, 2048, 4096, 8192)
SWEEP_PATHS = ("single-token kernel", "few-token kernel", "cuda-core", "tensor-core")


def sweep_flags(path: str) -> int:
    # MOE_FLAG_NO_DECODE_KERNEL, MOE_FLAG_NO_TENSOR_PREFILL, MOE_FLAG_NO_MULTI_DECODE
    no_decode, no_tensor, no_multi = 1, 2, 8
    return {"single-token kernel": no_multi, "few-token kernel": 0, "cuda-core": no_decode | no_tensor,
            "tensor-core": no_decode}[path]


def sweep_eligible(path: str, T: int) -> bool:
    """Whether a context pinned to `path` runs T tokens on that path."""
    if path == "single-token kernel":
        return T <= DISPATCH_SINGLE_MAX
    if path == "few-token kernel":
        return 2 <= T <= DISPATCH_FEW_MAX
    if path == "tensor-core":
        return T >= DISPATCH_TC_MIN
    return True


def default_path(T: int) -> str:
    if T == 1:
        return "single-token kernel"
    return "few-token kernel" if T <= DISPATCH_FEW_MAX else "tensor-core"


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
    ap.add_argument("--no-secondary", action="store_true", help="time the headline workload only")
    ap.add_argument("--no-cpu", action="store_true", help="leave out the oracle's CPU baselines")
    ap.add_argument("--l2-policy", default="stream", choices=sorted(L2_MODES),
                    help="L2 mode of the decode kernels' weight copies for the timed steps (the other mode is "
                         "timed too, for the l2_residency entry)")
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
    torch.cuda.set_device(local_rank)
    head = measure(args, cfg, rank, world, local_rank, dist_on, with_cpu=(rank == 0 and world == 1
                                                                        and not args.no_cpu))
    if rank == 0:
        out = {
            "metric": METRIC, "value": head["value"], "unit": "tok/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": head["dtype"],
            "data": "synthetic (seeded counter-hash weights, N(0,1) bf16 tokens)",
            "config": head["config"], "roofline": head["roofline"], "step_roofline": head["step_roofline"],
            "e2e": head["e2e"], "gpu_launches": head["gpu_launches"], "clocks": head["clocks"],
        }
        if "cpu_baseline" in head:
            out["cpu_baseline"] = head["cpu_baseline"]
        if "l2_residency" in head:
            out["l2_residency"] = head["l2_residency"]
        if world == 1 and not args.no_secondary and args.layers is None:
            out["secondary"] = {}
            for name in SECONDARY:
                if name == cfg.name:
                    continue
                out["secondary"][name] = measure(args, synth.CONFIGS[name], rank, world, local_rank, dist_on,
                                                 with_cpu=not args.no_cpu)
        print(json.dumps(out))
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
