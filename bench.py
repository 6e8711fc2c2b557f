"""Benchmark of the ZONOS2 sparse MoE feed-forward path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

A step is one pass of the whole MoE layer over one batch of synthetic tokens, through libzmoe's
C-ABI: at decode sizes one zmoe_moe_layer call (router, dispatch, SwiGLU and combine in one
launch); at prefill sizes zmoe_route -> zmoe_permute -> zmoe_grouped_swiglu -> zmoe_combine.
The default (headline) workload is the largest single-GPU layer: T = 16384 tokens, d_model 2048,
d_ff 3072, 16 experts, top-2 with renormalised gates and a Zipf(1.2) logit skew, bf16 weights with
fp32 accumulation; the grouped SwiGLU is tensor-bound and is reported against the bf16 tensor
peak.  The same run also measures, and reports under "also", the decode step (T = 64, top-1:
HBM-bound; four copies of the weights, 2.4 GB, rotate so that no step finds them in L2), the
top-1 prefill layer with uneven loads, and the batch-1 24-layer decode stack (us/token).

Multi-GPU (torchrun, one rank per GPU): tokens are independent, so every rank runs its own
batch against replicated weights with no data-path collective (weak scaling); the time is
the max over ranks, taken from CUDA events.

``--impl reference`` times the fp64 CPU oracle (the baseline arm) on the same workload.
Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time
from datetime import timedelta

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_moe_decoder_b200.dp import job_rate, max_over_ranks, rank_token_seed  # noqa: E402

METRIC = "MoE-layer tokens/sec on 1 B200 and % of roofline (HBM GB/s or tensor TFLOP/s)"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--config", type=int, default=None, choices=[2, 3, 4, 5, 6, 7, 8],
                    help="one workload alone; default: the headline workload (4) with workloads 2, 3 and 5 "
                         "measured in the same run and reported under 'also'")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the oracle timing leg")
    ap.add_argument("--h-pair", action="store_true",
                    help="prefill: carry h as the bf16 pair with the bf16 down weights instead of f16 h with the "
                         "prepared f16 down weights")
    ap.add_argument("--weight-copies", type=int, default=0,
                    help="device copies of the layer weights used in rotation (0: 4 for the decode step, else 1)")
    return ap.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p["bf16_tflops"]),
                    bf16_tflops_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm_gbs=FALLBACK_HBM_GBS, bf16_tflops=FALLBACK_BF16_TFLOPS,
                    bf16_tflops_sustained=1400.0, source="fallback")


WORKLOADS = {
    8: "final MoE layer in W8A8 fp8: T=16384, d_model=2048, d_ff=3072, E=16, top-2, Zipf(1.2) logit skew; expert "
       "weights E4M3 with one fp32 scale per row, token and hidden rows E4M3 with a dynamic per-token scale, "
       "bf16 router, fp32 accumulate",
    7: "decode step with fp8 expert weights: one MoE layer, T=64, d_model=2048, d_ff=3072, E=16, top-1; expert "
       "weights E4M3 with one fp32 scale per row, bf16 router, f16 tensor-core operands, fp32 accumulate",
    2: "decode step: one MoE layer, T=64 tokens (64 streams x 1 position), d_model=2048, d_ff=3072, E=16, top-1, "
       "bf16 weights/activations, fp32 accumulate",
    3: "prefill MoE layer: T=16384 (8 x 2048), d_model=2048, d_ff=3072, E=16, top-1, b~N(0,0.5), bf16",
    4: "final MoE layer: T=16384, d_model=2048, d_ff=3072, E=16, top-2, Zipf(1.2) logit skew, bf16",
    5: "batch-1 decode stack: 9-codebook embedding sum + RMSNorm, 24 pre-norm MoE layers (d_model=2048, "
       "d_ff=3072, E=16, top-1, top-2 in the last), attention omitted, bf16, one token per step",
    6: "batch-1 full decoder FFN step: embedding sum + RMSNorm, 3 dense SwiGLU layers, the 24 MoE layers "
       "(E=16, top-1, top-2 in the last), 1 dense layer, final RMSNorm + 9 codebook heads (1025 x 2048) with "
       "greedy next frame; d_model=2048, d_ff=3072, pre-norm residual, attention omitted, bf16, one token per step",
}


# ---------------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"zmoe_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            with open(self.path) as fh:
                for line in fh:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) < 9:
                        continue
                    try:
                        sm.append(float(parts[1]))
                        smax.append(float(parts[2]))
                    except ValueError:
                        continue
                    for n, v in zip(names, parts[5:9]):
                        if v.lower() == "active":
                            reasons.add(n)
            os.unlink(self.path)
        except OSError:
            pass
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [v for v in sm if v > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------------------------
# the oracle leg (cpu_baseline and --impl reference)
# ---------------------------------------------------------------------------------------------

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_leg(L, budget_s: float, max_steps: int | None = None):
    """Times oracle.moe_layer on the workload's layer; returns (tokens/s, steps, seconds, sample text)."""
    import oracle
    if L.T > 1024:
        # bounded sample: the first 512 tokens of the batch (same weights, same routing rule)
        T_s = 512
        x = L.x[:T_s]
    else:
        T_s = L.T
        x = L.x
    steps, t0 = 0, time.perf_counter()
    while True:
        oracle.moe_layer(x, L.w_router, L.w_gate, L.w_up, L.w_down, L.k, L.sel_bias, L.logit_bias)
        steps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or (max_steps is not None and steps >= max_steps):
            break
    sample = (f"oracle.moe_layer (numpy float64) on {T_s} of the workload's {L.T} tokens with the full "
              f"16-expert weights, {steps} step(s), {el:.1f} s")
    return T_s * steps / el, steps, el, sample


def run_reference(args):
    """The oracle as it stands, on the host cores: W untimed + K timed steps, each step a bounded
    sample of the workload's tokens (rotating through the batch) sized so the run ends in ~2.5 min."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    if args.config is None:
        args.config = HEADLINE
    if args.config in (5, 6):
        return run_reference_stack(args)
    from moe_inputs import make_config
    L = make_config(2 if args.config == 7 else args.config)
    if args.config == 7:
        from moe_inputs import quantize_e4m3_rows
        Q = [quantize_e4m3_rows(w) for w in (L.w_gate, L.w_up, L.w_down)]

    def one(lo, n):
        idx = (np.arange(n) + lo) % L.T
        if args.config == 7:
            oracle.moe_layer_fp8(L.x[idx], L.w_router, Q[0][0], Q[0][1], Q[1][0], Q[1][1], Q[2][0], Q[2][1], L.k,
                                 sel_bias=L.sel_bias)
        else:
            oracle.moe_layer(L.x[idx], L.w_router, L.w_gate, L.w_up, L.w_down, L.k, L.sel_bias, L.logit_bias)

    t0 = time.perf_counter()
    one(0, min(L.T, 64))                                  # calibration on up to 64 tokens
    t_cal = (time.perf_counter() - t0) / min(L.T, 64)
    per_step = 150.0 / max(1, args.steps + args.warmup)
    n = int(max(1, min(L.T, per_step / max(t_cal, 1e-9))))
    for i in range(args.warmup):
        one(i * n, n)
    t0 = time.perf_counter()
    for i in range(args.steps):
        one((args.warmup + i) * n, n)
    el = time.perf_counter() - t0
    v = n * args.steps / el
    cores = blas_threads()
    sample = (f"oracle.moe_layer (numpy float64), {n} of the workload's {L.T} tokens per step "
              f"(rotating through the batch), full 16-expert weights, {args.steps} timed steps, {el:.1f} s")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOADS[args.config], "T": L.T, "d_model": L.d, "d_ff": L.f, "E": L.E,
                       "k": L.k, "tokens_per_step": n},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------------

def traffic_from_profiles(kernel_key: str):
    """Per-launch DRAM bytes recorded from an ncu capture, if the kernel source is unchanged since."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        entries = {}
        with open(path) as fh:
            for line in fh:
                if line.startswith("#") or "=" not in line:
                    continue
                k, v = line.strip().split("=", 1)
                entries[k.strip()] = v.strip()
        src = entries.get(f"{kernel_key}.source")
        want_hash = entries.get(f"{kernel_key}.sha256")
        if not src or not want_hash:
            return None
        with open(os.path.join(ROOT, src), "rb") as fh:
            if hashlib.sha256(fh.read()).hexdigest() != want_hash:
                return None
        return float(entries[f"{kernel_key}.bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def run_reference_stack(args):
    """The oracle stack (numpy float64) on a bounded number of tokens: experts are drawn on first use
    and kept, so later tokens time the arithmetic, not the drawing."""
    import oracle
    from moe_inputs import StackSpec
    spec = StackSpec() if args.config == 5 else StackSpec(n_dense_front=3, n_dense_back=1)
    cache = {}

    def expert(l, e):
        if (l, e) not in cache:
            cache[(l, e)] = spec.expert(l, e)
        return cache[(l, e)]

    layers = oracle_stack_layers(spec, expert)
    tables, g0 = spec.tables(), spec.gamma0()
    n = max(1, min(args.steps, 3))
    codes = spec.codes(n + 1)
    heads = (spec.heads(), spec.gamma_out()) if args.config == 6 else None

    def one(i):
        ref = oracle.decode_stack_step(codes[i:i + 1], tables, g0, layers, spec.eps)
        if heads is not None:
            oracle.output_heads(ref["h"], heads[0], heads[1], spec.eps)

    one(n)      # warm-up: draws experts
    t0 = time.perf_counter()
    for i in range(n):
        one(i)
    el = time.perf_counter() - t0
    v = n / el
    sample = (f"oracle.decode_stack_step (numpy float64), {n} token(s) through the {spec.total_layers}-layer stack "
              f"(experts drawn on first use, outside the timing where already drawn), {el:.1f} s")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": n, "warmup": 1, "ms_per_step": 1e3 * el / n, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOADS[args.config], "us_per_token": 1e6 * el / n, "batch": 1},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def oracle_stack_layers(spec, expert):
    """The oracle's per-layer description of the stack (a dense FFN layer has no router)."""
    layers = []
    for l in range(spec.total_layers):
        wr, sb, gm = spec.layer_small(l)
        layers.append(dict(w_router=wr, sel_bias=sb, gamma=gm, k=spec.k_of(l), experts=(lambda e, l=l: expert(l, e))))
    return layers


def run_stack(args):
    """Configuration 5: tokens/s (= 1 / s per token) of the 24-layer batch-1 stack; 6: the full 28-layer
    FFN stack (3 dense + 24 MoE + 1 dense).  Returns rank 0's JSON line (None on other ranks)."""
    import torch

    world, rank, local_rank = args.world, args.rank, args.local_rank
    from moe_inputs import StackSpec, bf16_bits, stack_expert_bits
    from sparse_moe_decoder_b200 import zmoe_get_device_errors
    from sparse_moe_decoder_b200.layer import stack_from_bits

    spec = StackSpec() if args.config == 5 else StackSpec(n_dense_front=3, n_dense_back=1)
    full = args.config == 6   # the full step: 28 FFN layers, then the codebook heads and the next frame
    st = stack_from_bits(bf16_bits(spec.tables()), spec.gamma0(), spec.layer_small, stack_expert_bits(spec),
                         spec.total_layers, spec.E, spec.d, spec.f, spec.k_of, spec.eps, T=1, E_of=spec.E_of,
                         heads_bits=bf16_bits(spec.heads()) if full else None,
                         gamma_out=spec.gamma_out() if full else None)
    n = args.warmup + args.steps
    codes = spec.codes(n + 1)
    if rank > 0:
        codes = np.random.default_rng(rank_token_seed(rank)).integers(0, 1024, size=codes.shape).astype(np.int32)
    codes_dev = torch.from_numpy(codes).cuda()
    stream = torch.cuda.current_stream()

    # touched experts of one step (the roofline's bytes)
    st.record_inputs = True
    st.step(codes_dev[n:n + 1])
    torch.cuda.synchronize()
    touched = sum(int(torch.unique(t).numel()) for t in st.layer_idx)
    st.record_inputs = False
    per_expert = 3 * spec.f * spec.d * 2
    alg_bytes = touched * per_expert + spec.n_layers * spec.E * spec.d * 2 + spec.n_codebooks * spec.d * 2
    if full:
        alg_bytes += spec.n_codebooks * spec.vocab_rows * spec.d * 2     # the heads, streamed once per step

    graph = None
    try:
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for _ in range(2):
                st.step()
        stream.wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            st.step()
        torch.cuda.synchronize()
    except Exception as exc:   # capture not possible here: run the same calls eagerly
        graph = None
        print(f"# CUDA graph capture unavailable ({type(exc).__name__}: {exc}); timing eager launches",
              file=sys.stderr)
        torch.cuda.synchronize()

    def step(i):
        st.ids.copy_(codes_dev[i:i + 1])
        if graph is not None:
            graph.replay()
        else:
            st.step()

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        ev0.record(stream)
        for i in range(args.steps):
            step(args.warmup + i)
        ev1.record(stream)
        torch.cuda.synchronize()
    elapsed_ms = ev0.elapsed_time(ev1)
    elapsed_ms, = max_over_ranks([elapsed_ms], "cuda")
    ms_per_step = elapsed_ms / args.steps
    value = job_rate(1, world, args.steps, elapsed_ms)

    # e2e: codes from pinned host memory each step, the final residual stream read back
    codes_host = torch.from_numpy(codes).pin_memory()
    h_host = torch.empty((1, spec.d), dtype=torch.float32).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        st.ids.copy_(codes_host[i:i + 1], non_blocking=True)
        if graph is not None:
            graph.replay()
        else:
            st.step()
        h_host.copy_(st.h, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    dev_errors = zmoe_get_device_errors()
    peaks = load_peaks()
    achieved = alg_bytes / (ms_per_step / 1e3) / 1e9
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        t0 = time.perf_counter()
        layers = oracle_stack_layers(spec, spec.expert)
        ref = oracle.decode_stack_step(codes[:1], spec.tables(), spec.gamma0(), layers, spec.eps)
        if full:
            oracle.output_heads(ref["h"], spec.heads(), spec.gamma_out(), spec.eps)
        el = time.perf_counter() - t0
        cpu = {"value": 1.0 / el, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"oracle.decode_stack_step (numpy float64) on one token through all {spec.total_layers} layers, "
                         f"drawing each touched expert's weights as it goes, {el:.1f} s"}
    used_graph = graph is not None
    graph = None          # release the graph before the process group goes away
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOADS[args.config], "us_per_token": ms_per_step * 1e3, "layers": spec.total_layers,
                       "d_model": spec.d, "d_ff": spec.f, "E": spec.E, "batch": 1,
                       "parallelism": f"dp{world} (replicated weights, no data-path collective)",
                       "l2": "inputs larger than L2 (14.5 GB of weights; ~0.9 GB read per token)",
                       "experts_touched_per_token": touched, "cuda_graph": used_graph},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                         "kernel": (f"whole decode step: one stack_kernel launch (embedding + RMSNorm, then "
                                    f"{spec.total_layers} pre-norm layers: router, SwiGLU, residual)"
                                    + (" + heads_kernel" if full else "")) if st.persistent else
                                   (f"whole decode step (embed + {spec.total_layers} x tiny_layer_kernel: pre-norm, "
                                    "router, SwiGLU and combine in one launch per layer)"),
                         "algorithmic_bytes_per_launch": alg_bytes, "peak_source": peaks["source"]},
            "cpu_baseline": cpu,
            "e2e": {"value": world * args.steps / (e2e_ms / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": spec.n_codebooks * 4, "d2h_bytes_per_step": spec.d * 4},
            "gpu_launches": ((1 if st.persistent else 1 + spec.total_layers) + (1 if full else 0)) * args.steps,
            "clocks": clk.summary(),
            "device_errors": dev_errors,
        }
        return line
    return None


def run_fp8(args):
    """Workload 7: the decode step (configuration 2's tokens and weights) with the expert weights stored
    as E4M3 codes + row scales, one zmoe_moe_layer_fp8 call per step."""
    import torch
    world, rank, local_rank = args.world, args.rank, args.local_rank
    from moe_inputs import make_config, quantize_e4m3_rows
    from sparse_moe_decoder_b200 import zmoe_get_device_errors, zmoe_moe_layer_fp8
    L = make_config(2)
    if rank > 0:
        from moe_inputs import round_to_bf16
        L.x = round_to_bf16(np.random.default_rng(rank_token_seed(rank)).standard_normal(L.x.shape, dtype=np.float32))
    Q = [quantize_e4m3_rows(w) for w in (L.w_gate, L.w_up, L.w_down)]
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    n_copies = args.weight_copies if args.weight_copies > 0 else 8     # 8 x 302 MB of codes > L2
    copies = [[dev(q).clone() for q, _ in Q] for _ in range(n_copies)]
    scales = [dev(sc) for _, sc in Q]
    w_r = torch.from_numpy(L.w_router).cuda().to(torch.bfloat16)
    sb = dev(L.sel_bias)
    x = torch.from_numpy(L.x).cuda().to(torch.bfloat16)
    T = L.T
    idx = torch.empty((T, 1), dtype=torch.int32, device="cuda")
    y = torch.empty((T, L.d), dtype=torch.float32, device="cuda")
    ws = torch.empty(int(__import__("sparse_moe_decoder_b200").zmoe.lib().zmoe_moe_layer_fp8_workspace_size(
        T, L.d, L.f, L.E, 1)), dtype=torch.uint8, device="cuda")

    def step(i, xin=None):
        c = copies[i % n_copies]
        return zmoe_moe_layer_fp8(w_r, c[0], scales[0], c[1], scales[1], c[2], scales[2], 1, x=x if xin is None else xin,
                                  sel_bias=sb, out=y, outs=dict(expert_idx=idx), workspace=ws)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    touched = int(torch.unique(idx).numel())
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        e0.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step(i)
            ev[i][1].record(stream)
        e1.record(stream)
        torch.cuda.synchronize()
    elapsed = e0.elapsed_time(e1)
    k_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    elapsed, k_ms = max_over_ranks([elapsed, k_ms], "cuda")
    value = job_rate(T, world, args.steps, elapsed)
    # e2e from pinned host memory
    xh = torch.from_numpy(L.x).to(torch.bfloat16).pin_memory()
    yh = torch.empty((T, L.d), dtype=torch.float32).pin_memory()
    xd = torch.empty_like(x)
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for i in range(args.steps):
        xd.copy_(xh, non_blocking=True)
        step(i, xd)
        yh.copy_(y, non_blocking=True)
    a1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = a0.elapsed_time(a1)
    e2e_ms, = max_over_ranks([e2e_ms], "cuda")
    errs = zmoe_get_device_errors()
    peaks = load_peaks()
    M = T
    alg = (touched * 3 * L.f * L.d + touched * (2 * L.f + L.d) * 4 + T * L.d * 2 + L.E * L.d * 2
           + 2 * M * L.d * 2 + 2 * (M * 2 * L.f * 2) + M * L.d * 4 + T * L.d * 4)
    achieved = alg / (k_ms / 1e3) / 1e9
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        t0, n = time.perf_counter(), 0
        while time.perf_counter() - t0 < args.cpu_seconds:
            oracle.moe_layer_fp8(L.x, L.w_router, Q[0][0], Q[0][1], Q[1][0], Q[1][1], Q[2][0], Q[2][1], 1,
                                 sel_bias=L.sel_bias)
            n += 1
        el = time.perf_counter() - t0
        cpu = {"value": T * n / el, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"oracle.moe_layer_fp8 (numpy float64) on the 64-token layer, {n} step(s), {el:.1f} s"}
    if rank == 0:
        return {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp8", "data": "synthetic",
            "config": {"workload": WORKLOADS[7], "T": T, "d_model": L.d, "d_ff": L.f, "E": L.E, "k": 1,
                       "parallelism": f"dp{world} (replicated weights, no data-path collective)",
                       "l2": f"fp8 weights rotated over {n_copies} device copies ({n_copies * 0.302:.1f} GB > 126 MB L2)",
                       "experts_touched": touched},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": traffic_from_profiles("moe_layer_fp8_cfg7"),
                         "kernel": "moe_layer_kernel<fp8>: router, dispatch, fp8 SwiGLU and combine in one launch",
                         "algorithmic_bytes_per_launch": alg, "peak_source": peaks["source"]},
            "cpu_baseline": cpu,
            "e2e": {"value": T * world * args.steps / (e2e_ms / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": T * L.d * 2, "d2h_bytes_per_step": T * L.d * 4},
            "gpu_launches": args.steps, "clocks": clk.summary(), "layer_ms_per_step": k_ms, "device_errors": errs,
        }
    return None


def run_layer(args):
    """Workloads 2-4: one MoE layer per step.  Returns rank 0's JSON line (None on other ranks)."""
    import torch
    import torch.distributed as dist

    world, rank, local_rank = args.world, args.rank, args.local_rank
    from moe_inputs import make_config
    from sparse_moe_decoder_b200 import MoELayerRunner, MoEWeights, zmoe_get_device_errors

    L = make_config(args.config)
    if rank > 0:
        # each rank its own tokens, replicated weights
        from moe_inputs import round_to_bf16
        rng = np.random.default_rng(rank_token_seed(rank))
        L.x = round_to_bf16(rng.standard_normal(L.x.shape, dtype=np.float32))
    dt = torch.bfloat16
    W0 = MoEWeights.from_host(L)
    n_copies = args.weight_copies if args.weight_copies > 0 else (4 if args.config == 2 else 1)
    Ws = [W0] + [MoEWeights(W0.w_router.clone(), W0.w_gate.clone(), W0.w_up.clone(), W0.w_down.clone(),
                            W0.sel_bias, W0.logit_bias, None, W0.k) for _ in range(n_copies - 1)]
    R = MoELayerRunner(L.T, L.E, L.d, L.f, L.k, dt)
    x = torch.from_numpy(L.x).to("cuda", dt)
    stream = torch.cuda.current_stream()

    # decode sizes: the whole layer is one zmoe_moe_layer call (one cooperative launch); prefill sizes
    # time the four entry points separately, with events around the grouped SwiGLU.  Prefill carries h in
    # f16 with the f16 down weights, prepared once here (a load-time conversion, outside the timing).
    fused = L.T * L.k < 64 * L.E
    f16h = not fused and not args.h_pair
    if f16h:
        for W in Ws:
            W.prepare_f16()
        torch.cuda.synchronize()

    def step(i):
        return R.run(x, Ws[i % n_copies])

    def layer_call(xin, W):
        return R.run_f16h(xin, W) if f16h else R.run(xin, W)

    for i in range(args.warmup):
        if fused:
            step(i)
        elif f16h:
            R.run_steps_f16h(x, Ws[i % n_copies])
        else:
            R.run_steps(x, Ws[i % n_copies])
    torch.cuda.synchronize()
    counts = np.bincount(R.idx.cpu().numpy().ravel(), minlength=L.E)
    experts_touched = int((counts > 0).sum())

    # timed region: K steps, per-step events around the grouped-SwiGLU call (dominant kernels)
    import sparse_moe_decoder_b200.zmoe as Z
    ev_ffn = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        ev0.record(stream)
        for i in range(args.steps):
            W = Ws[i % n_copies]
            if fused:
                ev_ffn[i][0].record(stream)
                R.run(x, W)
                ev_ffn[i][1].record(stream)
                continue
            Z.zmoe_route(x, W.w_router, W.k, W.logit_bias, W.sel_bias, outs=(R.idx, R.gates, R.margin))
            Z.zmoe_permute(R.idx, x, W.E, outs=R.perm_outs, workspace=R.perm_ws)
            ev_ffn[i][0].record(stream)
            if f16h:
                Z.zmoe_grouped_swiglu_f16h(R.perm_outs["x_perm"], R.perm_outs["offsets"], W.w_gate, W.w_up,
                                           W.w_down_f16, W.down_scale, h=R.h16, y_perm=R.y_perm)
            else:
                Z.zmoe_grouped_swiglu(R.perm_outs["x_perm"], R.perm_outs["offsets"], W.w_gate, W.w_up, W.w_down,
                                      h=R.h, y_perm=R.y_perm, workspace=R.ffn_ws)
            ev_ffn[i][1].record(stream)
            Z.zmoe_combine(R.y_perm, R.perm_outs["inv_perm"], R.gates, None, out=R.y)
        ev1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    elapsed_ms = ev0.elapsed_time(ev1)
    ffn_ms = statistics.mean(a.elapsed_time(b) for a, b in ev_ffn)
    elapsed_ms, ffn_ms = max_over_ranks([elapsed_ms, ffn_ms], "cuda")
    ms_per_step = elapsed_ms / args.steps
    value = job_rate(L.T, world, args.steps, elapsed_ms)

    # launches of libzmoe kernels per step
    n_assign = L.T * L.k
    launches_per_step = 1 if fused else 1 + (1 if n_assign <= 1024 else 4) + 2 + 1

    # e2e: the same layer through the public API (one zmoe_moe_layer call) from pinned host memory,
    # result read back
    x_host = torch.from_numpy(L.x).to(dt).pin_memory()
    y_host = torch.empty((L.T, L.d), dtype=torch.float32).pin_memory()
    x_dev = torch.empty_like(x)
    for i in range(min(3, args.warmup)):
        x_dev.copy_(x_host, non_blocking=True)
        layer_call(x_dev, Ws[i % n_copies])
        y_host.copy_(R.y, non_blocking=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        x_dev.copy_(x_host, non_blocking=True)
        layer_call(x_dev, Ws[i % n_copies])
        y_host.copy_(R.y, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms, = max_over_ranks([e2e_ms], "cuda")
    e2e_value = job_rate(L.T, world, args.steps, e2e_ms)
    h2d = x_host.numel() * x_host.element_size()
    d2h = y_host.numel() * y_host.element_size()

    dev_errors = zmoe_get_device_errors()

    # roofline of the dominant kernels (decode: the one layer launch; prefill: the grouped-SwiGLU
    # launches, gate/up then down)
    peaks = load_peaks()
    bpe = 2
    touched = int((counts > 0).sum())
    M = int(counts.sum())
    weight_bytes = touched * 3 * L.f * L.d * bpe
    h_cols = L.f if f16h else 2 * L.f
    act_bytes = M * L.d * bpe + 2 * (M * h_cols * bpe) + M * L.d * 4   # x_perm in, h out + in, y_perm out
    if fused:
        # the launch also reads x and W_r, writes and re-reads x_perm, and writes y
        act_bytes += L.T * L.d * bpe + L.E * L.d * bpe + M * L.d * bpe + L.T * L.d * 4
    alg_bytes = weight_bytes + act_bytes
    flops = 2.0 * M * 3 * L.d * L.f
    if fused:
        achieved = alg_bytes / (ffn_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic_from_profiles("grouped_swiglu_cfg2"),
                "kernel": "moe_layer_kernel: router, dispatch, SwiGLU and combine in one launch",
                "algorithmic_bytes_per_launch": alg_bytes, "peak_source": peaks["source"]}
    else:
        achieved = flops / (ffn_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"],
                "traffic": traffic_from_profiles(f"grouped_swiglu_cfg{args.config}"),
                "kernel": ("zmoe_grouped_swiglu_f16h (tc_ffn_kernel on CTA pairs: gate/up, then down over f16 h)"
                           if f16h else "zmoe_grouped_swiglu (tc_ffn_kernel on CTA pairs: gate/up, then down over "
                                        "the bf16 h pair)"),
                "algorithmic_flops_per_launch": flops, "peak_source": peaks["source"],
                "peak_kind": "burst (the SwiGLU is timed alone, between the other calls of the step)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, steps, el, sample = oracle_leg(L, args.cpu_seconds)
        cpu = {"value": v, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle", "sample": sample}

    if rank != 0:
        return None
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOADS[args.config], "T": L.T, "d_model": L.d, "d_ff": L.f, "E": L.E,
                   "k": L.k, "tokens_per_rank": L.T, "parallelism": f"dp{world} (replicated weights, no "
                   "data-path collective)",
                   "l2": (f"weights rotated over {n_copies} device copies ({n_copies * 0.604:.1f} GB > 126 MB L2)"
                          if n_copies > 1 else "inputs larger than L2 (one layer's weights: 604 MB, x and the "
                          "permuted rows another 0.2-0.3 GB)"),
                   "experts_touched": experts_touched,
                   "expert_loads": counts.tolist(),
                   "h": ("f16 (down weights converted once to f16 with a power-of-two scale per expert)" if f16h
                         else "bf16 pair (h_hi + h_lo)" if not fused else "bf16 pair")},
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "call": "zmoe_moe_layer_f16h" if f16h else "zmoe_moe_layer"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
        "ffn_ms_per_step": ffn_ms,
        "device_errors": dev_errors,
    }


def summary_of(line):
    """The keys of another workload's line that the headline line carries under 'also'."""
    if line is None:
        return None
    out = {"workload": line["config"]["workload"], "value": line["value"], "unit": line["unit"],
           "steps": line["steps"], "warmup": line["warmup"], "ms_per_step": line["ms_per_step"]}
    if "us_per_token" in line["config"]:
        out["us_per_token"] = line["config"]["us_per_token"]
    r = line.get("roofline") or {}
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic", "kernel"):
        if k in r:
            out[f"roofline_{k}"] = r[k]
    out["e2e_value"] = (line.get("e2e") or {}).get("value")
    out["clocks"] = line.get("clocks")
    out["gpu_launches"] = line.get("gpu_launches")
    out["device_errors"] = line.get("device_errors")
    return out


def run_w8a8(args):
    """Workload 8: configuration 4's tokens and weights with the expert weights as E4M3 codes + row scales,
    one zmoe_moe_layer_w8a8 call per step (router, permutation + token quantization, both E4M3 GEMMs on
    CTA pairs, hidden quantization, combine)."""
    import torch
    world, rank, local_rank = args.world, args.rank, args.local_rank
    from moe_inputs import make_config, quantize_e4m3_rows
    from sparse_moe_decoder_b200 import zmoe_get_device_errors, zmoe_moe_layer_w8a8
    L = make_config(4)
    if rank > 0:
        from moe_inputs import round_to_bf16
        L.x = round_to_bf16(np.random.default_rng(rank_token_seed(rank)).standard_normal(L.x.shape, dtype=np.float32))
    Q = [quantize_e4m3_rows(w) for w in (L.w_gate, L.w_up, L.w_down)]
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    qs = [dev(q) for q, _ in Q]
    sc = [dev(s_) for _, s_ in Q]
    w_r = torch.from_numpy(L.w_router).cuda().to(torch.bfloat16)
    lb = dev(L.logit_bias) if L.logit_bias is not None else None
    sb = dev(L.sel_bias) if L.sel_bias is not None else None
    x = torch.from_numpy(L.x).cuda().to(torch.bfloat16)
    T = L.T
    idx = torch.empty((T, L.k), dtype=torch.int32, device="cuda")
    y = torch.empty((T, L.d), dtype=torch.float32, device="cuda")
    ws = torch.empty(int(__import__("sparse_moe_decoder_b200").zmoe.lib().zmoe_moe_layer_w8a8_workspace_size(
        T, L.d, L.f, L.E, L.k)), dtype=torch.uint8, device="cuda")

    def step(xin=None):
        return zmoe_moe_layer_w8a8(w_r, qs[0], sc[0], qs[1], sc[1], qs[2], sc[2], L.k, x=x if xin is None else xin,
                                   logit_bias=lb, sel_bias=sb, out=y, outs=dict(expert_idx=idx), workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    elapsed, = max_over_ranks([e0.elapsed_time(e1)], "cuda")
    value = job_rate(T, world, args.steps, elapsed)
    xh = torch.from_numpy(L.x).to(torch.bfloat16).pin_memory()
    yh = torch.empty((T, L.d), dtype=torch.float32).pin_memory()
    xd = torch.empty_like(x)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(args.steps):
        xd.copy_(xh, non_blocking=True)
        step(xd)
        yh.copy_(y, non_blocking=True)
    a1.record(stream)
    torch.cuda.synchronize()
    e2e_ms, = max_over_ranks([a0.elapsed_time(a1)], "cuda")
    errs = zmoe_get_device_errors()
    peaks = load_peaks()
    M = T * L.k
    flops = 2.0 * M * 3 * L.d * L.f
    ms = elapsed / args.steps
    achieved = flops / (ms / 1e3) / 1e12
    fp8_peak = 2.0 * peaks["bf16_tflops"]
    if rank != 0:
        return None
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8 (e4m3 weights and activations)", "data": "synthetic",
        "config": {"workload": WORKLOADS[8], "T": T, "d_model": L.d, "d_ff": L.f, "E": L.E, "k": L.k,
                   "parallelism": f"dp{world} (replicated weights, no data-path collective)",
                   "l2": "inputs larger than L2 (302 MB of E4M3 weights, 0.5 GB of per-step activations)"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": fp8_peak, "unit": "TFLOP/s",
                     "frac": achieved / fp8_peak, "traffic": None,
                     "kernel": "whole zmoe_moe_layer_w8a8 call (route, permutation + token quantization, two E4M3 "
                               "GEMMs on CTA pairs, hidden quantization, combine) against the GEMMs' FLOPs",
                     "algorithmic_flops_per_launch": flops,
                     "peak_source": peaks["source"] + " bf16 burst x 2 (the recipe's nominal fp8 / bf16 ratio)"},
        "cpu_baseline": None,
        "e2e": {"value": job_rate(T, world, args.steps, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": T * L.d * 2, "d2h_bytes_per_step": T * L.d * 4, "call": "zmoe_moe_layer_w8a8"},
        # route, the permutation's count / scan / scatter, token quantization, gate/up, h quantization,
        # down, combine (plus one memset of the row maxima)
        "gpu_launches": 9 * args.steps, "clocks": clk.summary(), "device_errors": errs,
    }


def run_one(args):
    if args.config == 8:
        return run_w8a8(args)
    if args.config == 7:
        return run_fp8(args)
    if args.config >= 5:
        return run_stack(args)
    return run_layer(args)


HEADLINE = 4
ALSO = ((2, 200, 20), (3, None, None), (5, 100, 10), (6, 100, 10), (7, 200, 20), (8, None, None))   # (workload, min steps, min warm-up)


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    args.world = int(os.environ.get("WORLD_SIZE", "1"))
    args.rank = int(os.environ.get("RANK", "0"))
    args.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    torch.cuda.set_device(args.local_rank)
    if args.world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=600),
                                device_id=torch.device("cuda", args.local_rank))
    if args.config is not None:
        line = run_one(args)
    else:
        # the headline workload, then the others in the same run (same ranks, same collective steps)
        args.config = HEADLINE
        line = run_one(args)
        also = {}
        for cfg, min_steps, min_warm in ALSO:
            sub = argparse.Namespace(**vars(args))
            sub.config = cfg
            sub.no_cpu_baseline = True
            if min_steps:
                sub.steps = max(args.steps, min_steps)
                sub.warmup = max(args.warmup, min_warm)
            torch.cuda.empty_cache()
            also[f"workload_{cfg}"] = summary_of(run_one(sub))
        if line is not None:
            line["also"] = also
    if line is not None:
        print(json.dumps(line), flush=True)
    if args.world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
