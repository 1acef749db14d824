"""Throughput of the DeepSeekMoE layer forward on B200, one JSON line.

    python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl reference]

Default workload: the DeepSeek-V3-shaped prefill layer (T=8192, d=7168, 256 routed
+ 1 shared SwiGLU experts of d_ff=2048, sigmoid scores with a selection-only bias,
top-8 renormalised), synthetic seeded inputs and random weights of that shape.

A step is one whole layer forward (router, scores, top-k, gates, balance
statistics, permutation, gate/up and down grouped GEMMs, combine) over one batch of
T tokens already resident in HBM; with N GPUs every rank runs its own batch of T
tokens (weak scaling) and the balance statistics are all-reduced across ranks each
step. Timing: W untimed steps, then K steps between barrier + synchronize, CUDA
events on the launching stream, max over ranks. The 22.6 GB of expert weights a
step streams are far larger than L2, so no flush is needed between steps.

Reported alongside: the dominant kernel's roofline (mean in-region duration from
per-stage CUDA events; a tensor-bound kernel is divided by the measured burst bf16
figure when the timed region ran at the maximum SM clock, else by the sustained one,
and the other fractions are kept as extra keys), the same metric end to end through
dsmoe_forward_host with pinned host buffers (copies inside the timed region), the
oracle timed on the host's cores over a bounded sample, SM clocks sampled during the
timed region, and the number of kernel launches. At N=1 a "decode" block follows:
the V4-shaped decode batches (T=256 and T=16), timed the same way after the main
workload's tensors are released, with the HBM bytes they must move per step and their
fraction of the measured copy bandwidth.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "DeepSeekMoE layer fwd tokens/s; achieved TFLOP/s (% bf16 peak) / GB/s on 1 B200"
SCORE_NAMES = {0: "softmax", 1: "sigmoid", 2: "sqrt_softplus", 3: "hash"}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="v3_prefill")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=None, help="steps of the end-to-end leg (default: --steps)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample", type=int, default=None, help="tokens in the oracle's timed sample")
    ap.add_argument("--gemm", default="single", choices=["single", "pair"],
                    help="grouped-GEMM kernel: one CTA per tile (default) or CTA pairs")
    ap.add_argument("--decode", default="v4_decode_t256,v4_decode_t16",
                    help="decode workloads timed after the main one at N=1 (comma list; empty: none)")
    ap.add_argument("--decode-steps", type=int, default=20)
    ap.add_argument("--graph", action="store_true",
                    help="N=1: capture one forward in a CUDA graph after the warm-up and time its replays "
                         "(the device work is the same; host launch overhead leaves the timed region)")
    ap.add_argument("--backward", action="store_true",
                    help="time a training step instead (forward saving the pre-activations, gate, router, "
                         "expert input and weight gradients) and print one JSON line of stage times and rates")
    ap.add_argument("--role-cycles", action="store_true",
                    help="profiling run: load the role-cycle build of the library (build.py --role-cycles) and "
                         "print, per grouped-GEMM launch kind, the SM clock and the share of cycles each role "
                         "waited, instead of the benchmark line")
    return ap.parse_args()


SPEC_BF16_TFLOPS = 2250.0  # B200 dense bf16, nominal
SPEC_HBM_GBS = 8000.0      # B200 HBM3e, nominal
PEAK_CHOICE = ("tensor frac is against the burst cuBLAS figure when the timed region ran at the "
               "maximum SM clock (median within 3% of clocks.max.sm), else against the sustained one")


def tensor_peak_key(clock_info):
    """The measured bf16 peak to divide by: the burst figure (a GEMM timed alone, at full
    clock) when the timed region's median SM clock was at the maximum, else the
    sustained, power-capped one."""
    if clock_info and clock_info.get("sm_mhz") and clock_info.get("sm_max_mhz"):
        if clock_info["sm_mhz"] >= 0.97 * clock_info["sm_max_mhz"]:
            return "bf16_tflops"
        return "bf16_tflops_sustained"
    return "bf16_tflops"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


CSRC = "mixture_experts_layer_score_b200/csrc/"
# the sources that decide each stage's memory traffic: the kernel and, for the grouped
# GEMMs, the tile schedule
KERNEL_SOURCES = {"gemm_gate_up": ("gemm_sm100.cu", "grouped_tiles.cuh"),
                  "gemm_down": ("gemm_sm100.cu", "grouped_tiles.cuh"),
                  "router": ("router_sm100.cu",)}
PAIR_GEMM_SOURCES = {"gemm_gate_up": ("gemm_gateup_pair_sm100.cu", "grouped_tiles.cuh"),
                     "gemm_down": ("gemm_pair_sm100.cu", "grouped_tiles.cuh")}


def source_digest(stage, gemm="single"):
    """First 16 hex digits of the sha256 over the stage's kernel sources, in order."""
    import hashlib
    srcs = PAIR_GEMM_SOURCES[stage] if (gemm == "pair" and stage in PAIR_GEMM_SOURCES) else KERNEL_SOURCES[stage]
    h = hashlib.sha256()
    for src in srcs:
        with open(os.path.join(ROOT, CSRC + src), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def captured_traffic(stage, weight_bytes, gemm="single", workload=None):
    """DRAM bytes per launch of `stage` from the committed ncu summary
    (profiles/ncu_dram_traffic.txt): the captured launch's DRAM read+write bytes divided by
    the algorithmic weight bytes it streamed, scaled to this launch's weight bytes. A
    capture of the benchmarked workload itself is preferred (the scaling is then the
    identity); otherwise the first capture of the stage is scaled (its DRAM traffic is
    dominated by the expert weights and grows with them). None when the kernel sources
    changed since the capture or no capture is recorded."""
    path = os.path.join(ROOT, "profiles", "ncu_dram_traffic.txt")
    if not os.path.exists(path):
        return None
    digest = source_digest(stage, gemm)
    found = []
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 5 and not line.startswith("#") and parts[0] == stage and parts[1] == digest:
                found.append((parts[4] == workload, float(parts[2]) / float(parts[3])))
    if not found:
        return None
    same = [r for m, r in found if m]
    return (same[0] if same else found[0][1]) * weight_bytes


def config_block(cfg, n_gpus):
    return {"workload": cfg.name, "T_per_gpu": cfg.T, "global_batch": cfg.T * n_gpus, "d_model": cfg.d_model,
            "n_routed": cfg.n_routed, "top_k": cfg.top_k, "d_ff": cfg.d_ff, "n_shared": cfg.n_shared,
            "d_ff_shared": cfg.d_ff_shared, "score": SCORE_NAMES[cfg.score], "renormalize": cfg.renormalize,
            "parallelism": f"dp{n_gpus} (token shards, full weight replica per GPU)",
            "l2": f"no flush: inputs larger than L2 ({(cfg.routed_weight_bytes() + cfg.shared_weight_bytes()) / 1e9:.1f}"
                  " GB of expert weights streamed per step vs 126 MB L2)"}


# ----------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ----------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [c.strip() for c in line.split(",")]
                if len(p) >= 9:
                    rows.append(p)
        os.unlink(self.path)
        if not rows:
            return None

        def num(v):
            try:
                return float(v)
            except ValueError:
                return float("nan")

        sm = [num(r[1]) for r in rows]
        smax = max(num(r[2]) for r in rows)
        loaded = [v for v, r in zip(sm, rows) if num(r[3]) > 200.0] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded.sort()
        return {"sm_mhz": loaded[len(loaded) // 2], "sm_max_mhz": smax, "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------------------
# CPU oracle leg (bounded sample)
# ----------------------------------------------------------------------------------------
def default_cpu_sample(cfg):
    # about 10-30 s of the oracle on the GPU machine's host cores (V3: ~0.9 s per token)
    return 512 if cfg.d_model <= 1024 and cfg.T <= 4096 else (64 if cfg.d_model <= 2048 else 16)


def cpu_oracle_throughput(cfg, x_cpu, b_cpu, W_router_cpu, token_ids_cpu, expert_source, n_tokens, seed=0):
    """Time the oracle, as it stands, on a sample of n_tokens tokens of the workload (their
    own batch: router, scores, top-k, statistics, experts, combine). Expert weights are
    fetched to host memory before the clock starts. Returns (tokens/s, seconds, threads)."""
    import numpy as np
    from oracle import dsmoe_oracle as O
    T = x_cpu.shape[0]
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(T, size=min(n_tokens, T), replace=False))
    inp = {"x": x_cpu[rows], "W_router": W_router_cpu, "b": b_cpu,
           "token_ids": None if token_ids_cpu is None else token_ids_cpu[rows]}
    r = O.route(cfg, inp)
    need = sorted(set(np.asarray(r["idx"]).ravel().tolist()))
    cache = {}
    for e in need:
        cache[e] = expert_source(e)
    shared = [expert_source(("s", s)) for s in range(cfg.n_shared)]

    inp_w = dict(inp)
    inp_w["W_gate"] = {e: cache[e][0] for e in need}
    inp_w["W_up"] = {e: cache[e][1] for e in need}
    inp_w["W_down"] = {e: cache[e][2] for e in need}
    inp_w["Ws_gate"] = [s[0] for s in shared]
    inp_w["Ws_up"] = [s[1] for s in shared]
    inp_w["Ws_down"] = [s[2] for s in shared]
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    O.forward(cfg, inp_w)
    dt = time.perf_counter() - t0
    return len(rows) / dt, dt, threads, len(rows)


# ----------------------------------------------------------------------------------------
# reference arm: the oracle on the host's cores
# ----------------------------------------------------------------------------------------
def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np
    import torch
    import workloads as W
    inp = W.make_inputs(cfg, seed=0, device="cpu", with_weights=False)
    n = args.cpu_sample or max(1, default_cpu_sample(cfg) // 4)

    def src(key):
        if isinstance(key, tuple):
            return tuple(W.expert_matrix(cfg, w, key[1], 0, "cpu") for w in ("Ws_gate", "Ws_up", "Ws_down"))
        return tuple(W.expert_matrix(cfg, w, key, 0, "cpu") for w in ("W_gate", "W_up", "W_down"))

    times, toks = [], 0
    threads = 1
    for step in range(args.warmup + args.steps):
        tps, dt, threads, m = cpu_oracle_throughput(cfg, inp["x"], inp["b"], inp["W_router"], inp["token_ids"],
                                                    src, n, seed=step)
        if step >= args.warmup:
            times.append(dt)
            toks += m
    value = toks / sum(times)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(cfg, 1),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": f"{n} tokens of the workload per step, full layer (float64 oracle)"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------------------
# native arm
# ----------------------------------------------------------------------------------------
def run_native(args, cfg):
    import numpy as np
    import torch
    import torch.distributed as dist
    import workloads as W
    import mixture_experts_layer_score_b200 as M
    from mixture_experts_layer_score_b200.sharded import global_balance_stats

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch N>1 with torch.distributed.run")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", rank=rank, world_size=world, timeout=timedelta(seconds=300),
                                device_id=dev)

    # inputs: every rank holds the same weights and its own batch of T tokens
    inp = W.make_inputs(cfg, seed=0, device=dev, with_weights=True)
    if rank > 0:
        inp["x"] = W.normal_bf16((cfg.T, cfg.d_model), 1.0, 0, "x", rank, dev)
        if inp["token_ids"] is not None:
            g = torch.Generator(device=dev)
            g.manual_seed(W.derive_seed(0, "token_ids", rank))
            inp["token_ids"] = torch.randint(0, W.TOKEN_VOCAB, (cfg.T,), generator=g, device=dev,
                                             dtype=torch.int64).to(torch.int32)
    layer = M.DSMoE(M.cfg_from(cfg, cfg.T), inp, device=local)
    M.dsmoe_set_gemm_kernel(layer.handle, M.DSMOE_GEMM_SINGLE if args.gemm == "single" else M.DSMOE_GEMM_PAIR)
    out = layer.alloc_outputs(cfg.T)
    T_total = cfg.T * world
    stream = torch.cuda.current_stream(dev)

    def step():
        layer.forward(inp["x"], token_ids=inp["token_ids"], out=out, stream=stream)
        if world > 1:
            global_balance_stats(layer.handle, T_total, out["counts"], out["P_sum"], out["f"], out["P"],
                                 stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    st = M.dsmoe_get_status(layer.handle)
    if st != M.DSMOE_OK:
        raise SystemExit(f"device status after warm-up: {M.dsmoe_last_error()}")

    # ---- timed region (device)
    M.dsmoe_set_timing(layer.handle, True)
    launches0 = M.dsmoe_launch_count(layer.handle)
    graph = None
    if args.graph and world == 1:
        # one untimed forward on the capture stream, then the capture with the stage events
        # (timing on): every replay records them again, into the one recorded slot
        M.dsmoe_set_timing(layer.handle, False)
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            layer.forward(inp["x"], token_ids=inp["token_ids"], out=out, stream=cap)
        stream.wait_stream(cap)
        M.dsmoe_set_timing(layer.handle, True)
        l0 = M.dsmoe_launch_count(layer.handle)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            layer.forward(inp["x"], token_ids=inp["token_ids"], out=out)
        per_forward = M.dsmoe_launch_count(layer.handle) - l0
        launches0 = M.dsmoe_launch_count(layer.handle)
        step = graph.replay  # noqa: F811
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    ms = e0.elapsed_time(e1)
    clock_info = clocks.stop()
    launches = M.dsmoe_launch_count(layer.handle) - launches0
    if graph is not None:
        launches = per_forward * args.steps  # replays launch the captured kernels
    stage_ms = M.dsmoe_stage_times(layer.handle)
    M.dsmoe_set_timing(layer.handle, False)
    if world > 1:
        t = torch.tensor([ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    st = M.dsmoe_get_status(layer.handle)
    if st != M.DSMOE_OK:
        raise SystemExit(f"device status after the timed region: {M.dsmoe_last_error()}")
    ms_per_step = ms / args.steps
    value = T_total / (ms_per_step / 1e3)

    # ---- roofline of the dominant kernel
    peaks, peak_src = load_peaks()
    S = cfg.T * cfg.top_k
    # the routed experts' GEMMs (the shared experts' run as their own stage, beside routing)
    flops = {
        "gemm_gate_up": 2.0 * 2 * cfg.d_model * S * cfg.d_ff,
        "gemm_down": 2.0 * cfg.d_model * S * cfg.d_ff,
    }
    dom = max(flops, key=lambda k: stage_ms.get(k, 0.0))
    counts = out["counts"].cpu().numpy()
    touched = int((counts > 0).sum())
    weight_bytes = {"gemm_gate_up": 2 * cfg.d_model * touched * 2 * cfg.d_ff,
                    "gemm_down": 2 * cfg.d_model * touched * cfg.d_ff}
    dom_ms = stage_ms[dom]
    intensity = flops[dom] / max(weight_bytes[dom], 1)
    tensor_key = tensor_peak_key(clock_info)
    ridge = peaks[tensor_key] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if intensity >= ridge:
        achieved = flops[dom] / (dom_ms / 1e3) / 1e12
        peak = peaks[tensor_key]
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "frac_of_burst": achieved / peaks["bf16_tflops"],
                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                "frac_of_spec": achieved / SPEC_BF16_TFLOPS}
    else:
        achieved = weight_bytes[dom] / (dom_ms / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "frac_of_spec": achieved / SPEC_HBM_GBS}
    traffic = captured_traffic(dom, weight_bytes[dom], args.gemm, cfg.name)
    roof.update({"kernel": dom, "kernel_ms": dom_ms, "traffic": traffic,
                 "peak_source": f"{peak_src} ({tensor_key if roof['bound'] == 'tensor' else 'hbm_gbs'})",
                 "peak_choice": PEAK_CHOICE,
                 "algorithmic": {"flops": flops[dom], "weight_bytes": weight_bytes[dom]}})
    layer_flops = cfg.flops_per_token() * cfg.T
    layer_tflops = layer_flops / (ms_per_step / 1e3) / 1e12

    # ---- end to end through the C ABI with host buffers
    e2e_steps = args.e2e_steps or args.steps
    T, K, N, d = cfg.T, cfg.top_k, cfg.n_routed, cfg.d_model
    xh = inp["x"].cpu().pin_memory()
    idh = None if inp["token_ids"] is None else inp["token_ids"].cpu().pin_memory()
    hh = torch.empty((T, d), dtype=torch.bfloat16).pin_memory()
    th = torch.empty((T, K), dtype=torch.int32).pin_memory()
    gh = torch.empty((T, K), dtype=torch.float32).pin_memory()
    ch = torch.empty((N,), dtype=torch.int32).pin_memory()
    fh = torch.empty((N,), dtype=torch.float32).pin_memory()
    ph = torch.empty((N,), dtype=torch.float32).pin_memory()
    w = inp

    def e2e_step():
        # pipelined host entry point: this step's copies overlap the neighbouring steps'
        # forwards (two staging slots, the handle's copy stream)
        M.dsmoe_forward_host_async(layer.handle, T, xh, idh, w.get("W_router"), w.get("b"), w["W_gate"], w["W_up"],
                                   w["W_down"], w.get("Ws_gate"), w.get("Ws_up"), w.get("Ws_down"), hh, th, gh, ch,
                                   fh, ph, stream)

    for _ in range(2):
        e2e_step()
    M.dsmoe_host_sync(layer.handle)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    M.dsmoe_host_join(layer.handle, stream)  # the timed region ends after the last output copy
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    if world > 1:
        t = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    h2d = xh.numel() * 2 + (0 if idh is None else idh.numel() * 4)
    d2h = hh.numel() * 2 + th.numel() * 4 + gh.numel() * 4 + 3 * N * 4
    e2e = {"value": T_total / (e2e_ms / e2e_steps / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "api": "dsmoe_forward_host_async (pinned host buffers, copies overlapped "
                                             "with the neighbouring steps' forwards)"}

    # ---- CPU oracle baseline (rank 0, N=1 only)
    cpu_base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n = args.cpu_sample or default_cpu_sample(cfg)

        def src(key):
            if isinstance(key, tuple):
                s = key[1]
                return (inp["Ws_gate"][s].cpu(), inp["Ws_up"][s].cpu(), inp["Ws_down"][s].cpu())
            return (inp["W_gate"][key].cpu(), inp["W_up"][key].cpu(), inp["W_down"][key].cpu())

        tps, dt, threads, m = cpu_oracle_throughput(
            cfg, inp["x"].cpu(), None if inp["b"] is None else inp["b"].cpu(),
            None if inp["W_router"] is None else inp["W_router"].cpu(),
            None if inp["token_ids"] is None else inp["token_ids"].cpu(), src, n)
        cpu_base = {"value": tps, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                    "sample": f"{m} tokens of the workload as one batch, full layer, float64 oracle, {dt:.1f} s"}

    layer.close()
    # ---- decode (weight-streaming) workloads, N=1 only: the main workload's tensors are
    # released first; each is timed on its own with the same event and clock method
    decode = None
    if world == 1 and args.decode.strip():
        del inp, w, layer, out, xh, hh, th, gh, ch, fh, ph
        torch.cuda.empty_cache()
        decode = {}
        for name in [n.strip() for n in args.decode.split(",") if n.strip()]:
            decode[name] = time_decode(M, W, name, dev, stream, args.decode_steps, max(args.warmup, 3), peaks,
                                       peak_src)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; random weights of the layer's shape)",
                "config": dict(config_block(cfg, world), gemm_kernel=args.gemm,
                               launch="cuda graph replay" if graph is not None else "stream launches"),
                "roofline": roof,
                "cpu_baseline": cpu_base, "e2e": e2e, "gpu_launches": int(launches), "clocks": clock_info,
                "layer_tflops": layer_tflops, "stage_ms": stage_ms, "experts_touched": touched, "decode": decode}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def time_decode(M, W, name, dev, stream, steps, warmup, peaks, peak_src):
    """One decode-shaped workload (few tokens, hundreds of experts): the layer streams the
    weights of every expert some token picked, so it is HBM-bound. Returns its step time,
    tokens/s and the bytes that must cross HBM per step (weights of the touched routed
    experts and the shared experts, the router matrix, x read and h written) as GB/s and
    as fractions of the measured copy bandwidth and of the 8 TB/s nominal figure, plus
    the same for the gate/up GEMM alone (its weights over its event time)."""
    import torch
    cfg = W.get_config(name)
    inp = W.make_inputs(cfg, seed=0, device=dev, with_weights=True)
    layer = M.DSMoE(M.cfg_from(cfg, cfg.T), inp, device=dev.index)
    out = layer.alloc_outputs(cfg.T)
    for _ in range(warmup):
        layer.forward(inp["x"], token_ids=inp["token_ids"], out=out, stream=stream)
    torch.cuda.synchronize(dev)
    M.dsmoe_set_timing(layer.handle, True)
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        layer.forward(inp["x"], token_ids=inp["token_ids"], out=out, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    clock_info = clocks.stop()
    stage_ms = M.dsmoe_stage_times(layer.handle)
    st = M.dsmoe_get_status(layer.handle)
    if st != M.DSMOE_OK:
        raise SystemExit(f"device status after the {name} timed region: {M.dsmoe_last_error()}")
    touched = int((out["counts"] > 0).sum())
    layer.close()
    d, F, Fs, Ks = cfg.d_model, cfg.d_ff, cfg.d_ff_shared, cfg.n_shared
    w_gate_up = 2 * d * 2 * touched * F   # the routed gate/up stage (the shared experts run beside routing)
    w_shared = 2 * d * 3 * Ks * Fs
    w_down = 2 * d * touched * F
    router = 0 if cfg.score == W.ROUTE_HASH else cfg.n_routed * d * 2
    step_bytes = w_gate_up + w_down + w_shared + router + 2 * cfg.T * d * 2
    gbs = step_bytes / (ms / 1e3) / 1e9
    gu_gbs = w_gate_up / (stage_ms["gemm_gate_up"] / 1e3) / 1e9
    del inp, out
    torch.cuda.empty_cache()
    return {"T": cfg.T, "ms_per_step": ms, "tokens_per_s": cfg.T / (ms / 1e3), "experts_touched": touched,
            "bytes_per_step": step_bytes, "achieved_gbs": gbs, "frac": gbs / peaks["hbm_gbs"],
            "frac_of_spec": gbs / SPEC_HBM_GBS, "peak_gbs": peaks["hbm_gbs"], "peak_source": f"{peak_src} (hbm_gbs)",
            "gate_up": {"ms": stage_ms["gemm_gate_up"], "weight_bytes": w_gate_up, "achieved_gbs": gu_gbs,
                        "frac": gu_gbs / peaks["hbm_gbs"]},
            "stage_ms": stage_ms, "clocks": clock_info, "steps": steps, "warmup": warmup}


def run_backward(args, cfg):
    """One GPU: W warm-up and K timed training steps of the layer (an upstream gradient dh
    drawn once): the forward with the pre-activations saved, then dsmoe_backward_gates,
    dsmoe_backward_router (expert-level balance term, alpha 0.01), dsmoe_backward_experts
    and dsmoe_backward_weights, each bracketed by CUDA events on the launching stream.
    Prints one JSON line: per stage ms and its MMA work's TFLOP/s (the GEMM stages), the
    step's time and tokens/s; weight gradients are fp32, summed over the step's tokens.
    With --role-cycles (the profiling build) it also prints the weight-gradient GEMM's role
    counters over the timed steps."""
    if args.role_cycles:
        os.environ.setdefault("DSMOE_LIBRARY", os.path.join(ROOT, "mixture_experts_layer_score_b200",
                                                            "libdsmoe_rolecycles.so"))
    import numpy as np
    import torch
    import workloads as W
    import mixture_experts_layer_score_b200 as M
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = W.make_inputs(cfg, seed=0, device=dev, with_weights=True)
    T, d, N, K, F = cfg.T, cfg.d_model, cfg.n_routed, cfg.top_k, cfg.d_ff
    Ks, Fs = cfg.n_shared, cfg.d_ff_shared
    layer = M.DSMoE(M.cfg_from(cfg, T), inp, device=0)
    M.dsmoe_set_training(layer.handle, True)
    out = layer.alloc_outputs(T, with_scores=True)
    dh = W.normal_bf16((T, d), 1.0, 0, "dh", 0, dev)
    f32 = dict(dtype=torch.float32, device=dev)
    dg = torch.empty((T, K), **f32)
    dY = torch.empty((T * K, d), dtype=torch.bfloat16, device=dev)
    hash_route = cfg.score == W.ROUTE_HASH
    dl = torch.empty((T, N), **f32)
    dx_r = torch.zeros((T, d), **f32)
    dWr = torch.empty((N, d), **f32)
    dx = torch.empty((T, d), **f32)
    dW = [torch.empty(shp, **f32) for shp in ((N, F, d), (N, F, d), (N, d, F))]
    dWs = [torch.empty(shp, **f32) if Ks else None for shp in ((Ks, Fs, d), (Ks, Fs, d), (Ks, d, Fs))]
    stream = torch.cuda.current_stream(dev)
    names = ["forward", "gates", "router", "experts_input", "experts_weights"]
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
    acc = {n: 0.0 for n in names}

    def step(timed):
        if timed:
            ev[0].record(stream)
        layer.forward(inp["x"], token_ids=inp["token_ids"], out=out, stream=stream)
        if timed:
            ev[1].record(stream)
        M.dsmoe_backward_gates(layer.handle, T, dh, out["gates"], dg, dY, stream=stream)
        if timed:
            ev[2].record(stream)
        if not hash_route:
            M.dsmoe_backward_router(layer.handle, T, inp["x"], inp["W_router"], out["topk_idx"], out["gates"],
                                    out["scores"], dg, out["f"], 0.01, dl, dx_r, dWr, stream=stream)
        if timed:
            ev[3].record(stream)
        M.dsmoe_backward_experts(layer.handle, T, dh, dY, inp["W_gate"], inp["W_up"], inp["W_down"],
                                 inp.get("Ws_gate"), inp.get("Ws_up"), inp.get("Ws_down"), dx_r, dx, stream=stream)
        if timed:
            ev[4].record(stream)
        M.dsmoe_backward_weights(layer.handle, T, dh, dY, inp["x"], dW[0], dW[1], dW[2], dWs[0], dWs[1], dWs[2],
                                 stream=stream)
        if timed:
            ev[5].record(stream)

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize(dev)
    if args.role_cycles:
        M.dsmoe_gemm_role_cycles()  # clears the counters
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step(True)
        torch.cuda.synchronize(dev)  # read this step's stage events
        for i, n in enumerate(names):
            acc[n] += ev[i].elapsed_time(ev[i + 1]) / args.steps
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if M.dsmoe_get_status(layer.handle) != M.DSMOE_OK:
        raise SystemExit(f"device status: {M.dsmoe_last_error()}")
    roles = M.dsmoe_gemm_role_cycles().astype(np.float64) if args.role_cycles else None
    layer.close()
    S = T * K
    flops = {"forward": cfg.flops_per_token() * T,
             # dm = W_down^T dy (+ SiLU backward), then du = W_gate^T da + W_up^T db
             "experts_input": 2.0 * d * F * S * 3 + 2.0 * d * Ks * Fs * T * 3,
             # dW_down, dW_gate, dW_up
             "experts_weights": 2.0 * d * F * S * 3 + 2.0 * d * Ks * Fs * T * 3}
    step_ms = sum(acc.values())
    rec = {"metric": "DeepSeekMoE layer training step (forward + backward) tokens/s on 1 B200",
           "workload": cfg.name, "steps": args.steps, "warmup": args.warmup, "dtype": "bf16 (fp32 accumulation, "
           "fp32 weight gradients)", "step_ms": step_ms, "tokens_per_s": T / (step_ms / 1e3),
           "stage_ms": acc, "stage_tflops": {k: flops[k] / (acc[k] / 1e3) / 1e12 for k in flops},
           "step_tflops": sum(flops.values()) / (step_ms / 1e3) / 1e12,
           "note": "stage events on the launching stream, the host synchronising after each step"}
    print(json.dumps(rec), flush=True)
    if roles is not None:
        b = roles[M.ROLE_KINDS.index("weight_grad")]
        b = b[b[:, 0] > 0]
        cyc, ns = b[:, 0], b[:, 1]
        share = {n: float((b[:, i] / cyc).mean()) for i, n in enumerate(M.ROLE_SLOT_NAMES) if i >= 2 and n != "tiles"}
        print(json.dumps({"workload": cfg.name, "kind": "weight_grad", "ctas": int(b.shape[0]), "steps": args.steps,
                          "sm_mhz": float((cyc / ns).mean() * 1e3), "us_per_step": float(ns.max()) / args.steps / 1e3,
                          "tiles_per_cta": float(b[:, 8].mean() / args.steps), "share_of_cycles": share}), flush=True)
    return 0


def run_role_cycles(args, cfg):
    """One GPU: W warm-up forwards, then K forwards whose grouped-GEMM role counters
    (role_clock.cuh) are read back; one JSON line per launch kind with the mean over CTAs
    of each role's share of the CTA's cycles, the SM clock (cycles / ns), the launch time
    and the tensor work per clock cycle against the tensor cores' 8192 bf16 FLOP per SM
    per cycle (dense)."""
    os.environ.setdefault("DSMOE_LIBRARY", os.path.join(ROOT, "mixture_experts_layer_score_b200",
                                                        "libdsmoe_rolecycles.so"))
    import numpy as np
    import torch
    import workloads as W
    import mixture_experts_layer_score_b200 as M
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = W.make_inputs(cfg, seed=0, device=dev, with_weights=True)
    layer = M.DSMoE(M.cfg_from(cfg, cfg.T), inp, device=0)
    out = layer.alloc_outputs(cfg.T)
    for _ in range(args.warmup):
        layer.forward(inp["x"], token_ids=inp["token_ids"], out=out)
    torch.cuda.synchronize(dev)
    M.dsmoe_gemm_role_cycles()  # clears the counters
    for _ in range(args.steps):
        layer.forward(inp["x"], token_ids=inp["token_ids"], out=out)
    torch.cuda.synchronize(dev)
    rc = M.dsmoe_gemm_role_cycles().astype(np.float64)
    if M.dsmoe_get_status(layer.handle) != M.DSMOE_OK:
        raise SystemExit(f"device status: {M.dsmoe_last_error()}")
    slots = int(out["counts"].sum().item())
    layer.close()
    d, F, T = cfg.d_model, cfg.d_ff, cfg.T
    KsFs = cfg.n_shared * cfg.d_ff_shared
    flops = {"gemm_gate_up": 4.0 * d * F * slots, "gemm_down": 2.0 * d * F * slots,
             "shared_gate_up": 4.0 * d * KsFs * T, "shared_down": 2.0 * d * KsFs * T}
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    names = M.ROLE_SLOT_NAMES
    for k, kind in enumerate(M.ROLE_KINDS):
        b = rc[k]
        b = b[b[:, 0] > 0]
        if b.shape[0] == 0:
            continue
        cyc, ns = b[:, 0], b[:, 1]
        share = {n: float((b[:, i] / cyc).mean()) for i, n in enumerate(names) if i >= 2 and n != "tiles"}
        mhz = float((cyc / ns).mean() * 1e3)
        launch_s = float(ns.max()) / args.steps * 1e-9
        rec = {"workload": cfg.name, "kind": kind, "ctas": int(b.shape[0]), "steps": args.steps,
               "sm_mhz": mhz, "us_per_launch": launch_s * 1e6, "tiles_per_cta": float(b[:, 8].mean() / args.steps),
               "tflops": flops[kind] / launch_s / 1e12,
               "tensor_per_cycle": flops[kind] / launch_s / (mhz * 1e6 * sms * 8192),
               "share_of_cycles": share}
        print(json.dumps(rec), flush=True)
    return 0


def main():
    args = parse_args()
    import workloads as W
    cfg = W.get_config(args.workload)
    if args.impl == "reference":
        return run_reference(args, cfg)
    if args.backward:
        return run_backward(args, cfg)
    if args.role_cycles:
        return run_role_cycles(args, cfg)
    return run_native(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
