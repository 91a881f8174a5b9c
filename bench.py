"""Benchmark of the MoE layer forward on B200 (one JSON line on rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one forward pass of the whole layer (router, expert order, gate/up
GEMM + SwiGLU, down GEMM + modulation, combine) over one batch of synthetic
tokens.  The default workload is the XS.2-shaped prefill with skewed routing:
T=32768, d=2048, E=256, top-8, F=Fs=512, a Zipf-ranked router bias giving
the hottest expert 10x the mean load; --workload picks another one.  In the
same process, and with the same weights, two sub-records follow: "decode"
(T=64, one fresh batch per step, 1000 CUDA-graph replays) and
"c2_xs2_small" (T=4096, near-uniform routing), plus "permute" (the
materialised expert-order gather at the main batch's routing).  With N>1
(torchrun) every rank runs an independent replica on its own token batch:
the layer has no exchange step, so there is no collective on the data path.

`value` is device-timed tokens/s (max over ranks) with inputs resident in
HBM; `e2e` is the same metric through the C ABI with the token batch copied
from pinned host memory and the output copied back inside the timed region.
`roofline` is the dominant kernel's algorithmic bytes (or FLOPs) per launch
over its CUDA-event duration on the launching stream.  `cpu_baseline` is the
float64 CPU oracle timed on the host cores: whole batches up to T=4096, a
seeded 2048-token sample of larger ones (per-token time, extrapolated).
"""
import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer fwd tokens/s on 1 B200; expert-GEMM % bf16 peak; decode % HBM BW"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}
L2_BYTES = 126 * 2 ** 20


def load_peaks(path=None):
    """Roofline denominators: the measured figures where MEASURED_PEAKS.json gives them
    (numbers at the top level), the fallback figures for any it lacks; "source" names
    which were measured."""
    path = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    peaks = dict(FALLBACK_PEAKS)
    if not os.path.exists(path):
        return peaks
    try:
        with open(path) as f:
            got = json.load(f)
    except (OSError, ValueError):
        return peaks
    keys = ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")
    measured = [k for k in keys
                if isinstance(got, dict) and isinstance(got.get(k), (int, float)) and got[k] > 0]
    for k in measured:
        peaks[k] = float(got[k])
    if len(measured) == len(keys):
        peaks["source"] = "measured"
    elif measured:
        peaks["source"] = "measured " + ", ".join(measured) + "; fallback for the rest"
    return peaks


def _code_tokens(text):
    """C/C++/CUDA source with comments removed and whitespace collapsed, so that a
    comment-only edit leaves the hash (and the traffic keyed to it) unchanged."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (" ".join(line.split()) for line in "".join(out).splitlines())
    return "\n".join(line for line in lines if line)


# The sources the expert GEMM kernels are compiled from (the kernels whose ncu DRAM
# traffic profiles/ncu_traffic.json records), including the shared header of all kernels.
GEMM_SOURCES = ("gemm_common.cuh", "kernels.h", "moe_gemm.cu", "moe_gemm_pair.cu", "ptx.cuh",
                "status.cuh")


def kernel_sources_sha1():
    """Hash of the expert GEMM kernels' sources (code only: comments and blank space
    ignored, and the public header they include): DRAM traffic taken by ncu is valid only
    for these."""
    import hashlib
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "sparse_moe_layer_select_b200", "csrc")
    paths = [os.path.join(csrc, n) for n in GEMM_SOURCES] + [os.path.join(ROOT, "include", "moe.h")]
    for path in paths:
        with open(path, encoding="utf-8") as f:
            h.update(os.path.basename(path).encode() + b"\0" + _code_tokens(f.read()).encode())
    return h.hexdigest()


def measured_traffic(workload, stage, fp8=False):
    """dram__bytes_read.sum + dram__bytes_write.sum per launch of a stage's kernel, from the
    committed ncu summary, or None when absent or taken on other kernel sources."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    e = rec.get("entries", {}).get(f"{workload}{'/fp8' if fp8 else ''}/{stage}")
    if e is None or rec.get("sources_sha1") != kernel_sources_sha1():
        return None
    return e["dram_bytes_per_launch"]


def max_over_ranks(value, world, device="cuda"):
    """The largest of every rank's value (each rank calls it); the value itself for one rank."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_step, steps, world, seconds):
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return tokens_per_step * steps * world / seconds


def replica_seed(w, rank):
    """Seed of a replica's token batch: rank 0 uses the workload's seed, the others their own."""
    return w.seed + rank


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ----------------------------------------------------------------- work model

def stage_work(w, counts, fp8=False):
    """Algorithmic FLOPs and bytes per launch of each stage.

    "bytes" are the method's own bytes (the layer's inputs and outputs: every touched
    expert's weights once, the shared expert, the router, x and y), so that the stages sum
    to the layer's algorithmic traffic; "inter_bytes" are the intermediates the stage moves
    through HBM as built (h, the routed contributions, the shared output), reported
    separately.  No padding, no re-reads.  fp8: expert weights of one byte per element,
    plus one float32 scale per weight row."""
    T, d, E, k, F, Fs = w.T, w.d_model, w.E, w.k, w.F, w.Fs
    touched = int((np.asarray(counts) > 0).sum())
    bf = 2
    wb = 1 if fp8 else 2
    rows = T * k
    h_bytes = (rows * F + T * Fs) * bf
    slot_bytes = T * (k + (1 if Fs else 0)) * d * bf
    scales1 = 4 * (touched * 2 * F + 2 * Fs) if fp8 else 0
    scales2 = 4 * (touched * d + d) if fp8 else 0
    return {
        "router": {"flops": 2 * T * d * E, "bytes": T * d * bf + E * d * bf + T * k * 8,
                   "inter_bytes": 0},
        "index": {"flops": 0, "bytes": T * k * 4 * 3 + E * 8, "inter_bytes": 0},
        "gemm1_swiglu": {"flops": 4 * d * F * rows + 4 * d * Fs * T,
                         "bytes": touched * 2 * F * d * wb + 2 * Fs * d * wb + T * d * bf + scales1,
                         "inter_bytes": h_bytes, "x_bytes": T * d * bf},
        "gemm2_down_scale": {"flops": 2 * d * F * rows + 2 * d * Fs * T,
                             "bytes": touched * d * F * wb + d * Fs * wb + scales2,
                             "inter_bytes": h_bytes + slot_bytes},
        "combine": {"flops": 0, "bytes": T * d * bf, "inter_bytes": slot_bytes},
    }


def layer_bytes(work):
    """The layer's algorithmic bytes per step: the sum of the stages' method bytes with x
    counted once (the router and the gate/up GEMM both read it; the routing arrays, a few
    hundred KB, are counted where they are written and read)."""
    return sum(v["bytes"] for v in work.values()) - work["gemm1_swiglu"]["x_bytes"]


# ----------------------------------------------------------------- clocks

class ClockSampler:
    def __init__(self, index, path):
        self.path = path
        self.proc = None
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
             "utilization.gpu")
        try:
            self.f = open(path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def wait_first_sample(self, timeout=3.0):
        t0 = time.time()
        while self.proc is not None and time.time() - t0 < timeout:
            self.f.flush()
            if os.path.getsize(self.path) > 0:
                return
            time.sleep(0.05)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    util = float(parts[9])
                    clk = float(parts[1])
                    mx = float(parts[2])
                except ValueError:
                    continue
                if util < 50:  # idle samples say nothing about the clock under load
                    continue
                sm.append(clk)
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "window": "warm-up start to end of timed region, "
                                              "samples with utilization >= 50%"}


# ----------------------------------------------------------------- CPU baseline

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


# Tokens per oracle call for workloads whose full batch is too large to time on the host:
# the per-token time of such a sample, times T, stands for the whole batch ("extrapolated").
ORACLE_SAMPLE_TOKENS = 2048


def oracle_weights(h):
    """The oracle's weights widened once to float64 (outside any timed region), so that a
    timed call spends its time on the layer's arithmetic; the oracle takes float arrays as
    they are."""
    from oracle import moe_oracle as O
    return {k: (None if v is None else (O.bf16_to_f64(v) if v.dtype == np.uint16 else v))
            for k, v in h.items()}


def oracle_call(w, h64, x, fp8=None):
    """One timed oracle forward on the token rows x (bf16 bits); returns seconds."""
    from oracle import moe_oracle as O
    t0 = time.perf_counter()
    if fp8 is not None:
        O.moe_forward_fp8(x, h64["w_router"], fp8, w.k, router_bias=h64.get("router_bias"),
                          routed_scaling_factor=w.routed_scaling_factor)
    else:
        O.moe_forward(x, h64["w_router"], h64["w_gate"], h64["w_up"], h64["w_down"], w.k,
                      router_bias=h64.get("router_bias"), ws_gate=h64.get("ws_gate"),
                      ws_up=h64.get("ws_up"), ws_down=h64.get("ws_down"),
                      routed_scaling_factor=w.routed_scaling_factor)
    return time.perf_counter() - t0


def oracle_tokens(w, n, seed):
    """n seeded token rows of the workload's x (all T rows, in order, when n >= T): the
    same generator and element indices as the device batch."""
    from sparse_moe_layer_select_b200 import inputs as I
    if n >= w.T:
        return I.generate_numpy((w.T, w.d_model), w.seed, I.TID_X, w.sigma_x)
    rows = np.sort(np.random.default_rng(seed).choice(w.T, size=n, replace=False))
    return np.stack([I.generate_numpy((w.d_model,), w.seed, I.TID_X, w.sigma_x,
                                      start=int(r) * w.d_model) for r in rows])


def oracle_unit(w):
    """Tokens per timed oracle call: the whole batch when it is small (T <= 4096; a decode
    batch is one such call), else a seeded ORACLE_SAMPLE_TOKENS-token sample."""
    return w.T if w.T <= 4096 else ORACLE_SAMPLE_TOKENS


def cpu_baseline(w, h64, min_seconds=10.0, max_calls=16, fp8=None):
    """The float64 oracle, as it stands, on the host cores: repeated calls of oracle_unit(w)
    tokens (fresh seeded samples) until about min_seconds of CPU work; tokens per second."""
    n = oracle_unit(w)
    secs, toks, calls = 0.0, 0, 0
    while calls < max_calls and (secs < min_seconds or calls == 0):
        secs += oracle_call(w, h64, oracle_tokens(w, n, seed=1000 + calls), fp8=fp8)
        toks += n
        calls += 1
    full = n >= w.T
    what = (f"the whole batch of {w.T} tokens through the float64 oracle, {calls} call(s)"
            if full else
            f"{calls} seeded samples of {n} of the {w.T} tokens through the float64 oracle "
            f"(extrapolated: per-token time of the samples stands for the batch)")
    return {"value": toks / secs, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{what}; {secs:.1f} s, weights widened to float64 once, untimed"}


# ----------------------------------------------------------------- our arm

# Workloads measured beside the main one in the same process (as sub-records of its line)
# when they share its weights: the decode batch (the metric's HBM target) and the T=4096
# small batch.
EXTRA_WORKLOADS = ("c5_decode", "c2_xs2_small")


def shares_weights(a, b):
    keys = ("d_model", "num_experts", "moe_intermediate_size", "shared_intermediate_size",
            "sigma_w", "sigma_router", "seed")
    return all(getattr(a, k) == getattr(b, k) for k in keys)


class Bench:
    """Times one workload on one layer: warm-up, a CUDA-graph replay loop of K steps
    bracketed by events on the layer's stream, and a second, eagerly launched pass with an
    event at every stage boundary (events inside a captured graph cannot be timed)."""

    def __init__(self, M, torch, layer, w, x_buf, ring, world, rank, local, graph=True,
                 label="main"):
        self.M, self.torch, self.layer, self.w = M, torch, layer, w
        self.x_buf, self.ring = x_buf, ring
        self.world, self.rank, self.local = world, rank, local
        self.use_graph, self.label = graph, label
        self.y = torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda")
        self.stream = torch.cuda.current_stream()
        self.graph = None
        # inputs larger than L2 need no flush; smaller ones get one before every step
        resident = sum(t.numel() * t.element_size() for t in layer.W.values() if t is not None)
        self.flush = resident < 2 * L2_BYTES
        self.flush_buf = (torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device="cuda")
                          if self.flush else None)
        self.resident = resident

    def step(self, i, events=None):
        if self.ring is not None:  # a fresh batch every step (decode)
            self.x_buf.copy_(self.ring[i % self.ring.shape[0]], non_blocking=True)
        if self.graph is not None and events is None:
            self.graph.replay()
            return
        if events is not None:
            self.M.profile_next_forward(events)
        self.layer.forward(self.x_buf, self.y)

    def check_status(self):
        code, site = self.M.read_device_status(self.layer.ws)
        if code != 0:
            raise RuntimeError(f"{self.label}: device status {self.M.status_string(code)} "
                               f"at site {site}")

    def warm(self, warmup, min_seconds=0.3):
        torch = self.torch
        t_w = time.time()
        i = 0
        while i < warmup or time.time() - t_w < min_seconds:
            self.step(i)
            i += 1
            if i % 16 == 0:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        self.check_status()
        self.launches_per_step = self.M.last_launch_count() + (1 if self.ring is not None else 0)
        if self.use_graph:
            self.graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.graph):
                self.layer.forward(self.x_buf, self.y)
            for i in range(3):
                self.step(i)
            torch.cuda.synchronize()

    def timed(self, steps, ev=None):
        torch = self.torch
        if self.flush:
            total = 0.0
            for i in range(steps):
                self.flush_buf.fill_(i)
                s0 = torch.cuda.Event(enable_timing=True)
                s1 = torch.cuda.Event(enable_timing=True)
                s0.record(self.stream)
                self.step(i, None if ev is None else ev[i])
                s1.record(self.stream)
                s1.synchronize()
                total += s0.elapsed_time(s1) / 1e3
            return total
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(self.stream)
        for i in range(steps):
            self.step(i, None if ev is None else ev[i])
        t1.record(self.stream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / 1e3

    def run(self, steps, warmup, clock_path):
        """Warm-up and the timed steps with clock samples; then the stage-marked pass."""
        torch, M = self.torch, self.M
        clocks = ClockSampler(self.local, clock_path)
        clocks.wait_first_sample()
        self.warm(warmup)
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()
        elapsed = self.timed(steps)
        if self.world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        clk = clocks.stop()
        elapsed = max_over_ranks(elapsed, self.world)
        self.check_status()
        n_st = len(M.FORWARD_STAGES)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_st + 1)]
              for _ in range(steps)]
        marked = self.timed(steps, ev)
        stage_ms = {name: float(np.mean([ev[i][j].elapsed_time(ev[i][j + 1])
                                         for i in range(steps)]))
                    for j, name in enumerate(M.FORWARD_STAGES)}
        return {"elapsed": elapsed, "ms_per_step": elapsed / steps * 1e3, "stage_ms": stage_ms,
                "marked_ms": marked / steps * 1e3, "clocks": clk}


def roofline(work, stage_ms, peaks, stage):
    t = stage_ms[stage] / 1e3
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    ai = work[stage]["flops"] / max(work[stage]["bytes"], 1)
    if ai < ridge:
        roof = {"kernel": stage, "bound": "hbm", "achieved": work[stage]["bytes"] / t / 1e9,
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "algorithmic_bytes": work[stage]["bytes"]}
    else:
        roof = {"kernel": stage, "bound": "tensor", "achieved": work[stage]["flops"] / t / 1e12,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "algorithmic_flops": work[stage]["flops"]}
        # The GEMMs run back to back in the timed loop; under the 1 kW cap the clocks settle
        # below max (see "clocks"), which the sustained figure reflects.
        roof["peak_sustained"] = peaks["bf16_tflops_sustained"]
        roof["frac_of_sustained"] = roof["achieved"] / peaks["bf16_tflops_sustained"]
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["peak_source"] = peaks["source"] + " (burst)"
    return roof


def expert_gemm_summary(work, stage_ms, peaks):
    gemm_stages = ("gemm1_swiglu", "gemm2_down_scale")
    g_flops = sum(work[s]["flops"] for s in gemm_stages)
    g_time = sum(stage_ms[s] for s in gemm_stages) / 1e3
    tf = g_flops / g_time / 1e12
    gbs = sum(work[s]["bytes"] for s in gemm_stages) / g_time / 1e9
    return {"tflops": tf, "frac_of_bf16_peak": tf / peaks["bf16_tflops"],
            "frac_of_bf16_sustained": tf / peaks["bf16_tflops_sustained"],
            "hbm_gbs": gbs, "frac_of_hbm_peak": gbs / peaks["hbm_gbs"],
            "ms": g_time * 1e3}


def host_oracle_inputs(dev, P, torch):
    """Device weights copied to the host for the oracle, widened to float64 once."""
    h = {k: (P.to_numpy_bf16(v) if v is not None and v.dtype == torch.bfloat16 else
             (None if v is None else v.cpu().numpy()))
         for k, v in dev.items() if k != "x"}
    return oracle_weights(h)


def run_ours(args):
    import torch
    import torch.distributed as dist

    from sparse_moe_layer_select_b200 import inputs as I
    from sparse_moe_layer_select_b200 import moe as M
    from tests import parity as P  # bf16 -> numpy helper only

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    M.lib()
    peaks = load_peaks()

    w = I.get(args.workload)
    dev = I.device_inputs(w)
    if rank > 0:  # each replica routes its own tokens
        I.generate_cuda(dev["x"], replica_seed(w, rank), I.TID_X, w.sigma_x)
    decode = w.decode_batches > 0
    ring = I.device_decode_ring(w, min(w.decode_batches, 1000)) if decode else None
    flags = ((M.MOE_FLAG_GEMM_SINGLE_CTA if args.single_cta else 0)
             | (M.MOE_FLAG_GEMM_PAIR if args.pair else 0)
             | (M.MOE_FLAG_COMBINE_REDUCE if args.combine == "reduce" else 0)
             | (M.MOE_FLAG_FUSED_EXPERTS if args.fused else 0))
    layer = M.MoeLayer(dev, w.d_model, w.E, w.k, w.F, w.Fs, w.routed_scaling_factor,
                       max_tokens=w.T, flags=flags, fp8=args.fp8)
    clock_dir = os.environ.get("MOE_CLOCKS_DIR", "/tmp")
    main = Bench(M, torch, layer, w, dev["x"], ring, world, rank, local,
                 graph=not args.no_graph, label=w.name)
    steps = max(args.steps, 1)
    res = main.run(steps, args.warmup, os.path.join(clock_dir, f"clocks_{w.name}_r{rank}.csv"))
    counts = layer.routing["counts"].cpu().numpy()
    work = stage_work(w, counts, fp8=args.fp8)
    stage_ms = res["stage_ms"]
    dom = max(("gemm1_swiglu", "gemm2_down_scale"), key=lambda s: stage_ms[s])
    roof = roofline(work, stage_ms, peaks, dom)
    roof["traffic"] = measured_traffic(w.name, dom, fp8=args.fp8)
    expert = expert_gemm_summary(work, stage_ms, peaks)
    lb = layer_bytes(work)

    # end to end through the C ABI: pinned host batch in, host output back, every step
    e2e = None
    if not args.no_e2e:
        e2e = end_to_end(M, torch, layer, w, dev["x"], ring, steps, world,
                         copy_streams=args.copy_streams)

    # the materialised permutation (moe_permute with x_perm) at this batch's routing
    permute = None
    if not args.no_extras and not args.fp8:
        permute = time_permute(M, torch, layer, w, dev["x"], steps, peaks)

    # workloads sharing these weights, measured in the same process (decode: the metric's
    # HBM target, over its 1000 fresh batches)
    extras = {}
    if not args.no_extras and not args.fp8:
        for name in EXTRA_WORKLOADS:
            wx = I.get(name)
            if name == w.name or not shares_weights(w, wx):
                continue
            dx = dict(dev)
            dx["router_bias"] = None if I.router_bias(wx) is None else \
                torch.from_numpy(I.router_bias(wx)).cuda()
            dx["x"] = torch.empty((wx.T, wx.d_model), dtype=torch.bfloat16, device="cuda")
            I.generate_cuda(dx["x"], replica_seed(wx, rank), I.TID_X, wx.sigma_x)
            # the same prepared fp16 down projections as the main layer
            dx["w_down_f16"], dx["ws_down_f16"] = layer.W["w_down_f16"], layer.W.get("ws_down_f16")
            lx = M.MoeLayer(dx, wx.d_model, wx.E, wx.k, wx.F, wx.Fs, wx.routed_scaling_factor,
                            max_tokens=wx.T, flags=flags | M.MOE_FLAG_DOWN_F16, prepare=False)
            rx = I.device_decode_ring(wx, min(wx.decode_batches, 1000)) \
                if wx.decode_batches else None
            bx = Bench(M, torch, lx, wx, dx["x"], rx, world, rank, local,
                       graph=not args.no_graph, label=name)
            sx = args.decode_steps if wx.decode_batches else steps
            r = bx.run(sx, max(args.warmup, 10),
                       os.path.join(clock_dir, f"clocks_{name}_r{rank}.csv"))
            cx = lx.routing["counts"].cpu().numpy()
            wk = stage_work(wx, cx)
            rec = {"workload": name, "T": wx.T, "steps": sx,
                   "value": job_tokens_per_s(wx.T, sx, world, r["elapsed"]), "unit": "tokens/s",
                   "ms_per_step": r["ms_per_step"], "stages_ms": r["stage_ms"],
                   "stages_pass_ms_per_step": r["marked_ms"],
                   "expert_gemm": expert_gemm_summary(wk, r["stage_ms"], peaks),
                   "gpu_launches": bx.launches_per_step * sx, "clocks": r["clocks"],
                   "l2": "L2 flushed between steps" if bx.flush else
                         f"inputs larger than L2 ({bx.resident / 1e9:.2f} GB resident)"}
            byt = layer_bytes(wk)
            rec["layer_hbm"] = {"algorithmic_bytes_per_step": byt,
                                "touched_experts": int((cx > 0).sum()),
                                "gbs": byt / (r["elapsed"] / sx) / 1e9,
                                "frac_of_hbm_peak": byt / (r["elapsed"] / sx) / 1e9 / peaks["hbm_gbs"],
                                "peak_source": peaks["source"]}
            if wx.decode_batches:
                rec["fresh_batches"] = int(rx.shape[0])
            extras[name] = rec
            del lx, bx, rx, dx
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        h64 = host_oracle_inputs(dev, P, torch)
        fp8 = None
        if args.fp8:  # the oracle's own e4m3 weights (made once, not timed)
            from oracle import moe_oracle as O
            fp8 = O.quantize_experts_fp8(h64["w_gate"], h64["w_up"], h64["w_down"],
                                         h64.get("ws_gate"), h64.get("ws_up"), h64.get("ws_down"))
        cpu = cpu_baseline(w, h64, fp8=fp8)
        for name, rec in extras.items():
            wx = I.get(name)
            hx = dict(h64, router_bias=I.router_bias(wx))
            rec["cpu_baseline"] = cpu_baseline(wx, hx, min_seconds=3.0, max_calls=4)
        del h64

    line = {
        "metric": METRIC, "value": job_tokens_per_s(w.T, steps, world, res["elapsed"]),
        "unit": "tokens/s",
        "n_gpus": world, "steps": steps, "warmup": args.warmup,
        "ms_per_step": res["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3" if args.fp8 else "bf16",
        "data": "synthetic (seeded Philox normal, bf16)",
        "config": {"workload": w.name, "T": w.T, "d_model": w.d_model, "num_experts": w.E,
                   "num_experts_per_tok": w.k, "moe_intermediate_size": w.F,
                   "shared_intermediate_size": w.Fs, "routed_scaling_factor": w.routed_scaling_factor,
                   "router_bias": "zipf" if w.zipf_s else None, "parallelism": f"replicas x{world}",
                   "gemm_engine": ("single-CTA M=128" if args.single_cta or args.fp8 else
                                   "CTA-pair M=256" if args.pair else
                                   "auto (gate/up single-CTA; down on CTA pairs when T*k >= 256*E)"),
                   "experts": ("e4m3 weights, x and h with per-row fp32 scales" if args.fp8 else
                               "fused kernel: bf16 gate/up, fp16 h in tensor memory, fp16 "
                               "W_down copy" if args.fused else
                               "bf16 weights (fp16 copy of W_down), fp16 h"),
                   "combine": ("fp32 reduce-adds into token rows in the down GEMM, then bf16"
                               if args.combine == "reduce" or args.fused else
                               "fp16 contribution rows, deterministic fp32 sum per token"),
                   "l2": "L2 flushed between steps" if main.flush else
                         f"inputs larger than L2 ({main.resident / 1e9:.2f} GB resident)"},
        "roofline": roof, "expert_gemm": expert,
        "layer_hbm": {"algorithmic_bytes_per_step": lb,
                      "gbs": lb / (res["elapsed"] / steps) / 1e9,
                      "frac_of_hbm_peak": lb / (res["elapsed"] / steps) / 1e9 / peaks["hbm_gbs"]},
        "stages_ms": stage_ms, "stages_pass_ms_per_step": res["marked_ms"],
        "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": main.launches_per_step * steps, "clocks": res["clocks"],
        "cuda_graph": main.graph is not None,
    }
    if decode:
        line["decode_hbm"] = dict(line["layer_hbm"], touched_experts=int((counts > 0).sum()))
    if permute is not None:
        line["permute"] = permute
    for name, rec in extras.items():
        line["decode" if I.get(name).decode_batches else name] = rec
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def end_to_end(M, torch, layer, w, x_buf, ring, steps, world, copy_streams=1):
    """Through the public API with host buffers: every step copies its own input from
    pinned host memory and reads its own output back.  The input copy, the layer and the
    output copy run on their own streams with two device buffers, so step i's copies
    overlap the layer of steps i-1 / i+1; each copy is split into `copy_streams` row
    blocks on as many streams, so that several copy engines share a direction."""
    decode = ring is not None
    n_host = min(steps, 64) if decode else 1
    hx = torch.empty((n_host, w.T, w.d_model), dtype=torch.bfloat16, pin_memory=True)
    hx.copy_(ring[:n_host].cpu() if decode else x_buf.cpu().unsqueeze(0))
    hy = [torch.empty((w.T, w.d_model), dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    xd = [torch.empty_like(x_buf) for _ in range(2)]
    yd = [torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    nc = max(1, min(copy_streams, w.T))
    s_in = [torch.cuda.Stream() for _ in range(nc)]
    s_out = [torch.cuda.Stream() for _ in range(nc)]
    s_c = torch.cuda.current_stream()
    cuts = [w.T * c // nc for c in range(nc + 1)]

    def run_e2e(n):
        ev_in = [[torch.cuda.Event() for _ in range(nc)] for _ in range(n)]
        ev_c = [torch.cuda.Event() for _ in range(n)]
        ev_out = [[torch.cuda.Event() for _ in range(nc)] for _ in range(n)]
        for i in range(n):
            b = i % 2
            for c in range(nc):
                lo, hi = cuts[c], cuts[c + 1]
                if i >= 2:
                    s_in[c].wait_event(ev_c[i - 2])      # the layer of step i-2 has read xd[b]
                with torch.cuda.stream(s_in[c]):
                    xd[b][lo:hi].copy_(hx[i % n_host][lo:hi], non_blocking=True)
                ev_in[i][c].record(s_in[c])
                s_c.wait_event(ev_in[i][c])
            if i >= 2:
                for c in range(nc):
                    s_c.wait_event(ev_out[i - 2][c])  # yd[b] of step i-2 is back on the host
            layer.forward(xd[b], yd[b], stream=s_c)
            ev_c[i].record(s_c)
            for c in range(nc):
                lo, hi = cuts[c], cuts[c + 1]
                s_out[c].wait_event(ev_c[i])
                with torch.cuda.stream(s_out[c]):
                    hy[b][lo:hi].copy_(yd[b][lo:hi], non_blocking=True)
                ev_out[i][c].record(s_out[c])
        return [ev_out[-1][c] for c in range(nc)]

    run_e2e(2)
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(s_c)
    for st in s_in + s_out:
        st.wait_event(a)
    last = run_e2e(steps)
    for ev in last:
        s_c.wait_event(ev)
    b.record(s_c)
    torch.cuda.synchronize()
    te = max_over_ranks(a.elapsed_time(b) / 1e3, world)
    return {"value": job_tokens_per_s(w.T, steps, world, te), "unit": "tokens/s",
            "h2d_bytes_per_step": w.T * w.d_model * 2, "d2h_bytes_per_step": w.T * w.d_model * 2,
            "overlap": f"input copy, layer and output copy on their own streams, two buffers; "
                       f"each copy in {nc} row blocks on {nc} streams"}


def time_permute(M, torch, layer, w, x, steps, peaks):
    """moe_permute with the materialised gather x_perm[r] = x[perm[r] / k] on this batch's
    routing (left by the last forward): CUDA events on the launching stream around K calls.
    Bytes: every routed row read once and written once (2 * T*k * d * 2), plus the index's
    own reads and writes."""
    d = M.dims_for(w)
    ws = M.alloc_workspace(d)
    E, k, T = w.E, w.k, w.T
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    x_perm = torch.empty((T * k, w.d_model), dtype=torch.bfloat16, device="cuda")
    idx = layer.routing["topk_idx"][:T]
    for _ in range(3):
        M.permute(d, idx, counts, offsets, perm, ws, x=x, x_perm=x_perm)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        M.permute(d, idx, counts, offsets, perm, ws, x=x, x_perm=x_perm)
    t1.record(stream)
    torch.cuda.synchronize()
    code, site = M.read_device_status(ws)
    if code != 0:
        raise RuntimeError(f"permute: device status {M.status_string(code)} at site {site}")
    t = t0.elapsed_time(t1) / 1e3 / steps
    byt = 2 * T * k * w.d_model * 2 + T * k * 4 * 3 + E * 8
    out = {"ms": t * 1e3, "bytes": byt, "gbs": byt / t / 1e9,
           "frac_of_hbm_peak": byt / t / 1e9 / peaks["hbm_gbs"], "launches": M.last_launch_count(),
           "what": "moe_permute with x_perm: index builder + gather of every routed row"}
    del x_perm, ws
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------- reference arm

def run_reference(args):
    """The float64 CPU oracle, as it stands, on the host cores: each step one oracle call on
    oracle_unit(w) tokens of the workload (the same unit as this arm's cpu_baseline, so the
    two rates agree)."""
    world, rank, _ = dist_env()
    if rank != 0:
        return
    from sparse_moe_layer_select_b200 import inputs as I
    w = I.get(args.workload)
    try:
        import torch
        gpu = torch.cuda.is_available()
    except Exception:
        gpu = False
    if gpu:  # input generation only (the same bits as the host generator); timing is CPU-only
        from tests import parity as P
        h = {}
        for name, shape, tid, sigma in I.tensor_specs(w):
            if name != "x":
                t = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
                I.generate_cuda(t, w.seed, tid, sigma)
                h[name] = P.to_numpy_bf16(t)
                del t
        torch.cuda.synchronize()
    else:
        h = {name: I.generate_numpy_chunked(shape, w.seed, tid, sigma)
             for name, shape, tid, sigma in I.tensor_specs(w) if name != "x"}
    h["router_bias"] = I.router_bias(w)
    h64 = oracle_weights(h)
    n = oracle_unit(w)
    for i in range(args.warmup):
        oracle_call(w, h64, oracle_tokens(w, n, seed=100 + i))
    tot = 0.0
    for i in range(args.steps):
        tot += oracle_call(w, h64, oracle_tokens(w, n, seed=200 + i))
    v = n * args.steps / tot
    full = n >= w.T
    sample = (f"the whole batch of {w.T} tokens per step" if full else
              f"a seeded sample of {n} of the {w.T} tokens per step (per-token time stands for "
              f"the batch: extrapolated)")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded Philox normal, bf16)",
        "config": {"workload": w.name, "T": w.T, "d_model": w.d_model, "num_experts": w.E,
                   "num_experts_per_tok": w.k, "moe_intermediate_size": w.F,
                   "shared_intermediate_size": w.Fs,
                   "routed_scaling_factor": w.routed_scaling_factor,
                   "router_bias": "zipf" if w.zipf_s else None, "parallelism": "host cores"},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"{sample} through the float64 oracle; weights widened to "
                                   f"float64 once, untimed"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="c3_xs2_prefill_zipf")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the sub-records (decode, T=4096, materialised permute)")
    ap.add_argument("--decode-steps", type=int, default=1000,
                    help="timed graph replays of the decode sub-record (one fresh batch each)")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch each step's kernels instead of replaying a CUDA graph")
    ap.add_argument("--single-cta", action="store_true",
                    help="force the single-CTA (M=128) expert GEMM engine")
    ap.add_argument("--pair", action="store_true",
                    help="force the CTA-pair (M=256) expert GEMM engine")
    ap.add_argument("--combine", default="slots", choices=["slots", "reduce"],
                    help="slots: fp16 contribution rows + deterministic combine kernel; reduce: "
                         "the down GEMM adds into fp32 token rows (MOE_FLAG_COMBINE_REDUCE)")
    ap.add_argument("--fused", action="store_true",
                    help="the fused expert kernel (h in tensor memory; MOE_FLAG_FUSED_EXPERTS)")
    ap.add_argument("--copy-streams", type=int, default=1,
                    help="streams (row blocks) each end-to-end host<->device copy is split over "
                         "(2 or 4 measured slower than 1 at the T=32768 prefill)")
    ap.add_argument("--fp8", action="store_true",
                    help="FP8 (e4m3) expert weights: moe_prepare_fp8 + moe_forward_fp8")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
