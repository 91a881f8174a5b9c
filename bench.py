"""Benchmark of the MoE layer forward on B200 (one JSON line on rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one forward pass of the whole layer (router, expert order, gate/up
GEMM + SwiGLU, down GEMM + modulation, combine) over one batch of synthetic
tokens.  The default workload is the XS.2-shaped layer at T=4096
(d=2048, E=256, top-8, F=Fs=512); --workload picks another one.  With N>1
(torchrun) every rank runs an independent replica on its own token batch:
the layer has no exchange step, so there is no collective on the data path.

`value` is device-timed tokens/s (max over ranks) with inputs resident in
HBM; `e2e` is the same metric through the C ABI with the token batch copied
from pinned host memory and the output copied back inside the timed region.
`roofline` is the dominant kernel's algorithmic bytes (or FLOPs) per launch
over its CUDA-event duration on the launching stream.  `cpu_baseline` is the
float64 CPU oracle timed on a bounded sample of the same workload.
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


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    return dict(FALLBACK_PEAKS)


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
    """Algorithmic FLOPs and bytes per launch of each stage (no padding, no re-reads).
    fp8: expert weights of one byte per element (plus one float32 scale per row)."""
    T, d, E, k, F, Fs = w.T, w.d_model, w.E, w.k, w.F, w.Fs
    touched = int((np.asarray(counts) > 0).sum())
    bf = 2
    wb = 1 if fp8 else 2
    rows = T * k
    h_bytes = (rows * F + T * Fs) * bf
    scales = 4 * (touched * (2 * F + d) + 2 * Fs + d) if fp8 else 0
    return {
        "router": {"flops": 2 * T * d * E, "bytes": T * d * bf + E * d * bf + T * k * 8},
        "index": {"flops": 0, "bytes": T * k * 4 * 3 + E * 8},
        "gemm1_swiglu": {"flops": 4 * d * F * rows + 4 * d * Fs * T,
                         "bytes": touched * 2 * F * d * wb + 2 * Fs * d * wb + T * d * bf + h_bytes
                         + scales},
        "gemm2_down_scale": {"flops": 2 * d * F * rows + 2 * d * Fs * T,
                             "bytes": touched * d * F * wb + d * Fs * wb + h_bytes
                             + T * (k + (1 if Fs else 0)) * d * bf},
        "combine": {"flops": 0, "bytes": T * (k + (1 if Fs else 0)) * d * bf + T * d * bf},
    }


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


def oracle_sample(w, h_small, n_tokens, seed=7, fp8=None):
    """Time the oracle on n_tokens tokens of the workload (its x rows are regenerated on the host).
    fp8: the oracle's FP8 expert weights (the FP8 forward is timed then)."""
    from oracle import moe_oracle as O
    from sparse_moe_layer_select_b200 import inputs as I
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(w.T, size=min(n_tokens, w.T), replace=False))
    x = np.stack([I.generate_numpy((w.d_model,), w.seed, I.TID_X, w.sigma_x, start=int(r) * w.d_model)
                  for r in rows])
    t0 = time.perf_counter()
    if fp8 is not None:
        O.moe_forward_fp8(x, h_small["w_router"], fp8, w.k, router_bias=h_small.get("router_bias"),
                          routed_scaling_factor=w.routed_scaling_factor)
    else:
        O.moe_forward(x, h_small["w_router"], h_small["w_gate"], h_small["w_up"], h_small["w_down"],
                      w.k, router_bias=h_small.get("router_bias"), ws_gate=h_small.get("ws_gate"),
                      ws_up=h_small.get("ws_up"), ws_down=h_small.get("ws_down"),
                      routed_scaling_factor=w.routed_scaling_factor)
    return time.perf_counter() - t0, len(rows)


def cpu_sample_size(w):
    # about 10-30 s of float64 work on a many-core host
    per_tok = 6 * w.d_model * (w.F * w.k + w.Fs)
    return int(max(16, min(w.T, 4e12 / per_tok / 100)))


# ----------------------------------------------------------------- our arm

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

    w = I.get(args.workload)
    dev = I.device_inputs(w)
    if rank > 0:  # each replica routes its own tokens
        I.generate_cuda(dev["x"], replica_seed(w, rank), I.TID_X, w.sigma_x)
    decode = w.decode_batches > 0
    ring = I.device_decode_ring(w, min(w.decode_batches, 1000)) if decode else None
    layer = M.MoeLayer(dev, w.d_model, w.E, w.k, w.F, w.Fs, w.routed_scaling_factor,
                       max_tokens=w.T,
                       flags=(M.MOE_FLAG_GEMM_SINGLE_CTA if args.single_cta else 0)
                       | (M.MOE_FLAG_GEMM_PAIR if args.pair else 0), fp8=args.fp8)
    x_buf = dev["x"]
    y = torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()
    working_set = sum(t.numel() * t.element_size() for t in dev.values() if t is not None)
    flush = working_set < 2 * L2_BYTES
    flush_buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device="cuda") if flush else None

    graph = None

    def step(i, events=None):
        """One step: a graph replay when a graph is captured, else (and always for the
        stage-marked pass) the layer's kernels launched one by one."""
        if decode:
            x_buf.copy_(ring[i % ring.shape[0]], non_blocking=True)
        if graph is not None and events is None:
            graph.replay()
            return
        if events is not None:
            M.profile_next_forward(events)
        layer.forward(x_buf, y)

    clocks = ClockSampler(local, os.environ.get("MOE_CLOCKS_CSV", f"/tmp/clocks_rank{rank}.csv"))
    clocks.wait_first_sample()
    # warm-up: at least W steps and at least 0.3 s, so clocks settle under load
    t_w = time.time()
    i = 0
    while i < args.warmup or time.time() - t_w < 0.3:
        step(i)
        i += 1
        if i % 16 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    code, site = M.read_device_status(layer.ws)
    if code != 0:
        raise RuntimeError(f"device status {M.status_string(code)} at site {site}")
    launches_per_step = M.last_launch_count() + (1 if decode else 0)
    if not args.no_graph:
        # the layer is captured once in a CUDA graph and replayed per step (decode: per
        # fresh batch copied into the same input buffer)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            layer.forward(x_buf, y)
        for i in range(3):
            step(i)
        torch.cuda.synchronize()

    n_st = len(M.FORWARD_STAGES)

    def timed_loop(ev=None):
        """K steps bracketed by events on the layer's stream; ev: per-step stage markers."""
        if flush:
            total = 0.0
            for i in range(args.steps):
                flush_buf.fill_(i)
                s0 = torch.cuda.Event(enable_timing=True)
                s1 = torch.cuda.Event(enable_timing=True)
                s0.record(stream)
                step(i, None if ev is None else ev[i])
                s1.record(stream)
                s1.synchronize()
                total += s0.elapsed_time(s1) / 1e3
            return total
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(args.steps):
            step(i, None if ev is None else ev[i])
        t1.record(stream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / 1e3

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    # the timed steps carry no stage markers (events recorded between the layer's kernels);
    # a second, marked pass gives the stage times
    elapsed = timed_loop()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    elapsed = max_over_ranks(elapsed, world)
    code, site = M.read_device_status(layer.ws)
    if code != 0:
        raise RuntimeError(f"device status {M.status_string(code)} at site {site}")

    # stage times: K more steps, launched eagerly with an event at each stage boundary
    # (events recorded inside a captured graph cannot be timed)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_st + 1)]
          for _ in range(args.steps)]
    marked_elapsed = timed_loop(ev)
    stage_ms = {name: float(np.mean([ev[i][j].elapsed_time(ev[i][j + 1])
                                     for i in range(args.steps)]))
                for j, name in enumerate(M.FORWARD_STAGES)}
    marked_ms = marked_elapsed / args.steps * 1e3

    # end to end through the C ABI: pinned host batch in, host output back, every step
    e2e = None
    if not args.no_e2e:
        # Through the public API with host buffers: every step copies its own input from
        # pinned host memory and reads its own output back.  Three streams (input copy,
        # layer, output copy) and two device buffers overlap step i's copies with the
        # layer of steps i-1 / i+1.
        n_host = min(args.steps, 64) if decode else 1
        hx = torch.empty((n_host, w.T, w.d_model), dtype=torch.bfloat16, pin_memory=True)
        hx.copy_(ring[:n_host].cpu() if decode else x_buf.cpu().unsqueeze(0))
        hy = [torch.empty((w.T, w.d_model), dtype=torch.bfloat16, pin_memory=True)
              for _ in range(2)]
        xd = [torch.empty_like(x_buf) for _ in range(2)]
        yd = [torch.empty_like(y) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        s_c = stream

        def run_e2e(n):
            ev_in = [torch.cuda.Event() for _ in range(n)]
            ev_c = [torch.cuda.Event() for _ in range(n)]
            ev_out = [torch.cuda.Event() for _ in range(n)]
            for i in range(n):
                b = i % 2
                if i >= 2:
                    s_in.wait_event(ev_c[i - 2])      # the layer of step i-2 has read xd[b]
                with torch.cuda.stream(s_in):
                    xd[b].copy_(hx[i % n_host], non_blocking=True)
                ev_in[i].record(s_in)
                s_c.wait_event(ev_in[i])
                if i >= 2:
                    s_c.wait_event(ev_out[i - 2])     # yd[b] of step i-2 is back on the host
                layer.forward(xd[b], yd[b], stream=s_c)
                ev_c[i].record(s_c)
                s_out.wait_event(ev_c[i])
                with torch.cuda.stream(s_out):
                    hy[b].copy_(yd[b], non_blocking=True)
                ev_out[i].record(s_out)
            return ev_out[-1]

        run_e2e(2)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(s_in)
        s_c.wait_event(a)
        s_out.wait_event(a)
        last = run_e2e(args.steps)
        s_out.wait_event(last)
        b.record(s_out)
        torch.cuda.synchronize()
        te = max_over_ranks(a.elapsed_time(b) / 1e3, world)
        e2e = {"value": job_tokens_per_s(w.T, args.steps, world, te), "unit": "tokens/s",
               "h2d_bytes_per_step": w.T * w.d_model * 2, "d2h_bytes_per_step": w.T * w.d_model * 2,
               "overlap": "input copy, layer and output copy on three streams, two buffers"}

    peaks = load_peaks()
    counts = layer.routing["counts"].cpu().numpy()
    work = stage_work(w, counts, fp8=args.fp8)
    gemm_stages = ("gemm1_swiglu", "gemm2_down_scale")
    dom = max(gemm_stages, key=lambda s: stage_ms[s])
    t_dom = stage_ms[dom] / 1e3
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    ai = work[dom]["flops"] / max(work[dom]["bytes"], 1)
    if ai < ridge:
        roof = {"kernel": dom, "bound": "hbm", "achieved": work[dom]["bytes"] / t_dom / 1e9,
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "algorithmic_bytes": work[dom]["bytes"]}
    else:
        roof = {"kernel": dom, "bound": "tensor", "achieved": work[dom]["flops"] / t_dom / 1e12,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "algorithmic_flops": work[dom]["flops"]}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["peak_source"] = peaks["source"] + " (burst)"
    if roof["bound"] == "tensor":
        # The GEMMs run back to back for the whole timed loop; under the 1 kW cap the
        # clocks settle below max (see "clocks"), which the sustained figure reflects.
        roof["peak_sustained"] = peaks["bf16_tflops_sustained"]
        roof["frac_of_sustained"] = roof["achieved"] / peaks["bf16_tflops_sustained"]
    roof["traffic"] = measured_traffic(w.name, dom, fp8=args.fp8)
    g_flops = sum(work[s]["flops"] for s in gemm_stages)
    g_time = sum(stage_ms[s] for s in gemm_stages) / 1e3
    expert = {"tflops": g_flops / g_time / 1e12,
              "frac_of_bf16_peak": g_flops / g_time / 1e12 / peaks["bf16_tflops"],
              "frac_of_bf16_sustained": g_flops / g_time / 1e12 / peaks["bf16_tflops_sustained"],
              "hbm_gbs": sum(work[s]["bytes"] for s in gemm_stages) / g_time / 1e9}
    expert["frac_of_hbm_peak"] = expert["hbm_gbs"] / peaks["hbm_gbs"]

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        h_small = {k: (P.to_numpy_bf16(v) if v is not None and v.dtype == torch.bfloat16 else
                       (None if v is None else v.cpu().numpy()))
                   for k, v in dev.items() if k != "x"}
        n = cpu_sample_size(w) if args.cpu_tokens <= 0 else args.cpu_tokens
        fp8 = None
        if args.fp8:  # the oracle's own e4m3 weights (made once, not timed)
            from oracle import moe_oracle as O
            fp8 = O.quantize_experts_fp8(h_small["w_gate"], h_small["w_up"], h_small["w_down"],
                                         h_small.get("ws_gate"), h_small.get("ws_up"),
                                         h_small.get("ws_down"))
        secs, n = oracle_sample(w, h_small, n, fp8=fp8)
        cpu = {"value": n / secs, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"{n} seeded tokens of the same workload through the float64 oracle "
                         f"({secs:.1f} s)"}

    line = {
        "metric": METRIC, "value": job_tokens_per_s(w.T, args.steps, world, elapsed),
        "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": elapsed / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
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
                               "bf16 weights (fp16 copy of W_down), fp16 h"),
                   "l2": "L2 flushed between steps" if flush else
                         f"inputs larger than L2 ({working_set / 1e9:.2f} GB resident)"},
        "roofline": roof, "expert_gemm": expert,
        "stages_ms": stage_ms, "stages_pass_ms_per_step": marked_ms,
        "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps, "clocks": clk,
        "cuda_graph": graph is not None,
    }
    if decode:
        byt = sum(work[s]["bytes"] for s in work)
        line["decode_hbm"] = {"bytes_per_step": byt,
                              "gbs": byt / (elapsed / args.steps) / 1e9,
                              "frac_of_hbm_peak": byt / (elapsed / args.steps) / 1e9 / peaks["hbm_gbs"]}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ----------------------------------------------------------------- reference arm

def run_reference(args):
    """The float64 CPU oracle on the host cores, a bounded token sample per step."""
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
    n = max(8, cpu_sample_size(w) // 8) if args.cpu_tokens <= 0 else args.cpu_tokens
    for i in range(args.warmup):
        oracle_sample(w, h, max(8, n // 4), seed=100 + i)
    tot, toks = 0.0, 0
    for i in range(args.steps):
        s, k = oracle_sample(w, h, n, seed=200 + i)
        tot += s
        toks += k
    v = toks / tot
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
                         "sample": f"{n} seeded tokens per step through the float64 oracle"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="c2_xs2_small")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=0)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch each step's kernels instead of replaying a CUDA graph")
    ap.add_argument("--single-cta", action="store_true",
                    help="force the single-CTA (M=128) expert GEMM engine")
    ap.add_argument("--pair", action="store_true",
                    help="force the CTA-pair (M=256) expert GEMM engine")
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
