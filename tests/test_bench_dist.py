"""Host-side logic of the multi-GPU bench path (replicas), on CPU with gloo ranks."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, port, results):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=2)
    try:
        elapsed = 0.25 + 0.5 * rank                     # the slower rank sets the job time
        slowest = bench.max_over_ranks(elapsed, 2, device="cpu")
        value = bench.job_tokens_per_s(4096, 10, 2, slowest)
        results.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_with_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get() for _ in range(2))
    for rank, slowest, value in got:
        assert slowest == 0.75                            # max over the ranks, on every rank
        assert value == 4096 * 10 * 2 / 0.75              # all ranks' tokens / slowest time


def test_replica_seeds_differ_per_rank():
    sys.path.insert(0, ROOT)
    import bench
    from sparse_moe_layer_select_b200 import inputs as I
    w = I.get("c2_xs2_small")
    seeds = [bench.replica_seed(w, r) for r in range(8)]
    assert seeds[0] == w.seed and len(set(seeds)) == 8


@pytest.mark.parametrize("rank,world,lines", [(1, 2, 0), (0, 1, 1)])
def test_reference_arm_prints_on_rank_zero_only(rank, world, lines):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--workload", "c1_tiny"],
                       capture_output=True, text=True, env=env, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    out = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(out) == lines
    if lines:
        d = json.loads(out[0])
        assert d["impl"] == "reference" and d["config"]["workload"] == "c1_tiny"
        assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_source_hash_ignores_comments_but_not_code():
    sys.path.insert(0, ROOT)
    import bench
    base = 'int f(int a) {  // doubles a\n  return a * 2;  /* "x" */\n}\n'
    comments = '// header\nint f(int a) {\n\n  return a * 2;\n}\n/* trailer\n   two lines */\n'
    code = 'int f(int a) {\n  return a * 3;\n}\n'
    literal = 'const char *s = "// not a comment";\n'
    assert bench._code_tokens(base) == bench._code_tokens(comments)
    assert bench._code_tokens(base) != bench._code_tokens(code)
    assert "// not a comment" in bench._code_tokens(literal)


def test_stored_traffic_matches_the_sources():
    sys.path.insert(0, ROOT)
    import bench
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        stored = json.load(f)
    if stored.get("sources_sha1") != bench.kernel_sources_sha1():
        assert bench.measured_traffic("c3_xs2_prefill_zipf", "gemm1_swiglu") is None
    else:
        assert bench.measured_traffic("c3_xs2_prefill_zipf", "gemm1_swiglu") is not None


def test_stage_work_of_the_t4096_workload():
    """Algorithmic work behind the roofline numbers, against sums done by hand for the
    T=4096 XS.2 workload (d=2048, E=256, k=8, F=Fs=512) with every expert touched.  The
    stages' "bytes" are the method's own (weights once, x, y); the intermediates (h, the
    routed contributions, the shared output) are counted apart."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    from sparse_moe_layer_select_b200 import inputs as I
    w = I.get("c2_xs2_small")
    work = bench.stage_work(w, np.ones(256, dtype=np.int64))
    # W_gate + W_up of 256 experts (2 x 512 x 2048 bf16 each) = 1073741824, shared gate + up
    # 4194304, x 16777216
    assert work["gemm1_swiglu"]["bytes"] == 1073741824 + 4194304 + 16777216
    # h: 32768 routed + 4096 shared rows of 512 fp16
    assert work["gemm1_swiglu"]["inter_bytes"] == 37748736
    # 4 d F per routed row (gate and up, 2 flops per MAC) + the same per shared row
    assert work["gemm1_swiglu"]["flops"] == 4 * 2048 * 512 * (32768 + 4096)
    # W_down 536870912 + shared 2097152; h read, O and S written (9 rows of 2048 fp16 per token)
    assert work["gemm2_down_scale"]["bytes"] == 536870912 + 2097152
    assert work["gemm2_down_scale"]["inter_bytes"] == 37748736 + 4096 * 9 * 4096
    # y written
    assert work["combine"]["bytes"] == 4096 * 2048 * 2
    # the layer: 1.61 GB of expert weights + shared 6.3 MB + router 1 MB + x, y 33.6 MB
    # (+ the routing arrays, 0.66 MB)
    lb = bench.layer_bytes(work)
    assert lb == (1073741824 + 536870912 + 3 * 2097152 + 1048576 + 2 * 16777216
                  + 4096 * 8 * 8 + 4096 * 8 * 12 + 256 * 8)
    assert 1.64e9 < lb < 1.66e9
    # half the expert weight bytes with e4m3, plus a float32 scale per weight row
    f8 = bench.stage_work(w, np.ones(256, dtype=np.int64), fp8=True)
    assert f8["gemm1_swiglu"]["bytes"] == (1073741824 + 4194304) // 2 + 16777216 + \
        4 * (256 * 2 * 512 + 2 * 512)
    assert f8["gemm2_down_scale"]["bytes"] == (536870912 + 2097152) // 2 + 4 * (256 * 2048 + 2048)


def test_peaks_measured_where_given_fallback_for_the_rest(tmp_path):
    sys.path.insert(0, ROOT)
    import bench
    full = tmp_path / "full.json"
    full.write_text(json.dumps({"hbm_gbs": 6537.3, "bf16_tflops": 1602.0,
                                "bf16_tflops_sustained": 1391.0, "clocks": {"sm": 1965}}))
    p = bench.load_peaks(str(full))
    assert (p["hbm_gbs"], p["bf16_tflops"], p["bf16_tflops_sustained"]) == (6537.3, 1602.0, 1391.0)
    assert p["source"] == "measured"
    part = tmp_path / "part.json"
    part.write_text(json.dumps({"hbm_gbs": 6537.3, "bf16_tflops": "n/a"}))
    p = bench.load_peaks(str(part))
    assert p["hbm_gbs"] == 6537.3
    assert p["bf16_tflops"] == bench.FALLBACK_PEAKS["bf16_tflops"]
    assert p["bf16_tflops_sustained"] == bench.FALLBACK_PEAKS["bf16_tflops_sustained"]
    assert p["source"].startswith("measured hbm_gbs") and "fallback" in p["source"]
    bad = tmp_path / "bad.json"
    bad.write_text("{not json")
    assert bench.load_peaks(str(bad)) == bench.FALLBACK_PEAKS
    assert bench.load_peaks(str(tmp_path / "missing.json")) == bench.FALLBACK_PEAKS
