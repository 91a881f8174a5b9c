"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Selection: bit-exact index sets and counts except the exempt near-ties
(tests/parity.py); weights within 1e-5; output within relative Frobenius
1e-2 and |dy| <= 2e-2 (|y| + 0.05) per element.  Permutation: bit-exact.
"""
import numpy as np
import pytest

from oracle import moe_oracle as O
from sparse_moe_layer_select_b200 import inputs as I
from sparse_moe_layer_select_b200 import moe as M
from tests import gpu_common as G
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    torch.cuda.set_device(0)
    from sparse_moe_layer_select_b200 import build as B
    B.build()
    yield


# ------------------------------------------------------------------ generator

def test_cuda_generator_matches_numpy_bit_for_bit():
    import torch
    for tid, sigma, start in [(0, 1.0, 0), (3, 0.02, 12345), (5, 0.015, 7), (101, 1.0, 0)]:
        n = 1 << 20
        t = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        I.generate_cuda(t, 0, tid, sigma, start=start)
        got = P.to_numpy_bf16(t)
        ref = I.generate_numpy((n,), 0, tid, sigma, start=start)
        assert np.array_equal(got, ref), (tid, int((got != ref).sum()))


# ------------------------------------------------------------------ tiny workload

def _small(w):
    h = I.host_inputs(w)
    return h, G.host_to_device(h)


def test_tiny_forward_matches_oracle():
    w = I.get("c1_tiny")
    h, dev = _small(w)
    y, routing, _ = G.run_forward(w, dev)
    ref = G.oracle_forward(w, h)
    G.check_routing(routing["topk_idx"].cpu().numpy(), routing["topk_w"].cpu().numpy(), ref, w.k)
    G.check_output(G.y_numpy(y), ref["y"], what="c1")
    counts, offsets, perm = O.expert_order(ref["topk_idx"], w.E)
    assert np.array_equal(routing["counts"].cpu().numpy(), counts)
    assert np.array_equal(routing["offsets"].cpu().numpy(), offsets)
    assert np.array_equal(routing["perm"].cpu().numpy(), perm)


@pytest.mark.parametrize("flags", [M.MOE_FLAG_ROUTER_CUDA_CORE, M.MOE_FLAG_ROUTER_TENSOR])
@pytest.mark.parametrize("T", [1, 64, 127, 128, 129, 1000])
def test_router_paths_match_oracle(flags, T):
    import torch
    w = I.get("c1_tiny").with_(T=T)
    h, dev = _small(w)
    dims = M.dims_for(w, flags=flags)
    ws = M.alloc_workspace(dims)
    idx = torch.empty((T, w.k), dtype=torch.int32, device="cuda")
    wt = torch.empty((T, w.k), dtype=torch.float32, device="cuda")
    M.route(dims, dev["x"], dev["w_router"], None, idx, wt, ws)
    torch.cuda.synchronize()
    assert M.read_device_status(ws)[0] == 0
    ridx, rw, scores, _ = O.route(h["x"], h["w_router"], None, w.k)
    ref = {"topk_idx": ridx, "topk_w": rw, "scores": scores}
    G.check_routing(idx.cpu().numpy(), wt.cpu().numpy(), ref, w.k)


ENGINES = [M.MOE_FLAG_GEMM_PAIR, M.MOE_FLAG_GEMM_SINGLE_CTA]  # CTA-pair (M = 256), single CTA (M = 128)


@pytest.mark.parametrize("engine", ENGINES)
@pytest.mark.parametrize("T", [1, 127, 128, 129, 255, 256, 257, 1000])
def test_ragged_and_multi_tile_forward(T, engine):
    w = I.get("c1_tiny").with_(T=T)
    h, dev = _small(w)
    y, routing, _ = G.run_forward(w, dev, flags=engine)
    ref = G.oracle_forward(w, h)
    G.check_routing(routing["topk_idx"].cpu().numpy(), routing["topk_w"].cpu().numpy(), ref, w.k)
    G.check_output(G.y_numpy(y), ref["y"], what=f"T={T}")


@pytest.mark.parametrize("T", [1024, 1500])
def test_auto_engines_mixed_and_equal_to_forced(T):
    """T*k >= 256*E: by default the gate/up GEMM runs on single CTAs (128-row tile list) and the
    down GEMM on CTA pairs (256-row tile list).  Checked against the oracle, and against both
    forced engines bit for bit: every engine runs the same K order of fp32 MMA accumulation."""
    w = I.get("c1_tiny").with_(T=T)
    assert w.T * w.k >= 256 * w.E
    h, dev = _small(w)
    y, routing, _ = G.run_forward(w, dev, flags=0)
    ref = G.oracle_forward(w, h)
    G.check_routing(routing["topk_idx"].cpu().numpy(), routing["topk_w"].cpu().numpy(), ref, w.k)
    G.check_output(G.y_numpy(y), ref["y"], what=f"auto T={T}")
    import torch
    bits = y.view(torch.int16).cpu().numpy()
    for engine in ENGINES:
        y2, _, _ = G.run_forward(w, dev, flags=engine)
        assert np.array_equal(y2.view(torch.int16).cpu().numpy(), bits), engine


def _mask_run(w, h, dev, mask, flags=0):
    import torch
    dims = M.dims_for(w, flags=flags)
    ws = M.alloc_workspace(dims)
    ws.fill_(0xFF)
    routing = M.alloc_routing(dims)
    y = torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda")
    M.forward(dims, dev, dev["x"], y, routing, ws, token_mask=torch.from_numpy(mask).cuda())
    torch.cuda.synchronize()
    assert M.read_device_status(ws)[0] == 0
    return y, routing


@pytest.mark.parametrize("engine", [0] + ENGINES)
@pytest.mark.parametrize("T,frac", [(300, 0.3), (1500, 0.5), (257, 1.0), (129, 0.0)])
def test_padding_mask_forward(T, frac, engine):
    """Padding tokens (mask 0) are not routed: MOE_NOT_ROUTED ids, zero weights, no expert
    rows, y = shared expert only; the other tokens match the oracle as without a mask."""
    w = I.get("c1_tiny").with_(T=T)
    h, dev = _small(w)
    rng = np.random.default_rng(T)
    mask = (rng.random(T) >= frac).astype(np.uint8)
    y, routing = _mask_run(w, h, dev, mask, engine)
    ref = O.moe_forward(h["x"], h["w_router"], h["w_gate"], h["w_up"], h["w_down"], w.k,
                        ws_gate=h["ws_gate"], ws_up=h["ws_up"], ws_down=h["ws_down"],
                        routed_scaling_factor=w.routed_scaling_factor, token_mask=mask)
    gidx = routing["topk_idx"].cpu().numpy()
    gw = routing["topk_w"].cpu().numpy()
    pad = mask == 0
    assert np.all(gidx[pad] == M.MOE_NOT_ROUTED) and np.all(gw[pad] == 0.0)
    keep = ~pad
    if keep.any():
        G.check_routing(gidx[keep], gw[keep], {"topk_idx": ref["topk_idx"][keep],
                                               "topk_w": ref["topk_w"][keep],
                                               "scores": ref["scores"][keep]}, w.k)
    c, o, p = O.expert_order(gidx, w.E)
    assert np.array_equal(routing["counts"].cpu().numpy(), c)
    assert np.array_equal(routing["offsets"].cpu().numpy(), o)
    assert np.array_equal(routing["perm"].cpu().numpy()[:o[-1]], p)
    G.check_output(G.y_numpy(y), ref["y"], what=f"mask T={T} frac={frac}")


@pytest.mark.parametrize("T,router", [(3000, M.MOE_FLAG_ROUTER_CUDA_CORE),
                                      (12000, M.MOE_FLAG_ROUTER_TENSOR)])
def test_padding_mask_multi_chunk_index(T, router):
    """Masked batches whose T * k entries span several index chunks, with the logits from
    either router (one plane at T=3000 on CUDA cores, K-sliced planes summed by the select
    kernel at T=12000): padding tokens are left unrouted, routed tokens match the oracle."""
    w = I.get("c1_tiny").with_(T=T)
    h, dev = _small(w)
    mask = (np.random.default_rng(T).random(T) >= 0.3).astype(np.uint8)
    y, routing = _mask_run(w, h, dev, mask, router)
    ref = O.moe_forward(h["x"], h["w_router"], h["w_gate"], h["w_up"], h["w_down"], w.k,
                        ws_gate=h["ws_gate"], ws_up=h["ws_up"], ws_down=h["ws_down"],
                        routed_scaling_factor=w.routed_scaling_factor, token_mask=mask)
    gidx = routing["topk_idx"].cpu().numpy()
    gw = routing["topk_w"].cpu().numpy()
    pad = mask == 0
    assert np.all(gidx[pad] == M.MOE_NOT_ROUTED) and np.all(gw[pad] == 0.0)
    keep = ~pad
    G.check_routing(gidx[keep], gw[keep], {"topk_idx": ref["topk_idx"][keep],
                                           "topk_w": ref["topk_w"][keep],
                                           "scores": ref["scores"][keep]}, w.k)
    same = np.ones(T, dtype=bool)
    same[keep] = P.same_selection_mask(gidx[keep], ref["topk_idx"][keep])
    G.check_output(G.y_numpy(y), ref["y"], rows_ok=same, what=f"mask, multi-chunk index T={T}")


def test_padding_mask_permute_and_gather():
    import torch
    w = I.get("c1_tiny").with_(T=500)
    h, dev = _small(w)
    ridx = O.route(h["x"], h["w_router"], None, w.k)[0]
    ridx[::3] = M.MOE_NOT_ROUTED
    dims = M.dims_for(w)
    ws = M.alloc_workspace(dims)
    idx = torch.from_numpy(ridx.astype(np.int32)).cuda()
    counts = torch.empty(w.E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(w.E + 1, dtype=torch.int32, device="cuda")
    perm = torch.full((w.T * w.k,), -7, dtype=torch.int32, device="cuda")
    xp = torch.zeros((w.T * w.k, w.d_model), dtype=torch.bfloat16, device="cuda")
    M.permute(dims, idx, counts, offsets, perm, ws, x=dev["x"], x_perm=xp)
    torch.cuda.synchronize()
    assert M.read_device_status(ws)[0] == 0
    c, o, p = O.expert_order(ridx, w.E)
    n = int(o[-1])
    assert np.array_equal(counts.cpu().numpy(), c) and np.array_equal(offsets.cpu().numpy(), o)
    got = perm.cpu().numpy()
    assert np.array_equal(got[:n], p) and np.all(got[n:] == -7)   # rows past offsets[E] untouched
    xpn = P.to_numpy_bf16(xp)
    assert np.array_equal(xpn[:n], h["x"][p // w.k]) and np.all(xpn[n:] == 0)


@pytest.mark.parametrize("flags", [M.MOE_FLAG_ROUTER_CUDA_CORE, M.MOE_FLAG_ROUTER_TENSOR,
                                   M.MOE_FLAG_ROUTER_TENSOR | M.MOE_FLAG_GEMM_PAIR])
def test_selection_only_bias(flags):
    """Auxiliary-loss-free variant: a per-expert bias on the sigmoid scores chooses the experts,
    the weights are the unbiased scores normalised over them."""
    import torch
    w = I.get("c1_tiny").with_(T=1100)
    h, dev = _small(w)
    rng = np.random.default_rng(77)
    b = (rng.standard_normal(w.E) * 0.05).astype(np.float32)
    dev = dict(dev, router_bias=torch.from_numpy(b).cuda())
    dims = M.dims_for(w, flags=flags | M.MOE_FLAG_BIAS_SELECTION_ONLY)
    ws = M.alloc_workspace(dims)
    ws.fill_(0xFF)
    routing = M.alloc_routing(dims)
    y = torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda")
    M.forward(dims, dev, dev["x"], y, routing, ws)
    torch.cuda.synchronize()
    assert M.read_device_status(ws)[0] == 0
    ref = O.moe_forward(h["x"], h["w_router"], h["w_gate"], h["w_up"], h["w_down"], w.k,
                        ws_gate=h["ws_gate"], ws_up=h["ws_up"], ws_down=h["ws_down"],
                        routed_scaling_factor=w.routed_scaling_factor,
                        selection_bias=b.astype(np.float64))
    gidx = routing["topk_idx"].cpu().numpy()
    G.check_routing(gidx, routing["topk_w"].cpu().numpy(), ref, w.k)
    plain = O.route(h["x"], h["w_router"], None, w.k)[0]
    assert (np.sort(gidx, 1) != np.sort(plain, 1)).any(axis=1).mean() > 0.05  # the bias acts
    same = P.same_selection_mask(gidx, ref["topk_idx"])
    G.check_output(G.y_numpy(y), ref["y"], rows_ok=same, what="selection-only bias")


def test_fp8_weight_quantization_matches_oracle():
    """moe_prepare_fp8: e4m3 codes and row scales equal the oracle's (codes of +0 and -0 are
    both accepted for zero)."""
    w = I.get("c1_tiny").with_(d_model=256, moe_intermediate_size=256, shared_intermediate_size=128)
    h, dev = _small(w)
    Q, (code, _) = M.prepare_fp8(M.dims_for(w), dev)
    assert code == 0
    ref = O.quantize_experts_fp8(h["w_gate"], h["w_up"], h["w_down"], h["ws_gate"], h["ws_up"],
                                 h["ws_down"])
    for name, key, skey in (("gate", "w_gate", "s_gate"), ("up", "w_up", "s_up"),
                            ("down", "w_down", "s_down"), ("s_gate", "ws_gate", "ss_gate"),
                            ("s_up", "ws_up", "ss_up"), ("s_down", "ws_down", "ss_down")):
        rc, rs = ref[name]
        gc = Q[key].cpu().numpy().reshape(rc.shape)
        gs = Q[skey].cpu().numpy().reshape(rs.shape)
        assert np.array_equal(gs.view(np.uint32), rs.astype(np.float32).view(np.uint32)), name
        zero = (O.e4m3_value(gc) == 0) & (O.e4m3_value(rc) == 0)
        assert np.all((gc == rc) | zero), name


@pytest.mark.parametrize("T", [64, 300])
def test_fp8_forward_matches_fp8_oracle(T):
    """moe_forward_fp8 against the oracle of the same FP8 method (e4m3 weights, x and h with
    per-row scales)."""
    import torch
    w = I.get("c1_tiny").with_(T=T, d_model=256, moe_intermediate_size=256,
                               shared_intermediate_size=128)
    h, dev = _small(w)
    layer = M.MoeLayer(dev, w.d_model, w.E, w.k, w.F, w.Fs, w.routed_scaling_factor,
                       max_tokens=w.T, fp8=True)
    y = layer.forward(dev["x"])
    torch.cuda.synchronize()
    assert M.read_device_status(layer.ws)[0] == 0
    fp8 = O.quantize_experts_fp8(h["w_gate"], h["w_up"], h["w_down"], h["ws_gate"], h["ws_up"],
                                 h["ws_down"])
    ref = O.moe_forward_fp8(h["x"], h["w_router"], fp8, w.k,
                            routed_scaling_factor=w.routed_scaling_factor)
    gidx = layer.routing["topk_idx"][:T].cpu().numpy()
    G.check_routing(gidx, layer.routing["topk_w"][:T].cpu().numpy(), ref, w.k)
    same = P.same_selection_mask(gidx, ref["topk_idx"])
    G.check_output(G.y_numpy(y), ref["y"], rows_ok=same, what=f"fp8 T={T}")


@pytest.mark.parametrize("Fs", [0, 512])
def test_fp8_xs2_widths_full_oracle(Fs):
    """FP8 experts at the XS.2 widths (d=2048, F=512; 16 experts, top-4 keep the float64
    oracle's weight quantization short), T=600 (ragged tiles everywhere), with and without
    the shared expert."""
    import torch
    w = I.get("c2_xs2_small").with_(T=600, num_experts=16, num_experts_per_tok=4,
                                    shared_intermediate_size=Fs)
    h, dev = _small(w)
    layer = M.MoeLayer(dev, w.d_model, w.E, w.k, w.F, w.Fs, w.routed_scaling_factor,
                       max_tokens=w.T, fp8=True)
    y = layer.forward(dev["x"])
    torch.cuda.synchronize()
    assert M.read_device_status(layer.ws)[0] == 0
    fp8 = O.quantize_experts_fp8(h["w_gate"], h["w_up"], h["w_down"], h.get("ws_gate"),
                                 h.get("ws_up"), h.get("ws_down"))
    ref = O.moe_forward_fp8(h["x"], h["w_router"], fp8, w.k,
                            routed_scaling_factor=w.routed_scaling_factor)
    gidx = layer.routing["topk_idx"][:w.T].cpu().numpy()
    G.check_routing(gidx, layer.routing["topk_w"][:w.T].cpu().numpy(), ref, w.k)
    same = P.same_selection_mask(gidx, ref["topk_idx"])
    G.check_output(G.y_numpy(y), ref["y"], rows_ok=same, what=f"fp8 xs2 Fs={Fs}")


def test_fp8_decode_matches_fp8_oracle():
    import torch
    w = I.get("c5_decode")
    dev = I.device_inputs(w)
    h = G.device_to_host(dev)
    layer = M.MoeLayer(dev, w.d_model, w.E, w.k, w.F, w.Fs, w.routed_scaling_factor,
                       max_tokens=w.T, fp8=True)
    ring = I.device_decode_ring(w, 2)
    fp8 = O.quantize_experts_fp8(h["w_gate"], h["w_up"], h["w_down"], h["ws_gate"], h["ws_up"],
                                 h["ws_down"])
    for i in range(2):
        y = layer.forward(ring[i])
        torch.cuda.synchronize()
        assert M.read_device_status(layer.ws)[0] == 0
        xi = P.to_numpy_bf16(ring[i])
        ref = O.moe_forward_fp8(xi, h["w_router"], fp8, w.k,
                                routed_scaling_factor=w.routed_scaling_factor)
        gidx = layer.routing["topk_idx"][:w.T].cpu().numpy()
        G.check_routing(gidx, layer.routing["topk_w"][:w.T].cpu().numpy(), ref, w.k)
        same = P.same_selection_mask(gidx, ref["topk_idx"])
        G.check_output(G.y_numpy(y), ref["y"], rows_ok=same, what=f"fp8 decode batch {i}")


def test_permute_materialised_gather_and_counts():
    import torch
    w = I.get("c1_tiny").with_(T=1000)
    h, dev = _small(w)
    ridx = O.route(h["x"], h["w_router"], None, w.k)[0]
    dims = M.dims_for(w)
    ws = M.alloc_workspace(dims)
    idx = torch.from_numpy(ridx.astype(np.int32)).cuda()
    counts = torch.empty(w.E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(w.E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(w.T * w.k, dtype=torch.int32, device="cuda")
    xp = torch.empty((w.T * w.k, w.d_model), dtype=torch.bfloat16, device="cuda")
    M.permute(dims, idx, counts, offsets, perm, ws, x=dev["x"], x_perm=xp)
    torch.cuda.synchronize()
    assert M.read_device_status(ws)[0] == 0
    c, o, p = O.expert_order(ridx, w.E)
    assert np.array_equal(counts.cpu().numpy(), c)
    assert np.array_equal(offsets.cpu().numpy(), o)
    assert np.array_equal(perm.cpu().numpy(), p)
    assert np.array_equal(P.to_numpy_bf16(xp), h["x"][p // w.k])


def test_bad_expert_id_sets_bounds_status():
    import torch
    w = I.get("c1_tiny")
    dims = M.dims_for(w)
    ws = M.alloc_workspace(dims)
    idx = torch.zeros((w.T, w.k), dtype=torch.int32, device="cuda")
    idx[5, 2] = w.E  # out of range
    counts = torch.empty(w.E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(w.E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(w.T * w.k, dtype=torch.int32, device="cuda")
    M.permute(dims, idx, counts, offsets, perm, ws)
    code, site = M.read_device_status(ws)
    assert code == M.MOE_ERR_DEVICE_BOUNDS and site == 20


def test_device_wait_timeout_is_reported_and_context_survives():
    import torch
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    M.selftest_bounded_wait(ws, 2000)
    code, site = M.read_device_status(ws)
    assert code == M.MOE_ERR_DEVICE_TIMEOUT and site == 90
    # the context is still usable: a normal layer call succeeds afterwards
    w = I.get("c1_tiny")
    h, dev = _small(w)
    y, _, _ = G.run_forward(w, dev)
    G.check_output(G.y_numpy(y), G.oracle_forward(w, h)["y"], what="after timeout")


# ------------------------------------------------------------------ special cases

def test_no_shared_expert():
    w = I.get("c1_tiny").with_(T=300, shared_intermediate_size=0)
    h, dev = _small(w)
    y, _, _ = G.run_forward(w, dev)
    ref = G.oracle_forward(w, h)
    assert np.array_equal(ref["Sh"], np.zeros_like(ref["Sh"]))
    G.check_output(G.y_numpy(y), ref["y"], what="Fs=0")


def test_zero_shared_weights_isolate_routed_path():
    import torch
    w = I.get("c1_tiny").with_(T=200)
    h, dev = _small(w)
    for key in ("ws_gate", "ws_up", "ws_down"):
        h[key] = np.zeros_like(h[key])
        dev[key] = torch.zeros_like(dev[key])
    y, _, _ = G.run_forward(w, dev)
    ref = G.oracle_forward(w, h)
    G.check_output(G.y_numpy(y), 2.5 * ref["R"], what="shared=0")


@pytest.mark.parametrize("E,k", [(2, 1), (2, 2), (4, 1), (4, 3), (8, 1), (8, 4), (8, 8), (16, 16),
                                 (24, 5), (40, 16), (300, 8), (512, 16)])
def test_small_expert_counts_and_k_extremes(E, k):
    w = I.get("c1_tiny").with_(T=257, num_experts=E, num_experts_per_tok=k)
    h, dev = _small(w)
    y, routing, _ = G.run_forward(w, dev)
    ref = G.oracle_forward(w, h)
    G.check_routing(routing["topk_idx"].cpu().numpy(), routing["topk_w"].cpu().numpy(), ref, k)
    G.check_output(G.y_numpy(y), ref["y"], what=f"E={E},k={k}")


@pytest.mark.parametrize("engine", ENGINES)
def test_m1_top16_unit_scale(engine):
    """The M.1 configuration of the layer: top-16, routed scale 1.0 (ragged tiles, full oracle)."""
    w = I.get("c1_tiny").with_(T=700, num_experts=64, num_experts_per_tok=16,
                               routed_scaling_factor=1.0)
    h, dev = _small(w)
    y, routing, _ = G.run_forward(w, dev, flags=engine)
    ref = G.oracle_forward(w, h)
    G.check_routing(routing["topk_idx"].cpu().numpy(), routing["topk_w"].cpu().numpy(), ref, w.k)
    G.check_output(G.y_numpy(y), ref["y"], what="top-16, scale 1")


@pytest.mark.parametrize("flags", [M.MOE_FLAG_ROUTER_CUDA_CORE, M.MOE_FLAG_ROUTER_TENSOR])
def test_exact_ties_go_to_lower_expert_index(flags):
    import torch
    w = I.get("c1_tiny").with_(T=256)
    h, _ = _small(w)
    wr = h["w_router"].copy()
    wr[9] = wr[2]   # experts 2 and 9, and 5 and 14, have identical logits for every token
    wr[14] = wr[5]
    h["w_router"] = wr
    dev = G.host_to_device(h)
    y, routing, ws = G.run_forward(w, dev, flags=flags)
    off = M.logits_offset(M.dims_for(w, flags=flags))
    logits = ws[off:off + w.T * w.E * 4].view(torch.float32).view(w.T, w.E).cpu().numpy()
    assert np.array_equal(logits[:, 2], logits[:, 9]) and np.array_equal(logits[:, 5], logits[:, 14])
    idx = routing["topk_idx"].cpu().numpy()
    ref = G.oracle_forward(w, h)
    for t in range(w.T):
        s_ = set(idx[t].tolist())
        assert not (9 in s_ and 2 not in s_) and not (14 in s_ and 5 not in s_), (t, idx[t])
    G.check_routing(idx, routing["topk_w"].cpu().numpy(), ref, w.k)
    G.check_output(G.y_numpy(y), ref["y"], what="ties")


ROUTERS = [M.MOE_FLAG_ROUTER_CUDA_CORE, M.MOE_FLAG_ROUTER_TENSOR]


@pytest.mark.parametrize("router", ROUTERS)
def test_more_than_32_experts_in_the_refine_band(router):
    """40 of 64 experts share one router row, so for every token the k-th and (k+1)-th
    places (k = 8) lie among 40 exactly tied experts: more than a warp's worth of band
    members, which the select kernel re-decides through its streamed fallback.  Inputs are
    small dyadic numbers, so every logit is exact in fp32 and float64 on both sides; the
    tied experts' logit (8) is far above every other expert's.  The oracle gives the 8
    lowest ids among the tied ones, in ascending id (equal scores), each with weight 1/8."""
    import torch
    T, d, E, k = 200, 256, 64, 8
    w = I.get("c1_tiny").with_(T=T, d_model=d, num_experts=E, num_experts_per_tok=k)
    rng = np.random.default_rng(40)
    h = I.host_inputs(w)
    x = rng.integers(-1, 2, size=(T, d)).astype(np.float64)
    x[:, 0] = 1.0
    wr = rng.integers(-1, 2, size=(E, d)).astype(np.float64) * 2.0 ** -4
    wr[:, 0] = 0.0
    tied = np.arange(10, 50)
    wr[tied] = 0.0
    wr[tied, 0] = 8.0
    h["x"] = I.f64_to_bf16_bits(x)
    h["w_router"] = I.f64_to_bf16_bits(wr)
    dev = G.host_to_device(h)
    y, routing, ws = G.run_forward(w, dev, flags=router)
    ref = G.oracle_forward(w, h)
    want = np.tile(np.arange(10, 10 + k), (T, 1))
    assert np.array_equal(ref["topk_idx"], want)
    idx = routing["topk_idx"].cpu().numpy()
    assert np.array_equal(idx, want), idx[:3]
    assert np.array_equal(routing["topk_w"].cpu().numpy(), np.full((T, k), 0.125, np.float32))
    off = M.logits_offset(M.dims_for(w, flags=router))
    logits = ws[off:off + T * E * 4].view(torch.float32).view(T, E).cpu().numpy()
    assert np.array_equal(logits[:, tied], np.full((T, tied.size), 8.0, np.float32))
    G.check_output(G.y_numpy(y), ref["y"], what="40-way tie")


@pytest.mark.parametrize("router,engine", [(M.MOE_FLAG_ROUTER_CUDA_CORE, M.MOE_FLAG_GEMM_SINGLE_CTA),
                                           (M.MOE_FLAG_ROUTER_TENSOR, M.MOE_FLAG_GEMM_PAIR)])
def test_unnormalised_weights(router, engine):
    """norm_topk_prob = 0: every weight is the selected expert's own sigmoid score (the
    oracle's branch is pinned by a plain-Python evaluation); the routed sum uses them as
    they are."""
    w = I.get("c1_tiny").with_(T=300)
    h, dev = _small(w)
    y, routing, _ = G.run_forward(w, dev, flags=router | engine, norm_topk_prob=0)
    ref = G.oracle_forward(w, h, norm_topk_prob=False)
    assert np.all(np.abs(ref["topk_w"].sum(axis=1) - 1.0) > 1e-3)
    G.check_routing(routing["topk_idx"].cpu().numpy(), routing["topk_w"].cpu().numpy(), ref, w.k)
    G.check_output(G.y_numpy(y), ref["y"], what="norm_topk_prob=0")


@pytest.mark.parametrize("engine", ENGINES)
@pytest.mark.parametrize("d", [64, 192, 320])
def test_d_model_multiple_of_64(d, engine):
    """d_model only a multiple of 64: the down projection runs on 64-column N tiles (and
    the router on 3 or 5 K blocks); ragged token tiles, full oracle."""
    w = I.get("c1_tiny").with_(T=300, d_model=d)
    h, dev = _small(w)
    y, routing, _ = G.run_forward(w, dev, flags=engine)
    ref = G.oracle_forward(w, h)
    G.check_routing(routing["topk_idx"].cpu().numpy(), routing["topk_w"].cpu().numpy(), ref, w.k)
    G.check_output(G.y_numpy(y), ref["y"], what=f"d={d}")


@pytest.mark.parametrize("flags", [M.MOE_FLAG_ROUTER_CUDA_CORE, M.MOE_FLAG_ROUTER_TENSOR])
def test_router_logits_error_against_float64(flags):
    """fp32 logits of both router paths against the oracle's float64 logits (XS.2 widths)."""
    import torch
    w = I.get("c2_xs2_small").with_(T=2048)
    dev = {"x": torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda"),
           "w_router": torch.empty((w.E, w.d_model), dtype=torch.bfloat16, device="cuda")}
    I.generate_cuda(dev["x"], w.seed, I.TID_X, w.sigma_x)
    I.generate_cuda(dev["w_router"], w.seed, I.TID_W_ROUTER, w.sigma_router)
    dims = M.dims_for(w, flags=flags)
    ws = M.alloc_workspace(dims)
    idx = torch.empty((w.T, w.k), dtype=torch.int32, device="cuda")
    wt = torch.empty((w.T, w.k), dtype=torch.float32, device="cuda")
    M.route(dims, dev["x"], dev["w_router"], None, idx, wt, ws)
    torch.cuda.synchronize()
    off = M.logits_offset(dims)
    got = ws[off:off + w.T * w.E * 4].view(torch.float32).view(w.T, w.E).cpu().numpy()
    ref = O.router_logits(P.to_numpy_bf16(dev["x"]), P.to_numpy_bf16(dev["w_router"]), None)
    err = float(np.abs(got - ref).max())
    # the select kernel re-decides, on float64 logits, every token whose k-th and
    # (k+1)-th fp32 logits are within 2e-4; that is exact as long as the fp32
    # logit error stays below half of it (measured: ~1.2e-5 tensor, < 4e-6 CUDA core)
    assert err < 1e-4 / 4, err


@pytest.mark.parametrize("d", [4096, 7296])
def test_cuda_core_router_wide_rows(d):
    """The CUDA-core router stages 8 bf16 token rows per CTA in shared memory; beyond d = 3072
    that takes more than the default 48 KB (the opt-in launch attribute).  Against the oracle's
    float64 logits and routing, on a ragged batch (43 tokens: five full groups of 8 and 3)."""
    import torch
    w = I.get("c2_xs2_small").with_(T=43, d_model=d)
    h = {"x": I.generate_numpy((w.T, d), w.seed, I.TID_X, w.sigma_x),
         "w_router": I.generate_numpy((w.E, d), w.seed, I.TID_W_ROUTER, w.sigma_router)}
    dev = G.host_to_device(h)
    dims = M.dims_for(w, flags=M.MOE_FLAG_ROUTER_CUDA_CORE)
    ws = M.alloc_workspace(dims)
    idx = torch.empty((w.T, w.k), dtype=torch.int32, device="cuda")
    wt = torch.empty((w.T, w.k), dtype=torch.float32, device="cuda")
    M.route(dims, dev["x"], dev["w_router"], None, idx, wt, ws)
    torch.cuda.synchronize()
    code, site = M.read_device_status(ws)
    assert code == 0, (M.status_string(code), site)
    off = M.logits_offset(dims)
    got = ws[off:off + w.T * w.E * 4].view(torch.float32).view(w.T, w.E).cpu().numpy()
    ref_l = O.router_logits(h["x"], h["w_router"], None)
    assert float(np.abs(got - ref_l).max()) < 1e-4 / 4
    ref = O.route(h["x"], h["w_router"], None, w.k)
    G.check_routing(idx.cpu().numpy(), wt.cpu().numpy(),
                    {"topk_idx": ref[0], "topk_w": ref[1], "scores": ref[2]}, w.k)


@pytest.mark.parametrize("T", [1024, 4096, 6000, 10000])
def test_router_k_slices_against_float64(T):
    """The tensor-core router splits d into 4 slices (T <= 2304), 2 (T <= 9472) or none; the
    select kernel sums the slices' partial logits.  The summed logits against the oracle's
    float64 logits, and the routing against the oracle's, at each split (XS.2 widths)."""
    import torch
    w = I.get("c2_xs2_small").with_(T=T)
    dev = {"x": torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda"),
           "w_router": torch.empty((w.E, w.d_model), dtype=torch.bfloat16, device="cuda")}
    I.generate_cuda(dev["x"], w.seed, I.TID_X, w.sigma_x)
    I.generate_cuda(dev["w_router"], w.seed, I.TID_W_ROUTER, w.sigma_router)
    dims = M.dims_for(w, flags=M.MOE_FLAG_ROUTER_TENSOR)
    ws = M.alloc_workspace(dims)
    idx = torch.empty((w.T, w.k), dtype=torch.int32, device="cuda")
    wt = torch.empty((w.T, w.k), dtype=torch.float32, device="cuda")
    M.route(dims, dev["x"], dev["w_router"], None, idx, wt, ws)
    torch.cuda.synchronize()
    code, site = M.read_device_status(ws)
    assert code == 0, (M.status_string(code), site)
    off = M.logits_offset(dims)
    got = ws[off:off + w.T * w.E * 4].view(torch.float32).view(w.T, w.E).cpu().numpy()
    xh, wh = P.to_numpy_bf16(dev["x"]), P.to_numpy_bf16(dev["w_router"])
    ref_l = O.router_logits(xh, wh, None)
    assert float(np.abs(got - ref_l).max()) < 1e-4 / 4
    ref = O.route(xh, wh, None, w.k)
    G.check_routing(idx.cpu().numpy(), wt.cpu().numpy(),
                    {"topk_idx": ref[0], "topk_w": ref[1], "scores": ref[2]}, w.k)


def test_prepared_down_weights_match_per_call_conversion():
    import torch
    w = I.get("c1_tiny").with_(T=500)
    h, dev = _small(w)
    y1, _, _ = G.run_forward(w, dev)                      # converts W_down every call
    layer = M.MoeLayer(dev, w.d_model, w.E, w.k, w.F, w.Fs, w.routed_scaling_factor,
                       max_tokens=w.T)                    # prepared once
    y2 = layer.forward(dev["x"])
    torch.cuda.synchronize()
    assert np.array_equal(P.to_numpy_bf16(y1), P.to_numpy_bf16(y2))
    wd = h["w_down"].astype(np.uint32) << 16
    ref16 = wd.view(np.float32).astype(np.float16)
    assert np.array_equal(layer.W["w_down_f16"].cpu().numpy(), ref16)


def test_fp16_range_violation_is_reported():
    import torch
    w = I.get("c1_tiny")
    h, dev = _small(w)
    bad = dev["w_down"].clone()
    bad[3, 5, 7] = 1.0e6
    W = {"w_down": bad, "ws_down": dev["ws_down"]}
    code, site = M.prepare_down_f16(M.dims_for(w), W)
    assert code == M.MOE_ERR_DEVICE_BOUNDS and site == 32


@pytest.mark.parametrize("engine", ENGINES)
def test_maximum_skew_all_tokens_on_the_same_experts(engine):
    import torch
    w = I.get("c1_tiny").with_(T=1000)
    h, dev = _small(w)
    bias = np.zeros(w.E, dtype=np.float32)
    bias[[3, 7, 11, 12]] = 100.0   # every token selects experts 3, 7, 11, 12
    h["router_bias"] = bias
    dev["router_bias"] = torch.from_numpy(bias).cuda()
    y, routing, _ = G.run_forward(w, dev, flags=engine)
    counts = routing["counts"].cpu().numpy()
    assert counts[[3, 7, 11, 12]].tolist() == [1000] * 4 and counts.sum() == 4000
    ref = G.oracle_forward(w, h)
    G.check_output(G.y_numpy(y), ref["y"], what="max skew")


def test_output_guard_bands_untouched():
    import torch
    w = I.get("c1_tiny").with_(T=300)
    h, dev = _small(w)
    big = torch.full((w.T + 2, w.d_model), 7.0, dtype=torch.bfloat16, device="cuda")
    y_view = big[1:w.T + 1]
    dims = M.dims_for(w)
    ws = M.alloc_workspace(dims)
    routing = M.alloc_routing(dims)
    M.forward(dims, dev, dev["x"], y_view, routing, ws)
    torch.cuda.synchronize()
    assert bool((big[0] == 7.0).all()) and bool((big[-1] == 7.0).all())
    G.check_output(G.y_numpy(y_view), G.oracle_forward(w, h)["y"], what="guard")


def test_redundant_runs_are_bit_identical():
    """The same inputs five times: routing, permutation and y identical bit for bit."""
    import torch
    w = I.get("c1_tiny").with_(T=1000)
    _, dev = _small(w)
    outs = []
    for _ in range(5):
        y, routing, _ = G.run_forward(w, dev)
        outs.append((P.to_numpy_bf16(y), routing["topk_idx"].cpu().numpy(),
                     routing["topk_w"].cpu().numpy(), routing["perm"].cpu().numpy()))
    for o in outs[1:]:
        for a, b in zip(outs[0], o):
            assert np.array_equal(a, b)


# ------------------------------------------------------------------ full-size workloads

def _device_workload(w):
    dev = I.device_inputs(w)
    h = G.device_to_host(dev)
    return h, dev


@pytest.mark.parametrize("engine", ENGINES)
def test_xs2_dims_multi_tile_full_oracle(engine):
    """XS.2 widths at T=1000: every token through the oracle (ragged tiles everywhere)."""
    w = I.get("c2_xs2_small").with_(T=1000)
    h, dev = _device_workload(w)
    y, routing, _ = G.run_forward(w, dev, flags=engine)
    ref = G.oracle_forward(w, h)
    G.check_routing(routing["topk_idx"].cpu().numpy(), routing["topk_w"].cpu().numpy(), ref, w.k)
    same = P.same_selection_mask(routing["topk_idx"].cpu().numpy(), ref["topk_idx"])
    G.check_output(G.y_numpy(y), ref["y"], rows_ok=same, what="xs2 T=1000")


@pytest.mark.parametrize("name,n_sample", [("c2_xs2_small", 1024), ("c3_xs2_prefill_zipf", 1024),
                                           ("c4_m1_width", 256), ("c6_m1_top16", 256)])
def test_full_size_workloads(name, n_sample):
    """Routing and counts on every token; y on a seeded sample of tokens."""
    w = I.get(name)
    h, dev = _device_workload(w)
    y, routing, _ = G.run_forward(w, dev)
    gidx = routing["topk_idx"].cpu().numpy()
    gw = routing["topk_w"].cpu().numpy()
    ridx, rw, scores, _ = O.route(h["x"], h["w_router"], h["router_bias"], w.k)
    n_ex, n_diff = G.check_routing(gidx, gw, {"topk_idx": ridx, "topk_w": rw, "scores": scores},
                                   w.k)
    c, o, p = O.expert_order(gidx, w.E)   # the permutation of the (accepted) GPU selection
    assert np.array_equal(routing["counts"].cpu().numpy(), c)
    assert np.array_equal(routing["offsets"].cpu().numpy(), o)
    assert np.array_equal(routing["perm"].cpu().numpy(), p)
    if n_diff == 0:
        assert np.array_equal(c, np.bincount(ridx.reshape(-1), minlength=w.E))
    rng = np.random.default_rng(1234)
    rows = np.sort(rng.choice(w.T, size=n_sample, replace=False))
    ref = G.oracle_forward(w, h, rows=rows)
    same = P.same_selection_mask(gidx[rows], ref["topk_idx"])
    G.check_output(G.y_numpy(y)[rows], ref["y"], rows_ok=same, what=name)


@pytest.mark.parametrize("T,Fs", [(64, 512), (512, 512), (512, 0), (513, 512)])
def test_select_kernel_builds_the_decode_index(T, Fs):
    """T * k <= 4096 (one index chunk) and E <= 256: the router's selection kernel also builds
    the expert order and tile lists (its last CTA); T=513 takes the separate index kernels.
    counts / offsets / perm against the oracle's expert order of the GPU selection, the launch
    count, and y on a sample of tokens against the oracle (XS.2 widths, with and without the
    shared expert)."""
    w = I.get("c2_xs2_small").with_(T=T, shared_intermediate_size=Fs)
    h, dev = _device_workload(w)
    y, routing, _ = G.run_forward(w, dev)
    launches = M.last_launch_count()
    gidx = routing["topk_idx"].cpu().numpy()
    c, o, p = O.expert_order(gidx, w.E)
    assert np.array_equal(routing["counts"].cpu().numpy(), c)
    assert np.array_equal(routing["offsets"].cpu().numpy(), o)
    assert np.array_equal(routing["perm"].cpu().numpy(), p)
    ridx, rw, scores, _ = O.route(h["x"], h["w_router"], None, w.k)
    G.check_routing(gidx, routing["topk_w"].cpu().numpy(),
                    {"topk_idx": ridx, "topk_w": rw, "scores": scores}, w.k)
    rng = np.random.default_rng(7)
    rows = np.sort(rng.choice(w.T, size=min(w.T, 48), replace=False))
    ref = G.oracle_forward(w, h, rows=rows)
    same = P.same_selection_mask(gidx[rows], ref["topk_idx"])
    G.check_output(G.y_numpy(y)[rows], ref["y"], rows_ok=same, what=f"T={T} Fs={Fs}")
    # router logits, selection (+ index when fused), [the one-launch index builder], W_down
    # and (with a shared expert) its W_down converted to fp16 (bf16 weights passed),
    # gate/up, down, combine
    fused = T * w.k <= 4096
    expected = 2 + (0 if fused else 1) + (2 if Fs else 1) + 3
    assert launches == expected, (launches, expected)


def test_decode_fresh_batches():
    import torch
    w = I.get("c5_decode")
    dev = I.device_inputs(w)
    h = G.device_to_host(dev)
    layer = M.MoeLayer(dev, w.d_model, w.E, w.k, w.F, w.Fs, w.routed_scaling_factor,
                       max_tokens=w.T)
    ring = I.device_decode_ring(w, 3)
    for i in range(3):
        y = layer.forward(ring[i])
        torch.cuda.synchronize()
        hx = dict(h, x=P.to_numpy_bf16(ring[i]))
        assert np.array_equal(hx["x"], I.decode_batch_host(w, i))
        ref = G.oracle_forward(w, hx)
        idx = layer.routing["topk_idx"][:w.T].cpu().numpy()
        G.check_routing(idx, layer.routing["topk_w"][:w.T].cpu().numpy(), ref, w.k)
        same = P.same_selection_mask(idx, ref["topk_idx"])
        G.check_output(G.y_numpy(y), ref["y"], rows_ok=same, what=f"decode batch {i}")
