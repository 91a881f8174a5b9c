"""GPU parity of the reduce combine (MOE_FLAG_COMBINE_REDUCE) and of the fused
expert kernel (MOE_FLAG_FUSED_EXPERTS) against the oracle.

With the reduce combine the down GEMM adds every scaled routed row and every
shared-expert row straight into fp32 token rows (bulk reduce-adds at L2) and a
last kernel rounds them to bf16.  The fused kernel does the same from one
kernel that also runs the gate/up GEMM and keeps h in tensor memory.

The same rules as the default path: routing bit-exact up to the exempt
near-ties, y within relative Frobenius 1e-2 and |dy| <= 2e-2 (|y| + 0.05) per
element.  The order of a token's additions is not fixed, so repeated runs are
compared within the redundant-run bound |dy| <= 1e-3 (|y| + 0.05) instead of
bit for bit.
"""
import numpy as np
import pytest

from oracle import moe_oracle as O
from sparse_moe_layer_select_b200 import inputs as I
from sparse_moe_layer_select_b200 import moe as M
from tests import gpu_common as G
from tests import parity as P

pytestmark = pytest.mark.gpu

RED = M.MOE_FLAG_COMBINE_REDUCE
FUSED = M.MOE_FLAG_FUSED_EXPERTS
ENGINES = [M.MOE_FLAG_GEMM_PAIR, M.MOE_FLAG_GEMM_SINGLE_CTA]
# the reduce combine on both GEMM engines, and the fused kernel (one engine)
VARIANTS = [RED | M.MOE_FLAG_GEMM_PAIR, RED | M.MOE_FLAG_GEMM_SINGLE_CTA, FUSED]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    torch.cuda.set_device(0)
    from sparse_moe_layer_select_b200 import build as B
    B.build()
    yield


def _small(w):
    h = I.host_inputs(w)
    return h, G.host_to_device(h)


def _close(a, b, rel=1e-3):
    return np.all(np.abs(a - b) <= rel * (np.abs(b) + 0.05))


@pytest.mark.parametrize("flags", VARIANTS)
@pytest.mark.parametrize("T", [1, 129, 300, 1500])
def test_reduce_combine_matches_oracle(T, flags):
    w = I.get("c1_tiny").with_(T=T)
    h, dev = _small(w)
    y, routing, _ = G.run_forward(w, dev, flags=flags)
    ref = G.oracle_forward(w, h)
    G.check_routing(routing["topk_idx"].cpu().numpy(), routing["topk_w"].cpu().numpy(), ref, w.k)
    G.check_output(G.y_numpy(y), ref["y"], what=f"reduce T={T}")


@pytest.mark.parametrize("flags", VARIANTS)
def test_reduce_combine_xs2_dims_full_oracle(flags):
    w = I.get("c2_xs2_small").with_(T=1000)
    dev = I.device_inputs(w)
    h = G.device_to_host(dev)
    y, routing, _ = G.run_forward(w, dev, flags=flags)
    ref = G.oracle_forward(w, h)
    G.check_routing(routing["topk_idx"].cpu().numpy(), routing["topk_w"].cpu().numpy(), ref, w.k)
    same = P.same_selection_mask(routing["topk_idx"].cpu().numpy(), ref["topk_idx"])
    G.check_output(G.y_numpy(y), ref["y"], rows_ok=same, what="reduce xs2 T=1000")


@pytest.mark.parametrize("flags", [RED, FUSED])
@pytest.mark.parametrize("Fs", [0, 128])
def test_reduce_combine_padding_mask_and_no_shared_expert(Fs, flags):
    import torch
    w = I.get("c1_tiny").with_(T=400, shared_intermediate_size=Fs)
    h, dev = _small(w)
    mask = (np.random.default_rng(3).random(w.T) >= 0.4).astype(np.uint8)
    dims = M.dims_for(w, flags=flags)
    ws = M.alloc_workspace(dims)
    ws.fill_(0xFF)
    routing = M.alloc_routing(dims)
    y = torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda")
    M.forward(dims, dev, dev["x"], y, routing, ws, token_mask=torch.from_numpy(mask).cuda())
    torch.cuda.synchronize()
    assert M.read_device_status(ws)[0] == 0
    ref = O.moe_forward(h["x"], h["w_router"], h["w_gate"], h["w_up"], h["w_down"], w.k,
                        ws_gate=h.get("ws_gate"), ws_up=h.get("ws_up"), ws_down=h.get("ws_down"),
                        routed_scaling_factor=w.routed_scaling_factor, token_mask=mask)
    G.check_output(G.y_numpy(y), ref["y"], what=f"reduce mask Fs={Fs}")
    if Fs == 0:
        assert np.all(G.y_numpy(y)[mask == 0] == 0.0)


@pytest.mark.parametrize("flags", [RED, FUSED])
def test_reduce_combine_runs_agree_with_each_other_and_the_default_path(flags):
    """Five runs of the same inputs: routing and permutation identical bit for bit, y within
    the redundant-run bound of each other and of the deterministic default combine."""
    import torch
    w = I.get("c1_tiny").with_(T=1000)
    _, dev = _small(w)
    y0, r0, _ = G.run_forward(w, dev)
    base = G.y_numpy(y0)
    outs = []
    for _ in range(5):
        y, routing, _ = G.run_forward(w, dev, flags=flags)
        outs.append((G.y_numpy(y), routing["topk_idx"].cpu().numpy(),
                     routing["perm"].cpu().numpy()))
    for yv, idx, perm in outs:
        assert np.array_equal(idx, r0["topk_idx"].cpu().numpy())
        assert np.array_equal(perm, r0["perm"].cpu().numpy())
        assert _close(yv, outs[0][0]) and _close(yv, base)
    torch.cuda.synchronize()


@pytest.mark.parametrize("flags", [RED, FUSED])
@pytest.mark.parametrize("name", ["c3_xs2_prefill_zipf", "c4_m1_width"])
def test_reduce_combine_full_size_sample(name, flags):
    """Full-size batches (T=32768 with the Zipf-ranked bias, hot experts at 10x the mean;
    the M.1 widths, whose F = 1024 runs in two parts in the fused kernel): y on a sample."""
    w = I.get(name)
    dev = I.device_inputs(w)
    h = G.device_to_host(dev)
    y, routing, _ = G.run_forward(w, dev, flags=flags)
    gidx = routing["topk_idx"].cpu().numpy()
    rows = np.sort(np.random.default_rng(99).choice(w.T, size=512, replace=False))
    ref = G.oracle_forward(w, h, rows=rows)
    same = P.same_selection_mask(gidx[rows], ref["topk_idx"])
    G.check_output(G.y_numpy(y)[rows], ref["y"], rows_ok=same, what=f"{name} sample")


@pytest.mark.parametrize("F,Fs", [(1024, 1024), (768, 256), (256, 1536)])
def test_fused_kernel_ffn_parts(F, Fs):
    """FFN widths above 512 run in equal parts of at most 512 columns (1024: 2 x 512, 768:
    2 x 384, 1536: 3 x 512) whose partial down projections add into the same rows."""
    w = I.get("c1_tiny").with_(T=300, moe_intermediate_size=F, shared_intermediate_size=Fs)
    h, dev = _small(w)
    y, routing, _ = G.run_forward(w, dev, flags=FUSED)
    ref = G.oracle_forward(w, h)
    G.check_routing(routing["topk_idx"].cpu().numpy(), routing["topk_w"].cpu().numpy(), ref, w.k)
    G.check_output(G.y_numpy(y), ref["y"], what=f"fused F={F} Fs={Fs}")
