"""GPU parity of the reduce combine (MOE_FLAG_COMBINE_REDUCE) and of the fused
expert kernel (MOE_FLAG_FUSED_EXPERTS) against the oracle.

With the reduce combine the down GEMM adds every scaled routed row and every
shared-expert row straight into fp32 token rows (bulk reduce-adds at L2) and a
last kernel rounds them to bf16.  The fused kernel does the same from one
kernel that also runs the gate/up GEMM and keeps h in tensor memory.

The same rules as the default path: routing bit-exact up to the exempt
near-ties, y within relative Frobenius 1e-2 and |dy| <= 2e-2 (|y| + 0.05) per
element.  The order of a token's additions is not fixed, so repeated runs are
compared up to one bf16 step per element instead of bit for bit.
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


def _bf16_steps_apart(a, b):
    """Per element, how many bf16 steps apart two bf16 tensors (bit patterns) are."""
    def ordered(u):
        u = u.astype(np.int32)
        return np.where(u & 0x8000, -(u & 0x7FFF), u)
    return np.abs(ordered(a) - ordered(b))


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
    """Five runs of the same inputs: routing and permutation identical bit for bit to each
    other and to the default path; y of any two runs at most one bf16 step apart per element
    (the fp32 sums differ in their last bits with the order of the additions, which can move
    the final rounding to bf16 by one step) and every run within the oracle's bound.
    (Against the default path, which rounds h and every contribution to fp16 where these
    keep fp32 sums, y differs at that rounding's level: both are held to the oracle's
    bound.)"""
    import torch
    w = I.get("c1_tiny").with_(T=1000)
    h, dev = _small(w)
    y0, r0, _ = G.run_forward(w, dev)
    ref = G.oracle_forward(w, h)
    outs = []
    for _ in range(5):
        y, routing, _ = G.run_forward(w, dev, flags=flags)
        outs.append((P.to_numpy_bf16(y), routing["topk_idx"].cpu().numpy(),
                     routing["perm"].cpu().numpy(), G.y_numpy(y)))
    for bits, idx, perm, yv in outs:
        assert np.array_equal(idx, r0["topk_idx"].cpu().numpy())
        assert np.array_equal(perm, r0["perm"].cpu().numpy())
        assert int(_bf16_steps_apart(bits, outs[0][0]).max()) <= 1
        G.check_output(yv, ref["y"], what="reduce run")
    G.check_output(G.y_numpy(y0), ref["y"], what="default run")
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


@pytest.mark.parametrize("F,Fs", [(1024, 1024), (768, 256), (256, 1536), (640, 128)])
def test_fused_kernel_ffn_parts(F, Fs):
    """FFN widths above 512 run in equal parts of whole 128-column chunks, at most 512
    columns each (narrower ones when the batch has few row tiles), whose partial down
    projections add into the same token rows."""
    w = I.get("c1_tiny").with_(T=300, moe_intermediate_size=F, shared_intermediate_size=Fs)
    h, dev = _small(w)
    y, routing, _ = G.run_forward(w, dev, flags=FUSED)
    ref = G.oracle_forward(w, h)
    G.check_routing(routing["topk_idx"].cpu().numpy(), routing["topk_w"].cpu().numpy(), ref, w.k)
    G.check_output(G.y_numpy(y), ref["y"], what=f"fused F={F} Fs={Fs}")
