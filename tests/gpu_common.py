"""Shared helpers of the GPU tests: inputs on both sides, oracle calls, checks."""
import numpy as np

from oracle import moe_oracle as O
from sparse_moe_layer_select_b200 import inputs as I
from sparse_moe_layer_select_b200 import moe as M
from tests import parity as P

WEIGHT_KEYS = ("w_router", "w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down")


def host_to_device(h):
    import torch
    out = {}
    for k, v in h.items():
        if v is None:
            out[k] = None
        elif v.dtype == np.uint16:
            out[k] = torch.from_numpy(np.ascontiguousarray(v).view(np.int16)).view(torch.bfloat16).cuda()
        else:
            out[k] = torch.from_numpy(np.ascontiguousarray(v)).cuda()
    return out


def device_to_host(dev):
    out = {}
    for k, v in dev.items():
        if v is None:
            out[k] = None
        elif str(v.dtype) == "torch.bfloat16":
            out[k] = P.to_numpy_bf16(v)
        else:
            out[k] = v.cpu().numpy()
    return out


def run_forward(w, dev, T=None, flags=0, x=None, norm_topk_prob=1):
    """One moe_forward call; returns (y, routing dict, ws)."""
    import torch
    T = w.T if T is None else T
    dims = M.dims_for(w, T=T, flags=flags, norm_topk_prob=norm_topk_prob)
    ws = M.alloc_workspace(dims)
    ws.fill_(0xFF)  # poison: reads of never-written workspace surface as NaN
    routing = M.alloc_routing(dims)
    x = dev["x"] if x is None else x
    y = torch.empty((T, w.d_model), dtype=torch.bfloat16, device="cuda")
    M.forward(dims, dev, x, y, routing, ws)
    torch.cuda.synchronize()
    code, site = M.read_device_status(ws)
    assert code == 0, f"device status {M.status_string(code)} at site {site}"
    return y, routing, ws


def oracle_forward(w, h, rows=None, routing=None, norm_topk_prob=True):
    x = h["x"] if rows is None else h["x"][rows]
    return O.moe_forward(x, h["w_router"], h["w_gate"], h["w_up"], h["w_down"], w.k,
                         router_bias=h.get("router_bias"), ws_gate=h.get("ws_gate"),
                         ws_up=h.get("ws_up"), ws_down=h.get("ws_down"),
                         routed_scaling_factor=w.routed_scaling_factor, routing=routing,
                         norm_topk_prob=norm_topk_prob)


def check_routing(gpu_idx, gpu_w, ref, k, max_diff_frac=1e-3):
    n_ex, n_diff, fails = P.compare_routing(gpu_idx, gpu_w, ref["topk_idx"], ref["topk_w"],
                                            ref["scores"], k)
    assert not fails, f"routing failures (first 5 of {len(fails)}): {fails[:5]}"
    assert n_diff <= max(1, max_diff_frac * len(gpu_idx)), (n_diff, n_ex)
    return n_ex, n_diff


def check_output(got, ref_y, rows_ok=None, what=""):
    ok, rel, ratio = P.output_ok(got, ref_y, rows_ok)
    assert ok, f"{what}: rel Frobenius {rel:.3e} (<= 1e-2), worst element ratio {ratio:.3f} (<= 1)"
    return rel, ratio


def y_numpy(y):
    return y.float().cpu().numpy().astype(np.float64)
