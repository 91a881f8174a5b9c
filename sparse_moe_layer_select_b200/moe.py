"""Python binding of the C ABI in include/moe.h (argument marshalling only).

Every step of the layer runs in the CUDA kernels of libmoe_b200.so; this
module only turns torch tensors into device pointers and checks status
codes.  There is no fallback: if the library is missing, importing the
functions raises.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED_SHAPE = 2
MOE_ERR_WORKSPACE_TOO_SMALL = 3
MOE_ERR_CUDA = 4
MOE_ERR_DEVICE_TIMEOUT = 5
MOE_ERR_DEVICE_BOUNDS = 6

MOE_FLAG_ROUTER_CUDA_CORE = 1
MOE_FLAG_ROUTER_TENSOR = 2
MOE_FLAG_DOWN_F16 = 4
MOE_FLAG_GEMM_SINGLE_CTA = 8
MOE_FLAG_GEMM_PAIR = 16
MOE_FLAG_BIAS_SELECTION_ONLY = 32
MOE_FLAG_FP8_EXPERTS = 64
MOE_FLAG_COMBINE_REDUCE = 128
MOE_FLAG_FUSED_EXPERTS = 256

# Every symbol the header declares (checked by the CPU tests).
EXPORTED = ["moe_workspace_size", "moe_route", "moe_permute", "moe_forward",
            "moe_read_device_status", "moe_selftest_bounded_wait", "moe_status_string",
            "moe_last_launch_count", "moe_profile_next_forward", "moe_prepare_down_f16",
            "moe_logits_offset", "moe_permute_static", "moe_route_masked",
            "moe_forward_masked", "moe_prepare_fp8", "moe_forward_fp8"]

# Expert id of a (token, slot) pair that is not routed (a padding token).
MOE_NOT_ROUTED = -1


class MoeError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({code})")


class moe_dims_t(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("T", ctypes.c_int32),
                ("d_model", ctypes.c_int32), ("num_experts", ctypes.c_int32),
                ("num_experts_per_tok", ctypes.c_int32), ("moe_intermediate_size", ctypes.c_int32),
                ("shared_intermediate_size", ctypes.c_int32),
                ("routed_scaling_factor", ctypes.c_float), ("norm_topk_prob", ctypes.c_int32),
                ("flags", ctypes.c_int32)]


class moe_weights_t(ctypes.Structure):
    _fields_ = [("w_router", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
                ("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p),
                ("w_down", ctypes.c_void_p), ("ws_gate", ctypes.c_void_p),
                ("ws_up", ctypes.c_void_p), ("ws_down", ctypes.c_void_p),
                ("w_down_f16", ctypes.c_void_p), ("ws_down_f16", ctypes.c_void_p)]


class moe_fp8_weights_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down",
                 "ws_gate", "ws_up", "ws_down", "ss_gate", "ss_up", "ss_down")]


class moe_routing_t(ctypes.Structure):
    _fields_ = [("topk_idx", ctypes.c_void_p), ("topk_w", ctypes.c_void_p),
                ("counts", ctypes.c_void_p), ("offsets", ctypes.c_void_p),
                ("perm", ctypes.c_void_p)]


_LIB = None


def lib():
    """The loaded C library (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} "
                               "(run python -m sparse_moe_layer_select_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        D = ctypes.POINTER(moe_dims_t)
        L.moe_workspace_size.restype = ctypes.c_size_t
        L.moe_workspace_size.argtypes = [D]
        L.moe_route.restype = ctypes.c_int
        L.moe_route.argtypes = [D, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.moe_permute.restype = ctypes.c_int
        L.moe_permute.argtypes = [D, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.moe_forward.restype = ctypes.c_int
        L.moe_forward.argtypes = [D, ctypes.POINTER(moe_weights_t), P, P,
                                  ctypes.POINTER(moe_routing_t), P, ctypes.c_size_t, P]
        L.moe_prepare_fp8.restype = ctypes.c_int
        L.moe_prepare_fp8.argtypes = [D, ctypes.POINTER(moe_weights_t),
                                      ctypes.POINTER(moe_fp8_weights_t), P, ctypes.c_size_t, P]
        L.moe_forward_fp8.restype = ctypes.c_int
        L.moe_forward_fp8.argtypes = [D, ctypes.POINTER(moe_weights_t),
                                      ctypes.POINTER(moe_fp8_weights_t), P, P,
                                      ctypes.POINTER(moe_routing_t), P, ctypes.c_size_t, P]
        L.moe_route_masked.restype = ctypes.c_int
        L.moe_route_masked.argtypes = [D, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.moe_forward_masked.restype = ctypes.c_int
        L.moe_forward_masked.argtypes = [D, ctypes.POINTER(moe_weights_t), P, P, P,
                                         ctypes.POINTER(moe_routing_t), P, ctypes.c_size_t, P]
        L.moe_read_device_status.restype = ctypes.c_int
        L.moe_read_device_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int32)]
        L.moe_selftest_bounded_wait.restype = ctypes.c_int
        L.moe_selftest_bounded_wait.argtypes = [P, ctypes.c_size_t, ctypes.c_uint32, P]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_last_launch_count.restype = ctypes.c_int32
        L.moe_last_launch_count.argtypes = []
        L.moe_prepare_down_f16.restype = ctypes.c_int
        L.moe_prepare_down_f16.argtypes = [D, P, P, P, P, P, ctypes.c_size_t, P]
        L.moe_permute_static.restype = ctypes.c_int
        L.moe_permute_static.argtypes = [D, P, P, P, P, P]
        L.moe_logits_offset.restype = ctypes.c_size_t
        L.moe_logits_offset.argtypes = [D]
        L.moe_profile_next_forward.restype = ctypes.c_int
        L.moe_profile_next_forward.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32]
        _LIB = L
    return _LIB


def status_string(code: int) -> str:
    return lib().moe_status_string(code).decode()


def make_dims(T, d_model, num_experts, num_experts_per_tok, moe_intermediate_size,
              shared_intermediate_size, routed_scaling_factor=2.5, norm_topk_prob=1, flags=0):
    return moe_dims_t(ctypes.sizeof(moe_dims_t), T, d_model, num_experts, num_experts_per_tok,
                      moe_intermediate_size, shared_intermediate_size, routed_scaling_factor,
                      norm_topk_prob, flags)


def dims_for(w, T=None, flags=0, norm_topk_prob=1):
    """moe_dims_t of an inputs.Workload (optionally with another token count)."""
    return make_dims(w.T if T is None else T, w.d_model, w.E, w.k, w.F, w.Fs,
                     w.routed_scaling_factor, norm_topk_prob, flags)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(code, where):
    if code != MOE_OK:
        raise MoeError(code, where)


def workspace_size(dims) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(dims)))


def alloc_workspace(dims, device="cuda"):
    import torch
    n = workspace_size(dims)
    if n == 0:
        raise MoeError(MOE_ERR_UNSUPPORTED_SHAPE, "moe_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def route(dims, x, w_router, bias, topk_idx, topk_w, ws, stream=None, token_mask=None):
    """moe_route, or moe_route_masked when a [T] uint8 token_mask (0 = padding) is given."""
    if token_mask is None:
        _check(lib().moe_route(ctypes.byref(dims), _p(x), _p(w_router), _p(bias), _p(topk_idx),
                               _p(topk_w), _p(ws), ws.numel(), _stream(stream)), "moe_route")
    else:
        _check(lib().moe_route_masked(ctypes.byref(dims), _p(x), _p(w_router), _p(bias),
                                      _p(token_mask), _p(topk_idx), _p(topk_w), _p(ws),
                                      ws.numel(), _stream(stream)), "moe_route_masked")


def permute(dims, topk_idx, counts, offsets, perm, ws, x=None, x_perm=None, stream=None):
    _check(lib().moe_permute(ctypes.byref(dims), _p(topk_idx), _p(counts), _p(offsets), _p(perm),
                             _p(x), _p(x_perm), _p(ws), ws.numel(), _stream(stream)),
           "moe_permute")


def weights_struct(W):
    return moe_weights_t(*[None if W.get(k) is None else W[k].data_ptr() for k in
                           ("w_router", "router_bias", "w_gate", "w_up", "w_down", "ws_gate",
                            "ws_up", "ws_down", "w_down_f16", "ws_down_f16")])


def prepare_down_f16(dims, W, stream=None):
    """fp16 copies of the down projections (moe_prepare_down_f16); adds them to W and
    returns the device status of the conversion."""
    import torch
    W["w_down_f16"] = torch.empty(W["w_down"].shape, dtype=torch.float16, device=W["w_down"].device)
    if W.get("ws_down") is not None:
        W["ws_down_f16"] = torch.empty(W["ws_down"].shape, dtype=torch.float16,
                                       device=W["ws_down"].device)
    hdr = torch.zeros(256, dtype=torch.uint8, device=W["w_down"].device)
    _check(lib().moe_prepare_down_f16(ctypes.byref(dims), _p(W["w_down"]), _p(W.get("ws_down")),
                                      _p(W["w_down_f16"]), _p(W.get("ws_down_f16")), _p(hdr), 256,
                                      _stream(stream)), "moe_prepare_down_f16")
    return read_device_status(hdr, stream)


FP8_FIELDS = ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down",
              "ws_gate", "ws_up", "ws_down", "ss_gate", "ss_up", "ss_down")


def prepare_fp8(dims, W, stream=None):
    """FP8 copies of the expert weights (moe_prepare_fp8): returns a dict of device tensors
    (e4m3 codes as uint8, float32 row scales) and the device status."""
    import torch
    dev = W["w_gate"].device
    E, F, d = W["w_gate"].shape
    Q = {"w_gate": torch.empty((E, F, d), dtype=torch.uint8, device=dev),
         "w_up": torch.empty((E, F, d), dtype=torch.uint8, device=dev),
         "w_down": torch.empty((E, d, F), dtype=torch.uint8, device=dev),
         "s_gate": torch.empty(E * F, dtype=torch.float32, device=dev),
         "s_up": torch.empty(E * F, dtype=torch.float32, device=dev),
         "s_down": torch.empty(E * d, dtype=torch.float32, device=dev)}
    if W.get("ws_gate") is not None:
        Fs = W["ws_gate"].shape[0]
        Q.update(ws_gate=torch.empty((Fs, d), dtype=torch.uint8, device=dev),
                 ws_up=torch.empty((Fs, d), dtype=torch.uint8, device=dev),
                 ws_down=torch.empty((d, Fs), dtype=torch.uint8, device=dev),
                 ss_gate=torch.empty(Fs, dtype=torch.float32, device=dev),
                 ss_up=torch.empty(Fs, dtype=torch.float32, device=dev),
                 ss_down=torch.empty(d, dtype=torch.float32, device=dev))
    hdr = torch.zeros(256, dtype=torch.uint8, device=dev)
    _check(lib().moe_prepare_fp8(ctypes.byref(dims), ctypes.byref(weights_struct(W)),
                                 ctypes.byref(fp8_struct(Q)), _p(hdr), 256, _stream(stream)),
           "moe_prepare_fp8")
    return Q, read_device_status(hdr, stream)


def fp8_struct(Q):
    return moe_fp8_weights_t(*[None if Q.get(k) is None else Q[k].data_ptr() for k in FP8_FIELDS])


def forward_fp8(dims, weights, fp8, x, y, routing, ws, stream=None):
    """moe_forward_fp8 (dims.flags must include MOE_FLAG_FP8_EXPERTS)."""
    ws_s = weights if isinstance(weights, moe_weights_t) else weights_struct(weights)
    q_s = fp8 if isinstance(fp8, moe_fp8_weights_t) else fp8_struct(fp8)
    r_s = routing if isinstance(routing, moe_routing_t) else routing_struct(routing)
    _check(lib().moe_forward_fp8(ctypes.byref(dims), ctypes.byref(ws_s), ctypes.byref(q_s), _p(x),
                                 _p(y), ctypes.byref(r_s), _p(ws), ws.numel(), _stream(stream)),
           "moe_forward_fp8")


def logits_offset(dims) -> int:
    return int(lib().moe_logits_offset(ctypes.byref(dims)))


def routing_struct(R):
    return moe_routing_t(*[R[k].data_ptr() for k in ("topk_idx", "topk_w", "counts", "offsets",
                                                     "perm")])


def forward(dims, weights, x, y, routing, ws, stream=None, token_mask=None):
    """moe_forward on torch tensors; weights/routing are dicts of tensors (or prebuilt structs).
    With a [T] uint8 token_mask (0 = padding token) it calls moe_forward_masked."""
    ws_s = weights if isinstance(weights, moe_weights_t) else weights_struct(weights)
    r_s = routing if isinstance(routing, moe_routing_t) else routing_struct(routing)
    if token_mask is None:
        _check(lib().moe_forward(ctypes.byref(dims), ctypes.byref(ws_s), _p(x), _p(y),
                                 ctypes.byref(r_s), _p(ws), ws.numel(), _stream(stream)),
               "moe_forward")
    else:
        _check(lib().moe_forward_masked(ctypes.byref(dims), ctypes.byref(ws_s), _p(x),
                                        _p(token_mask), _p(y), ctypes.byref(r_s), _p(ws),
                                        ws.numel(), _stream(stream)), "moe_forward_masked")


def alloc_routing(dims, device="cuda"):
    import torch
    T, k, E = dims.T, dims.num_experts_per_tok, dims.num_experts
    return {"topk_idx": torch.empty((T, k), dtype=torch.int32, device=device),
            "topk_w": torch.empty((T, k), dtype=torch.float32, device=device),
            "counts": torch.empty(E, dtype=torch.int32, device=device),
            "offsets": torch.empty(E + 1, dtype=torch.int32, device=device),
            "perm": torch.empty(T * k, dtype=torch.int32, device=device)}


def read_device_status(ws, stream=None):
    site = ctypes.c_int32(0)
    code = lib().moe_read_device_status(_p(ws), _stream(stream), ctypes.byref(site))
    return int(code), int(site.value)


def selftest_bounded_wait(ws, limit_us, stream=None):
    _check(lib().moe_selftest_bounded_wait(_p(ws), ws.numel(), limit_us, _stream(stream)),
           "moe_selftest_bounded_wait")


def profile_next_forward(events):
    """Arm per-kernel event recording for the next forward call (torch.cuda.Event list)."""
    if events is None:
        _check(lib().moe_profile_next_forward(None, 0), "moe_profile_next_forward")
        return
    import torch
    for e in events:  # torch creates the CUDA event handle on first record
        if e.cuda_event == 0:
            e.record(torch.cuda.current_stream())
    if any(e.cuda_event == 0 for e in events):
        raise RuntimeError("profile_next_forward: CUDA events were not created")
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    profile_next_forward._keep = arr
    _check(lib().moe_profile_next_forward(arr, len(events)), "moe_profile_next_forward")


# Stage names of the kernel-marker intervals recorded by moe_forward, in order.
FORWARD_STAGES = ("router", "index", "gemm1_swiglu", "gemm2_down_scale", "combine")


def last_launch_count() -> int:
    return int(lib().moe_last_launch_count())


class MoeLayer:
    """A layer instance: device weights, routing buffers and workspace, reused across calls."""

    def __init__(self, weights: dict, d_model, num_experts, num_experts_per_tok,
                 moe_intermediate_size, shared_intermediate_size, routed_scaling_factor=2.5,
                 max_tokens=1, flags=0, device="cuda", prepare=True, fp8=False):
        self.W = dict(weights)
        self.cfg = dict(d_model=d_model, num_experts=num_experts,
                        num_experts_per_tok=num_experts_per_tok,
                        moe_intermediate_size=moe_intermediate_size,
                        shared_intermediate_size=shared_intermediate_size,
                        routed_scaling_factor=routed_scaling_factor, flags=flags)
        self.device = device
        self.fp8 = None
        if fp8:  # one-time FP8 copies of the expert weights (model-load step)
            self.cfg["flags"] |= MOE_FLAG_FP8_EXPERTS
            self.fp8, (code, site) = prepare_fp8(self.dims(1), self.W)
            if code != MOE_OK:
                raise MoeError(code, f"moe_prepare_fp8 (site {site})")
            self._q_struct = fp8_struct(self.fp8)
        elif prepare:  # one-time fp16 copy of the down projections (model-load step)
            self.cfg["flags"] |= MOE_FLAG_DOWN_F16
            code, site = prepare_down_f16(self.dims(1), self.W)
            if code != MOE_OK:
                raise MoeError(code, f"moe_prepare_down_f16 (site {site})")
        self._ws_struct = weights_struct(self.W)
        self._reserve(max_tokens)

    def dims(self, T):
        c = self.cfg
        return make_dims(T, c["d_model"], c["num_experts"], c["num_experts_per_tok"],
                         c["moe_intermediate_size"], c["shared_intermediate_size"],
                         c["routed_scaling_factor"], 1, c["flags"])

    def _reserve(self, T):
        self.max_tokens = T
        d = self.dims(T)
        self.ws = alloc_workspace(d, self.device)
        self.routing = alloc_routing(d, self.device)
        self._r_struct = routing_struct(self.routing)

    def forward(self, x, y=None, stream=None, token_mask=None):
        import torch
        T = x.shape[0]
        if T > self.max_tokens:
            self._reserve(T)
        if y is None:
            y = torch.empty_like(x)
        d = self.dims(T)
        if self.fp8 is not None:
            if token_mask is not None:
                raise ValueError("the FP8-expert forward takes no token mask")
            forward_fp8(d, self._ws_struct, self._q_struct, x, y, self._r_struct, self.ws, stream)
        else:
            forward(d, self._ws_struct, x, y, self._r_struct, self.ws, stream,
                    token_mask=token_mask)
        return y
