"""Seeded synthetic inputs for the MoE layer: workload table and generator.

This module holds no arithmetic of the layer itself (no routing, no FFN).
It only says which tensors exist for each workload, how large they are and
how their values are drawn, so that the CUDA path and the CPU oracle can be
fed exactly the same bits.

Generator (one definition, two implementations that agree bit for bit):

* Counter-based uniform bits: Philox4x32-10 (Salmon, Moraes, Dror, Shaw,
  "Parallel random numbers: as easy as 1, 2, 3", SC'11).  The key is the
  64-bit seed, the counter is (block_lo, block_hi, tensor_id, 0), where
  block = element_index // 2.  One Philox call yields four 32-bit words.
* Normal deviates: element 2*block + h takes words (2h, 2h+1) as uniforms
  u_a = (w_a + 0.5) / 2**32 and u_b = (w_b + 0.5) / 2**32 and forms
  z = sqrt(-2 ln u_a) * cos(2 pi u_b) in float64 (the Box-Muller transform,
  cosine branch only).
* Scaling and storage: v = z * sigma in float64, rounded once, to nearest
  even, to bfloat16.  Tensors are returned as uint16 bit patterns.

``generate_numpy`` is the host implementation (slow, used for small tensors
and for cross-checking); ``generate_cuda`` runs the same definition in a
small CUDA kernel that lives in its own shared library, separate from the
MoE library, for the multi-gigabyte weight tensors.

Workloads follow the layer shapes of the Laguna XS.2 and M.1 models
(Laguna M.1/XS.2 Technical Report summary, §3.1; Laguna-M.1-base spec sheet,
"Mixture of experts" and "Shape" sections).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field

import numpy as np

# Tensor ids: the third Philox counter word, one per tensor of a workload.
TID_X = 0
TID_W_ROUTER = 1
TID_BIAS_PERM = 2
TID_W_GATE = 3
TID_W_UP = 4
TID_W_DOWN = 5
TID_WS_GATE = 6
TID_WS_UP = 7
TID_WS_DOWN = 8
TID_DECODE_BASE = 100  # decode batch i uses tensor id 100 + i

_MASK32 = 0xFFFFFFFF
_PHILOX_M0 = 0xD2511F53
_PHILOX_M1 = 0xCD9E8D57
_PHILOX_W0 = 0x9E3779B9
_PHILOX_W1 = 0xBB67AE85
_TWO_PI = 6.283185307179586


@dataclass(frozen=True)
class Workload:
    """One synthetic MoE-layer workload.

    Field names follow the model-config keys of the Laguna-M.1-base spec
    sheet ("Mixture of experts": num_experts, num_experts_per_tok,
    moe_intermediate_size, moe_routed_scaling_factor, norm_topk_prob).
    """

    name: str
    T: int
    d_model: int
    num_experts: int
    num_experts_per_tok: int
    moe_intermediate_size: int
    shared_intermediate_size: int
    sigma_x: float
    sigma_w: float
    sigma_router: float
    routed_scaling_factor: float = 2.5
    zipf_s: float = 0.0          # 0 = no router bias
    zipf_alpha: float = 0.0      # calibrated scale of the Zipf bias
    decode_batches: int = 0      # >0: a ring of fresh token batches
    seed: int = 0
    note: str = field(default="", compare=False)

    @property
    def E(self):
        return self.num_experts

    @property
    def k(self):
        return self.num_experts_per_tok

    @property
    def F(self):
        return self.moe_intermediate_size

    @property
    def Fs(self):
        return self.shared_intermediate_size

    def with_(self, **kw):
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    "c1_tiny": Workload("c1_tiny", T=64, d_model=256, num_experts=16, num_experts_per_tok=4,
                        moe_intermediate_size=128, shared_intermediate_size=128,
                        sigma_x=1.0, sigma_w=0.02, sigma_router=0.05,
                        note="tiny layer, T=64 d=256 E=16 top-4 F=Fs=128"),
    "c2_xs2_small": Workload("c2_xs2_small", T=4096, d_model=2048, num_experts=256,
                             num_experts_per_tok=8, moe_intermediate_size=512,
                             shared_intermediate_size=512, sigma_x=1.0, sigma_w=0.02,
                             sigma_router=0.02,
                             note="XS.2-shaped layer, T=4096, near-uniform routing"),
    "c3_xs2_prefill_zipf": Workload("c3_xs2_prefill_zipf", T=32768, d_model=2048,
                                    num_experts=256, num_experts_per_tok=8,
                                    moe_intermediate_size=512, shared_intermediate_size=512,
                                    sigma_x=1.0, sigma_w=0.02, sigma_router=0.02,
                                    zipf_s=1.1, zipf_alpha=-1.0,
                                    note="XS.2-shaped prefill, T=32768, Zipf-ranked router bias"),
    "c4_m1_width": Workload("c4_m1_width", T=16384, d_model=4096, num_experts=256,
                            num_experts_per_tok=8, moe_intermediate_size=1024,
                            shared_intermediate_size=1024, sigma_x=1.0, sigma_w=0.015,
                            sigma_router=0.02,
                            note="M.1-width layer, T=16384, d=4096, F=Fs=1024"),
    # M.1 as its spec sheet configures the layer (Mixture of experts: 16 experts
    # per token, routed scaling factor 1), at the M.1 widths of c4_m1_width.
    "c6_m1_top16": Workload("c6_m1_top16", T=16384, d_model=4096, num_experts=256,
                            num_experts_per_tok=16, moe_intermediate_size=1024,
                            shared_intermediate_size=1024, sigma_x=1.0, sigma_w=0.015,
                            sigma_router=0.02, routed_scaling_factor=1.0,
                            note="M.1-faithful layer: top-16 of 256, routed scale 1.0, "
                                 "T=16384, d=4096, F=Fs=1024"),
    "c5_decode": Workload("c5_decode", T=64, d_model=2048, num_experts=256,
                          num_experts_per_tok=8, moe_intermediate_size=512,
                          shared_intermediate_size=512, sigma_x=1.0, sigma_w=0.02,
                          sigma_router=0.02, decode_batches=1000,
                          note="decode-shaped, T=64, fresh batch per iteration"),
}


# The Zipf scale of the skewed prefill workload is written by
# oracle/calibrate_zipf.py (bisection on the oracle's routing, so that the
# hottest expert receives about 10x the mean load) into zipf_alpha.json.
def _load_calibrated_alpha():
    path = os.path.join(os.path.dirname(__file__), "zipf_alpha.json")
    if os.path.exists(path):
        import json
        with open(path) as f:
            return float(json.load(f)["alpha"])
    return None


_alpha = _load_calibrated_alpha()
if _alpha is not None:
    WORKLOADS["c3_xs2_prefill_zipf"] = WORKLOADS["c3_xs2_prefill_zipf"].with_(zipf_alpha=_alpha)


# --------------------------------------------------------------------------
# Philox4x32-10, host implementation (vectorised over counters)
# --------------------------------------------------------------------------

def philox4x32_10(c0, c1, c2, c3, k0: int, k1: int):
    """Philox4x32 with 10 rounds over uint32 counter arrays; returns 4 uint32 arrays."""
    M0 = np.uint64(_PHILOX_M0)
    M1 = np.uint64(_PHILOX_M1)
    m32 = np.uint64(_MASK32)
    s32 = np.uint64(32)
    c0 = np.asarray(c0, dtype=np.uint64)
    c1 = np.asarray(c1, dtype=np.uint64)
    c2 = np.asarray(c2, dtype=np.uint64)
    c3 = np.asarray(c3, dtype=np.uint64)
    for r in range(10):
        if r:
            k0 = (k0 + _PHILOX_W0) & _MASK32
            k1 = (k1 + _PHILOX_W1) & _MASK32
        p0 = M0 * c0
        p1 = M1 * c2
        n0 = (p1 >> s32) ^ c1 ^ np.uint64(k0)
        n1 = p1 & m32
        n2 = (p0 >> s32) ^ c3 ^ np.uint64(k1)
        n3 = p0 & m32
        c0, c1, c2, c3 = n0, n1, n2, n3
    return (c0.astype(np.uint32), c1.astype(np.uint32),
            c2.astype(np.uint32), c3.astype(np.uint32))


def f64_to_bf16_bits(v):
    """Round float64 values to bfloat16 (round to nearest, ties to even), once.

    Returns uint16 bit patterns.  Values below the bfloat16 normal range go
    through float32 first (never reached by the workloads' distributions).
    """
    v = np.asarray(v, dtype=np.float64)
    bits = v.view(np.uint64)
    lsb = (bits >> np.uint64(45)) & np.uint64(1)
    # half an ulp of bfloat16 (bit 44) minus one, plus the kept lsb: ties go to even
    rounded = (bits + np.uint64(0x0FFFFFFFFFFF) + lsb) & ~np.uint64(0x1FFFFFFFFFFF)
    f32 = rounded.view(np.float64).astype(np.float32)
    out = (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    tiny = np.abs(v) < 2.0 ** -126
    if np.any(tiny):
        t32 = v[tiny].astype(np.float32).view(np.uint32)
        t_lsb = (t32 >> np.uint32(16)) & np.uint32(1)
        out[tiny] = ((t32 + np.uint32(0x7FFF) + t_lsb) >> np.uint32(16)).astype(np.uint16)
    return out


def bf16_bits_to_f32(b):
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_f64_numpy(n: int, seed: int, tensor_id: int, start: int = 0):
    """Standard normal deviates (float64) for elements [start, start + n)."""
    if n <= 0:
        return np.zeros(0, dtype=np.float64)
    first_blk = start // 2
    last_blk = (start + n - 1) // 2
    blk = np.arange(first_blk, last_blk + 1, dtype=np.uint64)
    w0, w1, w2, w3 = philox4x32_10(blk & np.uint64(_MASK32), blk >> np.uint64(32),
                                   np.full(blk.shape, tensor_id, dtype=np.uint64),
                                   np.zeros(blk.shape, dtype=np.uint64),
                                   seed & _MASK32, (seed >> 32) & _MASK32)
    inv = 2.0 ** -32
    ua = np.empty(2 * blk.size, dtype=np.float64)
    ub = np.empty(2 * blk.size, dtype=np.float64)
    ua[0::2] = (w0.astype(np.float64) + 0.5) * inv
    ub[0::2] = (w1.astype(np.float64) + 0.5) * inv
    ua[1::2] = (w2.astype(np.float64) + 0.5) * inv
    ub[1::2] = (w3.astype(np.float64) + 0.5) * inv
    z = np.sqrt(-2.0 * np.log(ua)) * np.cos(_TWO_PI * ub)
    off = start - 2 * first_blk
    return z[off:off + n]


def generate_numpy(shape, seed: int, tensor_id: int, sigma: float, start: int = 0):
    """bfloat16 bits of sigma * N(0,1) for a tensor of ``shape`` (row-major).

    ``start`` offsets the element index, so a slice of a large tensor can be
    produced without generating the rest.
    """
    n = int(np.prod(shape)) if len(shape) else 1
    z = normal_f64_numpy(n, seed, tensor_id, start)
    return f64_to_bf16_bits(z * float(sigma)).reshape(shape)


def generate_numpy_chunked(shape, seed: int, tensor_id: int, sigma: float, chunk: int = 1 << 24):
    """generate_numpy for large tensors, drawn in slices to bound host memory."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for s in range(0, n, chunk):
        m = min(chunk, n - s)
        out[s:s + m] = generate_numpy((m,), seed, tensor_id, sigma, start=s)
    return out.reshape(shape)


def zipf_rank(E: int):
    """Popularity rank r_e in 1..E of each expert: a seed-1 Philox permutation."""
    e = np.arange(E, dtype=np.uint64)
    w0, _, _, _ = philox4x32_10(e, np.zeros_like(e), np.full(e.shape, TID_BIAS_PERM, np.uint64),
                                np.zeros_like(e), 1, 0)
    order = np.argsort(w0, kind="stable")
    rank = np.empty(E, dtype=np.int64)
    rank[order] = np.arange(1, E + 1)
    return rank


def zipf_bias(E: int, s: float, alpha: float):
    """Router bias b_e = -alpha * s * ln(r_e), float32 (a workload device, not part of the layer)."""
    r = zipf_rank(E).astype(np.float64)
    return (-alpha * s * np.log(r)).astype(np.float32)


# --------------------------------------------------------------------------
# Tensor recipe of a workload
# --------------------------------------------------------------------------

def tensor_specs(w: Workload):
    """(name, shape, tensor_id, sigma) for every bf16 tensor of the workload."""
    d, E, F, Fs = w.d_model, w.E, w.F, w.Fs
    specs = [
        ("x", (w.T, d), TID_X, w.sigma_x),
        ("w_router", (E, d), TID_W_ROUTER, w.sigma_router),
        ("w_gate", (E, F, d), TID_W_GATE, w.sigma_w),
        ("w_up", (E, F, d), TID_W_UP, w.sigma_w),
        ("w_down", (E, d, F), TID_W_DOWN, w.sigma_w),
    ]
    if Fs > 0:
        specs += [
            ("ws_gate", (Fs, d), TID_WS_GATE, w.sigma_w),
            ("ws_up", (Fs, d), TID_WS_UP, w.sigma_w),
            ("ws_down", (d, Fs), TID_WS_DOWN, w.sigma_w),
        ]
    return specs


def router_bias(w: Workload):
    if w.zipf_s <= 0.0:
        return None
    if w.zipf_alpha < 0:
        raise RuntimeError(f"{w.name}: Zipf scale not calibrated (run oracle/calibrate_zipf.py)")
    return zipf_bias(w.E, w.zipf_s, w.zipf_alpha)


def host_inputs(w: Workload):
    """All tensors of a workload as numpy arrays on the host (bf16 as uint16 bits).

    Only sensible for small workloads; large ones use ``device_inputs``.
    """
    out = {}
    for name, shape, tid, sigma in tensor_specs(w):
        out[name] = generate_numpy(shape, w.seed, tid, sigma)
    out["router_bias"] = router_bias(w)
    return out


def decode_batch_host(w: Workload, i: int):
    return generate_numpy((w.T, w.d_model), w.seed, TID_DECODE_BASE + i, w.sigma_x)


# --------------------------------------------------------------------------
# CUDA implementation of the same generator (separate shared library)
# --------------------------------------------------------------------------

_GEN_LIB = None


def _gen_lib():
    global _GEN_LIB
    if _GEN_LIB is None:
        path = os.path.join(os.path.dirname(__file__), "libmoe_gen.so")
        if not os.path.exists(path):
            raise RuntimeError(f"input generator library missing: {path} (run __graft_entry__.build())")
        lib = ctypes.CDLL(path)
        lib.moe_gen_normal_bf16.restype = ctypes.c_int
        lib.moe_gen_normal_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64,
                                            ctypes.c_uint32, ctypes.c_double, ctypes.c_int64,
                                            ctypes.c_void_p]
        _GEN_LIB = lib
    return _GEN_LIB


def generate_cuda(t, seed: int, tensor_id: int, sigma: float, start: int = 0):
    """Fill the contiguous CUDA tensor ``t`` (2-byte elements) with the generator's bf16 bits."""
    import torch
    assert t.is_cuda and t.is_contiguous() and t.element_size() == 2
    stream = torch.cuda.current_stream(t.device).cuda_stream
    rc = _gen_lib().moe_gen_normal_bf16(ctypes.c_void_p(t.data_ptr()), t.numel(), seed,
                                        tensor_id, float(sigma), start, ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"moe_gen_normal_bf16 failed with CUDA error {rc}")
    return t


def device_inputs(w: Workload, device="cuda"):
    """All tensors of a workload on the GPU (torch.bfloat16), drawn by the CUDA generator."""
    import torch
    out = {}
    for name, shape, tid, sigma in tensor_specs(w):
        t = torch.empty(shape, dtype=torch.bfloat16, device=device)
        generate_cuda(t, w.seed, tid, sigma)
        out[name] = t
    b = router_bias(w)
    out["router_bias"] = None if b is None else torch.from_numpy(b).to(device)
    return out


def device_decode_ring(w: Workload, n: int, device="cuda"):
    """A [n, T, d] ring of fresh decode batches (batch i uses tensor id 100 + i)."""
    import torch
    ring = torch.empty((n, w.T, w.d_model), dtype=torch.bfloat16, device=device)
    for i in range(n):
        generate_cuda(ring[i], w.seed, TID_DECODE_BASE + i, w.sigma_x)
    return ring


def get(name: str) -> Workload:
    return WORKLOADS[name]
