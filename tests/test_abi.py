"""The C ABI library: it builds, loads, exports every declared symbol, and its
host-side argument checks return the documented codes (no GPU needed: these
paths return before any CUDA call)."""
import ctypes
import os
import re

import pytest

from sparse_moe_layer_select_b200 import build as B
from sparse_moe_layer_select_b200 import moe as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    B.build()
    return M.lib()


def _declared_functions():
    with open(os.path.join(ROOT, "include", "moe.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(L):
    declared = _declared_functions()
    assert "moe_forward" in declared and "moe_route" in declared and "moe_permute" in declared
    for name in declared:
        assert hasattr(L, name), name
    assert sorted(M.EXPORTED) == declared


def test_generator_library_exports(L):
    import sparse_moe_layer_select_b200.inputs as I
    assert hasattr(I._gen_lib(), "moe_gen_normal_bf16")


def test_status_strings(L):
    for code, name in [(0, "MOE_OK"), (1, "MOE_ERR_INVALID_ARG"), (2, "MOE_ERR_UNSUPPORTED_SHAPE"),
                       (3, "MOE_ERR_WORKSPACE_TOO_SMALL"), (4, "MOE_ERR_CUDA"),
                       (5, "MOE_ERR_DEVICE_TIMEOUT"), (6, "MOE_ERR_DEVICE_BOUNDS")]:
        assert M.status_string(code) == name


def test_workspace_size_and_shape_limits(L):
    ok = M.make_dims(4096, 2048, 256, 8, 512, 512)
    n = M.workspace_size(ok)
    # slots alone: T * (k + 1) * d * 2 bytes
    assert n >= 4096 * 9 * 2048 * 2 and n % 256 == 0
    bad = [M.make_dims(64, 100, 16, 4, 128, 128),      # d not a multiple of 64
           M.make_dims(64, 96, 16, 4, 128, 128),       # d not a multiple of 64
           M.make_dims(64, 256, 16, 17, 128, 128),     # k > 16
           M.make_dims(64, 256, 4, 5, 128, 128),       # k > E
           M.make_dims(64, 256, 1024, 4, 128, 128),    # E > 512
           M.make_dims(64, 256, 16, 4, 96, 128),       # F not a multiple of 64
           M.make_dims(64, 256, 16, 4, 128, 32)]       # Fs not a multiple of 64
    for d in bad:
        assert M.workspace_size(d) == 0
    d = M.make_dims(64, 256, 16, 4, 128, 128)
    d.struct_size = 4
    assert M.workspace_size(d) == 0


def test_fused_and_reduce_combine_shape_rules_and_workspace(L):
    """The fused kernel needs F, Fs, d multiples of 128 (an FFN runs in equal parts of whole
    128-column chunks, at most 512 columns each: 640 as five parts of 128); its workspace
    holds no h and no fp16 contribution rows, only the fp32 token rows (so does the reduce
    combine's, which keeps h)."""
    F_ = M.MOE_FLAG_FUSED_EXPERTS
    R_ = M.MOE_FLAG_COMBINE_REDUCE
    for ok in [(4096, 2048, 256, 8, 512, 512), (64, 256, 16, 4, 1024, 1024),
               (64, 256, 16, 4, 768, 0), (64, 256, 16, 4, 1536, 128),
               (64, 256, 16, 4, 640, 128)]:
        assert M.workspace_size(M.make_dims(*ok, flags=F_)) > 0, ok
    for bad in [(64, 256, 16, 4, 192, 128),    # F not a multiple of 128
                (64, 256, 16, 4, 128, 320),    # Fs not a multiple of 128
                (64, 192, 16, 4, 128, 128)]:   # d not a multiple of 128
        assert M.workspace_size(M.make_dims(*bad, flags=F_)) == 0, bad
    T, d, E, k, F, Fs = 4096, 2048, 256, 8, 512, 512
    base = M.workspace_size(M.make_dims(T, d, E, k, F, Fs))
    red = M.workspace_size(M.make_dims(T, d, E, k, F, Fs, flags=R_))
    fus = M.workspace_size(M.make_dims(T, d, E, k, F, Fs, flags=F_))
    slots, yacc, h = T * (k + 1) * d * 2, T * d * 4, (T * k + T) * F * 2
    assert abs((base - red) - (slots - yacc)) < 4096
    assert abs((red - fus) - h) < 4096


def test_workspace_holds_one_logit_plane_per_router_slice(L):
    """The tensor-core router (T >= 1024 at E = 256) cuts d into 4 K slices up to 18 token
    tiles (T <= 2304), 2 up to 74 (T <= 9472), none above, and the workspace holds one fp32
    [T, E] logit plane per slice: the size jumps by about three planes at T = 1024 (no slices
    on the CUDA-core router below) and drops by about two planes just past T = 2304 and
    about one just past T = 9472; T = 4736 -> 4737 (37 -> 38 tiles) keeps two."""
    def ws(T):
        return M.workspace_size(M.make_dims(T, 2048, 256, 8, 512, 512))
    plane = lambda T: T * 256 * 4
    per_token = ws(2001) - ws(2000)          # growth of everything else, per token
    assert 0 < per_token < 200_000
    assert ws(1024) - ws(1023) > 3 * plane(1023) - 2 * per_token
    assert ws(2304) - ws(2305) > 2 * plane(2304) - 2 * per_token
    assert abs((ws(4737) - ws(4736)) - (per_token - 2 * 256 * 4)) < 4096
    assert ws(9472) - ws(9473) > plane(9472) - 2 * per_token
    # T = 2000 grows by four planes per token, T = 20000 by one (256-byte section alignment)
    assert abs((ws(20001) - ws(20000)) - (per_token - 3 * 256 * 4)) < 2048


def _call_forward(dims, x=256, y=512, ws=4096, ws_bytes=1 << 40, weights=None, routing=None):
    w = weights or M.moe_weights_t(1024, None, 2048, 4096, 8192, 16384, 32768, 65536)
    r = routing or M.moe_routing_t(1 << 20, 2 << 20, 3 << 20, 4 << 20, 5 << 20)
    return M.lib().moe_forward(ctypes.byref(dims), ctypes.byref(w), ctypes.c_void_p(x),
                               ctypes.c_void_p(y), ctypes.byref(r), ctypes.c_void_p(ws), ws_bytes,
                               None)


def test_argument_errors_return_before_any_launch(L):
    d = M.make_dims(64, 256, 16, 4, 128, 128)
    # fake device addresses are never dereferenced on these paths
    assert _call_forward(d, x=0) == M.MOE_ERR_INVALID_ARG
    assert _call_forward(d, x=256 + 8) == M.MOE_ERR_INVALID_ARG          # misaligned
    assert _call_forward(d, ws=4096 + 16) == M.MOE_ERR_INVALID_ARG       # ws not 256-aligned
    assert _call_forward(d, ws_bytes=1024) == M.MOE_ERR_WORKSPACE_TOO_SMALL
    bad = M.make_dims(64, 256, 16, 4, 128, 32)
    assert _call_forward(bad) == M.MOE_ERR_UNSUPPORTED_SHAPE
    w = M.moe_weights_t(1024, None, 2048, 4096, 8192, None, None, None)  # shared missing
    assert _call_forward(d, weights=w) == M.MOE_ERR_INVALID_ARG
    r = M.moe_routing_t(1 << 20, 2 << 20, 0, 4 << 20, 5 << 20)
    assert _call_forward(d, routing=r) == M.MOE_ERR_INVALID_ARG
    # forced tensor-core router with an E it cannot take
    f = M.make_dims(64, 256, 24, 4, 128, 128, flags=M.MOE_FLAG_ROUTER_TENSOR)
    assert _call_forward(f) == M.MOE_ERR_UNSUPPORTED_SHAPE
    # the CUDA-core router (small batches, or E outside the tensor router's range) stages
    # 8 bf16 token rows per CTA in 227 KB of shared memory: d <= 14528 on that path only
    wide = M.make_dims(64, 14592, 256, 8, 512, 512)
    assert M.workspace_size(wide) > 0                 # a permute-only caller can size it
    assert _call_forward(wide) == M.MOE_ERR_UNSUPPORTED_SHAPE
    assert _call_forward(M.make_dims(2048, 14592, 264, 8, 512, 512)) == M.MOE_ERR_UNSUPPORTED_SHAPE
    assert _call_forward(wide, x=0) == M.MOE_ERR_UNSUPPORTED_SHAPE  # shape checks come first


def _fp8_struct(missing=None):
    vals = {n: (1 << 24) + 4096 * i for i, n in enumerate(M.FP8_FIELDS)}
    if missing:
        vals[missing] = None
    return M.moe_fp8_weights_t(*[vals[n] for n in M.FP8_FIELDS])


def _call_forward_fp8(dims, q=None, x=256, y=512, ws=4096, ws_bytes=1 << 40):
    w = M.moe_weights_t(1024, None, 2048, 4096, 8192, 16384, 32768, 65536)
    r = M.moe_routing_t(1 << 20, 2 << 20, 3 << 20, 4 << 20, 5 << 20)
    q = q or _fp8_struct()
    return M.lib().moe_forward_fp8(ctypes.byref(dims), ctypes.byref(w), ctypes.byref(q),
                                   ctypes.c_void_p(x), ctypes.c_void_p(y), ctypes.byref(r),
                                   ctypes.c_void_p(ws), ws_bytes, None)


def test_fp8_argument_errors_return_before_any_launch(L):
    f8 = M.MOE_FLAG_FP8_EXPERTS
    d = M.make_dims(64, 256, 16, 4, 128, 128, flags=f8)
    # e4m3 rows of x and h on top of a workspace without the per-call fp16 copy of W_down
    assert M.workspace_size(d) > M.workspace_size(
        M.make_dims(64, 256, 16, 4, 128, 128, flags=M.MOE_FLAG_DOWN_F16))
    assert _call_forward_fp8(M.make_dims(64, 256, 16, 4, 128, 128)) == M.MOE_ERR_INVALID_ARG
    assert M.workspace_size(M.make_dims(64, 256, 16, 4, 192, 128, flags=f8)) == 0
    assert _call_forward_fp8(M.make_dims(64, 256, 16, 4, 192, 128, flags=f8)) == \
        M.MOE_ERR_UNSUPPORTED_SHAPE                                        # F % 128
    assert _call_forward_fp8(M.make_dims(64, 384, 16, 4, 128, 128, flags=f8)) == \
        M.MOE_ERR_UNSUPPORTED_SHAPE                                        # d % 256
    assert _call_forward_fp8(d, q=_fp8_struct("s_down")) == M.MOE_ERR_INVALID_ARG
    assert _call_forward_fp8(d, q=_fp8_struct("ss_gate")) == M.MOE_ERR_INVALID_ARG
    assert _call_forward_fp8(d, x=256 + 8) == M.MOE_ERR_INVALID_ARG
    # the 16-bit forward cannot use a workspace sized for FP8 without prepared fp16 W_down
    assert _call_forward(d) == M.MOE_ERR_INVALID_ARG
    assert _call_forward_fp8(M.make_dims(0, 256, 16, 4, 128, 128, flags=f8)) == M.MOE_OK


def test_zero_tokens_is_a_noop(L):
    d = M.make_dims(0, 256, 16, 4, 128, 128)
    assert _call_forward(d) == M.MOE_OK
    rc = L.moe_route(ctypes.byref(d), ctypes.c_void_p(256), ctypes.c_void_p(512), None,
                     ctypes.c_void_p(768), ctypes.c_void_p(1024), ctypes.c_void_p(4096),
                     1 << 30, None)
    assert rc == M.MOE_OK
    rc = L.moe_permute(ctypes.byref(d), ctypes.c_void_p(256), ctypes.c_void_p(512),
                       ctypes.c_void_p(768), ctypes.c_void_p(1024), None, None,
                       ctypes.c_void_p(4096), 1 << 30, None)
    assert rc == M.MOE_OK
    rc = L.moe_permute(ctypes.byref(d), ctypes.c_void_p(256), ctypes.c_void_p(512),
                       ctypes.c_void_p(768), ctypes.c_void_p(1024), ctypes.c_void_p(256), None,
                       ctypes.c_void_p(4096), 1 << 30, None)
    assert rc == M.MOE_ERR_INVALID_ARG  # x without x_perm
