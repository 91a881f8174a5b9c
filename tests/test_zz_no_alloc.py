"""moe_permute_static: the expert-order permutation without a workspace.

Callers that cannot allocate device memory (code inside another runtime's
memory pool, plugins whose host process owns all device memory, or work being
captured into a CUDA graph) get the permutation from this entry point, whose
scratch is a static device array inside the library.  Its output must be
identical to moe_permute's on the same input, call after call (the array keeps
the previous call's contents, which must not leak into the next one).
"""
import ctypes

import numpy as np
import pytest

from sparse_moe_layer_select_b200 import build as B
from sparse_moe_layer_select_b200 import moe as M


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _routing(T, E, k, seed):
    rng = np.random.default_rng(seed)
    # top-k sets as a router makes them: k distinct experts per token, skewed popularity
    pop = rng.dirichlet(np.full(E, 0.3))
    return np.stack([rng.choice(E, size=k, replace=False, p=pop) for _ in range(T)]).astype(np.int32)


def test_rejects_dims_beyond_the_static_scratch():
    B.build()
    L = M.lib()
    big = M.make_dims(262144, 2048, 256, 8, 512, 512)   # T*k = 2,097,152 pairs
    rc = L.moe_permute_static(ctypes.byref(big), ctypes.c_void_p(256), ctypes.c_void_p(512),
                              ctypes.c_void_p(768), ctypes.c_void_p(1024), None)
    assert rc == M.MOE_ERR_UNSUPPORTED_SHAPE


@pytest.mark.gpu
def test_static_scratch_permute_matches_workspace_permute_twice():
    import torch
    B.build()
    L = M.lib()
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    # two calls in a row with different sizes: the second must not see the first's scratch
    for (T, E, k, seed) in [(4096, 256, 8, 1), (1000, 64, 6, 2)]:
        idx = torch.from_numpy(_routing(T, E, k, seed)).cuda()
        dims = M.make_dims(T, 256, E, k, 128, 128)
        outs = []
        for use_static in (False, True):
            counts = torch.full((E,), -7, dtype=torch.int32, device="cuda")
            offsets = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
            perm = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
            if use_static:
                rc = L.moe_permute_static(ctypes.byref(dims), _p(idx), _p(counts), _p(offsets),
                                          _p(perm), ctypes.c_void_p(stream.cuda_stream))
                assert rc == M.MOE_OK, M.status_string(rc)
            else:
                ws = M.alloc_workspace(dims)
                M.permute(dims, idx, counts, offsets, perm, ws)
            torch.cuda.synchronize()
            outs.append((counts.cpu().numpy(), offsets.cpu().numpy(), perm.cpu().numpy()))
        for a, b in zip(outs[0], outs[1]):
            assert np.array_equal(a, b)
        assert outs[1][1][-1] == T * k and sorted(outs[1][2].tolist()) == list(range(T * k))
