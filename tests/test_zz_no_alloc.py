"""moe_route_static: the routing entry point for callers that cannot allocate
device memory (allocator callbacks, runtimes that own every device
allocation).  It keeps its scratch in a fixed array inside the library, so it
must give exactly what moe_route gives with a caller-provided workspace, call
after call, and refuse problems whose scratch would not fit.

This file is collected last on purpose: if it fails, a run stopped at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from fp8_moe_numerics_b200 import _lib, api, workloads


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def test_static_route_rejects_problems_beyond_its_scratch():
    from fp8_moe_numerics_b200 import build
    build.build()
    L = _lib.lib()
    buf = (ctypes.c_uint8 * 64)()
    p = ctypes.cast(buf, ctypes.c_void_p)
    T, E = 1 << 20, 1024                      # needs 16 MiB of scratch
    assert L.mx_route_workspace_bytes(T, E) > (1 << 20)
    cap = (T * 2 + 127 * E + 127) // 128 * 128
    assert L.moe_route_static(p, T, 2, E, cap, p, p, p, ctypes.c_void_p(0)) == _lib.MX_EINVAL


@pytest.mark.gpu
def test_static_route_matches_workspace_route_on_consecutive_calls(cuda):
    L = _lib.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, (T, k, E, kind, n_empty, seed) in enumerate([(3000, 8, 384, "zipf", 8, 5), (700, 2, 16, "uniform", 0, 6)]):
        ids = workloads.routing(T, k, E, kind, 1.2, n_empty, seed=seed).cuda()
        M_cap = api.max_routed_rows(T, k, E)
        ref = api.moe_route(ids, E, M_cap)
        seg = torch.full((E + 1,), -7, dtype=torch.int64, device="cuda")
        src = torch.full((M_cap,), -7, dtype=torch.int32, device="cuda")
        pos = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
        st = L.moe_route_static(_ptr(ids), T, k, E, M_cap, _ptr(seg), _ptr(src), _ptr(pos), stream)
        assert st == _lib.MX_OK, f"call {call}: status {st}"
        torch.cuda.synchronize()
        for got, want in zip((seg, src, pos), ref):
            assert torch.equal(got, want), f"call {call}"
