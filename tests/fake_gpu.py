"""A CPU stand-in for the GPU, for tests of host logic only.

Inside `fake_gpu()` torch's "cuda" device maps to the CPU (factory calls,
.cuda(), .to("cuda")), CUDA streams and events are inert stand-ins whose
timings read 1 ms, and the C library's compute entry points are recorded
instead of launched; moe_route fills its outputs with the routing the
oracle computes, since later host steps read them.  Size helpers
(mx_sf_bytes, mx_route_workspace_bytes) are the real library's.  Every patch
is undone on exit.  Nothing here computes any result of the method: outputs
of recorded calls stay zero.
"""
import contextlib
import ctypes
import types

import numpy as np
import torch
from torch.overrides import TorchFunctionMode


def _cpu(d):
    return "cpu" if d is not None and str(d).startswith("cuda") else d


class _CpuMode(TorchFunctionMode):
    def __torch_function__(self, func, types_, args=(), kwargs=None):
        kwargs = dict(kwargs or {})
        if func in (torch.Tensor.cuda, torch.Tensor.pin_memory):
            return args[0]
        if func is torch.Tensor.to:
            args = tuple(_cpu(a) if isinstance(a, (str, torch.device)) else a for a in args)
            kwargs.pop("non_blocking", None)
        if "device" in kwargs:
            kwargs["device"] = _cpu(kwargs["device"])
        kwargs.pop("pin_memory", None)
        if func is torch.empty:
            func = torch.zeros
        if func is torch.empty_like:
            func = torch.zeros_like
        return func(*args, **kwargs)


class _Stream:
    cuda_stream = 0

    def __init__(self, *a, **k):
        pass

    def synchronize(self):
        pass

    def wait_stream(self, s):
        pass

    def wait_event(self, e):
        pass


class _Event:
    def __init__(self, *a, **k):
        pass

    def record(self, s=None):
        pass

    def synchronize(self):
        pass

    def query(self):
        return True

    def elapsed_time(self, other):
        return 1.0


class _Lib:
    """The real library for size helpers, recorded no-ops for everything else."""

    def __init__(self, real, calls):
        self._real, self._calls = real, calls

    def __getattr__(self, name):
        if name in ("mx_sf_bytes", "mx_route_workspace_bytes", "mx_version", "mx_kernel_launches",
                    "mx_last_cuda_error"):
            return getattr(self._real, name)
        return lambda *a: self._calls.append(name) or 0


@contextlib.contextmanager
def fake_gpu(monkeypatch):
    from fp8_moe_numerics_b200 import _lib, api, build
    import oracle
    build.build()
    real = _lib.lib()
    calls = []
    gen = torch.Generator
    for name, value in [("is_available", lambda: True), ("synchronize", lambda *a, **k: None),
                        ("current_stream", lambda *a, **k: _Stream()), ("Stream", _Stream), ("Event", _Event),
                        ("stream", lambda s: contextlib.nullcontext()), ("current_device", lambda: 0),
                        ("set_device", lambda d: None),
                        ("get_device_properties", lambda *a, **k: types.SimpleNamespace(
                            multi_processor_count=148, name="stand-in", total_memory=180 << 30, major=10,
                            minor=0)),
                        ("mem_get_info", lambda *a, **k: (170 << 30, 180 << 30))]:
        monkeypatch.setattr(torch.cuda, name, value)
    monkeypatch.setattr(torch, "Generator", lambda device="cpu": gen(device=_cpu(device)))
    monkeypatch.setattr(torch.Tensor, "record_stream", lambda self, s: None)
    fake = _Lib(real, calls)
    monkeypatch.setattr(_lib, "_lib", fake)

    def call(name, *args):
        calls.append(name)

    monkeypatch.setattr(_lib, "call", call)
    monkeypatch.setattr(api, "_p", lambda t: ctypes.c_void_p(0 if t is None else t.data_ptr()))
    monkeypatch.setattr(api, "_s", lambda: ctypes.c_void_p(0))
    route = api.moe_route

    def routed(topk, E, M_cap=None, out=None, align=128):
        seg, src, pos = route(topk, E, M_cap, out, align)
        s, _, p = oracle.route(topk.numpy(), E, align)
        seg.copy_(torch.from_numpy(np.asarray(s, np.int64)))
        T, k = p.shape
        flat = np.full(src.numel(), -1, np.int32)
        flat[p.reshape(-1)] = np.arange(T * k, dtype=np.int32)
        src.copy_(torch.from_numpy(flat))
        pos.copy_(torch.from_numpy(np.asarray(p, np.int32)).reshape(pos.shape))
        return seg, src, pos

    monkeypatch.setattr(api, "moe_route", routed)
    mode = _CpuMode()
    with mode:
        yield calls
