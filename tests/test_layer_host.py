"""Host-side check of the expert-layer call sequence (no GPU).

ExpertLayer is run on CPU tensors with the binding's pointer check relaxed:
every call reaches the real C library, whose argument validation runs on the
host before the device check.  Valid arguments therefore return MX_ECUDA (no
CUDA device here), invalid ones MX_EINVAL -- so each call's shapes, strides,
alignment and sizes are checked against the ABI contract.
"""
import ctypes

import pytest
import torch

from fp8_moe_numerics_b200 import _lib, api, workloads
from fp8_moe_numerics_b200.layer import ExpertLayer


@pytest.fixture
def host_calls(monkeypatch):
    from fp8_moe_numerics_b200 import build
    build.build()
    calls = []

    def p(t):
        return ctypes.c_void_p(0 if t is None else t.data_ptr())

    def call(name, *args):
        st = getattr(_lib.lib(), name)(*args)
        calls.append((name, st))
        assert st != _lib.MX_EINVAL, f"{name} rejected its arguments"

    monkeypatch.setattr(api, "_p", p)
    monkeypatch.setattr(api, "_s", lambda: ctypes.c_void_p(0))
    monkeypatch.setattr(_lib, "call", call)
    monkeypatch.setattr(api.L, "call", call)
    return calls


def test_unfused_backward_sequence_passes_host_validation(host_calls):
    inp = workloads.layer_inputs("tiny_layer", device="cpu")
    c = inp["cfg"]
    L = ExpertLayer(inp["x"], inp["topk"], inp["w_comb"], inp["w1"], inp["w2"], inp["dout"], gated=c["gated"],
                    fuse_backward=False)
    L.step()
    names = [n for n, _ in host_calls]
    assert names.count("moe_dispatch_grad") == 1 and names.count("swiglu_bwd") == 1
    assert names.count("mxfp8_quantize") == 2 and len(names) == 22
    assert all(st == _lib.MX_ECUDA for _, st in host_calls)


@pytest.mark.parametrize("name", ["tiny_layer"])
def test_layer_sequence_passes_host_validation(host_calls, name):
    inp = workloads.layer_inputs(name, device="cpu")
    c = inp["cfg"]
    L = ExpertLayer(inp["x"], inp["topk"], inp["w_comb"], inp["w1"], inp["w2"], inp["dout"], gated=c["gated"])
    L.step()
    names = [n for n, _ in host_calls]
    assert names[0] == "moe_route" and names[-1] == "moe_combine"
    assert names.count("grouped_gemm_nvfp4") == 2 and names.count("grouped_gemm_mxfp8") == 4
    assert names.count("mxfp8_requant_transpose_sr") == 4
    assert names.count("swiglu_nvfp4_quantize") == 1 and "swiglu_fwd" not in names   # fused by default
    # the dispatch gradient fused into its quantiser by default
    assert names.count("moe_dispatch_grad_mxfp8_quantize") == 1 and "moe_dispatch_grad" not in names
    assert names.count("swiglu_bwd") == 1 and names.count("mxfp8_quantize") == 1
    assert len(names) == 21
    assert all(st == _lib.MX_ECUDA for _, st in host_calls)   # valid, and no device here


def test_s2f6_combine_sequence_passes_host_validation(host_calls):
    inp = workloads.layer_inputs("tiny_layer", device="cpu")
    c = inp["cfg"]
    L = ExpertLayer(inp["x"], inp["topk"], inp["w_comb"], inp["w1"], inp["w2"], inp["dout"], gated=c["gated"],
                    combine="s2f6")
    L.step()
    names = [n for n, _ in host_calls]
    assert names.count("grouped_gemm_nvfp4") == 1 and names.count("grouped_gemm_nvfp4_s2f6") == 1
    # the forward combine reads S2F6; the backward's un-permute of dX stays a bf16 combine
    assert names.count("moe_combine_s2f6") == 1 and names.count("moe_combine") == 1
    assert names.index("moe_combine_s2f6") == names.index("grouped_gemm_nvfp4_s2f6") + 1
    assert len(names) == 21
    assert all(st == _lib.MX_ECUDA for _, st in host_calls)


def test_unfused_swiglu_sequence_passes_host_validation(host_calls):
    inp = workloads.layer_inputs("tiny_layer", device="cpu")
    c = inp["cfg"]
    L = ExpertLayer(inp["x"], inp["topk"], inp["w_comb"], inp["w1"], inp["w2"], inp["dout"], gated=c["gated"],
                    fuse_swiglu=False)
    L.step()
    names = [n for n, _ in host_calls]
    assert "swiglu_nvfp4_quantize" not in names and names.count("swiglu_fwd") == 1
    assert names.count("nvfp4_quantize") == 4                   # tokens, W1, W2, activations
    assert len(names) == 22
    assert all(st == _lib.MX_ECUDA for _, st in host_calls)


@pytest.mark.parametrize("opts", [{}, {"fuse_swiglu": False}, {"combine": "s2f6"}, {"fuse_backward": False}])
def test_every_marked_stage_has_work_in_bench(host_calls, monkeypatch, opts):
    # bench.py turns the layer's stage marks into GB/s and TFLOP/s; a stage
    # without an entry in its work table would be reported without a rate
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench

    class FakeEvent:
        def __init__(self, **kw):
            pass

        def record(self, *a):
            pass

        def elapsed_time(self, other):
            return 1.0
    monkeypatch.setattr(torch.cuda, "Event", FakeEvent)
    inp = workloads.layer_inputs("tiny_layer", device="cpu")
    c = inp["cfg"]
    L = ExpertLayer(inp["x"], inp["topk"], inp["w_comb"], inp["w1"], inp["w2"], inp["dout"], gated=c["gated"],
                    **opts)
    L.step(record=True)
    stages = L.stage_times_ms()
    work = bench.stage_work(c, [c["T"] * c["k"] // c["E"]] * c["E"], L.M_cap)
    assert set(stages) <= set(work), set(stages) - set(work)
    assert {"gemm1", "gemm2", "requant_w1", "wgrad1"} <= set(stages)


def test_nvfp4_backward_sequence_passes_host_validation(host_calls):
    # the NVFP4 backward: routing padded to 256 rows, four NVFP4 backward GEMMs
    inp = workloads.layer_inputs("tiny_layer", device="cpu")
    c = inp["cfg"]
    L = ExpertLayer(inp["x"], inp["topk"], inp["w_comb"], inp["w1"], inp["w2"], inp["dout"], gated=c["gated"],
                    backward="nvfp4")
    assert L.M_cap % 256 == 0
    L.step()
    names = [n for n, _ in host_calls]
    assert names[0] == "moe_route_aligned" and names[-1] == "moe_combine"
    assert "grouped_gemm_mxfp8" not in names and "mxfp8_requant_transpose_sr" not in names
    assert names.count("grouped_gemm_nvfp4") == 4                 # GEMM1, GEMM2, dgrad2, dgrad1
    assert names.count("grouped_gemm_nvfp4_wgrad") == 2
    assert names.count("nvfp4_quantize_sr") == 2 and names.count("nvfp4_requant_transpose_sr") == 2
    assert names.count("nvfp4_quantize_transpose_segments") == 2
    assert names.count("nvfp4_requant_transpose_segments") == 2
    assert all(st == _lib.MX_ECUDA for _, st in host_calls)   # valid, and no device here
    # its stage marks all have a work entry in bench.py
    L2 = ExpertLayer(inp["x"], inp["topk"], inp["w_comb"], inp["w1"], inp["w2"], inp["dout"], gated=c["gated"],
                     backward="nvfp4")
    assert L2.backward_format == "nvfp4"
    with pytest.raises(ValueError, match="backward"):
        ExpertLayer(inp["x"], inp["topk"], inp["w_comb"], inp["w1"], inp["w2"], inp["dout"], gated=c["gated"],
                    backward="fp4")
