"""The Python binding's own checks, on the CPU.

The C library receives bare pointers and cannot see how large a buffer is, so
the binding checks each tensor's byte extent against the sizes include/mxmoe.h
gives, before any pointer is marshalled.  On the CPU the order shows which
check decided: a buffer one element short raises the size error, the same
call with every buffer large enough gets past the size checks and is then
refused because the tensors are not CUDA tensors.
"""
import pytest
import torch

from fp8_moe_numerics_b200 import api


@pytest.fixture(scope="module", autouse=True)
def built():
    from fp8_moe_numerics_b200 import build
    build.build()


def u8(*s):
    return torch.zeros(*s, dtype=torch.uint8)


def f32(*s):
    return torch.zeros(*s, dtype=torch.float32)


def bf16(*s):
    return torch.zeros(*s, dtype=torch.bfloat16)


def _size_error(fn, what):
    with pytest.raises(ValueError, match=f"^{what}: .* the call needs"):
        fn()


def _passes_size_checks(fn):
    with pytest.raises(ValueError, match="operates on CUDA tensors"):
        fn()


def test_nvfp4_quantize_outputs():
    x = bf16(256, 128)
    good = (u8(256, 64), u8(256 * 8), f32(256))
    _passes_size_checks(lambda: api.nvfp4_quantize(x, 1, api.MX_SF_MMA, out=good))
    _size_error(lambda: api.nvfp4_quantize(x, 1, api.MX_SF_MMA, out=(u8(256 * 64 - 1), good[1], good[2])), "codes")
    _size_error(lambda: api.nvfp4_quantize(x, 1, api.MX_SF_MMA, out=(good[0], u8(256 * 8 - 1), good[2])), "sf")
    _size_error(lambda: api.nvfp4_quantize(x, 1, api.MX_SF_MMA, out=(good[0], good[1], f32(255))), "outer")
    # per-expert outer scale: rows / group_rows floats
    _passes_size_checks(lambda: api.nvfp4_quantize(x, 128, api.MX_SF_MMA, out=(good[0], good[1], f32(2))))


def test_requant_inputs_and_outputs():
    rows, cols = 256, 128
    q = (u8(rows, cols // 2), u8(rows * cols // 16), f32(rows))
    out = (u8(cols, rows), u8(cols * rows // 32))
    _passes_size_checks(lambda: api.mxfp8_requant_transpose_sr(*q, rows, cols, out=out))
    _size_error(lambda: api.mxfp8_requant_transpose_sr(*q, rows, cols, out=(out[0], u8(cols * rows // 32 - 1))),
                "out e8m0")
    _size_error(lambda: api.mxfp8_requant_transpose_sr(q[0][:-1], q[1], q[2], rows, cols, out=out), "codes")
    _size_error(lambda: api.mxfp8_requant_transpose_sr(*q, rows, cols, rows_valid=torch.zeros(0, dtype=torch.int64),
                                                       out=out), "rows_valid")


def test_mxfp8_quantize_forms():
    x = bf16(256, 128)
    out = (u8(256, 128), u8(256 * 4), u8(128, 256), u8(128 * 8))
    _passes_size_checks(lambda: api.mxfp8_quantize(x, out=out))
    _size_error(lambda: api.mxfp8_quantize(x, out=(out[0], out[1], out[2], u8(128 * 8 - 1))), "col e8m0")
    _passes_size_checks(lambda: api.mxfp8_quantize(x, col=False, out=(out[0], out[1], None, None)))


def _nvfp4_operands(E, M, N, K):
    a = (u8(M, K // 2), u8(M * K // 16), f32(M))
    b = (u8(E * N, K // 2), u8(E * N * K // 16), f32(E))
    return a, b, torch.zeros(E + 1, dtype=torch.int64)


def test_grouped_gemm_nvfp4_operands():
    E, M, N, K = 3, 384, 256, 512
    a, b, seg = _nvfp4_operands(E, M, N, K)
    _passes_size_checks(lambda: api.grouped_gemm_nvfp4(a, b, seg, E, N, K, out=bf16(M, N)))
    _size_error(lambda: api.grouped_gemm_nvfp4(a, (b[0][:-1], b[1], b[2]), seg, E, N, K, out=bf16(M, N)), "b codes")
    _size_error(lambda: api.grouped_gemm_nvfp4(a, (b[0], b[1], f32(E - 1)), seg, E, N, K, out=bf16(M, N)), "b outer")
    _size_error(lambda: api.grouped_gemm_nvfp4(a, b, seg[:-1], E, N, K, out=bf16(M, N)), "seg")
    # an fp32 output needs twice the bytes of a bf16 one
    _size_error(lambda: api.grouped_gemm_nvfp4(a, b, seg, E, N, K, out=f32(M, N // 2)), "out")
    # the S2F6 epilogue's outputs
    _passes_size_checks(lambda: api.grouped_gemm_nvfp4_s2f6(a, b, seg, E, N, K, 1, 2,
                                                            out=(torch.zeros(M, N, dtype=torch.int8), u8(M, N // 32))))
    _size_error(lambda: api.grouped_gemm_nvfp4_s2f6(a, b, seg, E, N, K, 1, 2,
                                                    out=(torch.zeros(M, N, dtype=torch.int8), u8(M, N // 32 - 1))),
                "e8m0")


def test_grouped_gemm_mxfp8_modes():
    E, M, N, K = 2, 256, 128, 384
    seg = torch.zeros(E + 1, dtype=torch.int64)
    # DGRAD: A [M, K], B [N, E*K] -> [M, N]
    dA, dB = (u8(M, K), u8(M * K // 32)), (u8(N, E * K), u8(N * E * K // 32))
    _passes_size_checks(lambda: api.grouped_gemm_mxfp8(api.MX_GEMM_DGRAD, *dA, *dB, seg, E, M, N, K, out=bf16(M, N)))
    _size_error(lambda: api.grouped_gemm_mxfp8(api.MX_GEMM_DGRAD, *dA, dB[0][:, :-1].contiguous(), dB[1], seg, E, M, N,
                                               K, out=bf16(M, N)), "b codes")
    # WGRAD: A [N, M], B [K, M] -> [E, N, K]
    wA, wB = (u8(N, M), u8(N * M // 32)), (u8(K, M), u8(K * M // 32))
    _passes_size_checks(lambda: api.grouped_gemm_mxfp8(api.MX_GEMM_WGRAD, *wA, *wB, seg, E, M, N, K,
                                                       out=bf16(E, N, K)))
    _size_error(lambda: api.grouped_gemm_mxfp8(api.MX_GEMM_WGRAD, *wA, *wB, seg, E, M, N, K, out=bf16(E - 1, N, K)),
                "out")


def test_routing_and_glue_buffers():
    T, k, E = 64, 2, 4
    M = api.max_routed_rows(T, k, E)
    topk = torch.zeros(T, k, dtype=torch.int32)
    seg, src, pos = torch.zeros(E + 1, dtype=torch.int64), torch.zeros(M, dtype=torch.int32), \
        torch.zeros(T, k, dtype=torch.int32)
    ws = u8(4096)
    _passes_size_checks(lambda: api.moe_route(topk, E, out=(seg, src, pos, ws)))
    _size_error(lambda: api.moe_route(topk, E, out=(seg, src[:-1], pos, ws)), "src")
    D = 128
    w = f32(T, k)
    _passes_size_checks(lambda: api.moe_combine(bf16(M, D), pos, w, D, out=bf16(T, D)))
    _size_error(lambda: api.moe_combine(bf16(M, D), pos, f32(T, k - 1), D, out=bf16(T, D)), "w")
    _size_error(lambda: api.moe_dispatch_grad(bf16(T - 1, D), src, pos, w, out=bf16(M, D)), "dout")
    _size_error(lambda: api.nvfp4_gather_rows(u8(T, D // 2), u8(T * D // 16), f32(T), src, k, D,
                                              out=(u8(M, D // 2), u8(M * D // 16), f32(M - 1))), "out outer")
    F = 64
    _passes_size_checks(lambda: api.swiglu_fwd(bf16(M, 2 * F), F, True, out=bf16(M, F)))
    _size_error(lambda: api.swiglu_fwd(bf16(M, F), F, True, out=bf16(M, F)), "h")      # gated reads 2F columns
    _size_error(lambda: api.swiglu_bwd(bf16(M, 2 * F), bf16(M, F), F, True, out=bf16(M, F)), "dh")
    _size_error(lambda: api.swiglu_nvfp4_quantize(bf16(M, 2 * F), F, True, out=(u8(M, F // 2), u8(M * F // 16),
                                                                                 f32(M - 1))), "outer")


def test_s2f6_buffers():
    x = bf16(64, 128)
    _passes_size_checks(lambda: api.hadamard_s2f6_quantize(x, 1, 2, out=(torch.zeros(64, 128, dtype=torch.int8),
                                                                           u8(64, 4))))
    _size_error(lambda: api.hadamard_s2f6_quantize(x, 1, 2, out=(torch.zeros(64, 127, dtype=torch.int8), u8(64, 4))),
                "codes")
    pos = torch.zeros(16, 2, dtype=torch.int32)
    codes = torch.zeros(64, 128, dtype=torch.int8)
    _passes_size_checks(lambda: api.moe_combine_s2f6(codes, u8(64, 4), pos, f32(16, 2), 1, 2))
    _size_error(lambda: api.moe_combine_s2f6(codes, u8(64, 3), pos, f32(16, 2), 1, 2), "e8m0")


def test_input_types():
    with pytest.raises(ValueError, match="2-D bf16"):
        api.nvfp4_quantize(f32(128, 64))
    with pytest.raises(ValueError, match="2-D bf16"):
        api.mxfp8_quantize(bf16(128, 128, 1))
    with pytest.raises(ValueError, match="2-D bf16"):
        api.swiglu_nvfp4_quantize(torch.zeros(128, 128, dtype=torch.float16), 64)


def test_layer_rejects_mismatched_configuration():
    from fp8_moe_numerics_b200 import workloads
    from fp8_moe_numerics_b200.layer import ExpertLayer
    inp = workloads.layer_inputs("tiny_layer", device="cpu")
    args = (inp["x"], inp["topk"], inp["w_comb"], inp["w1"], inp["w2"], inp["dout"])
    with pytest.raises(ValueError, match="combine"):
        ExpertLayer(*args, combine="fp8")
    with pytest.raises(ValueError, match="rows per expert"):
        ExpertLayer(*args, gated=True)                  # w1 holds F rows per expert: an ungated layer


def test_nvfp4_backward_buffers():
    x = bf16(256, 128)
    good = (u8(256, 64), u8(256 * 8), f32(256))
    _passes_size_checks(lambda: api.nvfp4_quantize_sr(x, out=good))
    _size_error(lambda: api.nvfp4_quantize_sr(x, out=(good[0], u8(256 * 8 - 1), good[2])), "sf")
    # requantisation of a [256, 128] tensor: one expert, outer per output row
    q = (u8(256, 64), u8(256 * 8), f32(256))
    out = (u8(128, 128), u8(128 * 16), f32(128))
    _passes_size_checks(lambda: api.nvfp4_requant_transpose_sr(*q, 256, 128, out=out))
    _size_error(lambda: api.nvfp4_requant_transpose_sr(*q, 256, 128, out=(out[0], out[1], f32(127))), "out outer")
    # two experts of 128 rows with a per-expert outer scale: [2*128, 64] out, outer [2]
    out2 = (u8(256, 64), u8(256 * 8), f32(2))
    _passes_size_checks(lambda: api.nvfp4_requant_transpose_sr(*q, 256, 128, 128, experts=2,
                                                               out_outer_per_expert=True, out=out2))
    _size_error(lambda: api.nvfp4_requant_transpose_sr(*q, 256, 128, 128, experts=2, out_outer_per_expert=True,
                                                       out=(u8(256, 63), out2[1], out2[2])), "out codes")
    t = bf16(64, 48)
    _passes_size_checks(lambda: api.nvfp4_quantize_tile16(t, 32, out=(u8(64, 24), u8(4, 3), f32(2))))
    _size_error(lambda: api.nvfp4_quantize_tile16(t, 32, out=(u8(64, 24), u8(4, 2), f32(2))), "sf_tile")


def test_segment_transpose_buffers():
    M, C, E = 256, 128, 2
    seg = torch.zeros(E + 1, dtype=torch.int64)
    x = bf16(M, C)
    out = (u8(C, M // 2), u8(C * M // 16), f32(E * C))
    _passes_size_checks(lambda: api.nvfp4_quantize_transpose_segments(x, seg, E, True, out=out))
    _size_error(lambda: api.nvfp4_quantize_transpose_segments(x, seg, E, True, out=(out[0], out[1], f32(E))),
                "out outer")                                   # per (segment, row) needs E * C scales
    _size_error(lambda: api.nvfp4_quantize_transpose_segments(x, seg[:-1], E, True, out=out), "seg")
    q = (u8(M, C // 2), u8(M * C // 16), f32(M))
    _passes_size_checks(lambda: api.nvfp4_requant_transpose_segments(*q, M, C, seg, E, out=(out[0], out[1], f32(E))))
    _size_error(lambda: api.nvfp4_requant_transpose_segments(q[0][:-1], q[1], q[2], M, C, seg, E), "codes")


def test_nvfp4_wgrad_buffers():
    E, M, N, K = 2, 512, 128, 256
    seg = torch.zeros(E + 1, dtype=torch.int64)
    a = (u8(N, M // 2), u8(N * M // 16), f32(E * N))
    b = (u8(K, M // 2), u8(K * M // 16), f32(E))
    _passes_size_checks(lambda: api.grouped_gemm_nvfp4_wgrad(a, b, seg, E, N, K, out=f32(E, N, K)))
    _size_error(lambda: api.grouped_gemm_nvfp4_wgrad((a[0], a[1], f32(N)), b, seg, E, N, K, out=f32(E, N, K)),
                "a outer")                                     # one scale per (segment, row)
    _size_error(lambda: api.grouped_gemm_nvfp4_wgrad(a, b, seg, E, N, K, out=f32(E, N, K - 1)), "out")
