"""One expert layer's numerics, forward and backward, as a chain of C-ABI calls.

This is the whole hot path in order ([ai-primer] "Inkling 2 Small uses
four-bit training...", §NVFP4 forward, MXFP8 backward and §Stochastic rounding
across transposes):

  forward   route -> NVFP4 quantise tokens (per-token outer scale) -> gather
            into expert order -> NVFP4 quantise W1, W2 (per-expert outer
            scale) -> grouped NVFP4 GEMM1 -> SwiGLU + NVFP4 quantise (one kernel) ->
            grouped NVFP4 GEMM2 -> combine (with combine="s2f6", GEMM2's epilogue
            rotates each 32-column block by a random Hadamard transform and
            writes block-scaled S2F6, and the combine reads that:
            [ai-primer §Quantized NVLink and BBBK])
  backward  combine gradient -> MXFP8 quantise dY2 (row- and column-wise) ->
            requantise W2 and the saved activations (dequantise, transpose,
            MXFP8 with stochastic rounding) -> MXFP8 dgrad / wgrad GEMMs ->
            SwiGLU backward -> same for W1 and the saved tokens -> un-permute

All buffers are allocated once; `forward()` / `backward()` only enqueue
kernels on the current stream (no host synchronisation, no allocation), so a
step can be timed or captured.  Python here only sequences calls.
"""
from __future__ import annotations

import torch

from . import api
from .api import MX_GEMM_DGRAD, MX_GEMM_WGRAD, MX_ROUND_RNE, MX_ROUND_SR, MX_SF_MMA, MX_SF_ROWMAJOR


def nvfp4_gemm_flops(counts, N: int, K: int) -> int:
    """2 * sum_e m_e * N * K over true (unpadded) rows."""
    return 2 * int(sum(int(c) for c in counts)) * N * K


class ExpertLayer:
    """Buffers and call sequence of one MoE expert layer.

    x [T, D] bf16, topk [T, k] int32, w_comb [T, k] f32, w1 [E, 2F or F, D]
    bf16, w2 [E, D, F] bf16, dout [T, D] bf16, all on one CUDA device.
    `wgrad_dtype` is the dtype of dW1 / dW2 (bf16 or fp32).  `fuse_swiglu`
    quantises SwiGLU's output in the same kernel (the bf16 activation is then
    never written; `a` holds it only with fuse_swiglu=False).  `combine` is
    "bf16" (GEMM2 writes bf16 rows) or "s2f6" (GEMM2 writes rotated S2F6 rows,
    one byte per value plus one exponent per 32).  `backward` is "mxfp8" (the
    pages' recipe) or "nvfp4": the four backward GEMMs in NVFP4 with
    stochastically rounded operands (the pages' stated future work; routing
    then pads experts to 256 rows for the NVFP4 wgrad's K-stage).
    `fuse_backward` (MXFP8 backward) forms the dispatch gradient inside the
    gradient quantiser's kernel: the same codes, without the bf16 dy2
    (allocated only with fuse_backward=False or the NVFP4 backward).
    """

    S2F6_STREAM = 101                                   # Philox stream of the rotation's signs

    def __init__(self, x, topk, w_comb, w1, w2, dout, gated: bool = True, seed: int = 0,
                 wgrad_dtype=torch.bfloat16, out_dtype=torch.bfloat16, rbits: int = 16, combine: str = "bf16",
                 fuse_swiglu: bool = True, backward: str = "mxfp8", fuse_backward: bool = True):
        if combine not in ("bf16", "s2f6"):
            raise ValueError(f"combine must be 'bf16' or 's2f6', got {combine!r}")
        if backward not in ("mxfp8", "nvfp4"):
            raise ValueError(f"backward must be 'mxfp8' or 'nvfp4', got {backward!r}")
        self.backward_format = backward
        self.align = 256 if backward == "nvfp4" else 128
        self.combine = combine
        self.fuse_swiglu = fuse_swiglu
        self.fuse_backward = fuse_backward and backward == "mxfp8"
        dev = x.device
        self.dev = dev
        self.T, self.D = x.shape
        self.k = topk.shape[1]
        self.E, self.N1, _ = w1.shape
        self.F = w2.shape[2]
        self.gated = gated
        if self.N1 != (2 * self.F if gated else self.F):
            raise ValueError(f"w1 has {self.N1} rows per expert; {'2F' if gated else 'F'} = "
                             f"{2 * self.F if gated else self.F} expected")
        self.seed, self.rbits = seed, rbits
        self.x, self.topk, self.w_comb, self.w1, self.w2, self.dout = x, topk, w_comb, w1, w2, dout
        T, D, k, E, F, N1 = self.T, self.D, self.k, self.E, self.F, self.N1
        self.M_cap = M = api.max_routed_rows(T, k, E, self.align)
        e = lambda *s, dt=torch.uint8: torch.empty(*s, dtype=dt, device=dev)
        sfb = api.sf_bytes
        # routing
        self.seg = e(E + 1, dt=torch.int64)
        self.src = e(M, dt=torch.int32)
        self.pos = e(T, k, dt=torch.int32)
        self.route_ws = e(max(16, api.L.lib().mx_route_workspace_bytes(T, E)))
        self.rows_valid = self.seg[E:E + 1]
        # forward
        self.xq = (e(T, D // 2), e(sfb(T, D, 16, MX_SF_ROWMAJOR)), e(T, dt=torch.float32))
        self.xp = (e(M, D // 2), e(sfb(M, D, 16, MX_SF_MMA)), e(M, dt=torch.float32))
        self.w1q = (e(E * N1, D // 2), e(sfb(E * N1, D, 16, MX_SF_MMA)), e(E, dt=torch.float32))
        self.w2q = (e(E * D, F // 2), e(sfb(E * D, F, 16, MX_SF_MMA)), e(E, dt=torch.float32))
        self.h1 = e(M, N1, dt=out_dtype)
        self.a = e(M, F, dt=torch.bfloat16)
        self.aq = (e(M, F // 2), e(sfb(M, F, 16, MX_SF_MMA)), e(M, dt=torch.float32))
        if combine == "s2f6":
            self.y2s = (e(M, D, dt=torch.int8), e(M, D // 32))
        else:
            self.y2 = e(M, D, dt=out_dtype)
        self.out = e(T, D, dt=torch.bfloat16)
        # backward
        self.dy2 = None if self.fuse_backward else e(M, D, dt=torch.bfloat16)
        self.dy2q = (e(M, D), e(sfb(M, D, 32, MX_SF_MMA)), e(D, M), e(sfb(D, M, 32, MX_SF_MMA)))
        self.w2t = (e(F, E * D), e(sfb(F, E * D, 32, MX_SF_MMA)))
        self.da = e(M, F, dt=torch.bfloat16)
        self.at = (e(F, M), e(sfb(F, M, 32, MX_SF_MMA)))
        self.dw2 = e(E, D, F, dt=wgrad_dtype)
        self.dh1 = e(M, N1, dt=torch.bfloat16)
        self.dh1q = (e(M, N1), e(sfb(M, N1, 32, MX_SF_MMA)), e(N1, M), e(sfb(N1, M, 32, MX_SF_MMA)))
        self.w1t = (e(D, E * N1), e(sfb(D, E * N1, 32, MX_SF_MMA)))
        self.dxp = e(M, D, dt=torch.bfloat16)
        self.xt = (e(D, M), e(sfb(D, M, 32, MX_SF_MMA)))
        self.dw1 = e(E, N1, D, dt=wgrad_dtype)
        self.dx = e(T, D, dt=torch.bfloat16)
        if backward == "nvfp4":
            q4 = lambda r, c, n_outer: (e(r, c // 2), e(sfb(r, c, 16, MX_SF_MMA)), e(n_outer, dt=torch.float32))
            self.dy2n = q4(M, D, M)                     # dgrad2 A: dY2, per-token outer
            self.w2tn = q4(E * F, D, E)                 # dgrad2 B: stack of W2_e^T, per-expert outer
            self.dy2tn = q4(D, M, E * D)                # wgrad2 A: dY2^T, per (segment, row)
            self.atn = q4(F, M, E)                      # wgrad2 B: a^T, per segment
            self.dh1n = q4(M, N1, M)
            self.w1tn = q4(E * D, N1, E)
            self.dh1tn = q4(N1, M, E * N1)
            self.xtn = q4(D, M, E)
        self.marks = []

    # ------------------------------------------------------------------ timing
    def _mark(self, name: str, record: bool):
        if record:
            ev = torch.cuda.Event(enable_timing=True)
            ev.record()
            self.marks.append((name, ev))

    def reset_marks(self):
        self.marks = []

    # ------------------------------------------------------------------ I/O
    IO = ("x", "topk", "w_comb", "dout", "out", "dx")

    def io(self) -> dict:
        """The per-step inputs (x, topk, w_comb, dout) and outputs (out, dx)."""
        return {n: getattr(self, n) for n in self.IO}

    def bind_io(self, bufs: dict) -> None:
        """Point the next steps at other device tensors of the same shapes for
        the per-step inputs and outputs (weights and intermediates stay)."""
        for n in self.IO:
            t = bufs[n]
            if t.shape != getattr(self, n).shape or t.dtype != getattr(self, n).dtype:
                raise ValueError(f"{n}: {tuple(t.shape)} {t.dtype}, the layer was built for "
                                 f"{tuple(getattr(self, n).shape)} {getattr(self, n).dtype}")
            setattr(self, n, t)

    # ----------------------------------------------------------------- forward
    def forward(self, record: bool = False):
        T, D, k, E, F, N1, M = self.T, self.D, self.k, self.E, self.F, self.N1, self.M_cap
        self._mark("start", record)
        api.moe_route(self.topk, E, M, out=(self.seg, self.src, self.pos, self.route_ws), align=self.align)
        self._mark("route", record)
        api.nvfp4_quantize(self.x, 1, MX_SF_ROWMAJOR, out=self.xq)
        self._mark("quant_x", record)
        api.nvfp4_gather_rows(*self.xq, self.src, k, D, out=self.xp)
        self._mark("gather", record)
        api.nvfp4_quantize(self.w1.view(E * N1, D), N1, MX_SF_MMA, out=self.w1q)
        api.nvfp4_quantize(self.w2.view(E * D, F), D, MX_SF_MMA, out=self.w2q)
        self._mark("quant_w", record)
        api.grouped_gemm_nvfp4(self.xp, self.w1q, self.seg, E, N1, D, out=self.h1)
        self._mark("gemm1", record)
        if self.fuse_swiglu:
            api.swiglu_nvfp4_quantize(self.h1, F, self.gated, self.rows_valid, MX_SF_MMA, out=self.aq)
            self._mark("swiglu_quant", record)
        else:
            api.swiglu_fwd(self.h1, F, self.gated, self.rows_valid, out=self.a)
            self._mark("swiglu", record)
            api.nvfp4_quantize(self.a, 1, MX_SF_MMA, out=self.aq)
            self._mark("quant_a", record)
        if self.combine == "s2f6":
            api.grouped_gemm_nvfp4_s2f6(self.aq, self.w2q, self.seg, E, D, F, self.seed, self.S2F6_STREAM,
                                        out=self.y2s)
            self._mark("gemm2", record)
            api.moe_combine_s2f6(*self.y2s, self.pos, self.w_comb, self.seed, self.S2F6_STREAM, out=self.out)
        else:
            api.grouped_gemm_nvfp4(self.aq, self.w2q, self.seg, E, D, F, out=self.y2)
            self._mark("gemm2", record)
            api.moe_combine(self.y2, self.pos, self.w_comb, D, out=self.out)
        self._mark("combine", record)
        return self.out

    # ---------------------------------------------------------------- backward
    def backward(self, record: bool = False):
        if self.backward_format == "nvfp4":
            return self._backward_nvfp4(record)
        T, D, k, E, F, N1, M = self.T, self.D, self.k, self.E, self.F, self.N1, self.M_cap
        s, R = self.seed, self.rbits
        self._mark("bwd_start", record)
        if self.fuse_backward:
            api.moe_dispatch_grad_mxfp8_quantize(self.dout, self.src, self.w_comb, k, self.rows_valid, out=self.dy2q)
            self._mark("dispatch_grad_quant", record)
        else:
            api.moe_dispatch_grad(self.dout, self.src, self.pos, self.w_comb, out=self.dy2)
            self._mark("dispatch_grad", record)
            api.mxfp8_quantize(self.dy2, rows_valid=self.rows_valid, rounding=MX_ROUND_RNE, out=self.dy2q)
            self._mark("quant_dy2", record)
        api.mxfp8_requant_transpose_sr(*self.w2q, E * D, F, D, MX_SF_MMA, None, s, 1, R, out=self.w2t)
        self._mark("requant_w2", record)
        api.grouped_gemm_mxfp8(MX_GEMM_DGRAD, self.dy2q[0], self.dy2q[1], *self.w2t, self.seg, E, M, F, D, out=self.da)
        self._mark("dgrad2", record)
        api.mxfp8_requant_transpose_sr(*self.aq, M, F, 1, MX_SF_MMA, self.rows_valid, s, 2, R, out=self.at)
        self._mark("requant_a", record)
        api.grouped_gemm_mxfp8(MX_GEMM_WGRAD, self.dy2q[2], self.dy2q[3], *self.at, self.seg, E, M, D, F, out=self.dw2)
        self._mark("wgrad2", record)
        api.swiglu_bwd(self.h1, self.da, F, self.gated, self.rows_valid, out=self.dh1)
        self._mark("swiglu_bwd", record)
        api.mxfp8_quantize(self.dh1, rows_valid=self.rows_valid, rounding=MX_ROUND_RNE, out=self.dh1q)
        self._mark("quant_dh1", record)
        api.mxfp8_requant_transpose_sr(*self.w1q, E * N1, D, N1, MX_SF_MMA, None, s, 3, R, out=self.w1t)
        self._mark("requant_w1", record)
        api.grouped_gemm_mxfp8(MX_GEMM_DGRAD, self.dh1q[0], self.dh1q[1], *self.w1t, self.seg, E, M, D, N1,
                               out=self.dxp)
        self._mark("dgrad1", record)
        api.mxfp8_requant_transpose_sr(*self.xp, M, D, 1, MX_SF_MMA, self.rows_valid, s, 4, R, out=self.xt)
        self._mark("requant_x", record)
        api.grouped_gemm_mxfp8(MX_GEMM_WGRAD, self.dh1q[2], self.dh1q[3], *self.xt, self.seg, E, M, N1, D,
                               out=self.dw1)
        self._mark("wgrad1", record)
        api.moe_combine(self.dxp, self.pos, None, D, out=self.dx)
        self._mark("unpermute", record)
        return self.dx, self.dw1, self.dw2

    def _backward_nvfp4(self, record: bool):
        """The four backward GEMMs in NVFP4: dgrad as the forward grouped GEMM
        with B the requantised stack of W_e^T; wgrad on the transposes with
        outer scales per expert segment.  Every operand is rounded
        stochastically (its own Philox stream)."""
        D, E, F, N1, M = self.D, self.E, self.F, self.N1, self.M_cap
        s, R, SR = self.seed, self.rbits, MX_ROUND_SR
        self._mark("bwd_start", record)
        api.moe_dispatch_grad(self.dout, self.src, self.pos, self.w_comb, out=self.dy2)
        self._mark("dispatch_grad", record)
        api.nvfp4_quantize_sr(self.dy2, 1, SR, s, 11, R, MX_SF_MMA, out=self.dy2n)
        self._mark("quant_dy2", record)
        api.nvfp4_requant_transpose_sr(*self.w2q, E * D, F, D, MX_SF_MMA, E, True, SR, s, 12, R, MX_SF_MMA,
                                       out=self.w2tn)
        self._mark("requant_w2", record)
        api.grouped_gemm_nvfp4(self.dy2n, self.w2tn, self.seg, E, F, D, out=self.da)
        self._mark("dgrad2", record)
        api.nvfp4_quantize_transpose_segments(self.dy2, self.seg, E, True, SR, s, 13, R, MX_SF_MMA, out=self.dy2tn)
        api.nvfp4_requant_transpose_segments(*self.aq, M, F, self.seg, E, False, 1, MX_SF_MMA, SR, s, 14, R,
                                             MX_SF_MMA, out=self.atn)
        self._mark("requant_a", record)
        api.grouped_gemm_nvfp4_wgrad(self.dy2tn, self.atn, self.seg, E, D, F, out=self.dw2)
        self._mark("wgrad2", record)
        api.swiglu_bwd(self.h1, self.da, F, self.gated, self.rows_valid, out=self.dh1)
        self._mark("swiglu_bwd", record)
        api.nvfp4_quantize_sr(self.dh1, 1, SR, s, 15, R, MX_SF_MMA, out=self.dh1n)
        self._mark("quant_dh1", record)
        api.nvfp4_requant_transpose_sr(*self.w1q, E * N1, D, N1, MX_SF_MMA, E, True, SR, s, 16, R, MX_SF_MMA,
                                       out=self.w1tn)
        self._mark("requant_w1", record)
        api.grouped_gemm_nvfp4(self.dh1n, self.w1tn, self.seg, E, D, N1, out=self.dxp)
        self._mark("dgrad1", record)
        api.nvfp4_quantize_transpose_segments(self.dh1, self.seg, E, True, SR, s, 17, R, MX_SF_MMA, out=self.dh1tn)
        api.nvfp4_requant_transpose_segments(*self.xp, M, D, self.seg, E, False, 1, MX_SF_MMA, SR, s, 18, R,
                                             MX_SF_MMA, out=self.xtn)
        self._mark("requant_x", record)
        api.grouped_gemm_nvfp4_wgrad(self.dh1tn, self.xtn, self.seg, E, N1, D, out=self.dw1)
        self._mark("wgrad1", record)
        api.moe_combine(self.dxp, self.pos, None, D, out=self.dx)
        self._mark("unpermute", record)
        return self.dx, self.dw1, self.dw2

    def step(self, record: bool = False):
        self.forward(record)
        return self.backward(record)

    def stage_times_ms(self) -> dict:
        """Device time (ms) of each stage, summed over the recorded steps: the
        interval between a mark and the one before it is charged to the later
        mark's name (call after synchronising)."""
        out = {}
        for (_, a), (name, b) in zip(self.marks, self.marks[1:]):
            if name in ("start", "bwd_start"):                 # boundaries, not stages
                continue
            out[name] = out.get(name, 0.0) + a.elapsed_time(b)
        return out


def host_stream_steps(layer: ExpertLayer, host_in: dict, host_out: dict, steps: int) -> None:
    """Run `steps` layer steps whose inputs come from pinned host memory and
    whose outputs go back to it, every step copying its own inputs and results.

    host_in holds pinned x, topk, w_comb, dout; host_out pinned out, dx.  Two
    device buffer sets alternate between steps.  A host-to-device stream fills
    a step's forward inputs (x, topk, w_comb) and then its upstream gradient
    (dout), so the forward starts before dout has arrived; a device-to-host
    stream drains the forward output as soon as the forward ends (beside the
    backward) and dx after the backward.  The copy engines work beside the
    SMs, so only the first step's forward inputs and the last step's dx are
    not hidden behind kernels.  Everything is enqueued; the caller synchronises.
    """
    cs = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    up.wait_stream(cs)                                     # earlier work on the buffers comes first
    own = layer.io()
    sets = [own, {n: torch.empty_like(t) for n, t in own.items()}]
    for t in list(own.values()) + list(sets[1].values()):
        t.record_stream(up)                                # used beside the allocating stream
        t.record_stream(down)
    ev = lambda: [torch.cuda.Event() for _ in range(2)]
    fwd_ready, bwd_ready, in_free = ev(), ev(), ev()
    out_ready, out_free, dx_ready, dx_free = ev(), ev(), ev(), ev()
    for i in range(steps):
        b = i % 2
        buf = sets[b]
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(in_free[b])                  # step i-2 has read this set
            for n in ("x", "topk", "w_comb"):
                buf[n].copy_(host_in[n], non_blocking=True)
            fwd_ready[b].record(up)
            buf["dout"].copy_(host_in["dout"], non_blocking=True)
            bwd_ready[b].record(up)
        layer.bind_io(buf)
        cs.wait_event(fwd_ready[b])
        if i >= 2:
            cs.wait_event(out_free[b])                     # step i-2's output is on the host
        layer.forward()
        out_ready[b].record(cs)
        with torch.cuda.stream(down):
            down.wait_event(out_ready[b])
            host_out["out"].copy_(buf["out"], non_blocking=True)
            out_free[b].record(down)
        cs.wait_event(bwd_ready[b])
        if i >= 2:
            cs.wait_event(dx_free[b])                      # step i-2's dx is on the host
        layer.backward()
        in_free[b].record(cs)
        dx_ready[b].record(cs)
        with torch.cuda.stream(down):
            down.wait_event(dx_ready[b])
            host_out["dx"].copy_(buf["dx"], non_blocking=True)
            dx_free[b].record(down)
    cs.wait_stream(down)
    layer.bind_io(own)

