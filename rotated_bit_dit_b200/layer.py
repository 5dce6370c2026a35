"""RotatedLowBitLinear: one quantized linear of the diffusion transformer.

Holds the offline-packed weights (INT4 packed or per-row INT8), their scales,
the optional low-rank factors, bias and gate configuration, and runs a call as
two launches on the current stream: the rotate+quantise prologue (with the
low-rank down product when a branch is present) and the low-bit GEMM with its
fused epilogue.  Buffers are allocated with torch (device memory plumbing);
every arithmetic step runs in librbd.so.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _binding as B


class RotatedLowBitLinear:
    def __init__(self, weight: torch.Tensor, bits: int = 4, scale_group: int = 0, rot_group: int = 256,
                 bias: Optional[torch.Tensor] = None, l1: Optional[torch.Tensor] = None,
                 l2: Optional[torch.Tensor] = None, gate_mode: int = 0, gate_cols=(0, 0),
                 gate: Optional[torch.Tensor] = None, code_format: Optional[int] = None):
        """weight bf16 [N, K] (CUDA); l1 bf16 [K, r], l2 bf16 [r, N] (the branch adds (x l1) l2).
        code_format: how the activation codes are stored between the two kernels; by default
        E4M3 for INT4 with group-64 scales (the FP8 tensor-core GEMM), INT8 otherwise."""
        if weight.dtype != torch.bfloat16 or not weight.is_cuda:
            raise ValueError("weight must be a CUDA bf16 tensor")
        self.N, self.K = weight.shape
        self.bits, self.scale_group, self.rot_group = bits, scale_group, rot_group
        if code_format is None:
            code_format = B.CODES_E4M3 if (bits == 4 and scale_group == 64) else B.CODES_INT8
        self.code_format = code_format
        G = self.K // 64 if scale_group else 1
        dev = weight.device
        self.sw = torch.empty((self.N, G) if scale_group else (self.N,), dtype=torch.float32, device=dev)
        w = weight.contiguous()
        if bits == 4:
            self.wq = torch.empty((self.N, self.K // 2), dtype=torch.uint8, device=dev)
            B.rbd_pack_weights_int4(w, self.wq, self.sw, rot_group, scale_group)
        elif bits == 8:
            self.wq = torch.empty((self.N, self.K), dtype=torch.int8, device=dev)
            B.rbd_pack_weights_int8(w, self.wq, self.sw, rot_group, scale_group)
        else:
            raise ValueError("bits must be 4 or 8")
        self.bias = bias.contiguous() if bias is not None else None
        self.l1t = l1.t().contiguous() if l1 is not None else None
        self.l2t = l2.t().contiguous() if l2 is not None else None
        self.rank = 0 if l1 is None else int(l1.shape[1])
        self.gate_mode, self.gate_cols = gate_mode, gate_cols
        self.gate = gate.contiguous() if gate is not None else None
        self._bufs = {}
        self._host_pipes = {}   # forward_host: streams and staging buffers per (device, chunk, residual)

    def buffers(self, M: int, device):
        """The call's intermediates (codes, scales, low-rank Ld) for M tokens, kept per
        (M, device, current stream): calls queued on different streams never share them, so
        one stream's prologue cannot overwrite codes another stream's GEMM has yet to read."""
        key = (M, str(device), torch.cuda.current_stream(device).cuda_stream)
        if key not in self._bufs:
            G = self.K // 64 if self.scale_group else 1
            codes = torch.empty((M, self.K), dtype=torch.int8, device=device)
            sx = torch.empty((M, G) if self.scale_group else (M,), dtype=torch.float32, device=device)
            ld = torch.empty((M, self.rank), dtype=torch.bfloat16, device=device) if self.rank else None
            self._bufs[key] = (codes, sx, ld)
        return self._bufs[key]

    def __call__(self, x: torch.Tensor, residual: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None, acc_debug: Optional[torch.Tensor] = None) -> torch.Tensor:
        codes, sx, ld = self.buffers(x.shape[0], x.device)
        return self._run(x, codes, sx, ld, residual, out, acc_debug)

    def _run(self, x, codes, sx, ld, residual=None, out=None, acc_debug=None) -> torch.Tensor:
        M = x.shape[0]
        cf = self.code_format
        if self.rank:
            B.rbd_lowrank_fused(x, codes, sx, self.l1t, ld, self.bits, self.rot_group, self.scale_group,
                                code_format=cf)
        else:
            B.rbd_rot_quant_act(x, codes, sx, self.bits, self.rot_group, self.scale_group, code_format=cf)
        if out is None:
            out = torch.empty((M, self.N), dtype=torch.bfloat16, device=x.device)
        epi = B.make_epilogue(self.bias, ld, self.l2t, self.gate_mode, self.gate_cols, self.gate, residual,
                              acc_debug)
        if self.bits == 4:
            B.rbd_w4a4_linear(codes, sx, self.wq, self.sw, out, self.scale_group, epi, self.rot_group,
                              code_format=cf)
        else:
            B.rbd_w8a8_linear(codes, sx, self.wq, self.sw, out, self.scale_group, epi, self.rot_group)
        return out

    def forward_host(self, xh: torch.Tensor, yh: torch.Tensor, residual_h: Optional[torch.Tensor] = None,
                     chunk: int = 1024, device=None) -> torch.Tensor:
        """The layer on host-resident tokens: xh bf16 [M, K] and yh bf16 [M, N] in pinned host memory
        (residual_h likewise [M, N] for the gated residual).  Tokens are independent, so the call
        streams `chunk`-token slices through two CUDA streams: the host-to-device copy of slice i + 1
        and the device-to-host copy of slice i - 1 run on the copy engines while slice i computes.
        Every output element is computed exactly as by __call__ (bit-identical).  Ordered after the
        work already queued on the current stream; the current stream waits for the result."""
        if not (xh.is_pinned() and yh.is_pinned()) or (residual_h is not None and not residual_h.is_pinned()):
            raise ValueError("host tensors must be pinned")
        dev = torch.device(device) if device is not None else self.wq.device
        M = xh.shape[0]
        cur = torch.cuda.current_stream(dev)
        streams, staged = self._host_pipeline(dev, chunk, residual_h is not None)
        start = torch.cuda.Event()
        start.record(cur)
        for s in streams:
            s.wait_event(start)
        for i, m0 in enumerate(range(0, M, chunk)):
            m = min(M, m0 + chunk) - m0
            s = streams[i % 2]
            xd, yd, rd, codes, sx, ld = staged[i % 2]
            with torch.cuda.stream(s):
                xd[:m].copy_(xh[m0:m0 + m], non_blocking=True)
                r = None
                if rd is not None:
                    rd[:m].copy_(residual_h[m0:m0 + m], non_blocking=True)
                    r = rd[:m]
                self._run(xd[:m], codes[:m], sx[:m], ld[:m] if ld is not None else None, r, yd[:m])
                yh[m0:m0 + m].copy_(yd[:m], non_blocking=True)
        for s in streams:
            cur.wait_stream(s)
        return yh

    def _host_pipeline(self, dev, chunk: int, with_residual: bool):
        """The two streams of forward_host and, per stream, its own input, output, residual and
        intermediate buffers; created once per (device, chunk, residual) and reused.  Reuse is
        safe: a buffer is only touched on its own stream, every call makes its streams wait for
        the caller's stream first, and the caller's stream waits for them at the end."""
        key = (str(dev), chunk, with_residual)
        if key not in self._host_pipes:
            G = self.K // 64 if self.scale_group else 1
            streams = [torch.cuda.Stream(device=dev) for _ in range(2)]
            staged = []
            for _ in streams:
                staged.append((
                    torch.empty((chunk, self.K), dtype=torch.bfloat16, device=dev),
                    torch.empty((chunk, self.N), dtype=torch.bfloat16, device=dev),
                    torch.empty((chunk, self.N), dtype=torch.bfloat16, device=dev) if with_residual else None,
                    torch.empty((chunk, self.K), dtype=torch.int8, device=dev),
                    torch.empty((chunk, G) if self.scale_group else (chunk,), dtype=torch.float32, device=dev),
                    torch.empty((chunk, self.rank), dtype=torch.bfloat16, device=dev) if self.rank else None))
            self._host_pipes[key] = (streams, staged)
        return self._host_pipes[key]
