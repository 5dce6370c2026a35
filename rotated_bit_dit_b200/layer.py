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
                 gate: Optional[torch.Tensor] = None):
        """weight bf16 [N, K] (CUDA); l1 bf16 [K, r], l2 bf16 [r, N] (the branch adds (x l1) l2)."""
        if weight.dtype != torch.bfloat16 or not weight.is_cuda:
            raise ValueError("weight must be a CUDA bf16 tensor")
        self.N, self.K = weight.shape
        self.bits, self.scale_group, self.rot_group = bits, scale_group, rot_group
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

    def buffers(self, M: int, device):
        key = (M, str(device))
        if key not in self._bufs:
            G = self.K // 64 if self.scale_group else 1
            codes = torch.empty((M, self.K), dtype=torch.int8, device=device)
            sx = torch.empty((M, G) if self.scale_group else (M,), dtype=torch.float32, device=device)
            ld = torch.empty((M, self.rank), dtype=torch.bfloat16, device=device) if self.rank else None
            self._bufs[key] = (codes, sx, ld)
        return self._bufs[key]

    def __call__(self, x: torch.Tensor, residual: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None, acc_debug: Optional[torch.Tensor] = None) -> torch.Tensor:
        M = x.shape[0]
        codes, sx, ld = self.buffers(M, x.device)
        if self.rank:
            B.rbd_lowrank_fused(x, codes, sx, self.l1t, ld, self.bits, self.rot_group, self.scale_group)
        else:
            B.rbd_rot_quant_act(x, codes, sx, self.bits, self.rot_group, self.scale_group)
        if out is None:
            out = torch.empty((M, self.N), dtype=torch.bfloat16, device=x.device)
        epi = B.make_epilogue(self.bias, ld, self.l2t, self.gate_mode, self.gate_cols, self.gate, residual,
                              acc_debug)
        fn = B.rbd_w4a4_linear if self.bits == 4 else B.rbd_w8a8_linear
        fn(codes, sx, self.wq, self.sw, out, self.scale_group, epi, self.rot_group)
        return out
