"""INT8 attention (SageAttention v1 scheme) over the library's two calls.

int8_attention(q, k, v, heads) prepares the operands (key smoothing, INT8 codes
with a scale per token and head, fp16 transposed values) and runs the
attention kernel; buffers are allocated with torch (device memory plumbing),
every arithmetic step runs in librbd.so.  Source: "Krea 2 Turbo OrbitQuant
W4A4", "Fused transformer" (Q.K^T in INT8, P.V in FP16).
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _binding as B


def attention_operands(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, heads: int):
    """Allocate and fill (qc, sq, kc, sk, vt) for q [Tq, >=H*128], k / v [Tk, >=H*128] (bf16, CUDA)."""
    Tq, Tk = q.shape[0], k.shape[0]
    dev = q.device
    tkp = (Tk + 7) // 8 * 8
    qc = torch.empty((heads, Tq, 128), dtype=torch.int8, device=dev)
    sq = torch.empty((heads, Tq), dtype=torch.float32, device=dev)
    kc = torch.empty((heads, Tk, 128), dtype=torch.int8, device=dev)
    sk = torch.empty((heads, tkp), dtype=torch.float32, device=dev)
    vt = torch.empty((heads, 128, tkp), dtype=torch.float16, device=dev)
    work = torch.empty((B.rbd_attn_workspace_bytes(Tk, heads),), dtype=torch.uint8, device=dev)
    B.rbd_attn_quant(q, k, v, heads, qc, sq, kc, sk, vt, work)
    return qc, sq, kc, sk, vt


def int8_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, heads: int,
                   out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """o bf16 [Tq, heads*128] = softmax(Q K'^T / sqrt(128)) V with INT8 Q.K'^T (K' the smoothed keys)
    and FP16 P.V."""
    qc, sq, kc, sk, vt = attention_operands(q, k, v, heads)
    if out is None:
        out = torch.empty((q.shape[0], heads * 128), dtype=torch.bfloat16, device=q.device)
    B.rbd_attn_int8(qc, sq, kc, sk, vt, out)
    return out
