"""Int4KVCache: a ring of INT4 key (or value) slots driven by rbd_kv4_encode / rbd_kv4_decode.

The cache offers the three operations a serving loop performs on a KV cache -- appending a
slice, evicting the oldest tokens, reading a slice back -- ("lab", Study 6: the serving loop touches the
four-bit cache only through these, so it can stand where a bf16 cache tensor stood).  Only the ring's
bookkeeping lives here; encoding and decoding run in librbd.so.  Token 0 of the cache is the
oldest one held; slots are reused in ring order, so a write never moves existing codes.  Token
slices index it like a tensor: cache[a:b] reads, cache[a:b] = x overwrites, cache[len(cache):] = x
appends.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _binding as B


class Int4KVCache:
    def __init__(self, capacity: int, heads: int, groups_per_band: int = 1, device=None):
        """capacity: token slots; heads: heads of 128 channels per token; groups_per_band 1, 2
        or 4 (3, 6 or 12 scale groups per head)."""
        if capacity <= 0 or heads <= 0:
            raise ValueError("capacity and heads must be positive")
        if groups_per_band not in (1, 2, 4):
            raise ValueError("groups_per_band must be 1, 2 or 4")
        self.capacity, self.heads, self.groups_per_band = capacity, heads, groups_per_band
        dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.codes = torch.zeros((capacity, heads, 64), dtype=torch.uint8, device=dev)
        self.scales = torch.zeros((capacity, heads, 3 * groups_per_band), dtype=torch.float32, device=dev)
        self.start = 0   # slot of the oldest token held
        self.size = 0    # tokens held

    def write(self, x: torch.Tensor) -> None:
        """Append the tokens of x (bf16 [T, heads * 128], row stride may be larger).  When the
        ring is full the oldest tokens are evicted first (rolling)."""
        self._check_slice(x)
        t = x.shape[0]
        if t > self.capacity:
            raise ValueError("slice longer than the cache")
        # the ring's bookkeeping moves only once the encode has been accepted: a refused call
        # (bad stride, alignment, device) leaves the held tokens as they were
        overflow = max(self.size + t - self.capacity, 0)
        start = (self.start + overflow) % self.capacity
        size = self.size - overflow
        slot0 = (start + size) % self.capacity
        B.rbd_kv4_encode(x, self.codes, self.scales, self.groups_per_band, slot0)
        self.start, self.size = start, size + t

    def overwrite(self, first: int, x: torch.Tensor) -> None:
        """Re-encode held tokens first .. first + T - 1 (0 = the oldest held) from x (bf16
        [T, heads * 128]); the ring's start and size do not change."""
        self._check_slice(x)
        if first < 0 or first + x.shape[0] > self.size:
            raise ValueError("overwrite outside the tokens held")
        B.rbd_kv4_encode(x, self.codes, self.scales, self.groups_per_band, (self.start + first) % self.capacity)

    def _check_slice(self, x: torch.Tensor) -> None:
        if x.dtype != torch.bfloat16 or x.dim() != 2 or x.shape[1] != self.heads * 128:
            raise ValueError("x must be bf16 [T, heads * 128]")
        if x.device != self.codes.device:
            raise ValueError(f"x is on {x.device}, the cache on {self.codes.device}")

    def __len__(self) -> int:
        return self.size

    def _span(self, key) -> tuple:
        if not isinstance(key, slice):
            raise TypeError("the cache is indexed by token slices")
        a, b, step = key.indices(self.size)
        if step != 1:
            raise ValueError("slices of the cache have step 1")
        return a, max(b - a, 0)

    def __getitem__(self, key) -> torch.Tensor:
        """cache[a:b] decodes tokens a .. b - 1 (Python slice rules, 0 = the oldest held)."""
        a, n = self._span(key)
        return self.read(a, n)

    def __setitem__(self, key, x: torch.Tensor) -> None:
        """cache[a:b] = x re-encodes held tokens a .. b - 1; cache[len(cache):] = x appends (rolling)."""
        if isinstance(key, slice) and key.start == self.size and key.stop is None and key.step is None:
            self.write(x)
            return
        a, n = self._span(key)
        if n != x.shape[0]:
            raise ValueError("slice and x differ in token count")
        self.overwrite(a, x)

    def evict(self, n: int) -> None:
        """Drop the n oldest tokens (their slots are reused by later writes)."""
        if n < 0 or n > self.size:
            raise ValueError("cannot evict more tokens than the cache holds")
        self.start = (self.start + n) % self.capacity
        self.size -= n

    def read(self, first: int = 0, count: Optional[int] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Decode tokens first .. first + count - 1 (0 = the oldest held) into out (bf16
        [count, heads * 128]; allocated when not given)."""
        count = self.size - first if count is None else count
        if first < 0 or count < 0 or first + count > self.size:
            raise ValueError("read outside the tokens held")
        if out is None:
            out = torch.empty((count, self.heads * 128), dtype=torch.bfloat16, device=self.codes.device)
        elif out.dtype != torch.bfloat16 or out.dim() != 2 or out.shape[0] < count or out.shape[1] != self.heads * 128:
            raise ValueError("out must be bf16 [>= count, heads * 128]")
        elif out.device != self.codes.device:
            raise ValueError(f"out is on {out.device}, the cache on {self.codes.device}")
        if count:
            slot0 = (self.start + first) % self.capacity
            B.rbd_kv4_decode(self.codes, self.scales, out[:count], self.groups_per_band, slot0)
        return out
