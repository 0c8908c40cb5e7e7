"""Canary-padded output buffers: a kernel gets a tensor that is the interior
of a larger buffer whose margins (or padding heads) hold a sentinel bit
pattern; after the call every sentinel must be intact, or the kernel wrote
out of bounds.  The sentinels are NaN payloads (floating point) and 0xA5
(bytes); the tests also check the outputs are finite, so no kernel result
can look like a sentinel."""

from __future__ import annotations

import math

import torch

MARGIN_BYTES = 256  # keeps the interior 16-byte (TMA) aligned
_INT_VIEW = {torch.bfloat16: (torch.int16, 0x7FA5), torch.float32: (torch.int32, 0x7FC0DEAD),
             torch.uint8: (torch.uint8, 0xA5)}


class Canvas:
    """A contiguous tensor `t` of `shape` inside a buffer with sentinel margins."""

    def __init__(self, shape, dtype, device):
        self.int_dtype, self.sentinel = _INT_VIEW[dtype]
        esize = torch.empty((), dtype=dtype).element_size()
        self.m = MARGIN_BYTES // esize
        self.n = math.prod(shape)
        self.base = torch.empty(self.n + 2 * self.m, dtype=dtype, device=device)
        self.base.view(self.int_dtype).fill_(self.sentinel)
        self.t = self.base[self.m:self.m + self.n].view(shape)

    def intact(self) -> bool:
        ints = self.base.view(self.int_dtype)
        return bool((ints[:self.m] == self.sentinel).all()) and bool((ints[self.m + self.n:] == self.sentinel).all())


class HeadCanvas:
    """A strided bf16 tensor `t` ``[B, S, H, D]`` whose heads sit between a
    sentinel head on either side (the head stride is (H + 2) D)."""

    def __init__(self, B, S, H, D, device):
        self.base = torch.empty((B, S, H + 2, D), dtype=torch.bfloat16, device=device)
        self.base.view(torch.int16).fill_(_INT_VIEW[torch.bfloat16][1])
        self.t = self.base[:, :, 1:H + 1]
        self.H = H

    def intact(self) -> bool:
        ints = self.base.view(torch.int16)
        s = _INT_VIEW[torch.bfloat16][1]
        return bool((ints[:, :, 0] == s).all()) and bool((ints[:, :, self.H + 1] == s).all())
