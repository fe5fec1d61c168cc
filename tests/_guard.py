"""Guard bands around device buffers: a memory-safety check without a
sanitizer.

A guarded buffer is one uint8 allocation: GUARD bytes of PATTERN, the
buffer itself (256-byte aligned, viewed with its dtype and shape), then
GUARD bytes of PATTERN. After a call, any byte of either band that is no
longer PATTERN is a write outside the buffer.
"""

from __future__ import annotations

import math

import torch

GUARD = 4096
PATTERN = 0xA5


class Guarded:
    def __init__(self, shape, dtype, fill=None, device="cuda"):
        shape = tuple(shape)
        itemsize = torch.empty((), dtype=dtype).element_size()
        self.n = max(1, math.prod(shape)) * itemsize
        self.raw = torch.full((GUARD + self.n + GUARD,), PATTERN, dtype=torch.uint8, device=device)
        self.t = self.raw[GUARD:GUARD + self.n].view(dtype)[:math.prod(shape)].view(shape)
        if fill is not None:
            self.t.fill_(fill)

    def check(self, what="buffer"):
        torch.cuda.synchronize()
        head = self.raw[:GUARD]
        tail = self.raw[GUARD + self.n:]
        assert bool((head == PATTERN).all()), f"write before the {what}"
        assert bool((tail == PATTERN).all()), f"write after the {what}"


def workspace(nbytes, device="cuda"):
    """A guarded float32 decode workspace of at least `nbytes` bytes,
    NaN-filled, whose status word (its first int32) is zero."""
    g = Guarded((max(nbytes // 4, 1),), torch.float32, fill=float("nan"), device=device)
    g.t[:1].view(torch.int32).zero_()
    return g


def status_word(ws: Guarded) -> int:
    """The decode status word of a guarded workspace (synchronises)."""
    torch.cuda.synchronize()
    return int(ws.t[:1].view(torch.int32).item())
