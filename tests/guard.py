"""Guard bands around output buffers: each tensor is a view into the middle of
a byte buffer whose first and last GUARD bytes hold a fill pattern, so a
kernel that writes outside the tensor leaves a mark the host can see.  (The
memory checker is not available on the GPUs these tests run on; this catches
out-of-bounds writes near a tensor's ends, where tails and padding rows
would put them.)"""

from __future__ import annotations

import torch

GUARD = 4096  # bytes on each side (a multiple of every element size and of 16)
FILL = 0xA5


def guarded(shape, dtype: torch.dtype, device) -> tuple[torch.Tensor, torch.Tensor]:
    """A contiguous tensor of `shape` and `dtype` inside a guarded byte
    buffer.  Returns (tensor, buffer); the tensor starts GUARD bytes in."""
    numel = 1
    for s in shape:
        numel *= int(s)
    nbytes = numel * torch.empty((), dtype=dtype).element_size()
    buf = torch.full((GUARD + nbytes + GUARD,), FILL, dtype=torch.uint8, device=device)
    t = buf[GUARD:GUARD + nbytes].view(dtype).view(tuple(shape))
    return t, buf


def intact(buf: torch.Tensor) -> bool:
    """True if both guard bands still hold the fill pattern."""
    return bool((buf[:GUARD] == FILL).all()) and bool((buf[-GUARD:] == FILL).all())
