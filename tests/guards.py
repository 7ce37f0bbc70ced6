"""Canary guard bands around device output buffers: the output is a view into a
larger buffer whose margins hold a sentinel bit pattern, checked after a call
(an out-of-range write by a kernel changes a margin)."""
import math

import torch

PAD_BYTES = 256  # keeps the inner view 16-byte aligned


def guarded(shape, dtype, device="cuda"):
    """(inner view of `shape`, check()) for a fresh buffer with sentinel margins."""
    n = math.prod(shape)
    item = torch.empty((), dtype=dtype).element_size()
    pad = PAD_BYTES // item
    raw = torch.empty((n + 2 * pad) * item, dtype=torch.uint8, device=device)
    raw.fill_(0xA5)  # sentinel byte: not a value any kernel writes on purpose into a margin
    buf = raw.view(dtype)
    inner = buf[pad: pad + n].view(shape)

    def check():
        torch.cuda.synchronize()
        margins = torch.cat([raw[: pad * item], raw[(pad + n) * item:]])
        assert bool((margins == 0xA5).all()), "a kernel wrote outside its output buffer"

    return inner, check
