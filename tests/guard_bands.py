"""Guard bands around output buffers: the output is a contiguous slice in
the middle of a larger buffer whose margins hold a sentinel; after the call
the margins must be untouched (a store past either end of an output shows
up there)."""
import torch

PAD = 64          # rows of margin on each side (dim 0)


def guarded(shape, dtype, fill, device):
    """(buffer, view): view has `shape` and is contiguous; the buffer has PAD
    extra rows of `fill` before and after it."""
    n = shape[0]
    buf = torch.full((PAD + n + PAD,) + tuple(shape[1:]), fill, dtype=dtype,
                     device=device)
    return buf, buf[PAD:PAD + n]


def margins_intact(buf, fill):
    """True when the PAD rows at both ends of buf still hold `fill`."""
    n = buf.shape[0] - 2 * PAD
    want = torch.full_like(buf[:PAD], fill)
    return bool(torch.equal(buf[:PAD], want) and torch.equal(buf[PAD + n:], want))
