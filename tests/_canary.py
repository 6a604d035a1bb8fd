"""Guard regions around output buffers, the out-of-bounds write check that stands in for a
memory sanitizer.

guarded_empty() returns an output tensor that is a view into a larger buffer: GUARD bytes
before it and GUARD bytes after it hold a fixed byte pattern.  After a call,
guards_intact() checks that the pattern is unchanged, so a kernel that wrote past either
end of that output is caught.  GUARD is a multiple of 512 bytes, so the view keeps the
allocation's alignment and a kernel takes the same path as on a plain tensor."""

GUARD = 1024
PATTERN = 0xA5


def guarded_empty(shape, dtype, device):
    """(buffer, view): view has `shape` and `dtype`; the buffer holds it between two guard
    regions filled with PATTERN (the view itself starts out filled with PATTERN too)."""
    import torch
    es = torch.empty((), dtype=dtype).element_size()
    if GUARD % es:
        raise ValueError("guard size must be a multiple of the element size")
    count = 1
    for s in shape:
        count *= int(s)
    g = GUARD // es
    buf = torch.empty(2 * g + count, dtype=dtype, device=device)
    buf.view(torch.uint8).fill_(PATTERN)
    return buf, buf[g:g + count].view(*shape)


def guards_intact(buf) -> bool:
    """True when both guard regions of a buffer from guarded_empty() still hold PATTERN."""
    import torch
    b = buf.view(torch.uint8)
    return bool((b[:GUARD] == PATTERN).all().item() and (b[-GUARD:] == PATTERN).all().item())
