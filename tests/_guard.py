"""Guard regions around device buffers (test infrastructure).

compute-sanitizer is not available on the GPU pool, so out-of-bounds writes
are caught this way: every output buffer a test hands to the library is a
view into a larger allocation whose bytes before and after it hold a known
pattern, checked after the call.
"""
from __future__ import annotations

import torch

GUARD_BYTES = 4096
PATTERN = 0xA5


class Guarded:
    """``numel`` elements of ``dtype`` with GUARD_BYTES of PATTERN on each side.

    ``fill`` sets the inner bytes (0xFF makes an fp32/fp16 NaN, so outputs
    the call never writes show up).  ``intact()`` says whether both guards
    still hold the pattern."""

    def __init__(self, numel: int, dtype, device="cuda", fill: int = 0xFF, shape=None):
        esz = torch.empty((), dtype=dtype).element_size()
        self.nbytes = numel * esz
        self.buf = torch.full((2 * GUARD_BYTES + self.nbytes,), PATTERN, dtype=torch.uint8, device=device)
        self.buf[GUARD_BYTES: GUARD_BYTES + self.nbytes] = fill
        inner = self.buf[GUARD_BYTES: GUARD_BYTES + self.nbytes].view(dtype)
        self.t = inner.view(shape) if shape is not None else inner

    def intact(self) -> bool:
        head = self.buf[:GUARD_BYTES]
        tail = self.buf[GUARD_BYTES + self.nbytes:]
        return bool((head == PATTERN).all().item() and (tail == PATTERN).all().item())
