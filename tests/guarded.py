"""Guard-banded device buffers: a stand-in for a memory checker.

Every buffer handed to the library sits between two guard bands of canary
bytes; after the call the bands must still hold the canary, so a kernel that
writes past either end of an output, of the activations it quantises or of
its workspace is caught.  The payload starts at a 4096-byte offset inside a
fresh allocation, so its alignment is that of a plain torch allocation.
"""
from __future__ import annotations

import numpy as np

GUARD_BYTES = 4096
CANARY = 0xA5


class Guarded:
    """A [GUARD | payload | GUARD] uint8 allocation; `.t` is the payload tensor."""

    def __init__(self, torch, shape, dtype, fill=None, device="cuda"):
        self.torch = torch
        shape = tuple(int(s) for s in shape)
        item = torch.empty((), dtype=dtype).element_size()
        self.nbytes = int(np.prod(shape)) * item if shape else item
        pad = (-self.nbytes) % 256
        self.raw = torch.full((GUARD_BYTES + self.nbytes + pad + GUARD_BYTES,), CANARY, dtype=torch.uint8,
                              device=device)
        body = self.raw[GUARD_BYTES:GUARD_BYTES + self.nbytes]
        self.t = body.view(dtype).view(shape)
        if fill is not None:
            self.t.copy_(fill if isinstance(fill, torch.Tensor) else torch.as_tensor(fill).to(dtype))
        self.tail_start = GUARD_BYTES + self.nbytes

    def intact(self) -> bool:
        self.torch.cuda.synchronize()
        head = self.raw[:GUARD_BYTES]
        tail = self.raw[self.tail_start:]
        return bool((head == CANARY).all().item()) and bool((tail == CANARY).all().item())

    def check(self, what="buffer"):
        assert self.intact(), f"a kernel wrote outside {what} (guard band changed)"


def guarded_workspace(torch, bn, M, N, K):
    """A guard-banded workspace of exactly bitnet_workspace_bytes(M, N, K) bytes (at least 256)."""
    n = max(256, bn.bitnet_workspace_bytes(M, N, K))
    return Guarded(torch, (n,), torch.uint8)
