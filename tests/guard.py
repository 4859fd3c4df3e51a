"""Guard canaries around device buffers (the GPU tests' overrun check).

Every guarded buffer sits in the middle of a larger allocation whose first and
last PAD bytes hold a fixed byte pattern; after the calls, any byte of those
margins that changed means a kernel wrote outside the buffer it was given.  The
buffer itself starts out holding the same pattern (garbage to the callee), so a
kernel that fails to write part of its output is caught by the parity checks.
"Attention matrix view: make only frame-0 query rows dense" s4: the block
kernels write whole blocks, so a ragged last block is where an overrun lands.
"""
import numpy as np
import torch

PAD = 4096
FILL = 0xA5


class Guard:
    def __init__(self, device="cuda"):
        self.device = device
        self.bufs = []

    def alloc(self, shape, dtype, name):
        """A contiguous tensor of `shape` / `dtype` with PAD canary bytes on each side."""
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        raw = torch.full((PAD + n + PAD,), FILL, dtype=torch.uint8, device=self.device)
        t = raw[PAD:PAD + n].view(dtype).view(tuple(shape))
        self.bufs.append((name, raw, n))
        return t

    def bytes(self, n, name):
        return self.alloc((max(int(n), 1),), torch.uint8, name)

    def check(self):
        """Assert that no canary byte changed (synchronises the device first)."""
        torch.cuda.synchronize()
        for name, raw, n in self.bufs:
            for part, seg in (("before", raw[:PAD]), ("after", raw[PAD + n:])):
                bad = (seg != FILL).nonzero()
                assert bad.numel() == 0, "%s: %d canary bytes %s the buffer overwritten (first at %d)" % (
                    name, bad.numel(), part, int(bad[0]))
