"""Guard bands around device buffers (the race / out-of-bounds check used in
place of a sanitizer): a region of `nbytes` at a 4 KiB offset inside one
allocation, with 4 KiB of a fixed byte pattern before and after it.  A
region may hold a row-strided matrix whose padding columns also keep the
pattern; `intact()` checks every byte outside the writable part."""
import torch

GUARD = 4096
PATTERN = 0xA5


class Canary:
    def __init__(self, nbytes: int, device):
        self.nbytes = nbytes
        self.buf = torch.full((GUARD + nbytes + GUARD,), PATTERN, dtype=torch.uint8, device=device)
        self.writable = torch.zeros(nbytes, dtype=torch.bool, device=device)

    def ptr(self) -> int:
        """Device address of the region (4 KiB past the allocation's start, so 256-byte aligned)."""
        return self.buf.data_ptr() + GUARD

    def region(self) -> torch.Tensor:
        return self.buf[GUARD:GUARD + self.nbytes]

    def matrix(self, dtype, rows: int, cols: int, ld: int) -> torch.Tensor:
        """The region's start as a [rows, cols] matrix of `dtype` with row
        stride `ld` elements; those bytes become writable, the padding
        columns and anything past the last row stay guarded."""
        es = torch.empty(0, dtype=dtype).element_size()
        assert rows * ld * es <= self.nbytes and cols <= ld
        mask = torch.zeros(rows, ld * es, dtype=torch.bool, device=self.buf.device)
        mask[:, :cols * es] = True
        self.writable[:rows * ld * es] |= mask.flatten()
        return self.region()[:rows * ld * es].view(dtype).as_strided((rows, cols), (ld, 1))

    def zeroed(self) -> torch.Tensor:
        """The whole region, zero-filled and writable (a workspace)."""
        self.region().zero_()
        self.writable[:] = True
        return self.region()

    def intact(self) -> bool:
        """No byte outside the writable part changed: both guards and every padding byte."""
        b = self.buf
        guards = bool((b[:GUARD] == PATTERN).all()) and bool((b[GUARD + self.nbytes:] == PATTERN).all())
        pad = self.region()[~self.writable]
        return guards and bool((pad == PATTERN).all())
