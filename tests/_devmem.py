"""Addresses for the host-side argument checks of the C ABI.

The checks under test return before anything is launched, so without a GPU any
non-null, suitably aligned value exercises them.  Where a GPU is visible, every
address handed to the library points into one real, zero-filled device buffer
instead: if a host check ever regressed and a kernel did launch, it would read
zero lengths and zero table entries from memory it owns, never an invented
address.  Each region is 256-byte aligned and large enough for every shape the
checks describe.
"""
from __future__ import annotations

import ctypes

REGION = 32 << 20  # bytes per region
_NREGIONS = 12


class DevMem:
    def __init__(self):
        self.buf = None
        try:
            import torch
            if torch.cuda.is_available():
                self.buf = torch.zeros(REGION * _NREGIONS + 256, dtype=torch.uint8,
                                       device="cuda")
        except Exception:  # pragma: no cover - torch always imports here
            self.buf = None
        self._base = None
        if self.buf is not None:
            p = self.buf.data_ptr()
            self._base = (p + 255) // 256 * 256
        self._next = 0

    @property
    def on_gpu(self) -> bool:
        return self.buf is not None

    def region(self, offset: int = 0) -> ctypes.c_void_p:
        """A fresh region (zero-filled device memory on a GPU), plus ``offset`` bytes."""
        i = self._next % _NREGIONS
        self._next += 1
        if self._base is None:
            return ctypes.c_void_p(4096 * (i + 1) + offset)
        return ctypes.c_void_p(self._base + i * REGION + offset)


_shared = None


def devmem() -> DevMem:
    global _shared
    if _shared is None:
        _shared = DevMem()
    return _shared
