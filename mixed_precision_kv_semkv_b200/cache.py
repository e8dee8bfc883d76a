"""Device buffers of one layer's packed cache, allocated with torch (plumbing only).

SemkvCache sizes every buffer with semkv_cache_bytes, allocates it on the GPU and fills the
semkv_cache_t descriptor that the C entry points take.
"""
from __future__ import annotations

from . import _lib


def capacities(T: int, p: float, extra: int = 0, window: int = 0):
    """(cap_hi, cap_lo, T_cap) for a prefill of T tokens at fraction p (plus a recent window of
    `window` tokens on the finer grid) and `extra` appends (the library's semkv_capacities)."""
    _, ch, cl, tc = _lib.semkv_capacities(T, p, window, extra)
    return ch, cl, tc


class SemkvCache:
    """One layer's cache: device buffers + the semkv_cache_t descriptor.  window, clip, L_hi_v,
    L_lo_v and k_per_channel select the quantizer variants (recent tokens forced onto the finer
    grid; clipped group range; V level counts of their own; per-channel K grids); 0 is the plain
    method."""

    def __init__(self, B: int, H: int, Hq: int, G: int, L_hi: int, L_lo: int, cap_hi: int, cap_lo: int,
                 T_cap: int, D: int = 128, device="cuda", window: int = 0, clip: float = 0.0, L_hi_v: int = 0,
                 L_lo_v: int = 0, k_per_channel: int = 0):
        import torch

        self.struct = _lib.CacheStruct(B=B, H=H, Hq=Hq, D=D, G=G, L_hi=L_hi, L_lo=L_lo, cap_hi=cap_hi,
                                       cap_lo=cap_lo, T_cap=T_cap, window=window, clip=clip, L_hi_v=L_hi_v,
                                       L_lo_v=L_lo_v, k_per_channel=int(k_per_channel))
        sizes = _lib.semkv_cache_bytes(self.struct)
        self.sizes = dict(zip(_lib.BUF_NAMES, sizes))
        self.bufs = {}
        for name, nbytes in self.sizes.items():
            dtype = torch.float32 if name == "tau" else torch.int32
            t = torch.empty(max(nbytes // 4, 1), dtype=dtype, device=device)
            self.bufs[name] = t
            setattr(self.struct, name, int(t.data_ptr()))
        self.bufs["status"].zero_()
        self.shape = dict(B=B, H=H, Hq=Hq, D=D, G=G, L_hi=L_hi, L_lo=L_lo, cap_hi=cap_hi, cap_lo=cap_lo,
                          T_cap=T_cap, window=window, clip=clip, L_hi_v=L_hi_v or L_hi, L_lo_v=L_lo_v or L_lo,
                          k_per_channel=int(k_per_channel))

    @classmethod
    def for_prefill(cls, B, H, Hq, G, L_hi, L_lo, T, p, extra=0, device="cuda", window=0, clip=0.0, L_hi_v=0,
                    L_lo_v=0, k_per_channel=0):
        ch, cl, tc = capacities(T, p, extra, window)
        return cls(B, H, Hq, G, L_hi, L_lo, ch, cl, tc, device=device, window=window, clip=clip, L_hi_v=L_hi_v,
                   L_lo_v=L_lo_v, k_per_channel=k_per_channel)

    def __getattr__(self, name):
        shape = self.__dict__.get("shape", {})
        if name in shape:
            return shape[name]
        raise AttributeError(name)

    @property
    def packed_bytes(self) -> int:
        """Bytes of the buffers that hold the compressed cache (codes, scales/zeros, bitmap)."""
        names = ("k_hi", "v_hi", "kz_hi", "vz_hi", "k_lo", "v_lo", "kz_lo", "vz_lo", "bitmap")
        return sum(self.sizes[n] for n in names)

    def workspace(self):
        import torch

        nbytes = _lib.semkv_workspace_bytes(self.struct)
        return torch.empty(max(nbytes, 4), dtype=torch.uint8, device=self.bufs["status"].device)

    def poison(self):
        """Fill every buffer except the status word with 0xFF bytes (NaN as fp16/fp32), so that a
        read of bytes the library never wrote shows up in tests."""
        for name, t in self.bufs.items():
            if name != "status":
                t.view(__import__("torch").int32).fill_(-1)
        return self

    def status(self) -> int:
        """Read the device status word (synchronizes)."""
        return int(self.bufs["status"].item())

    def clear_status(self):
        self.bufs["status"].zero_()
