"""Host-side helpers shared by the GPU tests: the documented scale-factor tiling, undone or applied
on numpy arrays, guard-zone buffers, and the per-expert tile bases of a grouped call.

The tiling is stated in include/macaq.h: rows padded to 128 and cut into 128 x 4 tiles, ordered
row-tile-major then by K-tile; inside a tile, row r and scale column c sit at byte
(r % 32) * 16 + (r // 32) * 4 + c.
"""
import numpy as np
import torch

GUARD = 4096
CANARY = 0xA5


def sf_index(sf_rows: np.ndarray, K: int) -> np.ndarray:
    """Byte offset of (SF row, scale column) for every row in sf_rows and every column."""
    r = np.asarray(sf_rows, dtype=np.int64)[:, None]
    c = np.arange(K // 32, dtype=np.int64)[None, :]
    rt, rr = r // 128, r % 128
    return (rt * (K // 128) + c // 4) * 512 + (rr % 32) * 16 + (rr // 32) * 4 + c % 4


def unswizzle(buf: np.ndarray, rows: int, K: int, sf_rows=None) -> np.ndarray:
    if sf_rows is None:
        sf_rows = np.arange(rows)
    return buf[sf_index(sf_rows, K)]


def swizzle(sf: np.ndarray, K: int) -> np.ndarray:
    """Row-major [rows, K/32] -> tiled buffer (padding rows 0)."""
    rows = sf.shape[0]
    padded = (rows + 127) // 128 * 128
    out = np.zeros(padded * (K // 32), np.uint8)
    out[sf_index(np.arange(rows), K)] = sf
    return out


def tile_bases(offsets) -> np.ndarray:
    off = np.asarray(offsets, dtype=np.int64)
    cnt = (np.diff(off) + 127) // 128
    return np.concatenate([[0], np.cumsum(cnt)])


def grouped_sf_rows(offsets) -> np.ndarray:
    """Padded SF row of every row of a grouped call."""
    off = np.asarray(offsets, dtype=np.int64)
    tb = tile_bases(off)
    rows = np.empty(off[-1], np.int64)
    for e in range(len(off) - 1):
        rows[off[e]:off[e + 1]] = tb[e] * 128 + np.arange(off[e + 1] - off[e])
    return rows


def grouped_padding_rows(offsets) -> np.ndarray:
    off = np.asarray(offsets, dtype=np.int64)
    tb = tile_bases(off)
    pads = []
    for e in range(len(off) - 1):
        me = off[e + 1] - off[e]
        pads.append(tb[e] * 128 + np.arange(me, (tb[e + 1] - tb[e]) * 128))
    return np.concatenate(pads) if pads else np.zeros(0, np.int64)


class Guarded:
    """A device byte buffer with canary zones on both sides (16-byte aligned payload)."""

    def __init__(self, nbytes: int, device="cuda", dtype=torch.uint8, shape=None):
        self.n = int(nbytes)
        self.raw = torch.full((self.n + 2 * GUARD,), CANARY, dtype=torch.uint8, device=device)
        view = self.raw[GUARD:GUARD + self.n]
        if dtype != torch.uint8:
            view = view.view(dtype)
        self.t = view.view(shape) if shape is not None else view

    def intact(self) -> bool:
        r = self.raw.cpu().numpy()
        return bool(np.all(r[:GUARD] == CANARY) and np.all(r[GUARD + self.n:] == CANARY))
