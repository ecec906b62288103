"""Test helpers: layout permutations and host<->device moves (no NVFP4 arithmetic)."""
import numpy as np


def tiled_index(rows_alloc: int, nsf: int) -> np.ndarray:
    """Flat offsets of scale (r, j) in the tensor-core atom layout, shape [rows_alloc, nsf].

    Layout (include/nvfp4.h): atoms of 128 rows x 4 scales = 512 bytes, ordered
    row-block-major; inside an atom (r%32)*16 + ((r%128)//32)*4 + j%4.
    """
    r = np.arange(rows_alloc, dtype=np.int64)[:, None]
    j = np.arange(nsf, dtype=np.int64)[None, :]
    return ((r // 128) * (nsf // 4) + j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (j % 4)


def untile(sf_flat: np.ndarray, rows_alloc: int, nsf: int) -> np.ndarray:
    return np.asarray(sf_flat).reshape(-1)[tiled_index(rows_alloc, nsf)]


def tile(sf_rm: np.ndarray) -> np.ndarray:
    rows, nsf = sf_rm.shape
    out = np.zeros(rows * nsf, dtype=np.uint8)
    out[tiled_index(rows, nsf)] = sf_rm
    return out


def slot_rows(offsets: np.ndarray):
    """Per routed row r, its row in the 128-aligned slot layout."""
    off = np.asarray(offsets, dtype=np.int64)
    counts = np.diff(off)
    padded = (counts + 127) // 128 * 128
    starts = np.concatenate([[0], np.cumsum(padded)])
    rows = []
    for g in range(len(counts)):
        rows.append(starts[g] + np.arange(counts[g]))
    return (np.concatenate(rows) if rows else np.zeros(0, np.int64)), starts


def to_dev(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def bf16_dev(bits: np.ndarray):
    import torch
    return to_dev(bits.astype(np.uint16).view(np.int16)).view(torch.bfloat16)


def to_np(t):
    import torch
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()
