"""The tensor-core scale-factor tile layout, as a plain index permutation.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

The block-scaled FP4 tensor-core instruction reads the scale factors of a
128-row operand slab for a 64-element K step (four E4M3 scales per row) as one
512-byte tile: 32 lines of 16 bytes, where line i holds, for the rows
i, i+32, i+64, i+96 in that order, the four scales of that row for the four
consecutive 16-element K blocks.  Tiles are stored K-step-major inside each
128-row slab, slabs one after another:

    byte(row, kb) = ((row // 128) * n_ksteps + kb // 4) * 512
                    + (row % 32) * 16 + ((row // 32) % 4) * 4 + kb % 4

with kb the 16-element block index along K and n_ksteps = cols / 64.  Rows
are padded to a multiple of 128 (padding bytes are unspecified).

MXFP4 scales (one UE8M0 per 32 elements) use the same tile with 32-element
blocks: four scales per row per 128-column K step, n_ksteps = cols / 128.  This is the
layout the pages leave open (they only fix group 16); it is the instruction's
own operand layout, so the GEMM can copy scale tiles without reshuffling.
"""
import numpy as np


def mma_sf_bytes(rows, cols, block=16):
    """Size in bytes of the tiled scale buffer for a [rows, cols] FP4 matrix."""
    assert cols % (4 * block) == 0
    rows_pad = -(-rows // 128) * 128
    return rows_pad * (cols // block)


def mma_sf_index(rows, cols, block=16):
    """int64 [rows, cols/block]: byte offset of each canonical scale in the
    tile layout (block = 16 for NVFP4, 32 for MXFP4)."""
    assert cols % (4 * block) == 0
    n_ksteps = cols // (4 * block)
    r = np.arange(rows, dtype=np.int64)[:, None]
    kb = np.arange(cols // block, dtype=np.int64)[None, :]
    return ((r // 128) * n_ksteps + kb // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + kb % 4


def sf_to_mma(sf, fill=0, block=16):
    """Canonical row-major scales uint8 [rows, cols/block] -> tile layout bytes."""
    sf = np.asarray(sf, dtype=np.uint8)
    rows, nblk = sf.shape
    cols = nblk * block
    out = np.full(mma_sf_bytes(rows, cols, block), fill, dtype=np.uint8)
    out[mma_sf_index(rows, cols, block)] = sf
    return out


def sf_from_mma(buf, rows, cols, block=16):
    """Tile layout bytes -> canonical row-major scales [rows, cols/block]."""
    buf = np.asarray(buf, dtype=np.uint8).reshape(-1)
    return buf[mma_sf_index(rows, cols, block)]
