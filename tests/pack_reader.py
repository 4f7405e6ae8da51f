"""Independent reader of the direct-palette pack (test infrastructure).

Reads a pack exactly as include/uw.h documents it and rebuilds every BF16 word
of W from it, so a pack written by the library can be checked against W
itself -- the plain definition -- instead of against another writer of the
same layout.  It shares no code with the library or with the oracle.

Documented layout, for a matrix of R rows and C columns (KB = C/64 k-blocks,
MT = ceil(R/128) row tiles, T = MT*KB tiles in (row tile, k-block) order):
  bodies  T x 12304 bytes; body t at byte 12304 t:
            [0, 8192)      sm bytes, row r, 16-byte chunk j at r*64 + 16*(j ^ ((r>>1)&3))
            [8192, 12288)  4-bit indices, row r, chunk j at 8192 + r*32 + 16*(j ^ ((r>>2)&1)),
                           element 2i in the low nibble of byte i of the row
            [12288, 12304) 128-bit mask, bit r = row r's group is verbatim
  tails   after the bodies: the verbatim rows of every tile in tile order and
          row order, 64 BF16 words (128 bytes) each;
  offs    uint32[T+1]: offs[t] = verbatim rows of all tiles before t.
The sm byte of element k is (mantissa_k << 1) | sign of element k^1.
"""
import numpy as np

BODY, IDX, MASK = 12304, 8192, 12288


def _gather_indices():
    r = np.arange(128)[:, None]
    b = np.arange(16)[None, :]
    sm = np.concatenate([r * 64 + 16 * (j ^ ((r >> 1) & 3)) + b for j in range(4)], axis=1)       # [128, 64]
    ix = np.concatenate([IDX + r * 32 + 16 * (j ^ ((r >> 2) & 1)) + b for j in range(2)], axis=1)  # [128, 32]
    return sm, ix


def unpack_to_w(rows, cols, palette, pack, offs):
    """Every BF16 word of W as uint16[rows, cols], read from `pack` / `offs`.
    Also asserts the layout's own invariants: sizes, zero rows past the
    matrix, and one tail row per mask bit."""
    pack = np.asarray(pack, dtype=np.uint8)
    offs = np.asarray(offs, dtype=np.int64)
    palette = np.asarray(palette, dtype=np.uint16)
    KB = cols // 64
    MT = -(-rows // 128)
    T = MT * KB
    assert offs.size == T + 1 and offs[0] == 0 and np.all(np.diff(offs) >= 0)
    assert pack.size == T * BODY + 128 * int(offs[-1])
    bodies = pack[:T * BODY].reshape(T, BODY)
    tails = pack[T * BODY:].view(np.uint16).reshape(-1, 64)
    sm_at, ix_at = _gather_indices()
    out = np.zeros((MT * 128, cols), dtype=np.uint16)
    for mt in range(MT):
        blk = bodies[mt * KB:(mt + 1) * KB]              # [KB, BODY]
        sm = blk[:, sm_at].astype(np.uint16)             # [KB, 128, 64]
        ix = blk[:, ix_at]                               # [KB, 128, 32]
        nib = np.empty((KB, 128, 64), dtype=np.uint8)
        nib[..., 0::2] = ix & 0xF
        nib[..., 1::2] = ix >> 4
        mant = sm >> 1
        sign = (sm & 1).reshape(KB, 128, 32, 2)[..., ::-1].reshape(KB, 128, 64)
        words = (sign << 15) | (palette[nib] << 7) | mant
        mask_words = blk[:, MASK:MASK + 16].copy().view(np.uint32)   # [KB, 4]
        bits = (mask_words[:, np.arange(128) // 32] >> (np.arange(128) % 32).astype(np.uint32)) & 1
        live = rows - mt * 128  # rows of this tile inside the matrix
        if live < 128:
            assert not sm[:, live:].any() and not ix[:, live:].any() and not bits[:, live:].any(), \
                "rows past the matrix must be zero"
        for kb in range(KB):
            t = mt * KB + kb
            vrows = np.flatnonzero(bits[kb])
            assert offs[t + 1] - offs[t] == vrows.size
            words[kb, vrows] = tails[offs[t]:offs[t + 1]]
        out[mt * 128:(mt + 1) * 128] = words.transpose(1, 0, 2).reshape(128, cols)
    return out[:rows]


def verbatim_rows_per_tile(vmask_groups: np.ndarray) -> np.ndarray:
    """pack offsets from a [rows, KB] verbatim-group mask: offs[t] = verbatim
    groups of all tiles before t, tiles in (row tile, k-block) order."""
    rows, KB = vmask_groups.shape
    MT = -(-rows // 128)
    padded = np.zeros((MT * 128, KB), dtype=np.int64)
    padded[:rows] = vmask_groups
    per_tile = padded.reshape(MT, 128, KB).sum(axis=1).reshape(-1)
    return np.concatenate([[0], np.cumsum(per_tile)]).astype(np.uint32)
