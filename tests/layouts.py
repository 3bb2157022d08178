"""Byte-layout permutations between the oracle's plain layouts and the
library's tile-major packed layouts (include/qlin.h, qlin_weights).  Pure
index shuffling: no arithmetic of the layer."""
import numpy as np


def _swizzle_rows(block: np.ndarray) -> np.ndarray:
    """Apply the 128-byte swizzle to a [rows][128] byte block: 16-byte chunk
    c of row r moves to chunk c ^ (r % 8)."""
    rows = block.shape[0]
    out = np.empty_like(block)
    chunks = block.reshape(rows, 8, 16)
    o = out.reshape(rows, 8, 16)
    for r in range(rows):
        for c in range(8):
            o[r, c ^ (r % 8)] = chunks[r, c]
    return out


def tile_w4(packed: np.ndarray, N: int, K: int) -> np.ndarray:
    """packed: uint8 [N][K/2] (row n = channel n) -> tiled uint8 bytes; the
    16-byte chunk c of row r of a block moves to chunk c ^ ((r // 2) % 4)."""
    TN, KB = -(-N // 128), -(-K // 128)
    full = np.zeros((TN * 128, KB * 64), np.uint8)
    full[:N, :K // 2] = packed
    t = np.ascontiguousarray(full.reshape(TN, 128, KB, 64).transpose(0, 2, 1, 3))
    out = np.empty_like(t)
    src = t.reshape(TN, KB, 128, 4, 16)
    dst = out.reshape(TN, KB, 128, 4, 16)
    for r in range(128):
        for c in range(4):
            dst[:, :, r, c ^ ((r // 2) % 4)] = src[:, :, r, c]
    return out.reshape(-1)


def tile_w8(q_nk: np.ndarray, N: int, K: int) -> np.ndarray:
    """q_nk: int8 [N][K] -> tiled, swizzled bytes (as uint8)."""
    TN, KB = -(-N // 128), -(-K // 128)
    full = np.zeros((TN * 128, KB * 128), np.uint8)
    full[:N, :K] = q_nk.view(np.uint8)
    t = np.ascontiguousarray(full.reshape(TN, 128, KB, 128).transpose(0, 2, 1, 3))
    out = np.empty_like(t)
    for a in range(TN):
        for b in range(KB):
            out[a, b] = _swizzle_rows(t[a, b])
    return out.reshape(-1)


def tile_wot(wot_n_i: np.ndarray, N: int, nO: int) -> np.ndarray:
    """wot_n_i: uint16 [N][nO] (W[O_i][n] at [n][i]) -> tiled, swizzled uint16."""
    TN, IB = -(-N // 128), -(-nO // 64)
    full = np.zeros((TN * 128, IB * 64), np.uint16)
    full[:N, :nO] = wot_n_i
    t = np.ascontiguousarray(full.reshape(TN, 128, IB, 64).transpose(0, 2, 1, 3))
    out = np.empty((TN, IB, 128, 128), np.uint8)
    for a in range(TN):
        for b in range(IB):
            out[a, b] = _swizzle_rows(t[a, b].view(np.uint8).reshape(128, 128))
    return out.reshape(-1).view(np.uint16)
