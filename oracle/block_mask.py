"""BlockMask construction in the oracle (test infrastructure only).

Definition followed: tensorplay.nn.attention page, BlockMask "Basics" and
"Details". A block counts as sparse only when every element in it is masked.
Details item 1 gives (kv_num_blocks, kv_indices) and item 2 gives
(full_kv_num_blocks, full_kv_indices), which hold the blocks with no masked
element. With separate_full_blocks=True (create_block_mask's default) the
first pair holds only the partial blocks.

Readings where the page is silent:

* Tiles are 128x128. A tile is classified by counting its allowed elements
  that lie inside [0, Q_LEN) x [0, KV_LEN). FULL means 128*128 allowed
  elements (so a tile that crosses the end of either sequence is never
  FULL). EMPTY means 0. Everything else is PARTIAL.
* Index lists are in ascending block order. Entries after the count (the
  page calls them "undefined") are 0.
* B or H <= 0 stands for "None" and broadcasts as size 1.
"""
from __future__ import annotations

import numpy as np

from . import masks


def tile_classes(tree, b: int, Q_LEN: int, KV_LEN: int, BLOCK: int = 128) -> np.ndarray:
    """int8 [QB, KB]: 0 = empty, 1 = partial, 2 = full, for batch row b.

    The mask is evaluated one block row of queries at a time (only to bound
    memory); each tile's allowed in-range elements are counted."""
    QB = -(-Q_LEN // BLOCK)
    KB = -(-KV_LEN // BLOCK)
    cls = np.zeros((QB, KB), dtype=np.int8)
    for qb in range(QB):
        rows = np.arange(qb * BLOCK, min(Q_LEN, (qb + 1) * BLOCK), dtype=np.int64)
        dense = masks.dense_mask(tree, b, Q_LEN, KV_LEN, rows=rows)
        padded = np.zeros((BLOCK, KB * BLOCK), dtype=bool)
        padded[:len(rows), :KV_LEN] = dense
        counts = padded.reshape(BLOCK, KB, BLOCK).sum(axis=(0, 2), dtype=np.int64)
        cls[qb, counts > 0] = 1
        cls[qb, counts == BLOCK * BLOCK] = 2
    return cls


def create_block_mask(tree, B: int, H: int, Q_LEN: int, KV_LEN: int, BLOCK: int = 128) -> dict:
    """The four BlockMask tensors as int32 numpy arrays of shape [B, H, QB(, KB)]."""
    Bm = B if B > 0 else 1
    Hm = H if H > 0 else 1
    QB = -(-Q_LEN // BLOCK)
    KB = -(-KV_LEN // BLOCK)
    kv_num = np.zeros((Bm, Hm, QB), np.int32)
    kv_idx = np.zeros((Bm, Hm, QB, KB), np.int32)
    full_num = np.zeros((Bm, Hm, QB), np.int32)
    full_idx = np.zeros((Bm, Hm, QB, KB), np.int32)
    for b in range(Bm):
        cls = tile_classes(tree, b, Q_LEN, KV_LEN, BLOCK)
        for qb in range(QB):
            part = np.nonzero(cls[qb] == 1)[0]
            full = np.nonzero(cls[qb] == 2)[0]
            kv_num[b, :, qb] = len(part)
            full_num[b, :, qb] = len(full)
            kv_idx[b, :, qb, :len(part)] = part
            full_idx[b, :, qb, :len(full)] = full
    return {
        "kv_num_blocks": kv_num,
        "kv_indices": kv_idx,
        "full_kv_num_blocks": full_num,
        "full_kv_indices": full_idx,
    }


def to_dense(bm: dict) -> np.ndarray:
    """Block-level dense map [B, H, QB, KB] using the reconstruction loop of the
    tensorplay.nn.attention page (BlockMask "Basics"), applied to both the
    partial and the full lists."""
    kv_num, kv_idx = bm["kv_num_blocks"], bm["kv_indices"]
    full_num, full_idx = bm["full_kv_num_blocks"], bm["full_kv_indices"]
    Bm, Hm, QB, KB = kv_idx.shape
    dense = np.zeros((Bm, Hm, QB, KB), np.int32)
    for b in range(Bm):
        for h in range(Hm):
            for row in range(QB):
                for j in range(kv_num[b, h, row]):
                    dense[b, h, row, kv_idx[b, h, row, j]] = 1
                for j in range(full_num[b, h, row]):
                    dense[b, h, row, full_idx[b, h, row, j]] = 1
    return dense


def sparsity(bm: dict) -> float:
    """Percentage of blocks not computed (tensorplay.nn.attention page, BlockMask.sparsity)."""
    total = bm["kv_indices"].size
    computed = int(bm["kv_num_blocks"].sum()) + int(bm["full_kv_num_blocks"].sum())
    return 100.0 * (1.0 - computed / total)


def q_side(bm: dict) -> dict:
    """The q-side lists of a BlockMask (tensorplay.nn.attention page, BlockMask
    "Details" items 3 and 4): for every kv block, the q blocks whose partial
    list (item 3: q_num_blocks, q_indices) or full list (item 4:
    full_q_num_blocks, full_q_indices) holds it. The page calls them the
    transpose of items 1 and 2. Lists are ascending; entries after the count
    are 0; the shapes are [B, H, KB] and [B, H, KB, QB]."""
    out = {}
    for src_num, src_idx, dst_num, dst_idx in (("kv_num_blocks", "kv_indices", "q_num_blocks", "q_indices"),
                                               ("full_kv_num_blocks", "full_kv_indices", "full_q_num_blocks",
                                                "full_q_indices")):
        num, idx = bm[src_num], bm[src_idx]
        Bm, Hm, QB, KB = idx.shape
        cols = [[[[] for _ in range(KB)] for _ in range(Hm)] for _ in range(Bm)]
        for b in range(Bm):
            for h in range(Hm):
                for qb in range(QB):
                    for j in range(num[b, h, qb]):
                        cols[b][h][idx[b, h, qb, j]].append(qb)
        q_num = np.zeros((Bm, Hm, KB), np.int32)
        q_idx = np.zeros((Bm, Hm, KB, QB), np.int32)
        for b in range(Bm):
            for h in range(Hm):
                for kb in range(KB):
                    lst = sorted(cols[b][h][kb])
                    q_num[b, h, kb] = len(lst)
                    q_idx[b, h, kb, :len(lst)] = lst
        out[dst_num] = q_num
        out[dst_idx] = q_idx
    return out
