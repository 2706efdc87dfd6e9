"""Dense boolean mask_mod evaluation in the oracle (test infrastructure only).

A mask_mod(b, h, q_idx, kv_idx) returns True where attention is allowed
(tensorplay.nn.attention page, create_block_mask, parameter "mask_mod").
None of the primitives here depends on the head h, so the dense mask of one
batch row is shared by every head.

Primitives:

* noop: always True (tensorplay.nn.attention page, noop_mask).
* causal: q_idx >= kv_idx (same page, create_block_mask "Example Usage").
* window(W): q_idx - kv_idx < W. The sliding window is named on the L-GATr
  page ("Why care about Attention Kernels?") and the transformerlab page
  ("local" and "local_flex" rows); the strict "<" follows the StreamingLLM
  workload's own statement of the window.
* prefix_lm(P): kv_idx < P or q_idx >= kv_idx (PrefixLM, L-GATr page, same
  section).
* sink(S): kv_idx < S (StreamingLLM "first-k sink tokens", transformerlab
  page, registry table).
* document(q_doc, kv_doc): q_doc[b, q_idx] == kv_doc[b, kv_idx]. This is the
  block-diagonal mask over concatenated events (L-GATr page, same section).

Combinators: ``and`` is the intersection of its children and ``or`` is the
union (tensorplay.nn.attention page, and_masks and or_masks).
"""
from __future__ import annotations

import numpy as np


def _doc_row(ids, b: int) -> np.ndarray:
    ids = np.asarray(ids)
    if ids.ndim == 1:
        return ids
    return ids[b if ids.shape[0] > 1 else 0]


def evaluate(tree, b: int, q_idx: np.ndarray, kv_idx: np.ndarray) -> np.ndarray:
    """Evaluate ``tree`` at broadcastable integer index arrays for batch b."""
    kind = tree[0]
    shape = np.broadcast_shapes(np.shape(q_idx), np.shape(kv_idx))
    if kind == "noop":
        return np.ones(shape, dtype=bool)
    if kind == "causal":
        return np.broadcast_to(q_idx >= kv_idx, shape)
    if kind == "window":
        return np.broadcast_to((q_idx - kv_idx) < int(tree[1]), shape)
    if kind == "prefix_lm":
        return np.broadcast_to((kv_idx < int(tree[1])) | (q_idx >= kv_idx), shape)
    if kind == "sink":
        return np.broadcast_to(kv_idx < int(tree[1]), shape)
    if kind == "document":
        qd = _doc_row(tree[1], b)
        kd = _doc_row(tree[2], b)
        return np.broadcast_to(qd[q_idx] == kd[kv_idx], shape)
    if kind == "and":
        out = np.ones(shape, dtype=bool)
        for child in tree[1:]:
            out = out & evaluate(child, b, q_idx, kv_idx)
        return out
    if kind == "or":
        out = np.zeros(shape, dtype=bool)
        for child in tree[1:]:
            out = out | evaluate(child, b, q_idx, kv_idx)
        return out
    raise ValueError(f"unknown mask kind {kind!r}")


def dense_mask(tree, b: int, Q_LEN: int, KV_LEN: int, rows=None) -> np.ndarray:
    """bool [len(rows), KV_LEN]: the mask of batch b (rows default to all of Q_LEN)."""
    if tree is None:
        tree = ("noop",)
    q_idx = np.arange(Q_LEN, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    kv_idx = np.arange(KV_LEN, dtype=np.int64)
    return np.array(evaluate(tree, b, q_idx[:, None], kv_idx[None, :]), dtype=bool)


def create_mask(tree, B: int, H: int, Q_LEN: int, KV_LEN: int) -> np.ndarray:
    """bool [B, H, Q_LEN, KV_LEN] (tensorplay.nn.attention page, create_mask)."""
    out = np.empty((B, H, Q_LEN, KV_LEN), dtype=bool)
    for b in range(B):
        out[b, :] = dense_mask(tree, b, Q_LEN, KV_LEN)[None]
    return out
