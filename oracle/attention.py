"""Block-sparse masked attention forward in fp64 (test infrastructure only).

This is the plain definition of what the block-sparse kernel computes. The
kernel reaches the same result faster by skipping tiles in which every
element is masked. Those tiles add nothing to the softmax, so skipping them
does not change the mathematics.

Passages followed:

* Attention is softmax(scale * Q K^T) V, computed without ever writing the
  full matrix (L-GATr page, "Why care about Attention Kernels?"). The oracle
  does write the full matrix, because it only has to be obviously correct.
* score_mod "changes the value of a score before the softmax" (attention-gym
  page, "A gallery that grew into a toolkit"). It receives the scaled score.
* mask_mod says which positions may attend. Masked scores are set to -inf
  (tensorplay.nn.attention page, create_block_mask).
* Layouts are q [B, Hq, M, D] and k/v [B, Hkv, N, D]. With MQA/GQA, query
  head hq reads kv head hq // (Hq / Hkv) (FlagAttention page, "Operator
  overview"; transformerlab page, _maybe_repeat_kv).
* ALiBi adds m_h * (j - i) for key j and query i (transformerlab page,
  "alibi" row). h is the query head and the default slopes are
  m_h = 2^(-8(h+1)/Hq).
* tanh soft-capping s -> cap * tanh(s / cap) is named on the L-GATr page
  ("Why care about Attention Kernels?").
* A row with no allowed key has output 0 and lse = -inf. lse is the natural
  log-sum-exp of the modified, masked scores.

Steps per (b, hq), applied to a chunk of query rows at a time:
1. Upcast to fp64 (bf16 -> fp64 is exact).
2. S = scale * Q K^T.
3. Apply the score mods in order.
4. Set S to -inf where the mask is False.
5. Take the row softmax, multiply by V and compute lse.
"""
from __future__ import annotations

import math

import numpy as np

from . import masks


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor
        import torch
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def default_alibi_slopes(Hq: int) -> np.ndarray:
    return np.asarray([2.0 ** (-8.0 * (h + 1) / Hq) for h in range(Hq)], dtype=np.float64)


def apply_score_mods(S: np.ndarray, score_mods, hq: int, Hq: int,
                     q_idx: np.ndarray, kv_idx: np.ndarray) -> np.ndarray:
    for mod in score_mods or ():
        kind = mod[0]
        if kind == "softcap":
            cap = float(mod[1])
            S = cap * np.tanh(S / cap)
        elif kind == "alibi":
            slopes = mod[1]
            slopes = default_alibi_slopes(Hq) if slopes is None else np.asarray(slopes, np.float64)
            S = S + slopes[hq] * (kv_idx[None, :].astype(np.float64) - q_idx[:, None].astype(np.float64))
        else:
            raise ValueError(f"unknown score_mod {kind!r}")
    return S


def attend_rows(q_rows: np.ndarray, K: np.ndarray, V: np.ndarray, *, b: int, hq: int, Hq: int,
                q_idx: np.ndarray, mask, score_mods, scale: float):
    """out [R, D] and lse [R] for query rows ``q_idx`` of (b, hq). All inputs are fp64."""
    N = K.shape[0]
    kv_idx = np.arange(N, dtype=np.int64)
    S = scale * (q_rows @ K.T)
    S = apply_score_mods(S, score_mods, hq, Hq, q_idx, kv_idx)
    allowed = masks.dense_mask(mask, b, int(q_idx.max()) + 1 if len(q_idx) else 0, N, rows=q_idx)
    S = np.where(allowed, S, -np.inf)
    any_allowed = allowed.any(axis=1)
    mx = np.where(any_allowed, np.max(S, axis=1), 0.0)
    P = np.exp(S - mx[:, None])            # exp(-inf) = 0 for masked entries
    l = P.sum(axis=1)
    out = np.zeros((len(q_idx), V.shape[1]), np.float64)
    out[any_allowed] = (P[any_allowed] @ V) / l[any_allowed, None]
    lse = np.full(len(q_idx), -np.inf)
    lse[any_allowed] = mx[any_allowed] + np.log(l[any_allowed])
    return out, lse


def resolve_scale(scale, D: int) -> float:
    """The fp32 softmax scale that a caller passes: a value <= 0 or None means 1/sqrt(D)."""
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(D)
    return float(np.float32(scale))


def flex_attention(q, k, v, mask=None, score_mods=(), scale=None, enable_gqa=False,
                   row_chunk: int = 1024):
    """(out [B,Hq,M,D], lse [B,Hq,M]) in fp64 for every (b, hq, query row)."""
    Q, K, V = _f64(q), _f64(k), _f64(v)
    B, Hq, M, D = Q.shape
    Hkv = K.shape[1]
    if Hq != Hkv and not enable_gqa:
        raise ValueError("Hq != Hkv requires enable_gqa")
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    group = Hq // Hkv
    sc = resolve_scale(scale, D)
    out = np.zeros((B, Hq, M, V.shape[-1]), np.float64)
    lse = np.zeros((B, Hq, M), np.float64)
    for b in range(B):
        for hq in range(Hq):
            hkv = hq // group
            for r0 in range(0, M, row_chunk):
                rows = np.arange(r0, min(M, r0 + row_chunk), dtype=np.int64)
                o, s = attend_rows(Q[b, hq, rows], K[b, hkv], V[b, hkv], b=b, hq=hq, Hq=Hq,
                                   q_idx=rows, mask=mask, score_mods=score_mods, scale=sc)
                out[b, hq, rows] = o
                lse[b, hq, rows] = s
    return out, lse


def flex_attention_sampled(q, k, v, samples, mask=None, score_mods=(), scale=None,
                           enable_gqa=False):
    """Outputs for selected (b, hq, q_idx) triples only: (out [S, D], lse [S])."""
    B, Hq, M, D = q.shape
    Hkv = k.shape[1]
    group = Hq // Hkv
    sc = resolve_scale(scale, D)
    outs = np.zeros((len(samples), v.shape[-1]), np.float64)
    lses = np.zeros(len(samples), np.float64)
    by_head: dict = {}
    for i, (b, hq, qi) in enumerate(samples):
        by_head.setdefault((int(b), int(hq)), []).append((i, int(qi)))
    for (b, hq), items in by_head.items():
        hkv = hq // group
        K = _f64(k[b, hkv])
        V = _f64(v[b, hkv])
        rows = np.asarray([qi for _, qi in items], np.int64)
        Qr = _f64(q[b, hq, rows])
        o, s = attend_rows(Qr, K, V, b=b, hq=hq, Hq=Hq, q_idx=rows, mask=mask,
                           score_mods=score_mods, scale=sc)
        for j, (i, _) in enumerate(items):
            outs[i] = o[j]
            lses[i] = s[j]
    return outs, lses


def flex_attention_varlen(q, k, v, cu_q, cu_k, causal=False, score_mods=(), scale=None, enable_gqa=False):
    """Attention over packed variable-length sequences (L-GATr "attention
    backends" page: packed events attend within their own event; the varlen
    kernels' cu_seqlens form). q [total_q, Hq, D], k/v [total_k, Hkv, D];
    sequence i holds q tokens cu_q[i]:cu_q[i+1] and k tokens cu_k[i]:cu_k[i+1].
    Each sequence is plain attention of its own tokens, computed by
    flex_attention on a [1, H, L, D] view, causal (kv <= q, positions within
    the sequence) when asked. Tokens past the last sequence attend to nothing.
    Returns (out [total_q, Hq, D], lse [Hq, total_q])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    cu_q = [int(x) for x in cu_q]
    cu_k = [int(x) for x in cu_k]
    Mt, Hq, D = q.shape
    out = np.zeros((Mt, Hq, v.shape[2]), np.float64)
    lse = np.full((Hq, Mt), -np.inf, np.float64)
    for i in range(len(cu_q) - 1):
        q0, q1, k0, k1 = cu_q[i], cu_q[i + 1], cu_k[i], cu_k[i + 1]
        if q1 <= q0:
            continue
        qs = q[q0:q1].transpose(1, 0, 2)[None]
        ks = k[k0:k1].transpose(1, 0, 2)[None]
        vs = v[k0:k1].transpose(1, 0, 2)[None]
        tree = ("causal",) if causal else None
        o, l = flex_attention(qs, ks, vs, tree, score_mods, scale, enable_gqa)
        out[q0:q1] = o[0].transpose(1, 0, 2)
        lse[:, q0:q1] = l[0]
    return out, lse
