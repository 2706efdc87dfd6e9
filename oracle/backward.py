"""Block-sparse masked attention backward in fp64 (test infrastructure only).

This is the plain definition of the gradients the block-sparse backward
kernels compute: with out the forward of ``oracle.attention`` and dout the
gradient arriving at out, dq, dk and dv are the gradients of the scalar
sum(out * dout) with respect to q, k and v. Tiles in which every element
is masked have P = 0 there and add nothing, so the kernels may skip them.

Passages followed:

* The FlagAttention page ("Operator overview") lists forward and backward
  for dense FlashAttention with q [B, Hq, M, D], k/v [B, Hkv, N, D] and
  MQA/GQA, and says that the kernels recompute intermediates instead of
  storing the attention matrix. The oracle stores it; it only has to be
  obviously correct.
* The tensorplay.nn.attention page, BlockMask "Details" items 3-4: the
  backward computes dK and dV by walking the mask along the query dimension
  (q_num_blocks / q_indices and their full counterparts).
* The forward (``oracle.attention``) fixes the rest: scale before score_mod,
  score_mod on every element, masked scores at -inf, rows with no allowed key
  give out = 0. Such a row passes no gradient anywhere.

Steps per (b, hq), for a chunk of query rows at a time, all in fp64:
1. S = scale * Q K^T; Z = score_mods(S) with the elementwise derivative
   dZ/dS (soft-cap: 1 - tanh^2(s / cap); ALiBi adds a constant: 1).
2. Masked Z = -inf; P = row softmax of Z (all-zero rows stay zero).
3. dV[hkv] += P^T dO and dP = dO V^T.
4. delta = rowsum(P * dP); dZ = P * (dP - delta); dS = dZ * dZ/dS.
5. dQ = scale * dS K and dK[hkv] += scale * dS^T Q.
With GQA, kv head hkv collects the gradients of every query head of its
group.
"""
from __future__ import annotations

import numpy as np

from . import masks
from .attention import _f64, default_alibi_slopes, resolve_scale


def score_mods_with_grad(S: np.ndarray, score_mods, hq: int, Hq: int, q_idx: np.ndarray,
                         kv_idx: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """(Z, dZ/dS) for the score mods applied in order to the scaled scores S."""
    Z = S
    dZ = np.ones_like(S)
    for mod in score_mods or ():
        kind = mod[0]
        if kind == "softcap":
            cap = float(mod[1])
            t = np.tanh(Z / cap)
            dZ = dZ * (1.0 - t * t)
            Z = cap * t
        elif kind == "alibi":
            slopes = mod[1]
            slopes = default_alibi_slopes(Hq) if slopes is None else np.asarray(slopes, np.float64)
            Z = Z + slopes[hq] * (kv_idx[None, :].astype(np.float64) - q_idx[:, None].astype(np.float64))
        else:
            raise ValueError(f"unknown score_mod {kind!r}")
    return Z, dZ


def backward_rows(q_rows: np.ndarray, do_rows: np.ndarray, K: np.ndarray, V: np.ndarray, *, b: int, hq: int,
                  Hq: int, q_idx: np.ndarray, mask, score_mods, scale: float):
    """Gradients from query rows ``q_idx`` of (b, hq): (dq [R, D], dk [N, D],
    dv [N, D]); dk and dv are this chunk's share of the kv head's gradient."""
    N = K.shape[0]
    kv_idx = np.arange(N, dtype=np.int64)
    S = scale * (q_rows @ K.T)
    Z, dZdS = score_mods_with_grad(S, score_mods, hq, Hq, q_idx, kv_idx)
    allowed = masks.dense_mask(mask, b, int(q_idx.max()) + 1 if len(q_idx) else 0, N, rows=q_idx)
    Z = np.where(allowed, Z, -np.inf)
    any_allowed = allowed.any(axis=1)
    mx = np.where(any_allowed, np.max(Z, axis=1), 0.0)
    E = np.exp(Z - mx[:, None])
    l = E.sum(axis=1)
    P = np.zeros_like(E)
    P[any_allowed] = E[any_allowed] / l[any_allowed, None]
    dv = P.T @ do_rows
    dP = do_rows @ V.T
    delta = np.sum(P * dP, axis=1)
    dS = P * (dP - delta[:, None]) * dZdS
    dq = scale * (dS @ K)
    dk = scale * (dS.T @ q_rows)
    return dq, dk, dv


def flex_attention_backward(q, k, v, dout, mask=None, score_mods=(), scale=None, enable_gqa=False,
                            row_chunk: int = 1024):
    """(dq [B,Hq,M,D], dk [B,Hkv,N,D], dv [B,Hkv,N,D]) in fp64."""
    Q, K, V, dO = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Hq, M, D = Q.shape
    Hkv = K.shape[1]
    if Hq != Hkv and not enable_gqa:
        raise ValueError("Hq != Hkv requires enable_gqa")
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    group = Hq // Hkv
    sc = resolve_scale(scale, D)
    dq = np.zeros_like(Q)
    dk = np.zeros_like(K)
    dv = np.zeros_like(V)
    for b in range(B):
        for hq in range(Hq):
            hkv = hq // group
            for r0 in range(0, M, row_chunk):
                rows = np.arange(r0, min(M, r0 + row_chunk), dtype=np.int64)
                gq, gk, gv = backward_rows(Q[b, hq, rows], dO[b, hq, rows], K[b, hkv], V[b, hkv], b=b, hq=hq,
                                           Hq=Hq, q_idx=rows, mask=mask, score_mods=score_mods, scale=sc)
                dq[b, hq, rows] = gq
                dk[b, hkv] += gk
                dv[b, hkv] += gv
    return dq, dk, dv


def backward_dq_sampled(q, k, v, dout, samples, mask=None, score_mods=(), scale=None):
    """dq rows for selected (b, hq, q_idx) triples: [S, D]. A query row's dq
    needs only its own row of P, so each sample costs O(N * D)."""
    B, Hq, M, D = q.shape
    group = Hq // k.shape[1]
    sc = resolve_scale(scale, D)
    out = np.zeros((len(samples), D), np.float64)
    for i, (b, hq, qi) in enumerate(samples):
        b, hq, qi = int(b), int(hq), int(qi)
        hkv = hq // group
        rows = np.asarray([qi], np.int64)
        gq, _, _ = backward_rows(_f64(q[b, hq, rows]), _f64(dout[b, hq, rows]), _f64(k[b, hkv]), _f64(v[b, hkv]),
                                 b=b, hq=hq, Hq=Hq, q_idx=rows, mask=mask, score_mods=score_mods, scale=sc)
        out[i] = gq[0]
    return out


def backward_dkv_sampled(q, k, v, dout, samples, mask=None, score_mods=(), scale=None, row_chunk: int = 1024):
    """(dk rows [S, D], dv rows [S, D]) for selected (b, hkv, kv_idx) triples.
    Only query rows whose mask allows kv_idx contribute; each needs its whole
    row of P, so a sample costs O(rows attending * N * D) per query head of
    the group."""
    B, Hq, M, D = q.shape
    Hkv = k.shape[1]
    group = Hq // Hkv
    sc = resolve_scale(scale, D)
    dks = np.zeros((len(samples), D), np.float64)
    dvs = np.zeros((len(samples), D), np.float64)
    for i, (b, hkv, j) in enumerate(samples):
        b, hkv, j = int(b), int(hkv), int(j)
        col = masks.evaluate(mask, b, np.arange(M, dtype=np.int64), np.int64(j)) if mask is not None \
            else np.ones(M, dtype=bool)
        rows_all = np.nonzero(col)[0].astype(np.int64)
        Kh, Vh = _f64(k[b, hkv]), _f64(v[b, hkv])
        for hq in range(hkv * group, (hkv + 1) * group):
            for r0 in range(0, len(rows_all), row_chunk):
                rows = rows_all[r0:r0 + row_chunk]
                _, gk, gv = backward_rows(_f64(q[b, hq, rows]), _f64(dout[b, hq, rows]), Kh, Vh, b=b, hq=hq,
                                          Hq=Hq, q_idx=rows, mask=mask, score_mods=score_mods, scale=sc)
                dks[i] += gk[j]
                dvs[i] += gv[j]
    return dks, dvs


def flex_attention_varlen_backward(q, k, v, dout, cu_q, cu_k, causal=False, score_mods=(), scale=None,
                                   enable_gqa=False):
    """Gradients (dq [total_q, Hq, D], dk, dv [total_k, Hkv, D]) of
    sum(out * dout) for the packed variable-length attention of
    ``oracle.attention.flex_attention_varlen``. Each sequence is an
    independent plain attention, so its gradients are flex_attention_backward
    of its own tokens on a [1, H, L, D] view; tokens outside every sequence
    get zero gradients."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    cu_q = [int(x) for x in cu_q]
    cu_k = [int(x) for x in cu_k]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for i in range(len(cu_q) - 1):
        q0, q1, k0, k1 = cu_q[i], cu_q[i + 1], cu_k[i], cu_k[i + 1]
        if q1 <= q0 or k1 <= k0:
            continue
        view = lambda x, a, b: x[a:b].transpose(1, 0, 2)[None]  # noqa: E731
        gq, gk, gv = flex_attention_backward(view(q, q0, q1), view(k, k0, k1), view(v, k0, k1),
                                             view(dout, q0, q1), ("causal",) if causal else None, score_mods,
                                             scale, enable_gqa)
        dq[q0:q1] = gq[0].transpose(1, 0, 2)
        dk[k0:k1] = gk[0].transpose(1, 0, 2)
        dv[k0:k1] = gv[0].transpose(1, 0, 2)
    return dq, dk, dv
