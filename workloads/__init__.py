"""Seeded synthetic workloads for block-sparse masked attention.

This module is shared by the oracle side and the CUDA side, so it holds no
attention or masking arithmetic. It only describes each workload as data and
draws the random inputs.

* A mask is a nested tuple tree:
  ``("noop",)``, ``("causal",)``, ``("window", W)``, ``("prefix_lm", P)``,
  ``("sink", S)``, ``("document", q_doc_ids, kv_doc_ids)`` (int32 arrays of
  shape [B, Q_LEN] and [B, KV_LEN]), ``("and", m1, m2, ...)`` and
  ``("or", m1, m2, ...)``.
* A score modifier is a list of ``("softcap", cap)`` and
  ``("alibi", slopes)`` entries, applied in list order. ``slopes`` is a
  float32 array [Hq], or None for the default geometric slopes.

The five workloads are the shapes the pages' examples use:

* the causal block-mask example (tensorplay.nn.attention page,
  create_block_mask "Example Usage");
* sliding window with soft-capping (L-GATr "attention backends" page,
  "Why care about Attention Kernels?");
* ALiBi (transformerlab page, attention registry table);
* packed documents with a block-diagonal mask (L-GATr page, block-diagonal
  xformers mask over concatenated events);
* the StreamingLLM sink + window pattern (transformerlab page, "sink" row).

Inputs are drawn as follows:

* Every q/k/v draw uses ``torch.Generator('cpu').manual_seed(seed)`` with
  seed = 1000 + workload index (1-based).
* q, then k, then v are drawn as float32 N(0, 1) and rounded to bfloat16.
* Document lengths come from ``numpy.random.default_rng(seed)``. They are
  uniform in [128, 4096] and drawn until the total reaches the packed
  length; the last document is truncated to fit.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Any

import numpy as np
import torch

BLOCK_SIZE = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int          # 1-based position in the workload list
    B: int
    Hq: int
    Hkv: int
    M: int              # Q_LEN
    N: int              # KV_LEN
    D: int
    mask: str           # symbolic mask kind, resolved by mask_tree()
    window: int = 0
    sink: int = 0
    softcap: float = 0.0
    alibi: bool = False

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def enable_gqa(self) -> bool:
        return self.Hq != self.Hkv


WORKLOADS = [
    Workload("causal_b1_h2_s256_d64", 1, 1, 2, 2, 256, 256, 64, "causal"),
    Workload("swa512_softcap30_b4_hq16_hkv4_s2048_d128", 2, 4, 16, 4, 2048, 2048, 128,
             "causal_window", window=512, softcap=30.0),
    Workload("causal_alibi_b8_h16_s4096_d64", 3, 8, 16, 16, 4096, 4096, 64, "causal",
             alibi=True),
    Workload("doc_causal_b1_h32_s16384_d128", 4, 1, 32, 32, 16384, 16384, 128,
             "doc_causal"),
    Workload("streaming_sink4_win1024_b2_hq32_hkv8_s32768_d128", 5, 2, 32, 8, 32768, 32768,
             128, "streaming", window=1024, sink=4),
]

BY_NAME = {w.name: w for w in WORKLOADS}


def get(index_or_name) -> Workload:
    if isinstance(index_or_name, int):
        return WORKLOADS[index_or_name - 1]
    return BY_NAME[index_or_name]


def document_lengths(total: int, seed: int, lo: int = 128, hi: int = 4096) -> list[int]:
    """Document lengths uniform in [lo, hi], drawn until they cover ``total``."""
    rng = np.random.default_rng(seed)
    lengths: list[int] = []
    covered = 0
    while covered < total:
        n = int(rng.integers(lo, hi + 1))
        n = min(n, total - covered)
        lengths.append(n)
        covered += n
    return lengths


def document_ids(lengths: list[int]) -> np.ndarray:
    """Per-position document ordinal for contiguous (packed) documents."""
    return np.repeat(np.arange(len(lengths), dtype=np.int32),
                     np.asarray(lengths, dtype=np.int64)).astype(np.int32)


def alibi_slopes(Hq: int) -> np.ndarray:
    """Slopes m_h = 2^(-8(h+1)/Hq) as float32. These are input data for the workload."""
    return np.asarray([2.0 ** (-8.0 * (h + 1) / Hq) for h in range(Hq)], dtype=np.float32)


def mask_tree(w: Workload, doc_ids: np.ndarray | None = None) -> tuple:
    if w.mask == "causal":
        return ("causal",)
    if w.mask == "causal_window":
        return ("and", ("causal",), ("window", w.window))
    if w.mask == "streaming":
        return ("and", ("causal",), ("or", ("sink", w.sink), ("window", w.window)))
    if w.mask == "doc_causal":
        assert doc_ids is not None
        ids = np.broadcast_to(doc_ids, (w.B, w.M)).astype(np.int32).copy()
        return ("and", ("document", ids, ids), ("causal",))
    raise ValueError(w.mask)


def score_mods(w: Workload) -> list:
    mods: list[Any] = []
    if w.softcap:
        mods.append(("softcap", float(w.softcap)))
    if w.alibi:
        mods.append(("alibi", alibi_slopes(w.Hq)))
    return mods


def qkv(w: Workload, seed_offset: int = 0, shapes: tuple | None = None):
    """q [B,Hq,M,D], k/v [B,Hkv,N,D] as contiguous bfloat16 CPU tensors."""
    g = torch.Generator("cpu").manual_seed(w.seed + seed_offset)
    qs = (w.B, w.Hq, w.M, w.D)
    ks = (w.B, w.Hkv, w.N, w.D)
    if shapes is not None:
        qs, ks = shapes
    q = torch.randn(qs, generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn(ks, generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn(ks, generator=g, dtype=torch.float32).to(torch.bfloat16)
    return q, k, v


def make(w: Workload, seed_offset: int = 0) -> dict:
    """Everything one run of workload ``w`` needs, on the CPU."""
    doc = None
    lengths = None
    if w.mask == "doc_causal":
        lengths = document_lengths(w.M, w.seed + seed_offset)
        doc = document_ids(lengths)
    q, k, v = qkv(w, seed_offset)
    return {
        "workload": w,
        "q": q, "k": k, "v": v,
        "mask": mask_tree(w, doc),
        "score_mods": score_mods(w),
        "scale": w.scale,
        "doc_lengths": lengths,
    }


def random_inputs(seed: int, B: int, Hq: int, Hkv: int, M: int, N: int, D: int):
    """Small fuzz-case q/k/v from one seed (same draw order as ``qkv``)."""
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn((B, Hq, M, D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn((B, Hkv, N, D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn((B, Hkv, N, D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    return q, k, v


def random_mask_tree(rng: np.random.Generator, B: int, M: int, N: int, depth: int = 2,
                     allow_document: bool = True) -> tuple:
    """A random composable mask tree over the primitive set (fuzz data only).

    All document leaves of one tree share one packing (one pair of id arrays),
    as a single sequence packing has one set of document boundaries."""
    L = max(M, N)
    docs = None
    if allow_document and L >= 2:
        cuts = np.sort(rng.choice(np.arange(1, L), size=min(3, L - 1), replace=False))
        ids = np.searchsorted(cuts, np.arange(L), side="right").astype(np.int32)
        docs = (np.broadcast_to(ids[:M], (B, M)).copy(), np.broadcast_to(ids[:N], (B, N)).copy())

    def leaf():
        kinds = ["noop", "causal", "window", "prefix_lm", "sink"]
        if docs is not None:
            kinds.append("document")
        kind = kinds[int(rng.integers(len(kinds)))]
        if kind in ("noop", "causal"):
            return (kind,)
        if kind == "window":
            return ("window", int(rng.integers(1, max(2, N))))
        if kind == "prefix_lm":
            return ("prefix_lm", int(rng.integers(0, N + 1)))
        if kind == "sink":
            return ("sink", int(rng.integers(0, max(1, N // 2))))
        return ("document", docs[0], docs[1])

    def node(d):
        if d == 0 or rng.random() < 0.3:
            return leaf()
        op = "and" if rng.random() < 0.5 else "or"
        n = int(rng.integers(2, 4))
        return (op,) + tuple(node(d - 1) for _ in range(n))

    return node(depth)


def grad_output(seed: int, B: int, Hq: int, M: int, D: int) -> torch.Tensor:
    """The gradient arriving at out for backward cases: float32 N(0, 1) rounded
    to bfloat16, [B, Hq, M, D], from its own seeded generator."""
    g = torch.Generator("cpu").manual_seed(seed)
    return torch.randn((B, Hq, M, D), generator=g, dtype=torch.float32).to(torch.bfloat16)
