"""Block-sparse masked-tile attention for NVIDIA B200 (sm_100a).

This is a thin Python binding over the C ABI in ``include/bsmt.h``
(``libbsmt.so``). It only marshals arguments. PyTorch supplies device
memory and the current CUDA stream; every step of the computation runs in
the library's CUDA kernels. If the library is missing, importing this module
raises.

The API follows the tensorplay.nn.attention page:

* ``create_block_mask(mask_mod, B, H, Q_LEN, KV_LEN, BLOCK_SIZE=128)``
  returns a ``BlockMask`` holding kv_num_blocks/kv_indices (partial blocks)
  and full_kv_num_blocks/full_kv_indices (full blocks).
* ``flex_attention(q, k, v, block_mask, score_mod, scale, enable_gqa)``
  returns ``(out, lse)``.
* ``flex_attention_backward(q, k, v, out, lse, dout, block_mask, ...)``
  returns ``(dq, dk, dv)``, the gradients of sum(out * dout).
* Mask builders: ``noop_mask``, ``causal``, ``sliding_window``,
  ``prefix_lm``, ``sink``, ``document``, ``and_masks`` and ``or_masks``.
* Score mods: ``softcap`` and ``alibi``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field
from typing import Iterable, Sequence

import torch

__all__ = [
    "BsmtError", "MaskMod", "ScoreMod", "BlockMask", "noop_mask", "causal", "sliding_window", "prefix_lm",
    "sink", "document", "and_masks", "or_masks", "softcap", "alibi", "create_block_mask", "flex_attention",
    "check_device_status", "library_path", "mask_from_tree", "score_mods_from_list", "splitkv_workspace_bytes",
    "flex_attention_host", "host_workspace_bytes", "flex_attention_varlen", "seqlens_to_doc_ids", "flex_attention_backward",
    "backward_workspace_bytes", "flex_attention_varlen_backward",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libbsmt.so")

# ------------------------------------------------------------------ C ABI
MAX_NODES = 64
MAX_SCORE_OPS = 2
(MASK_NOOP, MASK_CAUSAL, MASK_WINDOW, MASK_PREFIX_LM, MASK_SINK, MASK_DOCUMENT, MASK_AND, MASK_OR) = range(8)
SCORE_NONE, SCORE_SOFTCAP, SCORE_ALIBI = 0, 1, 2
STATUS_NAMES = {
    0: "OK", 1: "INVALID_ARGUMENT", 2: "SHAPE_MISMATCH", 3: "UNSUPPORTED", 4: "CUDA_ERROR",
    5: "DEVICE_TIMEOUT", 6: "DEVICE_BOUNDS", 7: "DEVICE_PRECONDITION",
}


class _MaskNode(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("arg", ctypes.c_int32)]


class _MaskSpec(ctypes.Structure):
    _fields_ = [("num_nodes", ctypes.c_int32), ("nodes", _MaskNode * MAX_NODES),
                ("q_doc_ids", ctypes.c_void_p), ("kv_doc_ids", ctypes.c_void_p), ("doc_batch", ctypes.c_int32)]


class _ScoreOp(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("value", ctypes.c_float), ("slopes", ctypes.c_void_p),
                ("head_offset", ctypes.c_int32), ("num_heads", ctypes.c_int32)]


class _ScoreSpec(ctypes.Structure):
    _fields_ = [("num_ops", ctypes.c_int32), ("ops", _ScoreOp * MAX_SCORE_OPS)]


class _BlockMaskQ(ctypes.Structure):
    _fields_ = [("q_num_blocks", ctypes.c_void_p), ("q_indices", ctypes.c_void_p),
                ("full_q_num_blocks", ctypes.c_void_p), ("full_q_indices", ctypes.c_void_p)]


class _BlockMask(ctypes.Structure):
    _fields_ = [("kv_num_blocks", ctypes.c_void_p), ("kv_indices", ctypes.c_void_p),
                ("full_kv_num_blocks", ctypes.c_void_p), ("full_kv_indices", ctypes.c_void_p),
                ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("QB", ctypes.c_int32), ("KB", ctypes.c_int32),
                ("Q_LEN", ctypes.c_int32), ("KV_LEN", ctypes.c_int32),
                ("BLOCK_Q", ctypes.c_int32), ("BLOCK_KV", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_PATH} is missing: build it with `python block_sparse_masked_tile_b200/build.py` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(_LIB_PATH)
    i64, i32, vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p
    lib.bsmt_block_mask_shape.argtypes = [i64, i64, i64, i64, i32, i32, ctypes.POINTER(i64)]
    lib.bsmt_block_mask_shape.restype = i32
    lib.bsmt_create_block_mask.argtypes = [ctypes.POINTER(_MaskSpec), i64, i64, i64, i64, i32, i32,
                                           ctypes.POINTER(_BlockMask), vp]
    lib.bsmt_create_block_mask.restype = i32
    lib.bsmt_flex_attention_fwd.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, i64, ctypes.POINTER(_BlockMask),
                                            ctypes.POINTER(_MaskSpec), ctypes.POINTER(_ScoreSpec), ctypes.c_float,
                                            i32, vp, vp, vp]
    lib.bsmt_flex_attention_fwd.restype = i32
    lib.bsmt_block_mask_transpose.argtypes = [ctypes.POINTER(_BlockMask), ctypes.POINTER(_BlockMaskQ), vp]
    lib.bsmt_block_mask_transpose.restype = i32
    lib.bsmt_block_mask_to_dense.argtypes = [ctypes.POINTER(_BlockMask), vp, vp]
    lib.bsmt_block_mask_to_dense.restype = i32
    lib.bsmt_splitkv_workspace_bytes.argtypes = [i64, i64, i64, i64, i32, ctypes.POINTER(i64)]
    lib.bsmt_splitkv_workspace_bytes.restype = i32
    lib.bsmt_flex_attention_fwd_splitkv.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, i64,
                                                    ctypes.POINTER(_BlockMask), ctypes.POINTER(_MaskSpec),
                                                    ctypes.POINTER(_ScoreSpec), ctypes.c_float, i32, i32, vp, i64,
                                                    vp, vp, vp]
    lib.bsmt_flex_attention_fwd_splitkv.restype = i32
    lib.bsmt_flex_attention_fwd_splitkv_static.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, i64,
                                                           ctypes.POINTER(_BlockMask), ctypes.POINTER(_MaskSpec),
                                                           ctypes.POINTER(_ScoreSpec), ctypes.c_float, i32, i32,
                                                           vp, vp, vp]
    lib.bsmt_flex_attention_fwd_splitkv_static.restype = i32
    lib.bsmt_flex_attention_host_workspace_bytes.argtypes = [i64, i64, i64, i64, i64, i64,
                                                             ctypes.POINTER(_MaskSpec), ctypes.POINTER(i64)]
    lib.bsmt_flex_attention_host_workspace_bytes.restype = i32
    lib.bsmt_flex_attention_host.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, i64, ctypes.POINTER(_MaskSpec),
                                             ctypes.POINTER(_ScoreSpec), ctypes.c_float, i32, i32, vp, i64, vp, vp,
                                             vp]
    lib.bsmt_flex_attention_host.restype = i32
    lib.bsmt_seqlens_to_doc_ids.argtypes = [vp, i32, i64, vp, vp]
    lib.bsmt_seqlens_to_doc_ids.restype = i32
    lib.bsmt_flex_attention_fwd_packed.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, ctypes.POINTER(_BlockMask),
                                                   ctypes.POINTER(_MaskSpec), ctypes.POINTER(_ScoreSpec),
                                                   ctypes.c_float, i32, vp, vp, vp]
    lib.bsmt_flex_attention_fwd_packed.restype = i32
    lib.bsmt_flex_attention_bwd_workspace_bytes.argtypes = [i64, i64, i64, ctypes.POINTER(i64)]
    lib.bsmt_flex_attention_bwd_workspace_bytes.restype = i32
    lib.bsmt_flex_attention_bwd.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64,
                                            ctypes.POINTER(_BlockMask), ctypes.POINTER(_BlockMaskQ),
                                            ctypes.POINTER(_MaskSpec), ctypes.POINTER(_ScoreSpec), ctypes.c_float, i32,
                                            vp, vp, vp, vp, i64, vp]
    lib.bsmt_flex_attention_bwd.restype = i32
    lib.bsmt_flex_attention_bwd_packed.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64,
                                                   ctypes.POINTER(_BlockMask), ctypes.POINTER(_BlockMaskQ),
                                                   ctypes.POINTER(_MaskSpec), ctypes.POINTER(_ScoreSpec),
                                                   ctypes.c_float, i32, vp, vp, vp, vp, i64, vp]
    lib.bsmt_flex_attention_bwd_packed.restype = i32
    lib.bsmt_selftest_wait_timeout.argtypes = [vp, vp]
    lib.bsmt_selftest_wait_timeout.restype = i32
    lib.bsmt_last_error.argtypes = []
    lib.bsmt_last_error.restype = ctypes.c_char_p
    lib.bsmt_check_device_status.argtypes = [vp]
    lib.bsmt_check_device_status.restype = i32
    lib.bsmt_version.argtypes = []
    lib.bsmt_version.restype = i32
    return lib


_lib = _load()


def library_path() -> str:
    return _LIB_PATH


class BsmtError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class BsmtValueError(ValueError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def _check(status: int) -> None:
    if status == 0:
        return
    msg = _lib.bsmt_last_error().decode(errors="replace")
    if status in (1, 2):
        raise BsmtValueError(status, msg)
    raise BsmtError(status, msg)


# BSMT_DEBUG_SYNC=1: after every kernel launch, wait for the stream and raise
# any device-side status (bounds, precondition, timeout) at the call that
# caused it, instead of at the next check_device_status.
_DEBUG_SYNC = os.environ.get("BSMT_DEBUG_SYNC", "0") == "1"


def _check_launch(status: int) -> None:
    _check(status)
    if _DEBUG_SYNC:
        _check(_lib.bsmt_check_device_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)))


def _stream_ptr(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


# ------------------------------------------------------------------ masks
@dataclass(frozen=True)
class MaskMod:
    """A composable mask_mod, stored as a postfix program of ABI nodes."""
    nodes: tuple = ()
    q_doc_ids: torch.Tensor | None = field(default=None, compare=False)
    kv_doc_ids: torch.Tensor | None = field(default=None, compare=False)

    def _spec(self, device: torch.device, B: int) -> tuple[_MaskSpec, list]:
        if len(self.nodes) > MAX_NODES:
            raise ValueError(f"mask program has {len(self.nodes)} nodes (at most {MAX_NODES})")
        spec = _MaskSpec()
        spec.num_nodes = len(self.nodes)
        for i, (kind, arg) in enumerate(self.nodes):
            spec.nodes[i].kind = kind
            spec.nodes[i].arg = arg
        keep = []
        if self.q_doc_ids is not None:
            qd = self.q_doc_ids.to(device=device, dtype=torch.int32).contiguous()
            kd = self.kv_doc_ids.to(device=device, dtype=torch.int32).contiguous()
            if qd.dim() == 1:
                qd = qd[None]
            if kd.dim() == 1:
                kd = kd[None]
            if qd.shape[0] != kd.shape[0]:
                raise ValueError("q_doc_ids and kv_doc_ids need the same batch extent")
            keep += [qd, kd]
            spec.q_doc_ids = qd.data_ptr()
            spec.kv_doc_ids = kd.data_ptr()
            spec.doc_batch = qd.shape[0]
        else:
            spec.doc_batch = 1
        return spec, keep


def _leaf(kind: int, arg: int = 0) -> MaskMod:
    return MaskMod(((kind, int(arg)),))


def noop_mask() -> MaskMod:
    return _leaf(MASK_NOOP)


def causal() -> MaskMod:
    return _leaf(MASK_CAUSAL)


_causal_mask = causal  # (flex_attention_varlen's causal flag shadows the name)


def sliding_window(window: int) -> MaskMod:
    """q_idx - kv_idx < window (combine with causal() for a causal band)."""
    return _leaf(MASK_WINDOW, window)


def prefix_lm(prefix: int) -> MaskMod:
    return _leaf(MASK_PREFIX_LM, prefix)


def sink(num_sink: int) -> MaskMod:
    return _leaf(MASK_SINK, num_sink)


def document(q_doc_ids: torch.Tensor, kv_doc_ids: torch.Tensor | None = None) -> MaskMod:
    """q_doc_ids[b, q_idx] == kv_doc_ids[b, kv_idx]; kv ids must be non-decreasing (packed documents)."""
    if kv_doc_ids is None:
        kv_doc_ids = q_doc_ids
    return MaskMod(((MASK_DOCUMENT, 0),), q_doc_ids, kv_doc_ids)


def _combine(op: int, mods: Sequence[MaskMod]) -> MaskMod:
    if not mods:
        raise ValueError("and_masks/or_masks need at least one mask")
    docs = [m for m in mods if m.q_doc_ids is not None]
    for m in docs[1:]:
        if m.q_doc_ids is not docs[0].q_doc_ids or m.kv_doc_ids is not docs[0].kv_doc_ids:
            raise ValueError("all document() masks in one program must share the same id tensors")
    nodes: list = []
    for m in mods:
        nodes.extend(m.nodes)
    nodes.append((op, len(mods)))
    d = docs[0] if docs else None
    return MaskMod(tuple(nodes), d.q_doc_ids if d else None, d.kv_doc_ids if d else None)


def and_masks(*mods: MaskMod) -> MaskMod:
    """Intersection of the given masks (tensorplay.nn.attention, and_masks)."""
    return _combine(MASK_AND, mods)


def or_masks(*mods: MaskMod) -> MaskMod:
    """Union of the given masks (tensorplay.nn.attention, or_masks)."""
    return _combine(MASK_OR, mods)


def mask_from_tree(tree, device=None, _cache=None) -> MaskMod:
    """Convert a nested tuple mask description (see ``workloads``) into a MaskMod.
    Document id arrays are placed on ``device`` when it is given. One program
    carries one (q, kv) document id pair: document leaves over different arrays
    raise ValueError."""
    if _cache is None:
        _cache = {}
    if tree is None:
        return noop_mask()
    kind = tree[0]
    if kind == "noop":
        return noop_mask()
    if kind == "causal":
        return causal()
    if kind == "window":
        return sliding_window(tree[1])
    if kind == "prefix_lm":
        return prefix_lm(tree[1])
    if kind == "sink":
        return sink(tree[1])
    if kind == "document":
        key = (id(tree[1]), id(tree[2]))
        if key not in _cache:
            qd = torch.as_tensor(tree[1], dtype=torch.int32)
            kd = qd if tree[2] is tree[1] else torch.as_tensor(tree[2], dtype=torch.int32)
            if device is not None:
                qd = qd.to(device)
                kd = qd if tree[2] is tree[1] else kd.to(device)
            _cache[key] = (qd, kd, tree[1], tree[2])  # the arrays stay referenced while cached
        qd, kd = _cache[key][:2]
        return document(qd, kd)
    if kind in ("and", "or"):
        children = [mask_from_tree(c, device, _cache) for c in tree[1:]]
        return (and_masks if kind == "and" else or_masks)(*children)
    raise ValueError(f"unknown mask kind {kind!r}")


# ------------------------------------------------------------- score mods
@dataclass(frozen=True)
class ScoreMod:
    kind: int
    value: float = 0.0
    slopes: torch.Tensor | None = field(default=None, compare=False)
    head_offset: int = 0   # ALiBi default slopes: model index of the call's first query head
    num_heads: int = 0     # ALiBi default slopes: the model's head count (0: the call's Hq)


def softcap(cap: float) -> ScoreMod:
    """s -> cap * tanh(s / cap)."""
    return ScoreMod(SCORE_SOFTCAP, float(cap))


def alibi(slopes: torch.Tensor | None = None, head_offset: int = 0, num_heads: int | None = None) -> ScoreMod:
    """s -> s + m_h * (kv_idx - q_idx). Without ``slopes`` the library uses
    m_h = 2^(-8(head_offset + h + 1) / num_heads) for the call's head h
    (num_heads defaults to the call's Hq), so a call on a slice of a model's
    heads gets those heads' slopes."""
    return ScoreMod(SCORE_ALIBI, 0.0, slopes, int(head_offset), 0 if num_heads is None else int(num_heads))


def score_mods_from_list(mods) -> list[ScoreMod]:
    out = []
    for m in mods or ():
        if m[0] == "softcap":
            out.append(softcap(m[1]))
        elif m[0] == "alibi":
            out.append(alibi(None if m[1] is None else torch.as_tensor(m[1], dtype=torch.float32)))
        else:
            raise ValueError(f"unknown score mod {m[0]!r}")
    return out


# -------------------------------------------------------------- BlockMask
@dataclass
class BlockMask:
    """Block-sparse mask in the tensorplay.nn.attention BlockMask format."""
    seq_lengths: tuple[int, int]
    kv_num_blocks: torch.Tensor
    kv_indices: torch.Tensor
    full_kv_num_blocks: torch.Tensor
    full_kv_indices: torch.Tensor
    BLOCK_SIZE: tuple[int, int]
    mask_mod: MaskMod

    @property
    def shape(self) -> tuple[int, int, int, int]:
        return tuple(self.kv_indices.shape)

    def _c(self) -> _BlockMask:
        c = _BlockMask()
        c.kv_num_blocks = self.kv_num_blocks.data_ptr()
        c.kv_indices = self.kv_indices.data_ptr()
        c.full_kv_num_blocks = self.full_kv_num_blocks.data_ptr()
        c.full_kv_indices = self.full_kv_indices.data_ptr()
        c.B, c.H, c.QB, c.KB = self.shape
        c.Q_LEN, c.KV_LEN = self.seq_lengths
        c.BLOCK_Q, c.BLOCK_KV = self.BLOCK_SIZE
        return c

    def q_side(self) -> dict:
        """The q-side lists (tensorplay.nn.attention, BlockMask "Details" items 3-4),
        computed on the GPU on first use and kept: q_num_blocks [B, H, KB],
        q_indices [B, H, KB, QB], full_q_num_blocks, full_q_indices."""
        cached = getattr(self, "_q_side", None)
        if cached is not None:
            return cached
        Bm, Hm, QB, KB = self.shape
        dev = self.kv_indices.device
        t = {"q_num_blocks": torch.empty((Bm, Hm, KB), dtype=torch.int32, device=dev),
             "q_indices": torch.empty((Bm, Hm, KB, QB), dtype=torch.int32, device=dev),
             "full_q_num_blocks": torch.empty((Bm, Hm, KB), dtype=torch.int32, device=dev),
             "full_q_indices": torch.empty((Bm, Hm, KB, QB), dtype=torch.int32, device=dev)}
        cq = _BlockMaskQ()
        cq.q_num_blocks = t["q_num_blocks"].data_ptr()
        cq.q_indices = t["q_indices"].data_ptr()
        cq.full_q_num_blocks = t["full_q_num_blocks"].data_ptr()
        cq.full_q_indices = t["full_q_indices"].data_ptr()
        c = self._c()
        with torch.cuda.device(dev):
            _check_launch(_lib.bsmt_block_mask_transpose(ctypes.byref(c), ctypes.byref(cq),
                                                  ctypes.c_void_p(_stream_ptr(dev))))
        self._q_side = t
        return t

    @property
    def q_num_blocks(self) -> torch.Tensor:
        return self.q_side()["q_num_blocks"]

    @property
    def q_indices(self) -> torch.Tensor:
        return self.q_side()["q_indices"]

    @property
    def full_q_num_blocks(self) -> torch.Tensor:
        return self.q_side()["full_q_num_blocks"]

    @property
    def full_q_indices(self) -> torch.Tensor:
        return self.q_side()["full_q_indices"]

    def to_dense(self) -> torch.Tensor:
        """int32 [B, H, QB, KB]: 1 where a row's partial or full list holds the block
        (the reconstruction loop of tensorplay.nn.attention, BlockMask "Basics")."""
        dev = self.kv_indices.device
        dense = torch.empty(self.shape, dtype=torch.int32, device=dev)
        c = self._c()
        with torch.cuda.device(dev):
            _check_launch(_lib.bsmt_block_mask_to_dense(ctypes.byref(c), ctypes.c_void_p(dense.data_ptr()),
                                                 ctypes.c_void_p(_stream_ptr(dev))))
        return dense

    @classmethod
    def from_kv_blocks(cls, kv_num_blocks: torch.Tensor, kv_indices: torch.Tensor,
                       full_kv_num_blocks: torch.Tensor | None = None, full_kv_indices: torch.Tensor | None = None,
                       BLOCK_SIZE: int | tuple[int, int] = 128, mask_mod: "MaskMod | None" = None,
                       seq_lengths: tuple[int, int] | None = None) -> "BlockMask":
        """A BlockMask from precomputed kv-side lists (tensorplay.nn.attention,
        BlockMask.from_kv_blocks); the q-side lists are generated on the GPU.
        Raises ValueError for lists of the wrong rank, dtype or shape."""
        bq, bkv = _block_pair(BLOCK_SIZE)
        if kv_indices.dim() != 4 or kv_num_blocks.dim() != 3:
            raise ValueError("kv_num_blocks must be [B, H, QB] and kv_indices [B, H, QB, KB]")
        if full_kv_num_blocks is None:
            full_kv_num_blocks = torch.zeros_like(kv_num_blocks)
            full_kv_indices = torch.zeros_like(kv_indices)
        for name, t in (("kv_num_blocks", kv_num_blocks), ("kv_indices", kv_indices),
                        ("full_kv_num_blocks", full_kv_num_blocks), ("full_kv_indices", full_kv_indices)):
            if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous int32 CUDA tensor")
        Bm, Hm, QB, KB = kv_indices.shape
        if (tuple(kv_num_blocks.shape) != (Bm, Hm, QB) or tuple(full_kv_num_blocks.shape) != (Bm, Hm, QB)
                or tuple(full_kv_indices.shape) != (Bm, Hm, QB, KB)):
            raise ValueError("BlockMask tensors disagree in shape")
        if seq_lengths is None:
            seq_lengths = (QB * bq, KB * bkv)
        if mask_mod is None:
            mask_mod = noop_mask()
        bm = cls(tuple(int(x) for x in seq_lengths), kv_num_blocks, kv_indices, full_kv_num_blocks,
                 full_kv_indices, (bq, bkv), mask_mod)
        bm.q_side()
        return bm

    def sparsity(self) -> float:
        """Percentage of blocks that are not computed (reads the counts back to the host)."""
        total = self.kv_indices.numel()
        if total == 0:
            return 0.0
        computed = int(self.kv_num_blocks.sum().item()) + int(self.full_kv_num_blocks.sum().item())
        return 100.0 * (1.0 - computed / total)


def _block_pair(BLOCK_SIZE) -> tuple[int, int]:
    if isinstance(BLOCK_SIZE, int):
        return BLOCK_SIZE, BLOCK_SIZE
    return int(BLOCK_SIZE[0]), int(BLOCK_SIZE[1])


def create_block_mask(mask_mod: MaskMod, B: int | None, H: int | None, Q_LEN: int, KV_LEN: int,
                      device="cuda", BLOCK_SIZE: int | tuple[int, int] = 128, out: BlockMask | None = None
                      ) -> BlockMask:
    """Build a BlockMask on the GPU (tensorplay.nn.attention, create_block_mask,
    separate_full_blocks=True). ``out`` reuses the tensors of an earlier BlockMask
    of the same shape."""
    device = torch.device(device)
    bq, bkv = _block_pair(BLOCK_SIZE)
    Bv = -1 if B is None else int(B)
    Hv = -1 if H is None else int(H)
    shape = (ctypes.c_int64 * 4)()
    _check(_lib.bsmt_block_mask_shape(Bv, Hv, int(Q_LEN), int(KV_LEN), bq, bkv, shape))
    shp = tuple(int(x) for x in shape)
    if out is not None and out.shape == shp:
        t = (out.kv_num_blocks, out.kv_indices, out.full_kv_num_blocks, out.full_kv_indices)
    else:
        t = (torch.empty(shp[:3], dtype=torch.int32, device=device),
             torch.empty(shp, dtype=torch.int32, device=device),
             torch.empty(shp[:3], dtype=torch.int32, device=device),
             torch.empty(shp, dtype=torch.int32, device=device))
    bm = BlockMask((int(Q_LEN), int(KV_LEN)), t[0], t[1], t[2], t[3], (bq, bkv), mask_mod)
    c = bm._c()
    with torch.cuda.device(device):
        spec, keep = mask_mod._spec(device, shp[0])
        _check_launch(_lib.bsmt_create_block_mask(ctypes.byref(spec), Bv, Hv, int(Q_LEN), int(KV_LEN), bq, bkv,
                                           ctypes.byref(c), ctypes.c_void_p(_stream_ptr(device))))
    # the marshalled spec and its device copies of document ids live as long as the mask
    bm._spec = spec
    bm._keep = keep
    return bm


def _score_spec(mods, device: torch.device, Hq: int) -> tuple[_ScoreSpec, list]:
    if mods is None:
        mods = []
    elif isinstance(mods, ScoreMod):
        mods = [mods]
    mods = list(mods)
    if len(mods) > MAX_SCORE_OPS:
        raise ValueError(f"at most {MAX_SCORE_OPS} score mods")
    spec = _ScoreSpec()
    spec.num_ops = len(mods)
    keep = []
    for i, m in enumerate(mods):
        spec.ops[i].kind = m.kind
        spec.ops[i].value = m.value
        spec.ops[i].head_offset = m.head_offset
        spec.ops[i].num_heads = m.num_heads
        if m.kind == SCORE_ALIBI and m.slopes is not None:
            s = m.slopes.to(device=device, dtype=torch.float32).contiguous()
            if s.numel() != Hq:
                raise ValueError(f"ALiBi slopes: {s.numel()} values for Hq={Hq}")
            keep.append(s)
            spec.ops[i].slopes = s.data_ptr()
    return spec, keep


def splitkv_workspace_bytes(B: int, Hq: int, M: int, D: int, num_splits: int) -> int:
    """Bytes of device workspace split-KV needs for these sizes (0 for one split)."""
    n = ctypes.c_int64(0)
    _check(_lib.bsmt_splitkv_workspace_bytes(int(B), int(Hq), int(M), int(D), int(num_splits), ctypes.byref(n)))
    return int(n.value)


class _FlexAttentionFn(torch.autograd.Function):
    """flex_attention as a differentiable op: the forward kernel, then
    flex_attention_backward for dq, dk and dv. lse is an output without a
    gradient."""

    @staticmethod
    def forward(ctx, q, k, v, block_mask, score_mod, scale, enable_gqa, out, lse):
        out, lse = _flex_attention_fwd(q, k, v, block_mask, score_mod, scale, enable_gqa, out, lse, 1, None)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.args = (block_mask, score_mod, scale, enable_gqa)
        ctx.mark_non_differentiable(lse)
        return out, lse

    @staticmethod
    def backward(ctx, dout, _dlse):
        q, k, v, out, lse = ctx.saved_tensors
        block_mask, score_mod, scale, enable_gqa = ctx.args
        if dout is None:
            return (None,) * 9
        dq, dk, dv = flex_attention_backward(q, k, v, out, lse, dout.to(torch.bfloat16).contiguous(), block_mask,
                                             score_mod, scale, enable_gqa)
        return dq, dk, dv, None, None, None, None, None, None


def flex_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block_mask: BlockMask | None = None,
                   score_mod: ScoreMod | Iterable[ScoreMod] | None = None, scale: float | None = None,
                   enable_gqa: bool = False, out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                   num_splits: int = 1, workspace: torch.Tensor | None = None):
    """Block-sparse masked attention forward. Returns (out bf16 [B,Hq,M,D], lse fp32 [B,Hq,M]).

    When autograd is on and q, k or v requires grad, the call is recorded
    for backpropagation: out's gradient flows to q, k and v through
    flex_attention_backward (one split only; lse has no gradient).

    num_splits > 1 runs split-KV: every row's kv blocks are cut into that many
    slices computed in parallel and merged exactly (for few q-blocks and long
    kv). ``workspace`` (a uint8 CUDA tensor of at least
    splitkv_workspace_bytes(...) bytes) is allocated when not given;
    ``workspace="static"`` uses the library's fixed device scratch instead and
    allocates nothing (bsmt_flex_attention_fwd_splitkv_static: sizes above the
    scratch are rejected, and calls that overlap in time race on it)."""
    if torch.is_grad_enabled() and any(t.requires_grad for t in (q, k, v)):
        if num_splits != 1:
            raise ValueError("split-KV has no backward; use num_splits=1 when q, k or v requires grad")
        return _FlexAttentionFn.apply(q, k, v, block_mask, score_mod, scale, enable_gqa, out, lse)
    return _flex_attention_fwd(q, k, v, block_mask, score_mod, scale, enable_gqa, out, lse, num_splits, workspace)


def _flex_attention_fwd(q, k, v, block_mask, score_mod, scale, enable_gqa, out, lse, num_splits, workspace):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16:
            raise ValueError(f"{name} must be bfloat16 (got {t.dtype})")
        if t.dim() != 4:
            raise ValueError(f"{name} must be 4-D [B, H, S, D]")
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if not (q.device == k.device == v.device):
        raise ValueError("q, k and v must be on the same device")
    B, Hq, M, D = q.shape
    Bk, Hkv, N, Dk = k.shape
    if k.shape != v.shape or Bk != B or Dk != D:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)}, k {tuple(k.shape)}, v {tuple(v.shape)}")
    device = q.device
    if out is None:
        out = torch.empty((B, Hq, M, D), dtype=torch.bfloat16, device=device)
    if lse is None:
        lse = torch.empty((B, Hq, M), dtype=torch.float32, device=device)
    if out.shape != (B, Hq, M, D) or out.dtype != torch.bfloat16 or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 [B, Hq, M, D] tensor")
    if lse.shape != (B, Hq, M) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 [B, Hq, M] tensor")
    with torch.cuda.device(device):
        sspec, keep_s = _score_spec(score_mod, device, Hq)
        bm_c = None
        mspec = None
        keep_m = []
        if block_mask is not None:
            bm_c = block_mask._c()
            mspec = getattr(block_mask, "_spec", None)
            if mspec is None:
                mspec, keep_m = block_mask.mask_mod._spec(device, int(block_mask.shape[0]))
        common = (q.data_ptr(), k.data_ptr(), v.data_ptr(), B, Hq, Hkv, M, N, D,
                  ctypes.byref(bm_c) if bm_c is not None else None,
                  ctypes.byref(mspec) if mspec is not None else None,
                  ctypes.byref(sspec), ctypes.c_float(0.0 if scale is None else float(scale)),
                  int(bool(enable_gqa)))
        if num_splits == 1:
            _check_launch(_lib.bsmt_flex_attention_fwd(*common, out.data_ptr(), lse.data_ptr(),
                                                ctypes.c_void_p(_stream_ptr(device))))
        elif isinstance(workspace, str) and workspace == "static":
            # the library's own device scratch: no allocation (overlapping calls race)
            _check_launch(_lib.bsmt_flex_attention_fwd_splitkv_static(
                *common, int(num_splits), out.data_ptr(), lse.data_ptr(), ctypes.c_void_p(_stream_ptr(device))))
        else:
            need = splitkv_workspace_bytes(B, Hq, M, D, num_splits)
            if workspace is None:
                workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=device)
            if not workspace.is_cuda or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
                raise ValueError("workspace must be a contiguous uint8 CUDA tensor")
            _check_launch(_lib.bsmt_flex_attention_fwd_splitkv(
                *common, int(num_splits), ctypes.c_void_p(workspace.data_ptr()), workspace.numel(),
                out.data_ptr(), lse.data_ptr(), ctypes.c_void_p(_stream_ptr(device))))
    del keep_s, keep_m
    return out, lse


def backward_workspace_bytes(B: int, Hq: int, M: int) -> int:
    """Bytes of device workspace flex_attention_backward needs (lse and delta per query row)."""
    n = ctypes.c_int64(0)
    _check(_lib.bsmt_flex_attention_bwd_workspace_bytes(int(B), int(Hq), int(M), ctypes.byref(n)))
    return int(n.value)


def flex_attention_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                            lse: torch.Tensor, dout: torch.Tensor, block_mask: BlockMask | None = None,
                            score_mod: ScoreMod | Iterable[ScoreMod] | None = None, scale: float | None = None,
                            enable_gqa: bool = False, workspace: torch.Tensor | None = None,
                            dq: torch.Tensor | None = None, dk: torch.Tensor | None = None,
                            dv: torch.Tensor | None = None):
    """Gradients (dq, dk, dv) of sum(out * dout) for the forward
    ``out, lse = flex_attention(q, k, v, block_mask, score_mod, scale, enable_gqa)``.
    Pass the same arguments as the forward plus its out and lse. dk and dv
    walk the block mask's q-side lists (computed on first use), dq its
    kv-side lists. ``workspace``: a uint8 CUDA tensor of at least
    backward_workspace_bytes(B, Hq, M) bytes, allocated when not given.
    ``dq``, ``dk``, ``dv``: output tensors to write (contiguous bf16 of q's and
    k's shapes), allocated when not given."""
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout)):
        if t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 4-D CUDA tensor")
    B, Hq, M, D = q.shape
    Bk, Hkv, N, Dk = k.shape
    if k.shape != v.shape or Bk != B or Dk != D:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)}, k {tuple(k.shape)}, v {tuple(v.shape)}")
    if out.shape != q.shape or dout.shape != q.shape:
        raise ValueError("out and dout must have q's shape")
    if lse.shape != (B, Hq, M) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 [B, Hq, M] tensor")
    device = q.device
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for name, t, ref in (("dq", dq, q), ("dk", dk, k), ("dv", dv, v)):
        if t.shape != ref.shape or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.device != device:
            raise ValueError(f"{name} must be a contiguous bf16 tensor of shape {tuple(ref.shape)} on {device}")
    need = backward_workspace_bytes(B, Hq, M)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=device)
    if not workspace.is_cuda or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous uint8 CUDA tensor")
    with torch.cuda.device(device):
        sspec, keep_s = _score_spec(score_mod, device, Hq)
        bm_c = bmq_c = mspec = None
        keep_m = []
        if block_mask is not None:
            bm_c = block_mask._c()
            qs = block_mask.q_side()
            bmq_c = _BlockMaskQ()
            bmq_c.q_num_blocks = qs["q_num_blocks"].data_ptr()
            bmq_c.q_indices = qs["q_indices"].data_ptr()
            bmq_c.full_q_num_blocks = qs["full_q_num_blocks"].data_ptr()
            bmq_c.full_q_indices = qs["full_q_indices"].data_ptr()
            mspec = getattr(block_mask, "_spec", None)
            if mspec is None:
                mspec, keep_m = block_mask.mask_mod._spec(device, int(block_mask.shape[0]))
        _check_launch(_lib.bsmt_flex_attention_bwd(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dout.data_ptr(), lse.data_ptr(),
            B, Hq, Hkv, M, N, D,
            ctypes.byref(bm_c) if bm_c is not None else None, ctypes.byref(bmq_c) if bmq_c is not None else None,
            ctypes.byref(mspec) if mspec is not None else None, ctypes.byref(sspec),
            ctypes.c_float(0.0 if scale is None else float(scale)), int(bool(enable_gqa)),
            dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ctypes.c_void_p(workspace.data_ptr()), workspace.numel(),
            ctypes.c_void_p(_stream_ptr(device))))
    del keep_s, keep_m
    return dq, dk, dv


def host_workspace_bytes(B: int, Hq: int, Hkv: int, M: int, N: int, D: int,
                         mask_mod: MaskMod | None = None) -> int:
    """Bytes of device workspace flex_attention_host needs
    (bsmt_flex_attention_host_workspace_bytes)."""
    spec = None
    if mask_mod is not None:
        spec, _ = mask_mod._spec(torch.device("cpu"), int(B))
    n = ctypes.c_int64(0)
    _check(_lib.bsmt_flex_attention_host_workspace_bytes(int(B), int(Hq), int(Hkv), int(M), int(N), int(D),
                                                         ctypes.byref(spec) if spec is not None else None,
                                                         ctypes.byref(n)))
    return int(n.value)


def flex_attention_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, mask_mod: MaskMod | None = None,
                        score_mod: ScoreMod | Iterable[ScoreMod] | None = None, scale: float | None = None,
                        enable_gqa: bool = False, device="cuda", out: torch.Tensor | None = None,
                        lse: torch.Tensor | None = None, chunks: int = 16, workspace: torch.Tensor | None = None):
    """flex_attention on host tensors (bsmt_flex_attention_host): q [B,Hq,M,D],
    k/v [B,Hkv,N,D] bf16 in CPU memory (pinned for full speed). The library
    copies the document ids and slopes in, builds the BlockMask of
    ``mask_mod`` on the device and pipelines about ``chunks`` independent
    pieces along (batch row, kv-head group): the host-to-device copy of piece
    i+1, the attention of piece i and the device-to-host copy of piece i-1 run
    at the same time. Document ids of ``mask_mod`` and ALiBi slopes are read
    from host memory (CUDA tensors are brought to the host first). Returns
    host (out bf16 [B,Hq,M,D], lse fp32 [B,Hq,M]) once the copies are done;
    ``out``/``lse`` may be given (pinned CPU tensors). ``workspace``: a uint8
    tensor on ``device`` of at least host_workspace_bytes(...) bytes,
    allocated when not given."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or t.dim() != 4 or t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 4-D CPU tensor")
    device = torch.device(device)
    B, Hq, M, D = q.shape
    _, Hkv, N, _ = k.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[3] != D:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)}, k {tuple(k.shape)}, v {tuple(v.shape)}")
    if Hkv < 1 or Hq % Hkv != 0:
        raise ValueError(f"Hq={Hq} is not a multiple of Hkv={Hkv}")
    if out is None:
        out = torch.empty((B, Hq, M, D), dtype=torch.bfloat16, pin_memory=True)
    if lse is None:
        lse = torch.empty((B, Hq, M), dtype=torch.float32, pin_memory=True)
    if (out.shape != (B, Hq, M, D) or lse.shape != (B, Hq, M) or out.is_cuda or lse.is_cuda
            or out.dtype != torch.bfloat16 or lse.dtype != torch.float32
            or not out.is_contiguous() or not lse.is_contiguous()):
        raise ValueError("out and lse must be contiguous CPU tensors: bf16 [B,Hq,M,D] and fp32 [B,Hq,M]")
    host = torch.device("cpu")
    mspec, keep_m = (None, []) if mask_mod is None else mask_mod._spec(host, B)
    sspec, keep_s = _score_spec(score_mod, host, Hq)
    need = host_workspace_bytes(B, Hq, Hkv, M, N, D, mask_mod)
    with torch.cuda.device(device):
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=device)
        if not workspace.is_cuda or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
            raise ValueError("workspace must be a contiguous uint8 CUDA tensor")
        stream = torch.cuda.current_stream(device)
        _check(_lib.bsmt_flex_attention_host(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), B, Hq, Hkv, M, N, D,
            ctypes.byref(mspec) if mspec is not None else None, ctypes.byref(sspec),
            ctypes.c_float(0.0 if scale is None else float(scale)), int(bool(enable_gqa)), int(chunks),
            ctypes.c_void_p(workspace.data_ptr()), workspace.numel(), out.data_ptr(), lse.data_ptr(),
            ctypes.c_void_p(stream.cuda_stream)))
        stream.synchronize()  # the host outputs are complete
        if _DEBUG_SYNC:
            _check(_lib.bsmt_check_device_status(ctypes.c_void_p(stream.cuda_stream)))
    del keep_s, keep_m
    return out, lse


def seqlens_to_doc_ids(cu_seqlens: torch.Tensor, total: int) -> torch.Tensor:
    """int32 [total] on the device: each packed token's sequence ordinal
    (bsmt_seqlens_to_doc_ids)."""
    cu = cu_seqlens.to(dtype=torch.int32).contiguous()
    if not cu.is_cuda or cu.dim() != 1 or cu.numel() < 1:
        raise ValueError("cu_seqlens must be a 1-D CUDA tensor with at least one entry")
    ids = torch.empty(int(total), dtype=torch.int32, device=cu.device)
    with torch.cuda.device(cu.device):
        _check_launch(_lib.bsmt_seqlens_to_doc_ids(ctypes.c_void_p(cu.data_ptr()), cu.numel() - 1, int(total),
                                            ctypes.c_void_p(ids.data_ptr()), ctypes.c_void_p(_stream_ptr(cu.device))))
    return ids


def _varlen_block_mask(cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor, M: int, N: int, causal: bool,
                       mods: list, device: torch.device) -> BlockMask:
    """The BlockMask of packed sequences over (total_q, total_k), B = H = 1:
    sequence ordinals as DOCUMENT ids, and CAUSAL when asked."""
    # Causal masking and ALiBi see packed positions. These equal positions
    # within the sequence only when q and k share cu_seqlens (the sequence
    # start cancels in kv_idx - q_idx).
    if (causal or any(m.kind == SCORE_ALIBI for m in mods)) and not (
            cu_seqlens_q is cu_seqlens_k or torch.equal(cu_seqlens_q, cu_seqlens_k)):
        raise ValueError("causal or ALiBi varlen attention needs q and k to share cu_seqlens")
    q_ids = seqlens_to_doc_ids(cu_seqlens_q, M)
    kv_ids = q_ids if (cu_seqlens_k is cu_seqlens_q and N == M) else seqlens_to_doc_ids(cu_seqlens_k, N)
    mm = document(q_ids, kv_ids)
    if causal:
        mm = and_masks(mm, _causal_mask())
    return create_block_mask(mm, 1, 1, M, N, device=device)


def _check_packed(**tensors) -> None:
    for name, t in tensors.items():
        if t.dtype != torch.bfloat16 or t.dim() != 3 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 3-D CUDA tensor [tokens, H, D]")


def _varlen_fwd(q, k, v, bm, mods, scale, enable_gqa, out, lse):
    M, Hq, D = q.shape
    N, Hkv, _ = k.shape
    device = q.device
    if out is None:
        out = torch.empty((M, Hq, D), dtype=torch.bfloat16, device=device)
    if lse is None:
        lse = torch.empty((Hq, M), dtype=torch.float32, device=device)
    if out.shape != (M, Hq, D) or lse.shape != (Hq, M):
        raise ValueError("out must be [total_q, Hq, D] and lse [Hq, total_q]")
    with torch.cuda.device(device):
        sspec, keep_s = _score_spec(mods, device, Hq)
        c = bm._c()
        _check_launch(_lib.bsmt_flex_attention_fwd_packed(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), Hq, Hkv, M, N, D, ctypes.byref(c), ctypes.byref(bm._spec),
            ctypes.byref(sspec), ctypes.c_float(0.0 if scale is None else float(scale)), int(bool(enable_gqa)),
            out.data_ptr(), lse.data_ptr(), ctypes.c_void_p(_stream_ptr(device))))
    del keep_s
    return out, lse


def _varlen_bwd(q, k, v, out, lse, dout, bm, mods, scale, enable_gqa):
    M, Hq, D = q.shape
    N, Hkv, _ = k.shape
    device = q.device
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(max(backward_workspace_bytes(1, Hq, M), 1), dtype=torch.uint8, device=device)
    with torch.cuda.device(device):
        sspec, keep_s = _score_spec(mods, device, Hq)
        c = bm._c()
        qs = bm.q_side()
        cq = _BlockMaskQ()
        cq.q_num_blocks = qs["q_num_blocks"].data_ptr()
        cq.q_indices = qs["q_indices"].data_ptr()
        cq.full_q_num_blocks = qs["full_q_num_blocks"].data_ptr()
        cq.full_q_indices = qs["full_q_indices"].data_ptr()
        _check_launch(_lib.bsmt_flex_attention_bwd_packed(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dout.data_ptr(), lse.data_ptr(), Hq, Hkv, M, N,
            D, ctypes.byref(c), ctypes.byref(cq), ctypes.byref(bm._spec), ctypes.byref(sspec),
            ctypes.c_float(0.0 if scale is None else float(scale)), int(bool(enable_gqa)), dq.data_ptr(),
            dk.data_ptr(), dv.data_ptr(), ctypes.c_void_p(ws.data_ptr()), ws.numel(),
            ctypes.c_void_p(_stream_ptr(device))))
    del keep_s
    return dq, dk, dv


class _FlexAttentionVarlenFn(torch.autograd.Function):
    """flex_attention_varlen as a differentiable op (lse has no gradient)."""

    @staticmethod
    def forward(ctx, q, k, v, bm, mods, scale, enable_gqa, out, lse):
        out, lse = _varlen_fwd(q, k, v, bm, mods, scale, enable_gqa, out, lse)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.args = (bm, mods, scale, enable_gqa)
        ctx.mark_non_differentiable(lse)
        return out, lse

    @staticmethod
    def backward(ctx, dout, _dlse):
        if dout is None:
            return (None,) * 9
        q, k, v, out, lse = ctx.saved_tensors
        bm, mods, scale, enable_gqa = ctx.args
        dq, dk, dv = _varlen_bwd(q, k, v, out, lse, dout.to(torch.bfloat16).contiguous(), bm, mods, scale,
                                 enable_gqa)
        return dq, dk, dv, None, None, None, None, None, None


def flex_attention_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens_q: torch.Tensor,
                          cu_seqlens_k: torch.Tensor, causal: bool = False,
                          score_mod: ScoreMod | Iterable[ScoreMod] | None = None, scale: float | None = None,
                          enable_gqa: bool = False, out: torch.Tensor | None = None, lse: torch.Tensor | None = None):
    """Attention over packed variable-length sequences (the cu_seqlens form):
    q [total_q, Hq, D], k/v [total_k, Hkv, D] bf16; token t of the pack
    belongs to sequence i for cu_seqlens[i] <= t < cu_seqlens[i+1], and attends
    only to keys of its own sequence. ``causal`` needs q and k to share
    cu_seqlens (equal lengths, top-left aligned). Returns (out [total_q, Hq, D],
    lse [Hq, total_q]).

    The sequence ordinals become DOCUMENT ids on the device, the BlockMask is
    built over the whole pack (B = H = 1), and the packed layout goes straight
    to the attention kernel through its tensor maps. With q, k or v requiring
    grad the call is recorded for backpropagation (the packed backward)."""
    _check_packed(q=q, k=k, v=v)
    M, Hq, D = q.shape
    N, Hkv, Dk = k.shape
    if v.shape != k.shape or Dk != D:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)}, k {tuple(k.shape)}, v {tuple(v.shape)}")
    mods = [score_mod] if isinstance(score_mod, ScoreMod) else list(score_mod or ())
    bm = _varlen_block_mask(cu_seqlens_q, cu_seqlens_k, M, N, causal, mods, q.device)
    if torch.is_grad_enabled() and any(t.requires_grad for t in (q, k, v)):
        return _FlexAttentionVarlenFn.apply(q, k, v, bm, mods, scale, enable_gqa, out, lse)
    return _varlen_fwd(q, k, v, bm, mods, scale, enable_gqa, out, lse)


def flex_attention_varlen_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                                   lse: torch.Tensor, dout: torch.Tensor, cu_seqlens_q: torch.Tensor,
                                   cu_seqlens_k: torch.Tensor, causal: bool = False,
                                   score_mod: ScoreMod | Iterable[ScoreMod] | None = None,
                                   scale: float | None = None, enable_gqa: bool = False):
    """Gradients (dq [total_q, Hq, D], dk, dv [total_k, Hkv, D]) of
    sum(out * dout) for ``out, lse = flex_attention_varlen(...)`` with the same
    arguments (bsmt_flex_attention_bwd_packed)."""
    _check_packed(q=q, k=k, v=v, out=out, dout=dout)
    M, Hq, D = q.shape
    N, Hkv, Dk = k.shape
    if v.shape != k.shape or Dk != D or out.shape != q.shape or dout.shape != q.shape:
        raise ValueError("shape mismatch among q, k, v, out and dout")
    if lse.shape != (Hq, M) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 [Hq, total_q] tensor")
    mods = [score_mod] if isinstance(score_mod, ScoreMod) else list(score_mod or ())
    bm = _varlen_block_mask(cu_seqlens_q, cu_seqlens_k, M, N, causal, mods, q.device)
    return _varlen_bwd(q, k, v, out, lse, dout, bm, mods, scale, enable_gqa)


def selftest_wait_timeout(device=None) -> dict:
    """Run the library's bounded-wait failure path on purpose
    (bsmt_selftest_wait_timeout) and return what the kernel saw. The device
    status word then holds DEVICE_TIMEOUT; check_device_status raises it."""
    device = torch.device("cuda") if device is None else torch.device(device)
    res = torch.full((3,), -1, dtype=torch.int32, device=device)
    with torch.cuda.device(device):
        _check(_lib.bsmt_selftest_wait_timeout(ctypes.c_void_p(res.data_ptr()), ctypes.c_void_p(_stream_ptr(device))))
        torch.cuda.current_stream(device).synchronize()
    r = res.cpu().tolist()
    return {"warp0_completed": r[0], "warp1_completed": r[1], "warp0_wait_us": r[2]}


def check_device_status(device=None) -> None:
    """Synchronize the current stream and raise if a kernel recorded a device-side error."""
    device = torch.device("cuda") if device is None else torch.device(device)
    with torch.cuda.device(device):
        _check(_lib.bsmt_check_device_status(ctypes.c_void_p(_stream_ptr(device))))
