"""Host-only checks of the C ABI: symbols, shape helper and argument errors.

None of these calls reaches a CUDA API. Every error is caught on the host
before any device work, so they run on a machine without a GPU.
"""
import ctypes
import os
import re

import pytest

import block_sparse_masked_tile_b200 as bsmt
from block_sparse_masked_tile_b200 import _BlockMask, _MaskSpec, _ScoreSpec, _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bsmt.h")

OK, INVALID, SHAPE, UNSUPPORTED = 0, 1, 2, 3
FAKE = 0x10000  # 16-byte aligned non-null address; never dereferenced by these calls


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:bsmt_status|const char\*|int32_t)\s+(bsmt_\w+)\s*\(", text, re.M)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert names == sorted(["bsmt_block_mask_shape", "bsmt_create_block_mask", "bsmt_flex_attention_fwd",
                            "bsmt_block_mask_transpose", "bsmt_block_mask_to_dense",
                            "bsmt_splitkv_workspace_bytes", "bsmt_flex_attention_fwd_splitkv",
                            "bsmt_flex_attention_fwd_splitkv_static", "bsmt_seqlens_to_doc_ids",
                            "bsmt_flex_attention_fwd_packed", "bsmt_flex_attention_bwd_workspace_bytes",
                            "bsmt_flex_attention_bwd", "bsmt_flex_attention_bwd_packed",
                            "bsmt_selftest_wait_timeout", "bsmt_flex_attention_host_workspace_bytes",
                            "bsmt_flex_attention_host",
                            "bsmt_last_error", "bsmt_check_device_status", "bsmt_version"])
    lib = ctypes.CDLL(bsmt.library_path())
    for n in names:
        assert hasattr(lib, n), n


def test_version():
    assert _lib.bsmt_version() == (2 << 16) | 1


def shape(*args):
    out = (ctypes.c_int64 * 4)()
    st = _lib.bsmt_block_mask_shape(*args, out)
    return st, tuple(out)


def test_block_mask_shape():
    assert shape(2, 32, 32768, 32768, 128, 128) == (OK, (2, 32, 256, 256))
    assert shape(0, -1, 300, 129, 128, 128) == (OK, (1, 1, 3, 2))
    assert shape(1, 1, 0, 0, 128, 128) == (OK, (1, 1, 0, 0))
    assert shape(1, 1, 256, 256, 64, 64)[0] == UNSUPPORTED
    assert shape(1, 1, -5, 256, 128, 128)[0] == INVALID
    assert b"128" in _lib.bsmt_last_error() or True


def spec_of(nodes, q_doc=None, kv_doc=None, doc_batch=1):
    s = _MaskSpec()
    s.num_nodes = len(nodes)
    for i, (k, a) in enumerate(nodes):
        s.nodes[i].kind = k
        s.nodes[i].arg = a
    s.q_doc_ids = q_doc
    s.kv_doc_ids = kv_doc
    s.doc_batch = doc_batch
    return s


def build(spec, B=1, H=1, M=0, N=0, bq=128, bkv=128):
    # M = 0 means there are no rows: a valid spec returns OK without touching the GPU
    out = _BlockMask()
    st = _lib.bsmt_create_block_mask(ctypes.byref(spec) if spec is not None else None, B, H, M, N, bq, bkv,
                                     ctypes.byref(out), None)
    return st, out


C, W, P, S, DOC, AND, OR = (bsmt.MASK_CAUSAL, bsmt.MASK_WINDOW, bsmt.MASK_PREFIX_LM, bsmt.MASK_SINK,
                           bsmt.MASK_DOCUMENT, bsmt.MASK_AND, bsmt.MASK_OR)


def test_create_block_mask_valid_specs_without_rows():
    for nodes in ([(C, 0)], [(C, 0), (W, 512), (AND, 2)], [(C, 0), (S, 4), (W, 1024), (OR, 2), (AND, 2)],
                  [(bsmt.MASK_NOOP, 0)], [(P, 7), (S, 1), (OR, 2)]):
        st, out = build(spec_of(nodes), M=0, N=100)
        assert st == OK, _lib.bsmt_last_error()
        assert (out.B, out.H, out.QB, out.KB, out.KV_LEN) == (1, 1, 0, 1, 100)


@pytest.mark.parametrize("nodes,code", [
    ([], INVALID),                                   # empty program
    ([(C, 0), (W, 3)], INVALID),                     # two values left
    ([(C, 0), (AND, 2)], INVALID),                   # operand underflow
    ([(C, 0), (AND, 0)], INVALID),                   # arity 0
    ([(99, 0)], INVALID),                            # unknown kind
    ([(DOC, 0)], INVALID),                           # document without id arrays
])
def test_create_block_mask_malformed(nodes, code):
    st, _ = build(spec_of(nodes), M=0, N=10)
    assert st == code
    assert _lib.bsmt_last_error()


def test_create_block_mask_alternatives_after_simplification():
    # AND of 5 binary ORs of CAUSAL and SINK(2) expands to 32 alternatives,
    # which collapse to {CAUSAL} and {SINK(2)}: one leaf of a kind per
    # alternative, and CAUSAL AND SINK lies inside both
    nodes = []
    for _ in range(5):
        nodes += [(C, 0), (S, 2), (OR, 2)]
    nodes.append((AND, 5))
    st, _ = build(spec_of(nodes), M=0, N=10)
    assert st == OK, _lib.bsmt_last_error()
    # an OR of 17 alternatives WINDOW(w) AND SINK(s) with w rising and s
    # falling: none contains another, so 17 remain (> 16)
    nodes = [n for i in range(17) for n in [(W, 10 + i), (S, 100 - i), (AND, 2)]] + [(OR, 17)]
    assert len(nodes) == 52
    st, _ = build(spec_of(nodes), M=0, N=10)
    assert st == UNSUPPORTED and "17 alternatives" in _lib.bsmt_last_error().decode()
    # 16 of them are accepted; a repeat of one adds nothing
    nodes = [n for i in range(16) for n in [(W, 10 + i), (S, 100 - i), (AND, 2)]]
    st, _ = build(spec_of(nodes + [(W, 10), (S, 100), (AND, 2), (OR, 17)]), M=0, N=10)
    assert st == OK, _lib.bsmt_last_error()
    # ... and one with a stricter window and sink than another lies inside it
    st, _ = build(spec_of(nodes + [(W, 9), (S, 99), (AND, 2), (OR, 17)]), M=0, N=10)
    assert st == OK, _lib.bsmt_last_error()


def test_create_block_mask_other_errors():
    assert build(None, M=0, N=10)[0] == INVALID
    assert build(spec_of([(C, 0)]), M=0, N=10, bq=64, bkv=64)[0] == UNSUPPORTED
    st, _ = build(spec_of([(DOC, 0)], FAKE, FAKE, doc_batch=3), B=2, M=0, N=10)
    assert st == SHAPE
    st, _ = build(spec_of([(DOC, 0)], FAKE + 2, FAKE, doc_batch=1), B=2, M=0, N=10)
    assert st == INVALID
    # rows present but output pointers missing
    st, _ = build(spec_of([(C, 0)]), M=256, N=256)
    assert st == INVALID


def attn(B=1, Hq=2, Hkv=2, M=256, N=256, D=64, bm=None, spec=None, score=None, scale=0.0, gqa=0,
         q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE):
    return _lib.bsmt_flex_attention_fwd(q, k, v, B, Hq, Hkv, M, N, D, bm, spec, score, ctypes.c_float(scale), gqa,
                                        out, lse, None)


def test_flex_attention_argument_errors():
    assert attn(D=96) == UNSUPPORTED
    assert attn(D=256) == UNSUPPORTED
    assert attn(Hq=3, Hkv=2, gqa=1) == SHAPE
    assert attn(Hq=4, Hkv=2, gqa=0) == SHAPE
    assert attn(Hkv=0) == SHAPE
    assert attn(M=-1) == INVALID
    assert attn(q=0) == INVALID
    assert attn(k=FAKE + 8) == INVALID
    assert attn(out=FAKE + 4) == INVALID
    assert attn(lse=FAKE + 2) == INVALID
    assert attn(scale=float("inf")) == INVALID
    assert attn(N=(1 << 31) - 255) == UNSUPPORTED  # kv positions must fit int32 with a tile to spare


def test_flex_attention_score_errors():
    sc = _ScoreSpec()
    sc.num_ops = 3
    assert attn(score=ctypes.byref(sc)) == INVALID
    sc.num_ops = 1
    sc.ops[0].kind = bsmt.SCORE_SOFTCAP
    sc.ops[0].value = -1.0
    assert attn(score=ctypes.byref(sc)) == INVALID
    sc.ops[0].kind = 42
    assert attn(score=ctypes.byref(sc)) == INVALID
    sc.num_ops = 2
    sc.ops[0].kind = bsmt.SCORE_SOFTCAP
    sc.ops[0].value = 3.0
    sc.ops[1].kind = bsmt.SCORE_SOFTCAP
    sc.ops[1].value = 3.0
    assert attn(score=ctypes.byref(sc)) == UNSUPPORTED
    sc.ops[1].kind = bsmt.SCORE_ALIBI
    sc.ops[1].slopes = FAKE + 1
    assert attn(score=ctypes.byref(sc)) == INVALID


def test_alibi_head_offset_checks():
    # default ALiBi slopes for heads [head_offset, head_offset + Hq) of a model
    # of num_heads heads: the range must lie inside the model
    sc = _ScoreSpec()
    sc.num_ops = 1
    sc.ops[0].kind = bsmt.SCORE_ALIBI
    for h0, nh, code in ((0, 0, OK), (0, 2, OK), (6, 8, OK), (1, 0, INVALID), (7, 8, INVALID),
                         (-1, 8, INVALID), (0, 1, INVALID)):
        sc.ops[0].head_offset, sc.ops[0].num_heads = h0, nh
        assert attn(M=0, score=ctypes.byref(sc)) == code, (h0, nh, _lib.bsmt_last_error())
    # with explicit slopes both fields are ignored
    sc.ops[0].slopes = FAKE
    sc.ops[0].head_offset, sc.ops[0].num_heads = 5, 1
    assert attn(M=0, score=ctypes.byref(sc)) == OK


def host_ws(B, Hq, Hkv, M, N, D, spec=None):
    n = ctypes.c_int64(-1)
    st = _lib.bsmt_flex_attention_host_workspace_bytes(B, Hq, Hkv, M, N, D,
                                                       ctypes.byref(spec) if spec is not None else None,
                                                       ctypes.byref(n))
    return st, n.value


def test_host_workspace_bytes():
    r = lambda x: (x + 255) // 256 * 256  # noqa: E731
    B, Hq, Hkv, M, N, D = 2, 32, 8, 32768, 32768, 128
    q, kv, l = B * Hq * M * D * 2, B * Hkv * N * D * 2, B * Hq * M * 4
    slopes = 2 * r(Hq * 4)
    assert host_ws(B, Hq, Hkv, M, N, D) == (OK, 2 * r(q) + 2 * r(kv) + r(l) + slopes)
    # a mask adds its four tensors at B = H = 1 (the mask depends on neither)
    QB = KB = 256
    mask = 2 * r(QB * 4) + 2 * r(QB * KB * 4)
    assert host_ws(B, Hq, Hkv, M, N, D, spec_of([(C, 0)])) == (OK, 2 * r(q) + 2 * r(kv) + r(l) + mask + slopes)
    # document ids that differ per batch row: the mask keeps B rows, plus the ids
    st, n = host_ws(2, 4, 4, 300, 500, 64, spec_of([(DOC, 0)], FAKE, FAKE, doc_batch=2))
    q, kv, l = 2 * 4 * 300 * 64 * 2, 2 * 4 * 500 * 64 * 2, 2 * 4 * 300 * 4
    mask = 2 * r(2 * 3 * 4) + 2 * r(2 * 3 * 4 * 4)
    assert (st, n) == (OK, 2 * r(q) + 2 * r(kv) + r(l) + mask + r(2 * 300 * 4) + r(2 * 500 * 4) + 2 * r(16))
    assert host_ws(2, 4, 4, 300, 500, 96)[0] == UNSUPPORTED
    assert host_ws(3, 4, 4, 300, 500, 64, spec_of([(DOC, 0)], FAKE, FAKE, doc_batch=2))[0] == SHAPE
    assert _lib.bsmt_flex_attention_host_workspace_bytes(1, 1, 1, 1, 1, 64, None, None) == INVALID


def host_call(B=1, Hq=2, Hkv=2, M=256, N=256, D=64, spec=None, score=None, gqa=0, ws=FAKE, ws_bytes=1 << 40,
              q=FAKE, out=FAKE, lse=FAKE):
    return _lib.bsmt_flex_attention_host(q, FAKE, FAKE, B, Hq, Hkv, M, N, D,
                                         ctypes.byref(spec) if spec is not None else None,
                                         ctypes.byref(score) if score is not None else None, ctypes.c_float(0.0),
                                         gqa, 16, ctypes.c_void_p(ws), ws_bytes, out, lse, None)


def test_host_entry_argument_errors():
    """Every check of the host-buffer entry point runs before anything is
    enqueued (the attention's own checks at the full size included)."""
    assert host_call(D=96) == UNSUPPORTED
    assert host_call(Hq=3, Hkv=2, gqa=1) == SHAPE
    assert host_call(Hq=4, Hkv=2, gqa=0) == SHAPE
    assert host_call(M=-1) == INVALID
    assert host_call(q=0) == INVALID
    assert host_call(ws=0) == INVALID
    assert host_call(ws=FAKE + 16) == INVALID                 # not 256-byte aligned
    assert host_call(ws_bytes=1000) == INVALID                # too small
    assert host_call(spec=spec_of([(C, 0), (AND, 2)])) == INVALID
    assert host_call(spec=spec_of([(DOC, 0)])) == INVALID    # document without ids
    assert host_call(N=(1 << 31) - 255) == UNSUPPORTED       # kv positions beyond int32
    sc = _ScoreSpec()
    sc.num_ops = 1
    sc.ops[0].kind = bsmt.SCORE_SOFTCAP
    sc.ops[0].value = -2.0
    assert host_call(score=sc) == INVALID
    assert host_call(B=0) == OK                                # nothing to compute, nothing enqueued
    assert host_call(M=0) == OK


def block_mask_c(B=1, H=1, QB=2, KB=2, M=256, N=256, bq=128):
    c = _BlockMask()
    c.kv_num_blocks = c.kv_indices = c.full_kv_num_blocks = c.full_kv_indices = FAKE
    c.B, c.H, c.QB, c.KB = B, H, QB, KB
    c.Q_LEN, c.KV_LEN = M, N
    c.BLOCK_Q = c.BLOCK_KV = bq
    return c


def test_flex_attention_block_mask_errors():
    assert attn(bm=ctypes.byref(block_mask_c(QB=3))) == SHAPE
    assert attn(bm=ctypes.byref(block_mask_c(N=200))) == SHAPE
    assert attn(bm=ctypes.byref(block_mask_c(B=2))) == SHAPE
    assert attn(bm=ctypes.byref(block_mask_c(H=3))) == SHAPE
    assert attn(bm=ctypes.byref(block_mask_c(bq=64))) == UNSUPPORTED
    bad = spec_of([(C, 0), (AND, 2)])
    assert attn(bm=ctypes.byref(block_mask_c()), spec=ctypes.byref(bad)) == INVALID
    c = block_mask_c()
    c.kv_indices = None
    assert attn(bm=ctypes.byref(c)) == INVALID


def test_flex_attention_empty_is_ok_without_launch():
    # B == 0 or M == 0: nothing to compute, nothing launched
    assert attn(B=0) == OK
    assert attn(M=0) == OK


def test_python_errors_map_to_value_error():
    with pytest.raises(ValueError):
        bsmt._check(SHAPE)
    with pytest.raises(RuntimeError):
        bsmt._check(UNSUPPORTED)


def test_transpose_and_to_dense_argument_errors():
    from block_sparse_masked_tile_b200 import _BlockMaskQ
    null = ctypes.c_void_p(0)
    assert _lib.bsmt_block_mask_transpose(None, ctypes.byref(_BlockMaskQ()), null) == INVALID
    assert _lib.bsmt_block_mask_to_dense(None, ctypes.c_void_p(FAKE), null) == INVALID
    bm = _BlockMask()
    bm.B, bm.H, bm.QB, bm.KB = 1, 1, -1, 4
    assert _lib.bsmt_block_mask_transpose(ctypes.byref(bm), ctypes.byref(_BlockMaskQ()), null) == INVALID
    bm.QB = 4
    assert _lib.bsmt_block_mask_transpose(ctypes.byref(bm), ctypes.byref(_BlockMaskQ()), null) == INVALID  # NULL lists
    bm.kv_num_blocks = bm.kv_indices = bm.full_kv_num_blocks = bm.full_kv_indices = FAKE
    assert _lib.bsmt_block_mask_transpose(ctypes.byref(bm), None, null) == INVALID
    assert _lib.bsmt_block_mask_transpose(ctypes.byref(bm), ctypes.byref(_BlockMaskQ()), null) == INVALID
    q = _BlockMaskQ()
    q.q_num_blocks = q.q_indices = q.full_q_num_blocks = q.full_q_indices = FAKE + 2  # misaligned
    assert _lib.bsmt_block_mask_transpose(ctypes.byref(bm), ctypes.byref(q), null) == INVALID
    q.q_num_blocks = q.q_indices = q.full_q_num_blocks = q.full_q_indices = FAKE
    bm.QB = 20000
    assert _lib.bsmt_block_mask_transpose(ctypes.byref(bm), ctypes.byref(q), null) == UNSUPPORTED
    assert _lib.bsmt_block_mask_to_dense(ctypes.byref(bm), None, null) == INVALID
    bm.QB, bm.KB = 4, 0  # no kv column: nothing to write, nothing launched
    assert _lib.bsmt_block_mask_transpose(ctypes.byref(bm), ctypes.byref(q), null) == OK
    assert _lib.bsmt_block_mask_to_dense(ctypes.byref(bm), None, null) == OK


def test_splitkv_workspace_and_argument_errors():
    n = ctypes.c_int64(-1)
    assert _lib.bsmt_splitkv_workspace_bytes(2, 4, 300, 128, 1, ctypes.byref(n)) == OK and n.value == 0
    assert _lib.bsmt_splitkv_workspace_bytes(2, 4, 300, 128, 8, ctypes.byref(n)) == OK
    o_bytes = (8 * 2 * 4 * 300 * 128 * 4 + 255) // 256 * 256
    assert n.value == o_bytes + 8 * 2 * 4 * 300 * 4
    assert _lib.bsmt_splitkv_workspace_bytes(2, 4, 300, 96, 8, ctypes.byref(n)) == UNSUPPORTED
    assert _lib.bsmt_splitkv_workspace_bytes(2, 4, 300, 128, 0, ctypes.byref(n)) == INVALID
    assert _lib.bsmt_splitkv_workspace_bytes(2, 4, 300, 128, 65, ctypes.byref(n)) == INVALID
    assert _lib.bsmt_splitkv_workspace_bytes(2, 4, 300, 128, 8, None) == INVALID
    f = _lib.bsmt_flex_attention_fwd_splitkv
    args = (FAKE, FAKE, FAKE, 1, 2, 2, 128, 4096, 128, None, None, None, ctypes.c_float(0.0), 0)
    null = ctypes.c_void_p(0)
    assert f(*args, 4, None, 1 << 30, FAKE, FAKE, null) == INVALID                  # no workspace
    assert f(*args, 4, ctypes.c_void_p(FAKE + 16), 1 << 30, FAKE, FAKE, null) == INVALID  # misaligned
    assert f(*args, 4, ctypes.c_void_p(FAKE), 1024, FAKE, FAKE, null) == INVALID    # too small
    assert f(*args, 0, ctypes.c_void_p(FAKE), 1 << 30, FAKE, FAKE, null) == INVALID  # no splits


def test_static_scratch_rejects_sizes_above_its_limit():
    f = _lib.bsmt_flex_attention_fwd_splitkv_static
    null = ctypes.c_void_p(0)
    # 64 splits x 16 x 64 heads x 4096 rows x 129 floats is far above 32 MiB; rejected before any CUDA call
    r = f(FAKE, FAKE, FAKE, 16, 64, 64, 4096, 8192, 128, None, None, None, ctypes.c_float(0.0), 0, 64,
          FAKE, FAKE, null)
    assert r == UNSUPPORTED
    assert "static" in _lib.bsmt_last_error().decode() and "workspace" in _lib.bsmt_last_error().decode()
    assert f(FAKE, FAKE, FAKE, 1, 2, 2, 128, 4096, 96, None, None, None, ctypes.c_float(0.0), 0, 4,
             FAKE, FAKE, null) == UNSUPPORTED  # D = 96


def test_varlen_argument_errors():
    null = ctypes.c_void_p(0)
    assert _lib.bsmt_seqlens_to_doc_ids(None, 2, 10, None, null) == INVALID
    assert _lib.bsmt_seqlens_to_doc_ids(ctypes.c_void_p(FAKE), -1, 10, ctypes.c_void_p(FAKE), null) == INVALID
    assert _lib.bsmt_seqlens_to_doc_ids(ctypes.c_void_p(FAKE + 2), 2, 10, ctypes.c_void_p(FAKE), null) == INVALID
    assert _lib.bsmt_seqlens_to_doc_ids(None, 0, 0, None, null) == OK  # nothing to write
    f = _lib.bsmt_flex_attention_fwd_packed
    assert f(FAKE, FAKE, FAKE, 4, 3, 128, 128, 128, None, None, None, ctypes.c_float(0.0), 1, FAKE, FAKE,
             null) == SHAPE  # Hq not a multiple of Hkv
    assert f(FAKE, FAKE, FAKE, 4, 4, 128, 128, 80, None, None, None, ctypes.c_float(0.0), 0, FAKE, FAKE,
             null) == UNSUPPORTED


def bwd(B=1, Hq=2, Hkv=2, M=256, N=256, D=64, bm=None, bmq=None, spec=None, score=None, scale=0.0, gqa=0,
        ptr=FAKE, lse=FAKE, ws=FAKE, ws_bytes=1 << 30):
    return _lib.bsmt_flex_attention_bwd(ptr, ptr, ptr, ptr, ptr, lse, B, Hq, Hkv, M, N, D, bm, bmq, spec, score,
                                        ctypes.c_float(scale), gqa, ptr, ptr, ptr, ws, ws_bytes, None)


def bwd_ws(B, Hq, M):
    n = ctypes.c_int64(0)
    assert _lib.bsmt_flex_attention_bwd_workspace_bytes(B, Hq, M, ctypes.byref(n)) == OK
    return n.value


def test_backward_workspace_bytes():
    # 8 bytes per padded query row, rounded to 256, plus 256 bytes of counters
    assert bwd_ws(2, 32, 32768) == 2 * 32 * 32768 * 8 + 256
    assert bwd_ws(1, 1, 1) == 128 * 8 + 256
    assert bwd_ws(1, 3, 0) == 256
    assert _lib.bsmt_flex_attention_bwd_workspace_bytes(1, 1, 1, None) == INVALID
    assert _lib.bsmt_flex_attention_bwd_workspace_bytes(-1, 1, 1, ctypes.byref(ctypes.c_int64())) == INVALID


def test_backward_argument_errors():
    """Every check of the backward entry point runs on the host before any
    CUDA call, so these need no GPU."""
    assert bwd(D=96) == UNSUPPORTED
    assert bwd(Hq=3, Hkv=2, gqa=1) == SHAPE
    assert bwd(Hq=4, Hkv=2, gqa=0) == SHAPE
    assert bwd(M=-1) == INVALID
    assert bwd(ptr=FAKE + 8) == INVALID                      # misaligned tensors
    assert bwd(lse=FAKE + 2) == INVALID
    assert bwd(scale=float("nan")) == INVALID
    assert bwd(N=65537 * 128) == UNSUPPORTED                 # block numbers beyond 16 bits
    assert bwd(M=65537 * 128) == UNSUPPORTED
    assert bwd(Hq=256, Hkv=1, gqa=1) == UNSUPPORTED         # a GQA group beyond 255 heads
    # a block mask without its q-side lists
    c = _BlockMask()
    c.kv_num_blocks = c.kv_indices = c.full_kv_num_blocks = c.full_kv_indices = FAKE
    c.B, c.H, c.QB, c.KB, c.Q_LEN, c.KV_LEN, c.BLOCK_Q, c.BLOCK_KV = 1, 1, 2, 2, 256, 256, 128, 128
    assert bwd(bm=ctypes.byref(c), spec=ctypes.byref(spec_of([(C, 0)]))) == INVALID
    assert "q-side" in _lib.bsmt_last_error().decode()
    cq = bsmt._BlockMaskQ()
    cq.q_num_blocks = cq.q_indices = cq.full_q_num_blocks = cq.full_q_indices = FAKE
    c.QB = 3  # shape fields that disagree with M
    assert bwd(bm=ctypes.byref(c), bmq=ctypes.byref(cq), spec=ctypes.byref(spec_of([(C, 0)]))) == SHAPE
    # a workspace that is too small or misaligned (checked before any launch)
    c.QB = 2
    assert bwd(bm=ctypes.byref(c), bmq=ctypes.byref(cq), spec=ctypes.byref(spec_of([(C, 0)])), ws_bytes=100) == INVALID
    assert bwd(ws=FAKE + 16) == INVALID
    # nothing to compute: no work and no CUDA call
    assert bwd(B=0) == OK
    assert bwd(M=0, N=0) == OK
