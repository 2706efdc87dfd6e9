"""Pins for the oracle's mask_mod evaluation and BlockMask construction.

Every expected value here comes from a closed form, from a numpy/scipy
library routine on a special case, or from the reconstruction loop on the
tensorplay.nn.attention page (BlockMask "Basics"). None comes from the oracle
itself.
"""
import numpy as np
import pytest
import scipy.linalg

from oracle import block_mask as obm
from oracle import masks as om

pytestmark = pytest.mark.filterwarnings("ignore")


def test_causal_is_lower_triangle():
    # causal mask_mod q_idx >= kv_idx (tensorplay.nn.attention, create_block_mask example)
    for M, N in [(7, 7), (5, 9), (9, 5)]:
        got = om.dense_mask(("causal",), 0, M, N)
        assert np.array_equal(got, np.tril(np.ones((M, N), bool)))


def test_noop_is_all_true():
    assert om.dense_mask(("noop",), 0, 4, 6).all()
    assert om.dense_mask(None, 0, 3, 3).all()


@pytest.mark.parametrize("W", [1, 2, 5, 17])
def test_causal_window_is_band(W):
    n = 40
    got = om.dense_mask(("and", ("causal",), ("window", W)), 0, n, n)
    band = np.tril(np.ones((n, n), bool)) & np.triu(np.ones((n, n), bool), -(W - 1))
    assert np.array_equal(got, band)
    # closed form: row i keeps min(i + 1, W) keys
    assert got.sum() == sum(min(i + 1, W) for i in range(n))


def test_window_alone_allows_future():
    n, W = 12, 3
    got = om.dense_mask(("window", W), 0, n, n)
    assert np.array_equal(got, np.triu(np.ones((n, n), bool), -(W - 1)))


@pytest.mark.parametrize("P", [0, 1, 4, 11, 30])
def test_prefix_lm_counts(P):
    n = 20
    got = om.dense_mask(("prefix_lm", P), 0, n, n)
    # closed form: row i keeps |{j < P} U {j <= i}| = max(min(P, n), i + 1) keys
    assert [int(r.sum()) for r in got] == [max(min(P, n), i + 1) for i in range(n)]


@pytest.mark.parametrize("S,W", [(4, 10), (1, 1), (0, 5), (7, 3)])
def test_sink_or_window_causal_counts(S, W):
    n = 50
    tree = ("and", ("causal",), ("or", ("sink", S), ("window", W)))
    got = om.dense_mask(tree, 0, n, n)
    # closed form per row: the window keeps min(i+1, W) keys; the sink adds the
    # keys j < S that lie left of the window, max(0, min(S, i + 1 - W)) of them
    expect = [min(i + 1, W) + max(0, min(S, i + 1 - W)) for i in range(n)]
    assert [int(r.sum()) for r in got] == expect


def test_and_or_are_set_operations():
    n = 16
    tri = np.tril(np.ones((n, n), bool))
    cols = np.broadcast_to(np.arange(n)[None, :] < 5, (n, n))
    got_or = om.dense_mask(("or", ("causal",), ("sink", 5)), 0, n, n)
    got_and = om.dense_mask(("and", ("causal",), ("sink", 5)), 0, n, n)
    assert np.array_equal(got_or, tri | cols)
    assert np.array_equal(got_and, tri & cols)
    # n-ary forms equal nested binary forms
    three = om.dense_mask(("and", ("causal",), ("sink", 9), ("window", 4)), 0, n, n)
    nested = om.dense_mask(("and", ("and", ("causal",), ("sink", 9)), ("window", 4)), 0, n, n)
    assert np.array_equal(three, nested)


def test_document_is_block_diagonal():
    lengths = [3, 1, 5, 2]
    ids = np.repeat(np.arange(len(lengths)), lengths).astype(np.int32)
    n = len(ids)
    got = om.dense_mask(("document", ids[None], ids[None]), 0, n, n)
    expect = scipy.linalg.block_diag(*[np.ones((L, L), bool) for L in lengths])
    assert np.array_equal(got, expect)
    got_c = om.dense_mask(("and", ("document", ids[None], ids[None]), ("causal",)), 0, n, n)
    expect_c = scipy.linalg.block_diag(*[np.tril(np.ones((L, L), bool)) for L in lengths])
    assert np.array_equal(got_c, expect_c)
    # closed form: sum of L(L+1)/2 allowed pairs
    assert got_c.sum() == sum(L * (L + 1) // 2 for L in lengths)


def test_document_single_doc_equals_causal():
    n = 33
    ids = np.zeros((1, n), np.int32)
    got = om.dense_mask(("and", ("document", ids, ids), ("causal",)), 0, n, n)
    assert np.array_equal(got, np.tril(np.ones((n, n), bool)))


# ---------------------------------------------------------------- BlockMask

@pytest.mark.parametrize("n", [1, 2, 5, 9])
def test_causal_block_mask_closed_form(n):
    L = 128 * n
    bm = obm.create_block_mask(("causal",), 1, 1, L, L)
    # diagonal tiles are partial, tiles left of it are full, the rest empty
    for i in range(n):
        assert bm["kv_num_blocks"][0, 0, i] == 1
        assert bm["kv_indices"][0, 0, i, 0] == i
        assert bm["full_kv_num_blocks"][0, 0, i] == i
        assert list(bm["full_kv_indices"][0, 0, i, :i]) == list(range(i))
        assert not bm["full_kv_indices"][0, 0, i, i:].any()
        assert not bm["kv_indices"][0, 0, i, 1:].any()
    assert bm["full_kv_num_blocks"].sum() == n * (n - 1) // 2
    assert bm["kv_num_blocks"].sum() == n


def test_sliding_window_block_counts():
    # causal and window 512 over 2048 tokens: row i has full tiles at distances
    # 1..3 and partial tiles at distances 0 and 4, giving 42 full and 28 partial
    n = 16
    bm = obm.create_block_mask(("and", ("causal",), ("window", 512)), 1, 1, 128 * n, 128 * n)
    for i in range(n):
        full = list(range(max(0, i - 3), i))
        part = sorted({i} | ({i - 4} if i >= 4 else set()))
        assert list(bm["full_kv_indices"][0, 0, i, :len(full)]) == full
        assert bm["full_kv_num_blocks"][0, 0, i] == len(full)
        assert list(bm["kv_indices"][0, 0, i, :len(part)]) == part
        assert bm["kv_num_blocks"][0, 0, i] == len(part)
    assert bm["full_kv_num_blocks"].sum() == 42
    assert bm["kv_num_blocks"].sum() == 28


def test_streaming_block_counts_closed_form():
    # causal and (kv < 4 or q - kv < 1024) over 32768 tokens: per row i, full
    # tiles at distances 1..7, partial at distance 0, at 8 (window edge) and
    # tile 0 when i >= 9 (the sink columns only)
    n = 256
    bm = obm.create_block_mask(("and", ("causal",), ("or", ("sink", 4), ("window", 1024))),
                               1, 1, 128 * n, 128 * n)
    full = [min(i, 7) for i in range(n)]
    part = [1 + (i >= 8) + (i >= 9) for i in range(n)]
    assert list(bm["full_kv_num_blocks"][0, 0]) == full
    assert list(bm["kv_num_blocks"][0, 0]) == part
    assert sum(full) == 1764 and sum(part) == 751


def test_reconstruction_loop_matches_tile_any():
    # tensorplay.nn.attention, BlockMask "Basics": the reconstruction loop over
    # the lists gives every tile with at least one allowed element
    rng = np.random.default_rng(3)
    M, N = 300, 420
    ids = np.repeat(np.arange(4), [70, 90, 100, 160]).astype(np.int32)
    trees = [("causal",), ("and", ("causal",), ("window", 130)),
             ("or", ("sink", 3), ("prefix_lm", 200)),
             ("and", ("document", ids[None, :M], ids[None, :N]), ("causal",))]
    for tree in trees:
        bm = obm.create_block_mask(tree, 1, 2, M, N)
        dense = om.dense_mask(tree, 0, M, N)
        QB, KB = -(-M // 128), -(-N // 128)
        any_map = np.zeros((QB, KB), np.int32)
        for i in range(QB):
            for j in range(KB):
                any_map[i, j] = int(dense[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128].any())
        rec = obm.to_dense(bm)
        for h in range(2):
            assert np.array_equal(rec[0, h], any_map)
        # lists are disjoint and ascending
        for i in range(QB):
            p = list(bm["kv_indices"][0, 0, i, :bm["kv_num_blocks"][0, 0, i]])
            f = list(bm["full_kv_indices"][0, 0, i, :bm["full_kv_num_blocks"][0, 0, i]])
            assert p == sorted(p) and f == sorted(f) and not set(p) & set(f)
    del rng


def test_ragged_edges_never_full():
    # a tile that crosses Q_LEN or KV_LEN is never FULL even under noop
    bm = obm.create_block_mask(("noop",), 1, 1, 200, 300)
    assert list(bm["full_kv_num_blocks"][0, 0]) == [2, 0]
    assert list(bm["kv_num_blocks"][0, 0]) == [1, 3]


def test_sparsity_percentage():
    bm = obm.create_block_mask(("causal",), 1, 1, 128 * 4, 128 * 4)
    # 10 of 16 tiles computed -> 37.5 % sparse
    assert obm.sparsity(bm) == pytest.approx(37.5)


def test_broadcast_b_h_none():
    bm = obm.create_block_mask(("causal",), 0, None or 0, 256, 256)
    assert bm["kv_indices"].shape == (1, 1, 2, 2)


def test_q_side_matches_tile_columns():
    # tensorplay.nn.attention, BlockMask "Details" items 3-4: the q-side lists
    # are the transpose of the kv-side ones; checked against the columns of the
    # brute-force tile classification, a path that never reads the kv lists
    ids = np.repeat(np.arange(3), [150, 200, 170]).astype(np.int32)
    M = N = 520
    trees = [("causal",), ("and", ("causal",), ("or", ("sink", 5), ("window", 200))),
             ("and", ("document", ids[None], ids[None]), ("causal",)), ("prefix_lm", 300)]
    for tree in trees:
        bm = obm.create_block_mask(tree, 1, 2, M, N)
        qs = obm.q_side(bm)
        cls = obm.tile_classes(tree, 0, M, N)
        QB, KB = cls.shape
        for h in range(2):
            for kb in range(KB):
                part = np.nonzero(cls[:, kb] == 1)[0]
                full = np.nonzero(cls[:, kb] == 2)[0]
                assert qs["q_num_blocks"][0, h, kb] == len(part)
                assert qs["full_q_num_blocks"][0, h, kb] == len(full)
                assert list(qs["q_indices"][0, h, kb, :len(part)]) == list(part)
                assert list(qs["full_q_indices"][0, h, kb, :len(full)]) == list(full)
                assert not qs["q_indices"][0, h, kb, len(part):].any()
                assert not qs["full_q_indices"][0, h, kb, len(full):].any()


def test_q_side_twice_is_the_identity():
    rng = np.random.default_rng(11)
    for _ in range(5):
        M, N = int(rng.integers(1, 700)), int(rng.integers(1, 700))
        tree = ("and", ("causal",), ("window", int(rng.integers(1, 400))))
        bm = obm.create_block_mask(tree, 2, 1, M, N)
        qs = obm.q_side(bm)
        back = obm.q_side({"kv_num_blocks": qs["q_num_blocks"], "kv_indices": qs["q_indices"],
                           "full_kv_num_blocks": qs["full_q_num_blocks"],
                           "full_kv_indices": qs["full_q_indices"]})
        assert np.array_equal(back["q_num_blocks"], bm["kv_num_blocks"])
        assert np.array_equal(back["q_indices"], bm["kv_indices"])
        assert np.array_equal(back["full_q_num_blocks"], bm["full_kv_num_blocks"])
        assert np.array_equal(back["full_q_indices"], bm["full_kv_indices"])


def test_create_mask_per_batch_documents_and_heads():
    # create_mask(mod_fn, B, H, Q_LEN, KV_LEN) returns the element mask of
    # shape (B, H, M, N) (tensorplay.nn.attention page, create_mask). With
    # document ids that differ per batch row, each [b, h] slice must be that
    # row's block-diagonal matrix (scipy.linalg.block_diag of all-ones
    # blocks, one per document) intersected with the lower triangle, the same
    # for every head.
    lens = [[3, 5, 4], [6, 6], [1, 2, 3, 6]]
    ids = np.stack([np.repeat(np.arange(len(L)), L) for L in lens]).astype(np.int32)
    B, H, L = 3, 2, 12
    tree = ("and", ("document", ids, ids), ("causal",))
    got = om.create_mask(tree, B, H, L, L)
    assert got.shape == (B, H, L, L) and got.dtype == bool
    for b in range(B):
        blocks = scipy.linalg.block_diag(*[np.ones((n, n), bool) for n in lens[b]]).astype(bool)
        want = blocks & np.tril(np.ones((L, L), bool))
        for h in range(H):
            assert np.array_equal(got[b, h], want), (b, h)
    # rows of different batch rows really differ (the per-row ids are used)
    assert not np.array_equal(got[0, 0], got[1, 0])
    # no mask at all: every element allowed, at a non-square shape
    assert om.create_mask(None, 1, 3, 5, 7).all()
