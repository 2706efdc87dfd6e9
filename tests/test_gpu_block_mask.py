"""GPU parity: the block-mask builder kernel vs the oracle, bit for bit."""
import numpy as np
import pytest
import torch

import block_sparse_masked_tile_b200 as bsmt
import workloads
from oracle import block_mask as obm
from tests.gpu_helpers import assert_block_mask_equal, block_mask_numpy, gpu_block_mask, within_dnf_limits

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("index", [1, 2, 3, 4, 5])
def test_workload_block_masks_bit_exact(index):
    w = workloads.get(index)
    data = workloads.make(w)
    tree = data["mask"]
    bm = gpu_block_mask(tree, w.B, w.Hq, w.M, w.N)
    got = block_mask_numpy(bm)
    if w.mask == "doc_causal":
        want = obm.create_block_mask(tree, w.B, 1, w.M, w.N)
    else:
        # the mask does not depend on b or h: the oracle builds one row, replicated
        want = obm.create_block_mask(tree, 1, 1, w.M, w.N)
    want = {k: np.broadcast_to(v, got[k].shape) for k, v in want.items()}
    assert_block_mask_equal(got, want)


@pytest.mark.parametrize("seed", range(24))
def test_random_specs_bit_exact(seed):
    rng = np.random.default_rng(100 + seed)
    B = int(rng.integers(1, 3))
    H = int(rng.integers(1, 4))
    M = int(rng.integers(1, 700))
    N = int(rng.integers(1, 700))
    tree = workloads.random_mask_tree(rng, B, M, N, depth=2)
    if not within_dnf_limits(tree):
        with pytest.raises(bsmt.BsmtError, match="UNSUPPORTED"):
            gpu_block_mask(tree, B, H, M, N)
        return
    bm = gpu_block_mask(tree, B, H, M, N)
    want = obm.create_block_mask(tree, B, H, M, N)
    assert_block_mask_equal(block_mask_numpy(bm), want)


@pytest.mark.parametrize("seed", range(12))
def test_deep_specs_bit_exact(seed):
    # programs four and five levels deep: most expand to more than 16
    # alternatives before the library's simplification (one leaf of a kind
    # per alternative, repeats and contained alternatives dropped), and the
    # simplified program must give the same tiles as the oracle's direct
    # evaluation of the tree
    rng = np.random.default_rng(700 + seed)
    B = int(rng.integers(1, 3))
    H = int(rng.integers(1, 3))
    M = int(rng.integers(1, 900))
    N = int(rng.integers(1, 900))
    while True:  # a program of 12 to 64 nodes
        tree = workloads.random_mask_tree(rng, B, M, N, depth=4 + seed % 2)
        if 12 <= len(bsmt.mask_from_tree(tree).nodes) <= bsmt.MAX_NODES:
            break
    if not within_dnf_limits(tree):
        with pytest.raises(bsmt.BsmtError, match="UNSUPPORTED"):
            gpu_block_mask(tree, B, H, M, N)
        return
    bm = gpu_block_mask(tree, B, H, M, N)
    want = obm.create_block_mask(tree, B, H, M, N)
    assert_block_mask_equal(block_mask_numpy(bm), want)


def _and_of_ors(L):
    ids = np.repeat(np.arange(4, dtype=np.int32), [L // 4, L // 4, L // 4, L - 3 * (L // 4)])[None]
    return ("and", ("or", ("causal",), ("sink", 64)), ("or", ("window", 300), ("prefix_lm", 200)),
            ("or", ("causal",), ("window", 500)), ("or", ("sink", 32), ("document", ids, ids)),
            ("or", ("causal",), ("prefix_lm", 100)))


def test_and_of_five_ors_bit_exact():
    # 2^5 = 32 alternatives when AND is distributed over OR, fewer once
    # simplified; the tiles must equal the oracle's direct evaluation
    L = 1000
    tree = _and_of_ors(L)
    assert within_dnf_limits(tree)
    bm = gpu_block_mask(tree, 1, 2, L, L)
    assert_block_mask_equal(block_mask_numpy(bm), obm.create_block_mask(tree, 1, 2, L, L))


def test_broadcast_none_b_h():
    tree = ("and", ("causal",), ("window", 300))
    bm = gpu_block_mask(tree, None, None, 1000, 1000)
    assert bm.shape == (1, 1, 8, 8)
    assert_block_mask_equal(block_mask_numpy(bm), obm.create_block_mask(tree, 1, 1, 1000, 1000))


def test_ragged_and_tiny():
    for M, N in [(1, 1), (1, 1000), (1000, 1), (129, 127), (128, 128), (5000, 300)]:
        for tree in [("noop",), ("causal",), ("or", ("sink", 3), ("prefix_lm", 50))]:
            bm = gpu_block_mask(tree, 1, 2, M, N)
            assert_block_mask_equal(block_mask_numpy(bm), obm.create_block_mask(tree, 1, 2, M, N))


def test_empty_lengths():
    bm = gpu_block_mask(("causal",), 1, 1, 0, 300)
    assert bm.shape == (1, 1, 0, 3)
    bm = gpu_block_mask(("causal",), 1, 1, 300, 0)
    assert bm.shape == (1, 1, 3, 0)
    assert bm.kv_num_blocks.cpu().tolist() == [[[0, 0, 0]]]
    assert bm.full_kv_num_blocks.cpu().tolist() == [[[0, 0, 0]]]


def test_long_rows_multiple_chunks():
    # KB = 600 > 256: several word chunks per row
    tree = ("and", ("causal",), ("or", ("sink", 200), ("window", 20000)))
    M = N = 600 * 128 - 50
    bm = gpu_block_mask(tree, 1, 1, M, N)
    assert_block_mask_equal(block_mask_numpy(bm), obm.create_block_mask(tree, 1, 1, M, N))


def test_unsorted_document_ids_are_reported():
    ids = torch.tensor([[0, 0, 1, 1, 0, 2, 2, 2]], dtype=torch.int32).repeat(1, 40)
    mm = bsmt.and_masks(bsmt.document(ids.cuda()), bsmt.causal())
    bsmt.create_block_mask(mm, 1, 1, ids.shape[1], ids.shape[1])
    with pytest.raises(RuntimeError, match="DEVICE_PRECONDITION"):
        bsmt.check_device_status()
    bsmt.check_device_status()  # the status word was cleared


def test_reuse_output_tensors():
    tree = ("causal",)
    mm = bsmt.mask_from_tree(tree)
    bm = bsmt.create_block_mask(mm, 1, 1, 512, 512)
    bm2 = bsmt.create_block_mask(mm, 1, 1, 512, 512, out=bm)
    assert bm2.kv_indices.data_ptr() == bm.kv_indices.data_ptr()
    assert_block_mask_equal(block_mask_numpy(bm2), obm.create_block_mask(tree, 1, 1, 512, 512))
    assert bm2.sparsity() == pytest.approx(obm.sparsity(obm.create_block_mask(tree, 1, 1, 512, 512)))
