"""GPU parity: the q-side BlockMask lists (transpose kernel), the block-level
dense map and BlockMask.from_kv_blocks vs the oracle, bit for bit."""
import numpy as np
import pytest
import torch

import block_sparse_masked_tile_b200 as bsmt
import workloads
from oracle import block_mask as obm
from tests.gpu_helpers import gpu_block_mask, within_dnf_limits

pytestmark = pytest.mark.gpu

Q_KEYS = ("q_num_blocks", "q_indices", "full_q_num_blocks", "full_q_indices")


def assert_q_side_equal(bm, want: dict):
    got = bm.q_side()
    bsmt.check_device_status()
    for key in Q_KEYS:
        g, w = got[key].cpu().numpy(), want[key]
        assert g.shape == w.shape, (key, g.shape, w.shape)
        if not np.array_equal(g, w):
            bad = np.argwhere(g != w)[:5]
            raise AssertionError(f"{key} differs at {bad.tolist()}")


@pytest.mark.parametrize("index", [1, 2, 3, 4, 5])
def test_workload_q_side_and_dense(index):
    w = workloads.get(index)
    tree = workloads.make(w)["mask"]
    bm = gpu_block_mask(tree, 1, 1, w.M, w.N)
    want = obm.create_block_mask(tree, 1, 1, w.M, w.N)
    assert_q_side_equal(bm, obm.q_side(want))
    dense = bm.to_dense()
    bsmt.check_device_status()
    assert np.array_equal(dense.cpu().numpy(), obm.to_dense(want))


@pytest.mark.parametrize("seed", range(12))
def test_random_specs_q_side(seed):
    rng = np.random.default_rng(300 + seed)
    B, H = int(rng.integers(1, 3)), int(rng.integers(1, 3))
    M, N = int(rng.integers(1, 900)), int(rng.integers(1, 900))
    tree = workloads.random_mask_tree(rng, B, M, N, depth=2)
    if not within_dnf_limits(tree):
        return
    bm = gpu_block_mask(tree, B, H, M, N)
    want = obm.create_block_mask(tree, B, H, M, N)
    assert_q_side_equal(bm, obm.q_side(want))
    assert np.array_equal(bm.to_dense().cpu().numpy(), obm.to_dense(want))


def test_many_q_blocks_and_full_batch():
    # QB = 300 (several bitmap words per column), B = 2, H = 3
    tree = ("and", ("causal",), ("or", ("sink", 64), ("window", 2000)))
    M = N = 300 * 128 - 17
    bm = gpu_block_mask(tree, 2, 3, M, N)
    want = obm.create_block_mask(tree, 1, 1, M, N)
    want = {k: np.broadcast_to(v, (2, 3) + v.shape[2:]).copy() for k, v in want.items()}
    assert_q_side_equal(bm, obm.q_side(want))


def test_from_kv_blocks_random_lists():
    # lists drawn here (any order, disjoint within a row), not by the builder
    rng = np.random.default_rng(7)
    Bm, Hm, QB, KB = 2, 2, 37, 45
    kv_num = np.zeros((Bm, Hm, QB), np.int32)
    kv_idx = np.zeros((Bm, Hm, QB, KB), np.int32)
    full_num = np.zeros((Bm, Hm, QB), np.int32)
    full_idx = np.zeros((Bm, Hm, QB, KB), np.int32)
    for b in range(Bm):
        for h in range(Hm):
            for qb in range(QB):
                perm = rng.permutation(KB)
                n1, n2 = int(rng.integers(0, KB // 2)), int(rng.integers(0, KB // 2))
                kv_num[b, h, qb], full_num[b, h, qb] = n1, n2
                kv_idx[b, h, qb, :n1] = perm[:n1]
                full_idx[b, h, qb, :n2] = perm[n1:n1 + n2]
    t = [torch.from_numpy(x).cuda() for x in (kv_num, kv_idx, full_num, full_idx)]
    bm = bsmt.BlockMask.from_kv_blocks(*t)
    want = {"kv_num_blocks": kv_num, "kv_indices": kv_idx, "full_kv_num_blocks": full_num,
            "full_kv_indices": full_idx}
    assert bm.seq_lengths == (QB * 128, KB * 128)
    assert_q_side_equal(bm, obm.q_side(want))
    assert np.array_equal(bm.to_dense().cpu().numpy(), obm.to_dense(want))
    with pytest.raises(ValueError):
        bsmt.BlockMask.from_kv_blocks(t[0], t[1][0])


def test_bad_lists_are_reported():
    """Counts above KB and indices outside [0, KB) are skipped before any access
    and reported as DEVICE_BOUNDS."""
    kv_num = torch.tensor([[[2, 1]]], dtype=torch.int32).cuda()
    kv_idx = torch.tensor([[[[0, 5], [1, 0]]]], dtype=torch.int32).cuda()   # 5 >= KB = 2
    full_num = torch.tensor([[[0, 9]]], dtype=torch.int32).cuda()           # 9 > KB
    full_idx = torch.zeros((1, 1, 2, 2), dtype=torch.int32).cuda()
    bm = bsmt.BlockMask.from_kv_blocks(kv_num, kv_idx, full_num, full_idx)
    with pytest.raises(RuntimeError, match="DEVICE_BOUNDS"):
        bsmt.check_device_status()
    bm.to_dense()
    with pytest.raises(RuntimeError, match="DEVICE_BOUNDS"):
        bsmt.check_device_status()
    bsmt.check_device_status()
