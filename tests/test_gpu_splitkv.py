"""GPU parity: split-KV forward (slices computed as separate units, merged by
their log-sum-exps) vs the fp64 oracle, on decode-like shapes (one or two
q-blocks, long kv) and on the edge cases of the slicing."""
import numpy as np
import pytest
import torch

import block_sparse_masked_tile_b200 as bsmt
import workloads
from oracle import attention as oa
from tests.gpu_helpers import assert_attention_close

pytestmark = pytest.mark.gpu


def run(seed, B, Hq, Hkv, M, N, D, tree, mods, splits, use_block_mask=True):
    q, k, v = workloads.random_inputs(seed, B, Hq, Hkv, M, N, D)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    bm = None
    if use_block_mask:
        bm = bsmt.create_block_mask(bsmt.mask_from_tree(tree, device="cuda"), B, Hq, M, N)
    smods = bsmt.score_mods_from_list(mods)
    out, lse = bsmt.flex_attention(qd, kd, vd, block_mask=bm, score_mod=smods, enable_gqa=Hq != Hkv,
                                   num_splits=splits)
    bsmt.check_device_status()
    ref_out, ref_lse = oa.flex_attention(q, k, v, tree if use_block_mask else None, mods, None, Hq != Hkv)
    assert_attention_close(out.float().cpu().numpy(), lse.cpu().numpy(), ref_out, ref_lse, f"splits={splits}")
    return out, lse, (qd, kd, vd, bm, smods)


@pytest.mark.parametrize("splits", [2, 5, 16])
def test_decode_like_no_mask(splits):
    run(1, 1, 8, 2, 128, 4000, 128, None, (), splits, use_block_mask=False)


@pytest.mark.parametrize("D", [64, 128])
def test_masks_and_score_mods(D):
    ids = np.repeat(np.arange(3), [900, 1100, 1000]).astype(np.int32)[None]
    cases = [(("and", ("causal",), ("or", ("sink", 4), ("window", 700))), ()),
             (("document", ids[:, :256], ids), (("softcap", 20.0),)),
             (("prefix_lm", 2000), (("alibi", None),))]
    for i, (tree, mods) in enumerate(cases):
        run(10 + i, 1, 4, 4, 256, 3000, D, tree, mods, 6)


def test_sink_tiles_split():
    # the window leaves kv-block 0 for q-blocks 3..7; slices cut the stream anywhere
    run(25, 1, 4, 2, 1024, 2048, 128, ("and", ("causal",), ("or", ("sink", 4), ("window", 256))), (), 3)


def test_more_splits_than_entries_and_ragged():
    # slices beyond the entry count are empty and must merge as nothing
    run(20, 2, 2, 1, 200, 300, 128, ("causal",), (), 9)
    run(21, 1, 2, 2, 77, 1111, 64, None, (), 64, use_block_mask=False)


def test_matches_plain_path():
    out, lse, (qd, kd, vd, bm, smods) = run(30, 1, 8, 8, 128, 8192, 128, ("noop",), (), 8)
    out1, lse1 = bsmt.flex_attention(qd, kd, vd, block_mask=bm, score_mod=smods)
    assert (out.float() - out1.float()).abs().max().item() < 2e-2
    assert (lse - lse1).abs().max().item() < 1e-3


def test_workspace_reuse_and_too_small():
    q, k, v = (t.cuda() for t in workloads.random_inputs(40, 1, 2, 2, 128, 2048, 128))
    need = bsmt.splitkv_workspace_bytes(1, 2, 128, 128, 4)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    o1, l1 = bsmt.flex_attention(q, k, v, num_splits=4, workspace=ws)
    o2, l2 = bsmt.flex_attention(q, k, v, num_splits=4, workspace=ws)
    bsmt.check_device_status()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    with pytest.raises(ValueError, match="workspace"):
        bsmt.flex_attention(q, k, v, num_splits=4, workspace=ws[:need // 2])
