"""GPU: the allocation-free split-KV entry point (static device scratch) gives
the same bits as the workspace form, on two calls in a row (the scratch is
reused), and agrees with the fp64 oracle."""
import pytest
import torch

import block_sparse_masked_tile_b200 as bsmt
import workloads
from oracle import attention as oa
from tests.gpu_helpers import assert_attention_close

pytestmark = pytest.mark.gpu


def test_static_scratch_matches_workspace_form_twice():
    cases = [(1, 8, 2, 128, 4000, 128, None, 8),
             (2, 4, 4, 256, 3000, 64, ("and", ("causal",), ("or", ("sink", 4), ("window", 700))), 6)]
    for seed, (B, Hq, Hkv, M, N, D, tree, S) in enumerate(cases):
        q, k, v = workloads.random_inputs(50 + seed, B, Hq, Hkv, M, N, D)
        qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
        bm = None if tree is None else bsmt.create_block_mask(bsmt.mask_from_tree(tree, device="cuda"), B, Hq, M, N)
        gqa = Hq != Hkv
        ref = bsmt.flex_attention(qd, kd, vd, block_mask=bm, enable_gqa=gqa, num_splits=S)
        for _ in range(2):  # two calls in a row reuse the same scratch
            got = bsmt.flex_attention(qd, kd, vd, block_mask=bm, enable_gqa=gqa, num_splits=S, workspace="static")
            bsmt.check_device_status()
            assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
        ro, rl = oa.flex_attention(q, k, v, tree, (), None, gqa)
        assert_attention_close(got[0].float().cpu().numpy(), got[1].cpu().numpy(), ro, rl, "static scratch")


def test_static_scratch_size_limit():
    q, k, v = (t.cuda() for t in workloads.random_inputs(60, 1, 32, 32, 4096, 128, 128))
    with pytest.raises(RuntimeError, match="UNSUPPORTED"):
        bsmt.flex_attention(q, k, v, num_splits=64, workspace="static")
