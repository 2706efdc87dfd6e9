"""GPU: flex_attention_host (host tensors, copies pipelined with the attention
of independent pieces) gives the same bits as the device path, and matches
the oracle where the score mod is per head (ALiBi)."""
import numpy as np
import pytest
import torch

import block_sparse_masked_tile_b200 as bsmt
import workloads
from oracle import attention as oa
from tests.gpu_helpers import assert_attention_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,Hq,Hkv,M,N,D,chunks", [(2, 8, 2, 300, 500, 128, 8), (3, 4, 4, 256, 256, 64, 5),
                                                   (1, 16, 4, 700, 900, 128, 3)])
def test_host_path_matches_device_path(B, Hq, Hkv, M, N, D, chunks):
    q, k, v = workloads.random_inputs(70, B, Hq, Hkv, M, N, D)
    tree = ("and", ("causal",), ("or", ("sink", 8), ("window", 200)))
    mm = bsmt.mask_from_tree(tree, device="cuda")
    gqa = Hq != Hkv
    out_h, lse_h = bsmt.flex_attention_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), mask_mod=mm,
                                            score_mod=bsmt.softcap(30.0), enable_gqa=gqa, chunks=chunks)
    bm = bsmt.create_block_mask(mm, B, Hq, M, N)
    out_d, lse_d = bsmt.flex_attention(q.cuda(), k.cuda(), v.cuda(), block_mask=bm, score_mod=bsmt.softcap(30.0),
                                       enable_gqa=gqa)
    bsmt.check_device_status()
    assert torch.equal(out_h, out_d.cpu()) and torch.equal(lse_h, lse_d.cpu())


def test_host_path_documents_per_batch_row_and_alibi():
    B, Hq, Hkv, M, N, D = 2, 4, 2, 384, 384, 64
    q, k, v = workloads.random_inputs(71, B, Hq, Hkv, M, N, D)
    ids = np.stack([np.repeat(np.arange(3), [100, 150, 134]), np.repeat(np.arange(2), [300, 84])]).astype(np.int32)
    tree = ("and", ("document", ids, ids), ("causal",))
    mm = bsmt.mask_from_tree(tree, device="cuda")
    out_h, lse_h = bsmt.flex_attention_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), mask_mod=mm,
                                            score_mod=bsmt.alibi(), enable_gqa=True, chunks=4)
    bsmt.check_device_status()
    ro, rl = oa.flex_attention(q, k, v, tree, (("alibi", None),), None, True)
    assert_attention_close(out_h.float().numpy(), lse_h.numpy(), ro, rl, "host path")
