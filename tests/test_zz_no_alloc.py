"""GPU: the allocation-free split-KV entry point.

bsmt_flex_attention_fwd_splitkv_static serves callers that cannot allocate
device memory (a server whose memory manager owns the whole device, a
plug-in whose host framework owns every allocation): it takes its split-KV
workspace from a static device array inside the library. These tests call it
through the C ABI (the binding's ``workspace="static"``) and check that it
gives the same bits as the workspace form on two calls in a row (the shared
scratch keeps the previous call's contents), that it agrees with the fp64
oracle, and that its size limit sits exactly where the workspace formula
puts it.
"""
import pytest
import torch

import block_sparse_masked_tile_b200 as bsmt
import workloads
from oracle import attention as oa
from tests.gpu_helpers import assert_attention_close

pytestmark = pytest.mark.gpu

SCRATCH = 32 << 20  # BSMT_SPLITKV_SCRATCH_BYTES


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


def test_static_scratch_size_limit_boundary():
    # 2 splits at D = 128: the workspace is 2 * M * 128 * 4 bytes of partial
    # outputs (a multiple of 256) plus 2 * M * 4 bytes of lse. M = 32513
    # needs 33,553,416 bytes (1016 under the scratch) and must run and match
    # the workspace form bit for bit; M = 32514 needs 16 bytes more than the
    # scratch holds and must be refused.
    D, S, N = 128, 2, 1024
    for M, fits in ((32513, True), (32514, False)):
        need = bsmt.splitkv_workspace_bytes(1, 1, M, D, S)
        assert (need <= SCRATCH) == fits, (M, need)
        q, k, v = (t.cuda() for t in workloads.random_inputs(61, 1, 1, 1, M, N, D))
        if fits:
            ref = bsmt.flex_attention(q, k, v, num_splits=S)
            got = bsmt.flex_attention(q, k, v, num_splits=S, workspace="static")
            bsmt.check_device_status()
            assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
        else:
            with pytest.raises(RuntimeError, match="UNSUPPORTED"):
                bsmt.flex_attention(q, k, v, num_splits=S, workspace="static")
