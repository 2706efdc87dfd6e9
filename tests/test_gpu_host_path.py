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


def test_host_entry_through_the_c_abi_matches_the_oracle():
    """bsmt_flex_attention_host called directly (ctypes, no binding logic):
    pinned host q/k/v in, pinned host out/lse back, a caller workspace, the
    StreamingLLM mask with GQA and ALiBi (default slopes, cut per piece) and
    more pieces than batch rows."""
    import ctypes
    B, Hq, Hkv, M, N, D = 2, 8, 2, 640, 640, 128
    q, k, v = workloads.random_inputs(72, B, Hq, Hkv, M, N, D)
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    oh = torch.empty((B, Hq, M, D), dtype=torch.bfloat16).pin_memory()
    lh = torch.empty((B, Hq, M), dtype=torch.float32).pin_memory()
    tree = ("and", ("causal",), ("or", ("sink", 4), ("window", 200)))
    mspec, keep = bsmt.mask_from_tree(tree)._spec(torch.device("cpu"), B)
    sspec, keep_s = bsmt._score_spec([bsmt.alibi()], torch.device("cpu"), Hq)
    n = ctypes.c_int64(0)
    assert bsmt._lib.bsmt_flex_attention_host_workspace_bytes(B, Hq, Hkv, M, N, D, ctypes.byref(mspec),
                                                              ctypes.byref(n)) == 0
    ws = torch.empty(n.value, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    st = bsmt._lib.bsmt_flex_attention_host(qh.data_ptr(), kh.data_ptr(), vh.data_ptr(), B, Hq, Hkv, M, N, D,
                                            ctypes.byref(mspec), ctypes.byref(sspec), ctypes.c_float(0.0), 1, 4,
                                            ctypes.c_void_p(ws.data_ptr()), ws.numel(), oh.data_ptr(),
                                            lh.data_ptr(), ctypes.c_void_p(stream.cuda_stream))
    assert st == 0, bsmt._lib.bsmt_last_error()
    stream.synchronize()
    bsmt.check_device_status()
    ro, rl = oa.flex_attention(q, k, v, tree, (("alibi", None),), None, True)
    assert_attention_close(oh.float().numpy(), lh.numpy(), ro, rl, "host entry")


def test_host_path_explicit_slopes_and_no_mask():
    B, Hq, Hkv, M, N, D = 1, 6, 3, 300, 400, 64
    q, k, v = workloads.random_inputs(73, B, Hq, Hkv, M, N, D)
    slopes = torch.tensor([0.5, 0.3, 0.2, 0.1, 0.05, 0.01], dtype=torch.float32)
    out_h, lse_h = bsmt.flex_attention_host(q.pin_memory(), k.pin_memory(), v.pin_memory(),
                                            score_mod=[bsmt.alibi(slopes), bsmt.softcap(20.0)], enable_gqa=True,
                                            chunks=3)
    out_d, lse_d = bsmt.flex_attention(q.cuda(), k.cuda(), v.cuda(), score_mod=[bsmt.alibi(slopes.cuda()),
                                                                                bsmt.softcap(20.0)],
                                       enable_gqa=True)
    bsmt.check_device_status()
    assert torch.equal(out_h, out_d.cpu()) and torch.equal(lse_h, lse_d.cpu())


def test_alibi_default_slopes_of_a_head_slice():
    """alibi(head_offset=h0, num_heads=Hq) on heads [h0, h1) gives the same
    bits as those heads of a call over all Hq heads: the library derives the
    default slopes of the slice."""
    B, Hq, Hkv, M, N, D = 1, 8, 2, 384, 384, 128
    q, k, v = (t.cuda() for t in workloads.random_inputs(74, B, Hq, Hkv, M, N, D))
    bm = bsmt.create_block_mask(bsmt.causal(), B, None, M, N)
    full_o, full_l = bsmt.flex_attention(q, k, v, block_mask=bm, score_mod=bsmt.alibi(), enable_gqa=True)
    for g0, g1 in ((0, 1), (1, 2)):
        h0, h1 = g0 * 4, g1 * 4
        o, l = bsmt.flex_attention(q[:, h0:h1].contiguous(), k[:, g0:g1].contiguous(), v[:, g0:g1].contiguous(),
                                   block_mask=bm, score_mod=bsmt.alibi(head_offset=h0, num_heads=Hq),
                                   enable_gqa=True)
        bsmt.check_device_status()
        assert torch.equal(o, full_o[:, h0:h1]) and torch.equal(l, full_l[:, h0:h1])
