"""Host logic of the Python binding on CPU: argument checks that must fail
loudly, with ValueError, before anything reaches the device.

None of these calls launches a kernel; each one stops at a check that runs
before the first CUDA call of its entry point.
"""
import pytest
import torch

import block_sparse_masked_tile_b200 as bsmt


def _bf16(*shape, dtype=torch.bfloat16):
    return torch.zeros(shape, dtype=dtype)


def test_mask_programs():
    with pytest.raises(ValueError, match="at least one mask"):
        bsmt.and_masks()
    with pytest.raises(ValueError, match="at least one mask"):
        bsmt.or_masks()
    a = torch.zeros(8, dtype=torch.int32)
    b = torch.zeros(8, dtype=torch.int32)
    with pytest.raises(ValueError, match="same id tensors"):
        bsmt.and_masks(bsmt.document(a), bsmt.document(b))
    with pytest.raises(ValueError, match="unknown mask kind"):
        bsmt.mask_from_tree(("diagonal",))
    # postfix programs: leaves first, then the operator with its arity
    m = bsmt.and_masks(bsmt.causal(), bsmt.or_masks(bsmt.sink(4), bsmt.sliding_window(1024)))
    assert m.nodes == ((bsmt.MASK_CAUSAL, 0), (bsmt.MASK_SINK, 4), (bsmt.MASK_WINDOW, 1024),
                       (bsmt.MASK_OR, 2), (bsmt.MASK_AND, 2))
    assert bsmt.mask_from_tree(("and", ("causal",), ("or", ("sink", 4), ("window", 1024)))).nodes == m.nodes
    # a program longer than the ABI's node array is refused when it is encoded
    big = bsmt.and_masks(*[bsmt.causal()] * bsmt.MAX_NODES)
    assert len(big.nodes) == bsmt.MAX_NODES + 1
    with pytest.raises(ValueError, match="nodes"):
        big._spec(torch.device("cpu"), 1)


def test_document_ids_need_one_batch_extent():
    m = bsmt.document(torch.zeros((2, 8), dtype=torch.int32), torch.zeros((3, 8), dtype=torch.int32))
    with pytest.raises(ValueError, match="batch extent"):
        m._spec(torch.device("cpu"), 2)


def test_score_mods():
    with pytest.raises(ValueError, match="unknown score mod"):
        bsmt.score_mods_from_list([("relu", None)])
    mods = bsmt.score_mods_from_list([("softcap", 30.0), ("alibi", None)])
    assert [m.kind for m in mods] == [bsmt.SCORE_SOFTCAP, bsmt.SCORE_ALIBI] and mods[0].value == 30.0
    with pytest.raises(ValueError, match="score mods"):
        bsmt._score_spec([bsmt.softcap(1.0)] * (bsmt.MAX_SCORE_OPS + 1), torch.device("cpu"), 4)
    with pytest.raises(ValueError, match="ALiBi slopes"):
        bsmt._score_spec([bsmt.alibi(torch.ones(3))], torch.device("cpu"), 4)
    spec, keep = bsmt._score_spec(bsmt.alibi(torch.ones(4)), torch.device("cpu"), 4)
    assert spec.num_ops == 1 and len(keep) == 1


def test_flex_attention_rejects_host_and_malformed_tensors():
    q = _bf16(1, 2, 128, 64)
    with pytest.raises(ValueError, match="bfloat16"):
        bsmt.flex_attention(_bf16(1, 2, 128, 64, dtype=torch.float32), q, q)
    with pytest.raises(ValueError, match="4-D"):
        bsmt.flex_attention(_bf16(2, 128, 64), q, q)
    with pytest.raises(ValueError, match="CUDA"):
        bsmt.flex_attention(q, q, q)


def test_split_kv_refuses_autograd():
    q = _bf16(1, 2, 128, 64).requires_grad_()
    with pytest.raises(ValueError, match="split-KV has no backward"):
        bsmt.flex_attention(q, q.detach(), q.detach(), num_splits=2)


def test_backward_rejects_host_tensors():
    t = _bf16(1, 2, 128, 64)
    with pytest.raises(ValueError, match="CUDA"):
        bsmt.flex_attention_backward(t, t, t, t, torch.zeros((1, 2, 128)), t)


def test_host_path_checks():
    q = _bf16(1, 4, 128, 64)
    kv = _bf16(1, 3, 128, 64)
    with pytest.raises(ValueError, match="CPU tensor"):
        bsmt.flex_attention_host(_bf16(1, 4, 128, 64, dtype=torch.float16), kv, kv)
    with pytest.raises(ValueError, match="shape mismatch"):
        bsmt.flex_attention_host(q, kv, _bf16(1, 3, 100, 64))
    with pytest.raises(ValueError, match="not a multiple"):
        bsmt.flex_attention_host(q, kv, kv)


def test_varlen_checks():
    with pytest.raises(ValueError, match="cu_seqlens"):
        bsmt.seqlens_to_doc_ids(torch.tensor([0, 5, 9], dtype=torch.int32), 9)
    cu_q = torch.tensor([0, 5, 9], dtype=torch.int32)
    cu_k = torch.tensor([0, 4, 9], dtype=torch.int32)
    # causal masking and ALiBi use packed positions, which only line up when q
    # and k share their sequence boundaries
    with pytest.raises(ValueError, match="share cu_seqlens"):
        bsmt._varlen_block_mask(cu_q, cu_k, 9, 9, True, [], torch.device("cpu"))
    with pytest.raises(ValueError, match="share cu_seqlens"):
        bsmt._varlen_block_mask(cu_q, cu_k, 9, 9, False, [bsmt.alibi()], torch.device("cpu"))
