"""GPU parity: rows longer than 1024 kv blocks (KV_LEN > 131072).

The forward's scheduler builds each unit's tile stream in windows of 1024 kv
blocks, starting at the unit's first listed block. A unit whose blocks span
more than one window goes out as several segments, in kv order, and the
consumers carry the online softmax from one segment to the next (the
flash-attention recurrence of the FlagAttention page, "Operator overview",
visits a row's tiles in order, and a segment boundary is just a point in that
order). These tests compare that path with the fp64 oracle: whole outputs
where the oracle is quick, sampled rows around window edges where it is not;
units whose q-blocks have tiles only in the first or only in the last
segment; split-KV slices that cut across segments; ragged last tiles; and
the static-scratch entry.
"""
import numpy as np
import pytest
import torch

import block_sparse_masked_tile_b200 as bsmt
import workloads
from oracle import attention as oa
from tests.gpu_helpers import LSE_TOL, OUT_TOL, assert_attention_close

pytestmark = pytest.mark.gpu

WINDOW = 1024 * 128  # kv positions of one window


def _gpu(q, k, v, tree, mods, splits=1, workspace=None):
    B, Hq, M, _ = q.shape
    N = k.shape[2]
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    bm = None if tree is None else bsmt.create_block_mask(bsmt.mask_from_tree(tree, device="cuda"), B, Hq, M, N)
    out, lse = bsmt.flex_attention(qd, kd, vd, block_mask=bm, score_mod=bsmt.score_mods_from_list(mods),
                                   enable_gqa=Hq != k.shape[1], num_splits=splits, workspace=workspace)
    bsmt.check_device_status()
    return out, lse


def _oracle_all(q, k, v, tree, mods):
    return oa.flex_attention(q, k, v, tree, mods, None, q.shape[1] != k.shape[1])


def _compare_all(ref, out, lse, what):
    assert_attention_close(out.float().cpu().numpy(), lse.cpu().numpy(), ref[0], ref[1], what)


def _compare_rows(q, k, v, tree, mods, out, lse, rows, what):
    B, Hq = q.shape[:2]
    samples = [(b, h, r) for b in range(B) for h in range(Hq) for r in rows]
    ref_out, ref_lse = oa.flex_attention_sampled(q, k, v, samples, tree, mods, None, Hq != k.shape[1])
    o = out.float().cpu().numpy()
    ls = lse.cpu().numpy()
    got_out = np.stack([o[b, h, r] for (b, h, r) in samples])
    got_lse = np.array([ls[b, h, r] for (b, h, r) in samples])
    assert_attention_close(got_out, got_lse, ref_out, ref_lse, what)


@pytest.mark.parametrize("D", [64, 128])
def test_no_mask_two_windows_ragged(D):
    # 140000 keys: 1094 kv blocks (the last one 96 keys), two segments per
    # unit; GQA; one split and three
    q, k, v = workloads.random_inputs(70 + D, 1, 4, 2, 300, 140000, D)
    ref = _oracle_all(q, k, v, None, ())
    for splits in (1, 3):
        out, lse = _gpu(q, k, v, None, (), splits)
        _compare_all(ref, out, lse, f"D={D} splits={splits}")


def test_causal_short_queries_one_window():
    # causal with 300 queries keeps kv blocks 0..2 of 1055: one window per unit
    tree = ("causal",)
    mods = (("softcap", 20.0),)
    q, k, v = workloads.random_inputs(80, 2, 2, 2, 300, 135000, 128)
    out, lse = _gpu(q, k, v, tree, mods)
    _compare_all(_oracle_all(q, k, v, tree, mods), out, lse, "causal, short queries")


def test_window_and_sink_across_the_window_edge():
    # M = N = 140000; rows past 131072 keep the sink block 0 and window
    # blocks beyond the first window: units of two segments, the first
    # holding the sink tile only
    tree = ("and", ("causal",), ("or", ("sink", 4), ("window", 2048)))
    mods = (("alibi", None),)
    q, k, v = workloads.random_inputs(81, 1, 2, 1, 140000, 140000, 64)
    rows = list(range(0, 40)) + list(range(WINDOW - 200, WINDOW + 200)) + list(range(139900, 140000))
    first = None
    for splits in (1, 4):
        out, lse = _gpu(q, k, v, tree, mods, splits)
        _compare_rows(q, k, v, tree, mods, out, lse, rows, f"window+sink splits={splits}")
        if first is None:
            first = (out, lse)
        else:  # the two paths agree everywhere, not only on the sampled rows
            assert (out.float() - first[0].float()).abs().max().item() <= OUT_TOL
            assert (lse - first[1]).abs().max().item() <= LSE_TOL


def test_document_spanning_the_window_edge():
    # one document runs from 120000 to 135000, across kv block 1024; the
    # others are short. Each unit's window starts at its first listed block.
    lengths = [5000, 60000, 55000, 15000, 3000, 12000]
    assert sum(lengths) == 150000 and sum(lengths[:3]) == 120000
    ids = np.repeat(np.arange(len(lengths)), lengths).astype(np.int32)[None]
    tree = ("and", ("document", ids, ids), ("causal",))
    q, k, v = workloads.random_inputs(82, 1, 1, 1, 150000, 150000, 128)
    rows = (list(range(120000, 120100)) + list(range(WINDOW - 100, WINDOW + 100)) +
            list(range(134900, 135100)) + list(range(149950, 150000)))
    for splits in (1, 2):
        out, lse = _gpu(q, k, v, tree, (), splits)
        _compare_rows(q, k, v, tree, (), out, lse, rows, f"document across the window edge, splits={splits}")


def test_q_blocks_in_different_segments():
    # Query document ids need not be sorted. Pair (0, 1): q-block 0 reads
    # document 0 (kv blocks 0..15) and q-block 1 document 2 (blocks
    # 1015..1031), so the unit's first segment holds q-block 0's tiles only
    # and its last q-block 1's; pair (2, 3) the other way round; q-block 4,
    # alone in its pair, mixes rows of both documents, so its row state
    # crosses the segments. GQA, soft-cap, and split-KV slices cut across the
    # segments.
    N = 132000
    kv_ids = np.repeat(np.array([0, 1, 2], np.int32), [2000, 128000, 2000])[None]
    blocks = [np.full(128, d, np.int32) for d in (0, 2, 2, 0)] + [np.tile(np.array([0, 2], np.int32), 64)]
    q_ids = np.concatenate(blocks)[None]
    tree = ("document", q_ids, kv_ids)
    mods = (("softcap", 25.0),)
    q, k, v = workloads.random_inputs(85, 1, 2, 1, 640, N, 128)
    ref = _oracle_all(q, k, v, tree, mods)
    for splits in (1, 3):
        out, lse = _gpu(q, k, v, tree, mods, splits)
        _compare_all(ref, out, lse, f"documents in different segments, splits={splits}")


def test_static_scratch_long_kv_matches_workspace_form():
    q, k, v = workloads.random_inputs(83, 1, 2, 2, 300, 140000, 128)
    ref = _gpu(q, k, v, None, (), 2)
    for _ in range(2):
        got = _gpu(q, k, v, None, (), 2, workspace="static")
        assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
    # the workspace does not grow with N
    assert bsmt.splitkv_workspace_bytes(1, 2, 300, 128, 2) == (2 * 600 * 128 * 4 + 255) // 256 * 256 + 2 * 600 * 4


def test_host_entry_long_rows():
    # the host-buffer entry over rows of more than one window: its pieces run
    # the same kernels, so the bits equal the device path's
    q, k, v = workloads.random_inputs(86, 1, 4, 2, 300, 140000, 64)
    tree = ("or", ("sink", 4), ("window", 3000))
    mm = bsmt.mask_from_tree(tree, device="cuda")
    out_h, lse_h = bsmt.flex_attention_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), mask_mod=mm,
                                            enable_gqa=True, chunks=2)
    bm = bsmt.create_block_mask(mm, 1, 4, 300, 140000)
    out_d, lse_d = bsmt.flex_attention(q.cuda(), k.cuda(), v.cuda(), block_mask=bm, enable_gqa=True)
    bsmt.check_device_status()
    assert torch.equal(out_h, out_d.cpu()) and torch.equal(lse_h, lse_d.cpu())
    _compare_all(_oracle_all(q, k, v, tree, ()), out_d, lse_d, "host entry, long rows")


def test_varlen_pack_longer_than_one_window():
    # 150 packed sequences, 160k tokens in all: the pack's kv blocks exceed
    # one window, each unit's listed blocks lie within its own sequences
    rng = np.random.default_rng(87)
    lens = rng.integers(300, 1900, size=150)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    total = int(cu[-1])
    assert total > WINDOW
    g = torch.Generator().manual_seed(88)
    q, k, v = (torch.randn((total, h, 64), generator=g).to(torch.bfloat16) for h in (4, 2, 2))
    cuq = torch.from_numpy(cu).cuda()
    out, lse = bsmt.flex_attention_varlen(q.cuda(), k.cuda(), v.cuda(), cuq, cuq, causal=True, enable_gqa=True)
    bsmt.check_device_status()
    ro, rl = oa.flex_attention_varlen(q, k, v, cu, cu, True, (), None, True)
    # out [total, Hq, D] and lse [Hq, total]; every causal row sees its own key
    assert np.abs(out.float().cpu().numpy() - ro).max() <= OUT_TOL
    got_l = lse.cpu().numpy()
    assert np.all(np.isfinite(rl)) and np.all(np.isfinite(got_l))
    assert np.abs(got_l - rl).max() <= LSE_TOL


def test_two_batch_rows_documents_per_row():
    # B = 2 with different document ids per batch row (doc_batch = 2) and GQA;
    # row 1's first document spans the window edge, row 0's does not
    N = 136000
    lens0 = [60000, 76000]
    lens1 = [120000, 16000]
    ids = np.stack([np.repeat(np.arange(2), lens0), np.repeat(np.arange(2), lens1)]).astype(np.int32)
    tree = ("and", ("document", ids, ids), ("causal",))
    q, k, v = workloads.random_inputs(89, 2, 2, 1, N, N, 64)
    rows = list(range(WINDOW - 64, WINDOW + 64)) + list(range(119900, 120100)) + list(range(135900, 136000))
    for splits in (1, 3):
        out, lse = _gpu(q, k, v, tree, (), splits)
        _compare_rows(q, k, v, tree, (), out, lse, rows, f"two batch rows, splits={splits}")
