"""GPU parity: the tcgen05 attention kernel vs the fp64 oracle.

Small cases are compared element by element over every output. The five
workloads are compared at full size: exhaustively where the oracle finishes
in seconds, otherwise on sampled query rows that the oracle computes one by
one. Sampled rows include the first and last row of several q-blocks.
Tolerances: out max-abs 2e-2, lse max-abs 1e-2, and -inf lse exactly where
the oracle has it.
"""
import numpy as np
import pytest
import torch

import block_sparse_masked_tile_b200 as bsmt
import workloads
from oracle import attention as oa
from tests.gpu_helpers import assert_attention_close, gpu_attention, within_dnf_limits

pytestmark = pytest.mark.gpu


def run_case(seed, B, Hq, Hkv, M, N, D, tree, mods, scale=None, mask_B=None, mask_H=None, use_block_mask=True):
    q, k, v = workloads.random_inputs(seed, B, Hq, Hkv, M, N, D)
    gqa = Hq != Hkv
    if use_block_mask and not within_dnf_limits(tree):
        with pytest.raises(bsmt.BsmtError, match="UNSUPPORTED"):
            gpu_attention(q, k, v, tree, mods, scale, gqa, mask_B, mask_H, use_block_mask)
        return None
    out, lse = gpu_attention(q, k, v, tree, mods, scale, gqa, mask_B, mask_H, use_block_mask)
    ref_out, ref_lse = oa.flex_attention(q, k, v, tree if use_block_mask else None, mods, scale, gqa)
    return assert_attention_close(out, lse, ref_out, ref_lse, f"seed={seed}")


def test_workload1_full():
    w = workloads.get(1)
    d = workloads.make(w)
    out, lse = gpu_attention(d["q"], d["k"], d["v"], d["mask"], d["score_mods"], w.scale, w.enable_gqa)
    ref_out, ref_lse = oa.flex_attention(d["q"], d["k"], d["v"], d["mask"], d["score_mods"], w.scale, w.enable_gqa)
    assert_attention_close(out, lse, ref_out, ref_lse, w.name)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("mods", [(), (("softcap", 30.0),), (("alibi", None),),
                                  (("softcap", 5.0), ("alibi", None)), (("alibi", None), ("softcap", 5.0))])
def test_score_mods(D, mods):
    run_case(7, 1, 2, 2, 384, 384, D, ("causal",), mods)


@pytest.mark.parametrize("D", [64, 128])
def test_dense_no_block_mask(D):
    run_case(11, 2, 2, 1, 256, 384, D, None, (), use_block_mask=False)


@pytest.mark.parametrize("M,N", [(300, 200), (129, 513), (1, 1), (100, 1000), (1000, 100)])
def test_ragged_lengths(M, N):
    run_case(13, 1, 2, 2, M, N, 128, ("and", ("causal",), ("window", 150)), ())
    run_case(14, 1, 1, 1, M, N, 64, None, (), use_block_mask=False)


@pytest.mark.parametrize("seed", range(16))
def test_random_masks_and_shapes(seed):
    rng = np.random.default_rng(500 + seed)
    D = int(rng.choice([64, 128]))
    Hkv = int(rng.integers(1, 3))
    Hq = Hkv * int(rng.choice([1, 2, 4]))
    B = int(rng.integers(1, 3))
    M = int(rng.integers(1, 800))
    N = int(rng.integers(1, 800))
    tree = workloads.random_mask_tree(rng, B, M, N, depth=2)
    mods = [(), (("softcap", 20.0),), (("alibi", None),)][int(rng.integers(3))]
    run_case(seed, B, Hq, Hkv, M, N, D, tree, mods)


@pytest.mark.parametrize("seed", range(8))
def test_deep_masks(seed):
    # four-level programs, simplified by the library before the kernels see
    # them (more than 4 alternatives take the kernel's general mask path)
    rng = np.random.default_rng(900 + seed)
    D = int(rng.choice([64, 128]))
    Hkv = int(rng.integers(1, 3))
    Hq = Hkv * int(rng.choice([1, 2]))
    M = int(rng.integers(100, 700))
    N = int(rng.integers(100, 700))
    tree = workloads.random_mask_tree(rng, 1, M, N, depth=4)
    mods = [(), (("softcap", 20.0),), (("alibi", None),)][int(rng.integers(3))]
    run_case(seed, 1, Hq, Hkv, M, N, D, tree, mods)


def test_and_of_five_ors():
    # 32 alternatives before the library's simplification
    from tests.test_gpu_block_mask import _and_of_ors
    run_case(77, 1, 4, 2, 1000, 1000, 128, _and_of_ors(1000), (("alibi", None),))


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("S", [1, 4, 31, 32, 33])
def test_sink_tiles(D, S):
    # Once the window no longer reaches kv-block 0, the sink tile allows only
    # its first S columns in every row of a q-block (StreamingLLM's shape at
    # several sink sizes).
    run_case(40 + S, 1, 2, 1, 1024, 1024, D, ("and", ("causal",), ("or", ("sink", S), ("window", 256))), ())


@pytest.mark.parametrize("mods", [(("softcap", 20.0),), (("alibi", None),), (("softcap", 5.0), ("alibi", None)),
                                  (("alibi", None), ("softcap", 5.0))])
def test_sink_tiles_score_mods_gqa_ragged(mods):
    run_case(50, 2, 4, 2, 1000, 1100, 128, ("and", ("causal",), ("or", ("sink", 8), ("window", 300))), mods)


@pytest.mark.parametrize("D", [64, 128])
def test_sink_only(D):
    # causal and sink(4) alone: each q-block has a single partial tile, which
    # both starts and finishes its O
    run_case(60, 1, 2, 2, 640, 640, D, ("and", ("causal",), ("sink", 4)), ())


def test_broadcast_block_mask():
    run_case(21, 2, 4, 2, 512, 512, 128, ("and", ("causal",), ("window", 200)), (), mask_B=None, mask_H=None)
    tree = ("and", ("causal",), ("window", 200))
    q, k, v = workloads.random_inputs(22, 2, 4, 2, 512, 512, 128)
    bm = bsmt.create_block_mask(bsmt.mask_from_tree(tree), None, None, 512, 512)
    out, lse = bsmt.flex_attention(q.cuda(), k.cuda(), v.cuda(), block_mask=bm, enable_gqa=True)
    bsmt.check_device_status()
    ro, rl = oa.flex_attention(q, k, v, tree, (), None, True)
    assert_attention_close(out.float().cpu().numpy(), lse.cpu().numpy(), ro, rl, "broadcast")


def test_fully_masked_rows():
    # window 0 with causal allows nothing: every row is 0 / -inf
    run_case(31, 1, 2, 2, 300, 300, 64, ("and", ("causal",), ("window", 0)), ())
    # a sink of zero tokens allows nothing either
    run_case(32, 1, 1, 1, 200, 200, 128, ("sink", 0), ())
    # mixed: document ids where some queries have a document that holds no key
    ids_q = np.repeat(np.arange(4), [50, 50, 50, 106]).astype(np.int32)[None]
    ids_kv = np.repeat(np.arange(3), [60, 60, 136]).astype(np.int32)[None]
    run_case(33, 1, 1, 1, 256, 256, 64, ("document", ids_q, ids_kv), ())


def test_empty_inputs():
    q, k, v = workloads.random_inputs(40, 1, 2, 2, 0, 64, 64)
    out, lse = bsmt.flex_attention(q.cuda(), k.cuda(), v.cuda())
    assert out.shape == (1, 2, 0, 64)
    q, k, v = workloads.random_inputs(41, 1, 2, 2, 70, 0, 64)
    out, lse = bsmt.flex_attention(q.cuda(), k.cuda(), v.cuda())
    bsmt.check_device_status()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))


def sampled_rows(rng, w, count):
    rows = []
    qbs = sorted(set([0, w.M // 128 - 1] + list(rng.integers(0, (w.M + 127) // 128, size=count // 4))))
    for qb in qbs:
        for r in (0, 127, int(rng.integers(1, 127))):
            rows.append((int(rng.integers(w.B)), int(rng.integers(w.Hq)), qb * 128 + r))
    while len(rows) < count:
        rows.append((int(rng.integers(w.B)), int(rng.integers(w.Hq)), int(rng.integers(w.M))))
    return rows


@pytest.mark.parametrize("index", [2, 3, 4, 5])
def test_workloads_full_size_sampled(index):
    w = workloads.get(index)
    d = workloads.make(w)
    out, lse = gpu_attention(d["q"], d["k"], d["v"], d["mask"], d["score_mods"], w.scale, w.enable_gqa)
    assert np.all(np.isfinite(out))
    rng = np.random.default_rng(index)
    samples = sampled_rows(rng, w, 96)
    so, sl = oa.flex_attention_sampled(d["q"], d["k"], d["v"], samples, d["mask"], d["score_mods"], w.scale,
                                       w.enable_gqa)
    go = np.stack([out[b, h, r] for b, h, r in samples])
    gl = np.array([lse[b, h, r] for b, h, r in samples])
    assert_attention_close(go, gl, so, sl, w.name)


def test_workload2_full_exhaustive():
    w = workloads.get(2)
    d = workloads.make(w)
    out, lse = gpu_attention(d["q"], d["k"], d["v"], d["mask"], d["score_mods"], w.scale, w.enable_gqa)
    ref_out, ref_lse = oa.flex_attention(d["q"], d["k"], d["v"], d["mask"], d["score_mods"], w.scale, w.enable_gqa)
    assert_attention_close(out, lse, ref_out, ref_lse, w.name)


def _compare_slices(out, lse, tasks, results, what):
    go = np.concatenate([out[b, hq, r0:r1] for (b, hq, r0, r1) in tasks])
    gl = np.concatenate([lse[b, hq, r0:r1] for (b, hq, r0, r1) in tasks])
    ro = np.concatenate([o for o, _ in results])
    rl = np.concatenate([l for _, l in results])
    assert_attention_close(go, gl, ro, rl, what)


def test_workload3_full_exhaustive():
    # causal + ALiBi at D = 64: every (b, hq) and every row, oracle in a pool
    from tests import oracle_pool
    w = workloads.get(3)
    d = workloads.make(w)
    out, lse = gpu_attention(d["q"], d["k"], d["v"], d["mask"], d["score_mods"], w.scale, w.enable_gqa)
    tasks = oracle_pool.row_tasks([(b, h) for b in range(w.B) for h in range(w.Hq)], w.M, w.M)
    res = oracle_pool.forward_rows(d["q"], d["k"], d["v"], tasks, d["mask"], d["score_mods"], w.scale)
    _compare_slices(out, lse, tasks, res, w.name)


def test_workload4_whole_heads():
    # document and causal: every row of four query heads
    from tests import oracle_pool
    w = workloads.get(4)
    d = workloads.make(w)
    out, lse = gpu_attention(d["q"], d["k"], d["v"], d["mask"], d["score_mods"], w.scale, w.enable_gqa)
    tasks = oracle_pool.row_tasks([(0, 0), (0, 11), (0, 20), (0, 31)], w.M, 4096)
    res = oracle_pool.forward_rows(d["q"], d["k"], d["v"], tasks, d["mask"], d["score_mods"], w.scale)
    _compare_slices(out, lse, tasks, res, w.name)


def test_workload5_whole_heads_and_transition_blocks():
    # StreamingLLM at full size: every row of two (b, hq) slices, one per
    # batch row and in different GQA groups, and every row of q-blocks 0-10
    # (where the window leaves the sink's block) for all four query heads of
    # one kv head
    from tests import oracle_pool
    w = workloads.get(5)
    d = workloads.make(w)
    out, lse = gpu_attention(d["q"], d["k"], d["v"], d["mask"], d["score_mods"], w.scale, w.enable_gqa)
    group = w.Hq // w.Hkv
    tasks = oracle_pool.row_tasks([(0, 3), (1, 30)], w.M, 4096)
    tasks += [(1, h, 0, 11 * 128) for h in range(5 * group, 6 * group)]
    res = oracle_pool.forward_rows(d["q"], d["k"], d["v"], tasks, d["mask"], d["score_mods"], w.scale)
    _compare_slices(out, lse, tasks, res, w.name)


def test_repeatable_and_deterministic():
    w = workloads.get(1)
    d = workloads.make(w)
    a = gpu_attention(d["q"], d["k"], d["v"], d["mask"], (), None, False)
    b = gpu_attention(d["q"], d["k"], d["v"], d["mask"], (), None, False)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_invalid_block_mask_is_reported():
    """Block indices outside [0, KB) and counts above KB are caught before any
    access: the kernel skips them and sets DEVICE_BOUNDS in the status word."""
    import dataclasses
    q, k, v = (t.cuda() for t in workloads.random_inputs(45, 1, 2, 2, 512, 512, 64))
    bm = bsmt.create_block_mask(bsmt.causal(), 1, 2, 512, 512)
    KB = bm.shape[-1]
    bad_index = dataclasses.replace(bm, kv_indices=bm.kv_indices.clone())
    bad_index.kv_indices[0, 0, 1, 0] = KB           # one past the last block
    bad_index.kv_indices[0, 1, 2, 0] = -1
    bad_count = dataclasses.replace(bm, full_kv_num_blocks=bm.full_kv_num_blocks.clone())
    bad_count.full_kv_num_blocks[0, 1, 3] = KB + 7
    for bad in (bad_index, bad_count):
        bsmt.flex_attention(q, k, v, block_mask=bad)
        with pytest.raises(RuntimeError, match="DEVICE_BOUNDS"):
            bsmt.check_device_status()
    # the word was cleared and a valid call afterwards is correct
    out, lse = bsmt.flex_attention(q, k, v, block_mask=bm)
    bsmt.check_device_status()
    ro, rl = oa.flex_attention(q.cpu(), k.cpu(), v.cpu(), ("causal",), (), None, False)
    assert_attention_close(out.float().cpu().numpy(), lse.cpu().numpy(), ro, rl, "after bounds error")


def test_wait_timeout_is_reported_and_context_survives():
    """Failure detection without a fault: a pipeline wait on an mbarrier that
    nothing arrives on gives up after its 2 s bound, records DEVICE_TIMEOUT in
    the status word, and the CTA's other wait returns too. The context stays
    usable: the word clears and the next attention call is correct."""
    r = bsmt.selftest_wait_timeout()
    assert r["warp0_completed"] == 0 and r["warp1_completed"] == 0
    assert 1_500_000 <= r["warp0_wait_us"] <= 10_000_000, r
    with pytest.raises(RuntimeError, match="DEVICE_TIMEOUT"):
        bsmt.check_device_status()
    bsmt.check_device_status()  # read and cleared
    run_case(47, 1, 2, 2, 384, 384, 128, ("causal",), ())


def test_debug_sync_raises_at_the_call():
    """With BSMT_DEBUG_SYNC=1 a device-side status is raised by the call that
    caused it (here a block index past KB), not at a later check."""
    import subprocess
    import sys
    code = ("import torch, block_sparse_masked_tile_b200 as bsmt\n"
            "q = torch.randn(1, 1, 256, 64, device='cuda').to(torch.bfloat16)\n"
            "bm = bsmt.create_block_mask(bsmt.causal(), 1, 1, 256, 256)\n"
            "bm.kv_indices[0, 0, 1, 0] = 99\n"
            "try:\n"
            "    bsmt.flex_attention(q, q, q, block_mask=bm)\n"
            "except RuntimeError as e:\n"
            "    print('raised', 'DEVICE_BOUNDS' in str(e))\n")
    import os
    env = dict(os.environ, BSMT_DEBUG_SYNC="1")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], env=env, cwd=root, capture_output=True, text=True, timeout=300)
    assert "raised True" in r.stdout, r.stdout + r.stderr
