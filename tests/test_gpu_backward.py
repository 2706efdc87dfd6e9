"""GPU parity: the tcgen05 attention backward (dq, dk, dv) vs the fp64 oracle.

The backward runs on the GPU forward's own out and lse, as a training step
would. Small cases are compared element by element over all of dq, dk and
dv. The four large workloads run at full size, and sampled rows are compared
with the oracle's one-row forms: dq rows, and dk/dv rows of chosen keys
(every query row that reaches the key contributes, so these are exact).

Tolerance, per tensor: max |gpu - oracle| <= 2e-2 * max(1, max |oracle|).
P and dS enter the tensor-core products as bf16 (relative rounding 2^-9),
delta comes from the bf16 forward output, and the results are rounded to
bf16; accumulation is fp32. Each of these is a few tenths of a percent of
the tensor's scale.
"""
import numpy as np
import pytest
import torch

import block_sparse_masked_tile_b200 as bsmt
import workloads
from oracle import backward as ob
from tests.gpu_helpers import gpu_block_mask, within_dnf_limits

pytestmark = pytest.mark.gpu

GRAD_TOL = 2e-2


def gpu_backward(q, k, v, dout, tree, mods, scale, gqa, use_block_mask=True, mask_B=None, mask_H=None):
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, dout))
    B, Hq, M, _ = q.shape
    N = k.shape[2]
    bm = None
    if use_block_mask:
        bm = gpu_block_mask(tree, B if mask_B is None else mask_B, Hq if mask_H is None else mask_H, M, N)
    sm = bsmt.score_mods_from_list(mods)
    out, lse = bsmt.flex_attention(qd, kd, vd, block_mask=bm, score_mod=sm, scale=scale, enable_gqa=gqa)
    dq, dk, dv = bsmt.flex_attention_backward(qd, kd, vd, out, lse, dod, block_mask=bm, score_mod=sm, scale=scale,
                                              enable_gqa=gqa)
    bsmt.check_device_status()
    return [t.float().cpu().numpy().astype(np.float64) for t in (dq, dk, dv)]


def assert_close(name, got, ref, what=""):
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite {name}"
    scale = max(1.0, float(np.abs(ref).max(initial=0.0)))
    err = float(np.abs(got - ref).max(initial=0.0))
    assert err <= GRAD_TOL * scale, (f"{what}: {name} max-abs {err:.3e} > {GRAD_TOL * scale:.3e} at "
                                     f"{np.unravel_index(np.abs(got - ref).argmax(), got.shape)}")
    return err / scale


def assert_grads_close(got, ref, what=""):
    return [assert_close(n, g, r, what) for n, g, r in zip(("dq", "dk", "dv"), got, ref)]


def run_case(seed, B, Hq, Hkv, M, N, D, tree, mods, scale=None, use_block_mask=True, mask_B=None, mask_H=None):
    q, k, v = workloads.random_inputs(seed, B, Hq, Hkv, M, N, D)
    dout = workloads.grad_output(seed + 7919, B, Hq, M, D)
    gqa = Hq != Hkv
    if use_block_mask and not within_dnf_limits(tree):
        return None
    got = gpu_backward(q, k, v, dout, tree, mods, scale, gqa, use_block_mask, mask_B, mask_H)
    ref = ob.flex_attention_backward(q, k, v, dout, tree if use_block_mask else None, mods, scale, gqa)
    return assert_grads_close(got, ref, f"seed={seed}")


def test_workload1_full():
    w = workloads.get(1)
    d = workloads.make(w)
    dout = workloads.grad_output(w.seed + 50, w.B, w.Hq, w.M, w.D)
    got = gpu_backward(d["q"], d["k"], d["v"], dout, d["mask"], d["score_mods"], w.scale, w.enable_gqa)
    ref = ob.flex_attention_backward(d["q"], d["k"], d["v"], dout, d["mask"], d["score_mods"], w.scale,
                                     w.enable_gqa)
    assert_grads_close(got, ref, w.name)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("mods", [(), (("softcap", 30.0),), (("alibi", None),),
                                  (("softcap", 5.0), ("alibi", None)), (("alibi", None), ("softcap", 5.0))])
def test_score_mods(D, mods):
    run_case(7, 1, 2, 2, 384, 384, D, ("causal",), mods)


@pytest.mark.parametrize("D", [64, 128])
def test_gqa_sliding_window(D):
    run_case(8, 2, 8, 2, 640, 640, D, ("and", ("causal",), ("window", 200)), (("softcap", 30.0),))


@pytest.mark.parametrize("D", [64, 128])
def test_dense_no_block_mask(D):
    run_case(11, 2, 2, 1, 256, 384, D, None, (), use_block_mask=False)
    run_case(12, 1, 2, 2, 200, 300, D, None, (), use_block_mask=False)


@pytest.mark.parametrize("M,N", [(300, 200), (129, 513), (1, 1), (100, 1000), (1000, 100)])
def test_ragged_lengths(M, N):
    run_case(13, 1, 2, 2, M, N, 128, ("and", ("causal",), ("window", 150)), ())
    run_case(14, 1, 1, 1, M, N, 64, ("prefix_lm", 70), (("alibi", None),))


def test_streaming_sink_window():
    run_case(15, 1, 4, 2, 2048, 2048, 128, ("and", ("causal",), ("or", ("sink", 4), ("window", 256))), ())


def test_document_causal():
    lengths = [300, 77, 500, 1, 400, 258]
    ids = workloads.document_ids(lengths)[None]
    run_case(16, 1, 2, 2, 1536, 1536, 128, ("and", ("document", ids, ids), ("causal",)), ())


@pytest.mark.parametrize("seed", range(10))
def test_random_masks_and_shapes(seed):
    rng = np.random.default_rng(900 + seed)
    D = int(rng.choice([64, 128]))
    Hkv = int(rng.integers(1, 3))
    Hq = Hkv * int(rng.choice([1, 2, 4]))
    B = int(rng.integers(1, 3))
    M = int(rng.integers(1, 700))
    N = int(rng.integers(1, 700))
    tree = workloads.random_mask_tree(rng, B, M, N, depth=2)
    mods = [(), (("softcap", 20.0),), (("alibi", None),)][int(rng.integers(3))]
    run_case(seed, B, Hq, Hkv, M, N, D, tree, mods)


@pytest.mark.parametrize("seed", range(4))
def test_deep_masks(seed):
    # four-level programs after the library's simplification, on both walks
    rng = np.random.default_rng(950 + seed)
    M = int(rng.integers(100, 600))
    N = int(rng.integers(100, 600))
    tree = workloads.random_mask_tree(rng, 1, M, N, depth=4)
    run_case(970 + seed, 1, 2, 1, M, N, 64, tree, ())


def test_broadcast_block_mask():
    run_case(21, 2, 4, 2, 512, 512, 128, ("and", ("causal",), ("window", 200)), (), mask_B=1, mask_H=1)


def test_fully_masked_rows_pass_no_gradient():
    run_case(31, 1, 2, 2, 300, 300, 64, ("and", ("causal",), ("window", 0)), ())
    ids_q = np.repeat(np.arange(4), [50, 50, 50, 106]).astype(np.int32)[None]
    ids_kv = np.repeat(np.arange(3), [60, 60, 136]).astype(np.int32)[None]
    run_case(33, 1, 1, 1, 256, 256, 64, ("document", ids_q, ids_kv), ())


def test_empty_inputs():
    for (M, N) in ((0, 64), (70, 0)):
        q, k, v = (t.cuda() for t in workloads.random_inputs(40, 1, 2, 2, M, N, 64))
        dout = workloads.grad_output(41, 1, 2, M, 64).cuda()
        out, lse = bsmt.flex_attention(q, k, v)
        dq, dk, dv = bsmt.flex_attention_backward(q, k, v, out, lse, dout)
        bsmt.check_device_status()
        assert torch.all(dq == 0) and torch.all(dk == 0) and torch.all(dv == 0)


def test_deterministic():
    q, k, v = (t.cuda() for t in workloads.random_inputs(50, 1, 4, 2, 700, 700, 128))
    dout = workloads.grad_output(51, 1, 4, 700, 128).cuda()
    bm = bsmt.create_block_mask(bsmt.causal(), 1, 4, 700, 700)
    out, lse = bsmt.flex_attention(q, k, v, block_mask=bm, enable_gqa=True)
    a = bsmt.flex_attention_backward(q, k, v, out, lse, dout, block_mask=bm, enable_gqa=True)
    b = bsmt.flex_attention_backward(q, k, v, out, lse, dout, block_mask=bm, enable_gqa=True)
    bsmt.check_device_status()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_invalid_q_side_list_is_reported():
    q, k, v = (t.cuda() for t in workloads.random_inputs(45, 1, 2, 2, 512, 512, 64))
    dout = workloads.grad_output(46, 1, 2, 512, 64).cuda()
    bm = bsmt.create_block_mask(bsmt.causal(), 1, 2, 512, 512)
    out, lse = bsmt.flex_attention(q, k, v, block_mask=bm)
    qs = bm.q_side()
    saved = qs["q_indices"].clone()
    qs["q_indices"][0, 1, 2, 0] = bm.shape[2] + 3  # past the last q-block
    bsmt.flex_attention_backward(q, k, v, out, lse, dout, block_mask=bm)
    with pytest.raises(RuntimeError, match="DEVICE_BOUNDS"):
        bsmt.check_device_status()
    qs["q_indices"].copy_(saved)
    got = [t.float().cpu().numpy() for t in bsmt.flex_attention_backward(q, k, v, out, lse, dout, block_mask=bm)]
    bsmt.check_device_status()
    ref = ob.flex_attention_backward(q.cpu(), k.cpu(), v.cpu(), dout.cpu(), ("causal",), (), None, False)
    assert_grads_close(got, ref, "after bounds error")


def dkv_samples(rng, w, count, lo=0):
    out = []
    for kb in sorted(set([w.N // 128 - 1, lo // 128 + 1] + list(rng.integers(lo // 128, w.N // 128, size=count)))):
        out.append((int(rng.integers(w.B)), int(rng.integers(w.Hkv)), kb * 128 + int(rng.integers(128))))
    return out[:count]


@pytest.mark.parametrize("index", [2, 3, 4, 5])
def test_workloads_full_size_sampled(index):
    w = workloads.get(index)
    d = workloads.make(w)
    dout = workloads.grad_output(w.seed + 50, w.B, w.Hq, w.M, w.D)
    dq, dk, dv = gpu_backward(d["q"], d["k"], d["v"], dout, d["mask"], d["score_mods"], w.scale, w.enable_gqa)
    for t in (dq, dk, dv):
        assert np.all(np.isfinite(t))
    rng = np.random.default_rng(100 + index)
    qs = [(int(rng.integers(w.B)), int(rng.integers(w.Hq)), int(r)) for r in
          [0, 127, 128, w.M - 1] + list(rng.integers(0, w.M, size=12))]
    ref_q = ob.backward_dq_sampled(d["q"], d["k"], d["v"], dout, qs, d["mask"], d["score_mods"], w.scale)
    assert_close("dq rows", np.stack([dq[b, h, r] for b, h, r in qs]), ref_q, w.name)
    # keys past the sink tokens: each is reached by at most a window of queries
    # (the sink keys, reached by every query, are covered by the small streaming case)
    ks = dkv_samples(rng, w, 3, lo=128 if w.mask == "streaming" else 0)
    ref_k, ref_v = ob.backward_dkv_sampled(d["q"], d["k"], d["v"], dout, ks, d["mask"], d["score_mods"], w.scale)
    assert_close("dk rows", np.stack([dk[b, h, j] for b, h, j in ks]), ref_k, w.name)
    assert_close("dv rows", np.stack([dv[b, h, j] for b, h, j in ks]), ref_v, w.name)


def _gpu_backward_full(w, d, dout):
    dq, dk, dv = gpu_backward(d["q"], d["k"], d["v"], dout, d["mask"], d["score_mods"], w.scale, w.enable_gqa)
    for t in (dq, dk, dv):
        assert np.all(np.isfinite(t))
    return dq, dk, dv


def test_workload3_backward_exhaustive():
    # causal + ALiBi at D = 64: all of dq, dk and dv, oracle in a pool
    from tests import oracle_pool
    w = workloads.get(3)
    d = workloads.make(w)
    dout = workloads.grad_output(w.seed + 50, w.B, w.Hq, w.M, w.D)
    dq, dk, dv = _gpu_backward_full(w, d, dout)
    tasks = oracle_pool.row_tasks([(b, h) for b in range(w.B) for h in range(w.Hq)], w.M, w.M)
    res = oracle_pool.backward_rows(d["q"], d["k"], d["v"], dout, tasks, d["mask"], d["score_mods"], w.scale,
                                    want_kv=True)
    ref_q = np.zeros_like(dq)
    ref_k, ref_v = np.zeros_like(dk), np.zeros_like(dv)
    group = w.Hq // w.Hkv
    for (b, hq, r0, r1), (gq, gk, gv) in zip(tasks, res):
        ref_q[b, hq, r0:r1] = gq
        ref_k[b, hq // group] += gk
        ref_v[b, hq // group] += gv
    assert_grads_close([dq, dk, dv], [ref_q, ref_k, ref_v], w.name)


@pytest.mark.parametrize("index", [4, 5])
def test_workload_dq_whole_heads(index):
    # every dq row of whole (b, hq) slices (and, for the streaming workload,
    # of q-blocks 0-10 for the four query heads of one kv head)
    from tests import oracle_pool
    w = workloads.get(index)
    d = workloads.make(w)
    dout = workloads.grad_output(w.seed + 50, w.B, w.Hq, w.M, w.D)
    dq, _, _ = _gpu_backward_full(w, d, dout)
    if index == 4:
        tasks = oracle_pool.row_tasks([(0, 0), (0, 11), (0, 20), (0, 31)], w.M, 4096)
    else:
        group = w.Hq // w.Hkv
        tasks = oracle_pool.row_tasks([(0, 3), (1, 30)], w.M, 4096)
        tasks += [(1, h, 0, 11 * 128) for h in range(5 * group, 6 * group)]
    res = oracle_pool.backward_rows(d["q"], d["k"], d["v"], dout, tasks, d["mask"], d["score_mods"], w.scale)
    got = np.concatenate([dq[b, hq, r0:r1] for (b, hq, r0, r1) in tasks])
    ref = np.concatenate([gq for gq, _, _ in res])
    assert_close("dq rows", got, ref, w.name)


def test_autograd_through_flex_attention():
    """q, k, v that require grad: flex_attention records the op and
    backpropagating sum(out * dout) gives the same bits as the direct
    backward call, and matches the oracle."""
    q, k, v = (t.cuda() for t in workloads.random_inputs(60, 1, 4, 2, 300, 300, 128))
    dout = workloads.grad_output(61, 1, 4, 300, 128).cuda()
    tree = ("and", ("causal",), ("window", 100))
    mods = (("softcap", 20.0),)
    bm = gpu_block_mask(tree, 1, 4, 300, 300)
    sm = bsmt.score_mods_from_list(mods)
    qg, kg, vg = (t.clone().requires_grad_(True) for t in (q, k, v))
    out, lse = bsmt.flex_attention(qg, kg, vg, block_mask=bm, score_mod=sm, enable_gqa=True)
    assert out.requires_grad and not lse.requires_grad
    (out.float() * dout.float()).sum().backward()
    bsmt.check_device_status()
    want = bsmt.flex_attention_backward(q, k, v, out.detach(), lse, dout, block_mask=bm, score_mod=sm,
                                        enable_gqa=True)
    for got, ref in zip((qg.grad, kg.grad, vg.grad), want):
        assert torch.equal(got, ref)
    oracle = ob.flex_attention_backward(q.cpu(), k.cpu(), v.cpu(), dout.cpu(), tree, mods, None, True)
    assert_grads_close([t.float().cpu().numpy() for t in (qg.grad, kg.grad, vg.grad)], oracle, "autograd")
    with pytest.raises(ValueError, match="split-KV"):
        bsmt.flex_attention(qg, kg, vg, block_mask=bm, enable_gqa=True, num_splits=2)


def test_one_buffer_boundary_forward_and_backward():
    """KV_LEN = 1024 kv blocks (the forward's one window) with GQA 2:1, so a
    dk/dv unit walks 2 heads x 1024 q-blocks = 2048 entries, exactly one
    buffer of the backward's scheduler. Sampled query rows are compared for
    out, lse and dq; dk/dv rows for keys near the end, which few queries
    reach under the causal mask."""
    from oracle import attention as oa
    from tests.gpu_helpers import assert_attention_close
    L, D = 1024 * 128, 64
    q, k, v = workloads.random_inputs(70, 1, 2, 1, L, L, D)
    dout = workloads.grad_output(71, 1, 2, L, D)
    qd, kd, vd, dd = (t.cuda() for t in (q, k, v, dout))
    bm = bsmt.create_block_mask(bsmt.causal(), 1, 2, L, L)
    out, lse = bsmt.flex_attention(qd, kd, vd, block_mask=bm, enable_gqa=True)
    dq, dk, dv = bsmt.flex_attention_backward(qd, kd, vd, out, lse, dd, block_mask=bm, enable_gqa=True)
    bsmt.check_device_status()
    rows = [(0, 0, 0), (0, 1, 1), (0, 0, 127), (0, 1, 128), (0, 0, L // 2 + 3), (0, 1, L - 1), (0, 0, L - 129)]
    so, sl = oa.flex_attention_sampled(q, k, v, rows, ("causal",), (), None, True)
    go = np.stack([out[b, h, r].float().cpu().numpy() for b, h, r in rows])
    gl = np.array([lse[b, h, r].item() for b, h, r in rows])
    assert_attention_close(go, gl, so, sl, "maximum length")
    ref_q = ob.backward_dq_sampled(q, k, v, dout, rows, ("causal",), (), None)
    assert_close("dq rows", np.stack([dq[b, h, r].float().cpu().numpy() for b, h, r in rows]), ref_q, "max")
    keys = [(0, 0, L - 1), (0, 0, L - 128), (0, 0, L - 700)]
    ref_k, ref_v = ob.backward_dkv_sampled(q, k, v, dout, keys, ("causal",), (), None)
    assert_close("dk rows", np.stack([dk[b, h, j].float().cpu().numpy() for b, h, j in keys]), ref_k, "max")
    assert_close("dv rows", np.stack([dv[b, h, j].float().cpu().numpy() for b, h, j in keys]), ref_v, "max")
