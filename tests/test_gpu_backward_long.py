"""GPU parity: backward units of more than one scheduler buffer.

A dk/dv unit (one kv-block) walks every listed q-block of every query head
of its GQA group; a dq unit (one q-block) walks its listed kv-blocks. One
buffer of the backward's scheduler holds 2048 such entries. Longer units go
out as several full buffers and a last one, and the MMA issuer, the loader
and the softmax warps carry the unit (its accumulators, its fixed tiles and
its row data) across them, so the result is the same sum over the unit's
tiles (tensorplay.nn.attention page, BlockMask "Details" items 3-4: dK and
dV walk the q-side lists, dQ the kv-side lists). These tests compare whole
gradients with the fp64 oracle on shapes whose units need two buffers:
  - dk/dv: 8 query heads per kv head over 300 q-blocks (2400 entries), the
    buffer boundary inside one head's list;
  - dq: 2056 kv-blocks per row (263,144 keys).
"""
import numpy as np
import pytest

import block_sparse_masked_tile_b200 as bsmt
import workloads
from oracle import backward as ob
from tests.test_gpu_backward import assert_grads_close, gpu_backward

pytestmark = pytest.mark.gpu


def _case(seed, Hq, Hkv, M, N, D, tree, mods, use_block_mask=True):
    q, k, v = workloads.random_inputs(seed, 1, Hq, Hkv, M, N, D)
    dout = workloads.grad_output(seed + 7919, 1, Hq, M, D)
    gqa = Hq != Hkv
    got = gpu_backward(q, k, v, dout, tree, mods, None, gqa, use_block_mask)
    ref = ob.flex_attention_backward(q, k, v, dout, tree if use_block_mask else None, mods, None, gqa)
    return assert_grads_close(got, ref, f"seed={seed}")


@pytest.mark.parametrize("D", [64, 128])
def test_dkdv_units_over_two_buffers_dense(D):
    # 300 q-blocks (the last one ragged) x 8 heads = 2400 entries per kv-block
    _case(90 + D, 8, 1, 300 * 128 - 37, 306, D, None, (), use_block_mask=False)


def test_dkdv_units_over_two_buffers_masked():
    # sink 4 + window 200 (with causal): queries past the window keep the sink
    # tile only, a partial tile in every q-block's list of kv-block 0; soft-cap
    tree = ("and", ("causal",), ("or", ("sink", 4), ("window", 200)))
    _case(93, 8, 1, 300 * 128 - 37, 306, 64, tree, (("softcap", 30.0),))


def test_dq_units_over_two_buffers():
    # 263,144 keys: 2056 kv-blocks per dq unit, the last one ragged; GQA 2:1.
    # prefix-LM 263,000: blocks 0..2054 listed (2054 partial), 2055 empty.
    N = 263144
    _case(94, 2, 1, 300, N, 64, ("prefix_lm", 263000), ())
    _case(95, 2, 1, 300, N, 64, None, (), use_block_mask=False)


def test_autograd_long_rows():
    # the differentiable call over rows of more than one forward window
    # (1094 kv-blocks); the backward's units fit one buffer here
    M, N, D = 256, 140000, 64
    q, k, v = workloads.random_inputs(96, 1, 16, 1, M, N, D)
    dout = workloads.grad_output(97, 1, 16, M, D)
    qd, kd, vd = (t.cuda().requires_grad_(True) for t in (q, k, v))
    out, _ = bsmt.flex_attention(qd, kd, vd, enable_gqa=True)
    out.backward(dout.cuda())
    bsmt.check_device_status()
    ref = ob.flex_attention_backward(q, k, v, dout, None, (), None, True)
    got = [t.grad.float().cpu().numpy().astype(np.float64) for t in (qd, kd, vd)]
    assert_grads_close(got, ref, "autograd long rows")


def test_dkdv_units_over_two_buffers_two_batch_rows_broadcast_mask():
    # B = 2 with a block mask built once for B = H = 1 (broadcast), GQA 8:1
    # over 260 q-blocks and 333 keys: kv-block 0 (the sink keys for most
    # queries, the window for the first ones) is listed for every q-block,
    # 2080 entries in two buffers; the others for the first q-blocks only
    tree = ("and", ("causal",), ("or", ("sink", 16), ("window", 1000)))
    M, N = 260 * 128, 333
    q, k, v = workloads.random_inputs(98, 2, 8, 1, M, N, 64)
    dout = workloads.grad_output(99, 2, 8, M, 64)
    got = gpu_backward(q, k, v, dout, tree, (), None, True, True, mask_B=1, mask_H=1)
    ref = ob.flex_attention_backward(q, k, v, dout, tree, (), None, True)
    assert_grads_close(got, ref, "two batch rows, broadcast mask")
