"""Pins for the oracle's attention backward.

The expected values come from sources other than the backward's formulas:

* Central finite differences of sum(out * dout), with out from the oracle's
  forward (itself pinned against torch SDPA and closed forms), on tiny
  inputs: every mask primitive, both score mods in both orders, GQA.
* torch autograd in fp64 through torch.nn.functional.scaled_dot_product_attention
  with a boolean mask and enable_gqa: the library special case with no
  score_mod.
* Invariants: the dV rows of a kv head sum to the dout rows of its group's
  non-empty query rows (each P row sums to 1); dS rows sum to zero, so
  without score mods the dK rows sum to zero; a query row with no allowed
  key gets dq = 0 and a key no query sees gets dk = dv = 0.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import attention as oa
from oracle import backward as ob
from oracle import masks


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float64)


def _loss(q, k, v, dout, mask, mods, scale, gqa):
    out, _ = oa.flex_attention(q, k, v, mask, mods, scale, gqa)
    return float(np.sum(out * dout))


def _fd_grad(x, f, h=1e-5):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = x[i]
        x[i] = old + h
        fp = f()
        x[i] = old - h
        fm = f()
        x[i] = old
        g[i] = (fp - fm) / (2 * h)
    return g


DOC = np.array([[0, 0, 0, 1, 1, 2, 2, 2, 2]])
CASES = [
    (None, ()),
    (("causal",), ()),
    (("and", ("causal",), ("window", 3)), (("softcap", 2.0),)),
    (("document", DOC, DOC), (("alibi", None),)),
    (("prefix_lm", 3), (("alibi", None), ("softcap", 1.5))),
    (("or", ("sink", 2), ("and", ("causal",), ("window", 2))), (("softcap", 1.5), ("alibi", [0.5, -0.25]))),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_finite_differences(case):
    mask, mods = CASES[case]
    B, Hq, Hkv, M, N, D = 1, 2, 1, 9, 9, 3
    q = _rand((B, Hq, M, D), 10 + case).numpy()
    k = _rand((B, Hkv, N, D), 20 + case).numpy()
    v = _rand((B, Hkv, N, D), 30 + case).numpy()
    dout = _rand((B, Hq, M, D), 40 + case).numpy()
    scale = 0.7
    dq, dk, dv = ob.flex_attention_backward(q, k, v, dout, mask, mods, scale, enable_gqa=True)
    f = lambda: _loss(q, k, v, dout, mask, mods, scale, True)  # noqa: E731
    np.testing.assert_allclose(dq, _fd_grad(q, f), atol=2e-8, rtol=0)
    np.testing.assert_allclose(dk, _fd_grad(k, f), atol=2e-8, rtol=0)
    np.testing.assert_allclose(dv, _fd_grad(v, f), atol=2e-8, rtol=0)


@pytest.mark.parametrize("mask", [None, ("causal",), ("and", ("causal",), ("window", 7))])
def test_equals_torch_autograd_sdpa(mask):
    B, Hq, Hkv, M, N, D = 2, 4, 2, 33, 33, 16
    q = _rand((B, Hq, M, D), 1).requires_grad_()
    k = _rand((B, Hkv, N, D), 2).requires_grad_()
    v = _rand((B, Hkv, N, D), 3).requires_grad_()
    dout = _rand((B, Hq, M, D), 4)
    scale = float(np.float32(0.3))
    dense = torch.from_numpy(masks.dense_mask(mask, 0, M, N))
    out = F.scaled_dot_product_attention(q, k, v, attn_mask=dense, scale=scale, enable_gqa=True)
    out.backward(dout)
    dq, dk, dv = ob.flex_attention_backward(q.detach(), k.detach(), v.detach(), dout, mask, (), 0.3, True)
    np.testing.assert_allclose(dq, q.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, k.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, v.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_invariants():
    B, Hq, Hkv, M, N, D = 1, 4, 2, 40, 50, 8
    q, k, v, dout = (_rand(s, 50 + i).numpy() for i, s in
                     enumerate(((B, Hq, M, D), (B, Hkv, N, D), (B, Hkv, N, D), (B, Hq, M, D))))
    # kv 45..49 are past every query's window end; query rows 0..2 see only
    # kv 0..2 through the sink, rows with q < 3 have their own keys too
    mask = ("and", ("causal",), ("or", ("sink", 3), ("window", 5)))
    dq, dk, dv = ob.flex_attention_backward(q, k, v, dout, mask, (), 0.4, True)
    allowed = masks.dense_mask(mask, 0, M, N)
    nonempty = allowed.any(axis=1)
    for hkv in range(Hkv):
        group = dout[0, 2 * hkv:2 * hkv + 2][:, nonempty].sum(axis=(0, 1))
        np.testing.assert_allclose(dv[0, hkv].sum(axis=0), group, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dk[0, hkv].sum(axis=0), 0.0, atol=1e-12)
    unseen = ~allowed.any(axis=0)
    assert unseen[45:].all()
    assert np.all(dk[:, :, unseen] == 0) and np.all(dv[:, :, unseen] == 0)
    # a mask with an empty row: document ids that no key carries
    qd = np.array([[0] * 10 + [7] * 30])
    kd = np.array([[0] * 50])
    dq2, _, _ = ob.flex_attention_backward(q, k, v, dout, ("document", qd, kd), (), 0.4, True)
    assert np.all(dq2[:, :, 10:] == 0)
    assert np.any(dq2[:, :, :10] != 0)


def test_sampled_equals_full():
    B, Hq, Hkv, M, N, D = 2, 4, 2, 70, 90, 8
    q, k, v, dout = (_rand(s, 60 + i).numpy() for i, s in
                     enumerate(((B, Hq, M, D), (B, Hkv, N, D), (B, Hkv, N, D), (B, Hq, M, D))))
    mask = ("and", ("causal",), ("window", 20))
    mods = (("softcap", 3.0), ("alibi", None))
    dq, dk, dv = ob.flex_attention_backward(q, k, v, dout, mask, mods, None, True)
    qs = [(0, 1, 5), (1, 3, 69), (1, 0, 0)]
    got = ob.backward_dq_sampled(q, k, v, dout, qs, mask, mods, None)
    np.testing.assert_allclose(got, np.stack([dq[s] for s in qs]), rtol=1e-12, atol=1e-13)
    ks = [(0, 0, 3), (1, 1, 60), (0, 1, 89)]
    gk, gv = ob.backward_dkv_sampled(q, k, v, dout, ks, mask, mods, None, row_chunk=7)
    np.testing.assert_allclose(gk, np.stack([dk[s] for s in ks]), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(gv, np.stack([dv[s] for s in ks]), rtol=1e-12, atol=1e-13)


def test_varlen_backward_equals_document_mask_form():
    """Packed sequences: the per-sequence backward equals the backward of the
    whole pack under the document mask (and causal when asked), which is the
    same attention written as one [1, H, T, D] problem."""
    lens_q = [5, 1, 7, 3]
    T = sum(lens_q) + 2  # two tokens past the last sequence
    cu = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int64)
    ids = np.full(T, len(lens_q), np.int32)
    for i in range(len(lens_q)):
        ids[cu[i]:cu[i + 1]] = i
    Hq, Hkv, D = 4, 2, 8
    q = _rand((T, Hq, D), 71).numpy()
    k = _rand((T, Hkv, D), 72).numpy()
    v = _rand((T, Hkv, D), 73).numpy()
    dout = _rand((T, Hq, D), 74).numpy()
    for causal in (False, True):
        for mods in ((), (("softcap", 3.0),)):
            got = ob.flex_attention_varlen_backward(q, k, v, dout, cu, cu, causal, mods, None, True)
            # the pack: tokens past the last sequence carry their own id and attend
            # nothing in the varlen form, so their rows are masked out here too
            ids_q = ids.copy()
            ids_q[cu[-1]:] = -1
            tree = ("document", ids_q[None], ids[None])
            if causal:
                tree = ("and", tree, ("causal",))
            pk = lambda x: x.transpose(1, 0, 2)[None]  # noqa: E731
            ref = ob.flex_attention_backward(pk(q), pk(k), pk(v), pk(dout), tree, mods, None, True)
            for g, r in zip(got, ref):
                np.testing.assert_allclose(g, r[0].transpose(1, 0, 2), rtol=1e-10, atol=1e-12)
            assert np.all(got[0][cu[-1]:] == 0) and np.all(got[1][cu[-1]:] == 0)
