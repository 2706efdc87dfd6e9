"""Pins for the oracle's attention forward.

The expected values come from sources other than the oracle:

* torch.nn.functional.scaled_dot_product_attention in fp64 on the CPU.
  This is the library special case where the mask is boolean and there is
  no score_mod.
* torch.logsumexp.
* Closed forms: the ALiBi geometric weights and the tanh(1) soft-cap
  worked case.
* Invariants: rows sum to 1, constant V gives a constant output, GQA equals
  explicitly repeated kv heads, and a row with every key masked gives 0 and
  -inf.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import attention as oa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float64)


def test_noop_equals_sdpa():
    q, k, v = _rand((2, 3, 37, 16), 1), _rand((2, 3, 45, 16), 2), _rand((2, 3, 45, 16), 3)
    out, lse = oa.flex_attention(q, k, v, None, (), scale=0.3)
    ref = F.scaled_dot_product_attention(q, k, v, scale=float(np.float32(0.3)))
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)
    s = float(np.float32(0.3)) * (q @ k.transpose(-1, -2))
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), rtol=1e-12, atol=1e-12)


def test_default_scale_is_rsqrt_d():
    q, k, v = _rand((1, 1, 8, 64), 4), _rand((1, 1, 8, 64), 5), _rand((1, 1, 8, 64), 6)
    out, _ = oa.flex_attention(q, k, v, None, ())
    ref = F.scaled_dot_product_attention(q, k, v, scale=float(np.float32(1 / 8)))
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_causal_equals_sdpa_is_causal():
    q, k, v = _rand((1, 2, 64, 32), 7), _rand((1, 2, 64, 32), 8), _rand((1, 2, 64, 32), 9)
    out, lse = oa.flex_attention(q, k, v, ("causal",), (), scale=0.25)
    ref = F.scaled_dot_product_attention(q, k, v, is_causal=True, scale=0.25)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)
    s = 0.25 * (q @ k.transpose(-1, -2))
    s = s.masked_fill(~torch.ones(64, 64, dtype=torch.bool).tril(), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), rtol=1e-12, atol=1e-12)


def test_band_mask_equals_sdpa_bool_mask():
    n, W = 80, 9
    q, k, v = _rand((1, 1, n, 8), 10), _rand((1, 1, n, 8), 11), _rand((1, 1, n, 8), 12)
    out, _ = oa.flex_attention(q, k, v, ("and", ("causal",), ("window", W)), (), scale=0.5)
    band = torch.ones(n, n, dtype=torch.bool).tril() & torch.ones(n, n, dtype=torch.bool).triu(-(W - 1))
    ref = F.scaled_dot_product_attention(q, k, v, attn_mask=band, scale=0.5)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_gqa_equals_sdpa_enable_gqa():
    q, k, v = _rand((1, 8, 20, 16), 13), _rand((1, 2, 24, 16), 14), _rand((1, 2, 24, 16), 15)
    out, _ = oa.flex_attention(q, k, v, None, (), scale=0.2, enable_gqa=True)
    ref = F.scaled_dot_product_attention(q, k, v, scale=float(np.float32(0.2)), enable_gqa=True)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)
    # explicit repeat of each kv head over its 4 query heads
    rep, _ = oa.flex_attention(q, k.repeat_interleave(4, 1), v.repeat_interleave(4, 1), None, (),
                               scale=0.2)
    np.testing.assert_allclose(out, rep, rtol=0, atol=0)
    with pytest.raises(ValueError):
        oa.flex_attention(q, k, v, None, (), enable_gqa=False)


def test_rows_sum_to_one_and_constant_v():
    n = 24
    q, k = _rand((1, 1, n, 8), 16), _rand((1, 1, n, 8), 17)
    eye = torch.eye(n, dtype=torch.float64)[None, None]        # V = I -> out = P
    tree = ("and", ("causal",), ("or", ("sink", 2), ("window", 5)))
    P, _ = oa.flex_attention(q, k, eye, tree, (), scale=1.0)
    np.testing.assert_allclose(P.sum(-1), 1.0, rtol=0, atol=1e-13)
    const = torch.full((1, 1, n, 8), 2.5, dtype=torch.float64)
    out, _ = oa.flex_attention(q, k, const, tree, (("softcap", 5.0),), scale=1.0)
    np.testing.assert_allclose(out, 2.5, rtol=0, atol=1e-13)


def test_fully_masked_rows_are_zero_and_minus_inf():
    q, k, v = _rand((1, 1, 10, 4), 18), _rand((1, 1, 10, 4), 19), _rand((1, 1, 10, 4), 20)
    # kv < 0 allows nothing; rows with q_idx < 3 of the OR below are masked too
    out, lse = oa.flex_attention(q, k, v, ("sink", 0), ())
    assert np.all(out == 0) and np.all(np.isneginf(lse))
    out, lse = oa.flex_attention(q, k, v, ("and", ("causal",), ("window", 0)), ())
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_alibi_closed_form_geometric_weights():
    # ALiBi m_h * (j - i) (transformerlab page, "alibi" row). With K = 0 every
    # score is 0, so the weights of causal row i are proportional to
    # exp(m (j - i)) for j <= i. One-hot values read the weights back.
    n, H = 12, 2
    q = _rand((1, H, n, n), 21)
    k = torch.zeros((1, H, n, n), dtype=torch.float64)
    v = torch.eye(n, dtype=torch.float64)[None, None].repeat(1, H, 1, 1)
    slopes = np.array([0.5, 0.125], np.float32)
    out, lse = oa.flex_attention(q, k, v, ("causal",), (("alibi", slopes),), scale=1.0)
    for h, m in enumerate(slopes.astype(np.float64)):
        r = math.exp(m)
        for i in range(n):
            denom = (r ** (i + 1) - 1) / (r - 1)
            for j in range(n):
                w = r ** j / denom if j <= i else 0.0
                assert out[0, h, i, j] == pytest.approx(w, rel=1e-12, abs=1e-15)
            # lse = log sum_{j<=i} exp(m (j - i)) = log((1 - e^{-m(i+1)}) / (1 - e^{-m}))
            assert lse[0, h, i] == pytest.approx(
                math.log((1 - math.exp(-m * (i + 1))) / (1 - math.exp(-m))), rel=1e-12)


def test_alibi_equals_sdpa_float_bias():
    # ALiBi adds m_h * (j - i) to the scaled score of query i and key j
    # (transformerlab page, "alibi" row). SDPA with a float attn_mask adds the
    # mask to scale * q.k before its softmax, so a bias tensor m_h * (j - i),
    # with -inf where a boolean mask forbids the pair, must give the same
    # attention. Several heads with different slopes, GQA and a sliding-window
    # causal mask check the head index, the sign and the masking together.
    B, Hq, Hkv, M, N, D = 2, 4, 2, 41, 53, 16
    q, k, v = _rand((B, Hq, M, D), 31), _rand((B, Hkv, N, D), 32), _rand((B, Hkv, N, D), 33)
    slopes = np.array([0.5, 0.25, 0.0625, 0.75], np.float32)
    sc = float(np.float32(0.2))
    tree = ("and", ("causal",), ("window", 17))
    out, lse = oa.flex_attention(q, k, v, tree, (("alibi", slopes),), scale=0.2, enable_gqa=True)
    i = torch.arange(M, dtype=torch.float64)[:, None]
    j = torch.arange(N, dtype=torch.float64)[None, :]
    allowed = (i >= j) & ((i - j) < 17)
    bias = torch.tensor(slopes, dtype=torch.float64)[:, None, None] * (j - i)[None]
    bias = bias.masked_fill(~allowed[None], float("-inf"))[None].expand(B, Hq, M, N)
    ref = F.scaled_dot_product_attention(q, k, v, attn_mask=bias, scale=sc, enable_gqa=True)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)
    kr = k.repeat_interleave(Hq // Hkv, dim=1)
    s = sc * (q @ kr.transpose(-1, -2)) + bias
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), rtol=1e-12, atol=1e-12)
    # the default slopes 2^(-8(h+1)/Hq) through the same float-bias form
    out_d, _ = oa.flex_attention(q, k, v, tree, (("alibi", None),), scale=0.2, enable_gqa=True)
    dflt = torch.tensor([2.0 ** (-8.0 * (h + 1) / Hq) for h in range(Hq)], dtype=torch.float64)
    bias_d = (dflt[:, None, None] * (j - i)[None]).masked_fill(~allowed[None], float("-inf"))[None]
    ref_d = F.scaled_dot_product_attention(q, k, v, attn_mask=bias_d.expand(B, Hq, M, N), scale=sc,
                                           enable_gqa=True)
    np.testing.assert_allclose(out_d, ref_d.numpy(), rtol=1e-12, atol=1e-12)


def test_alibi_default_slopes_and_zero_slopes():
    np.testing.assert_allclose(oa.default_alibi_slopes(16)[[0, 1, 15]],
                               [2 ** -0.5, 2 ** -1.0, 2 ** -8.0], rtol=1e-15)
    q, k, v = _rand((1, 2, 16, 8), 22), _rand((1, 2, 16, 8), 23), _rand((1, 2, 16, 8), 24)
    a, _ = oa.flex_attention(q, k, v, ("causal",), (("alibi", np.zeros(2, np.float32)),))
    b, _ = oa.flex_attention(q, k, v, ("causal",), ())
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-15)


def test_softcap_golden_tanh1():
    vals = {}
    with open(os.path.join(GOLDEN, "softcap_tanh1.txt")) as fh:
        for line in fh:
            if line.strip() and not line.startswith("#"):
                key, val = line.split()
                vals[key] = float(val)
    q = torch.tensor([[[[30.0]]]], dtype=torch.float64)
    k = torch.tensor([[[[1.0], [0.0]]]], dtype=torch.float64)
    v = torch.tensor([[[[1.0], [0.0]]]], dtype=torch.float64)
    out, lse = oa.flex_attention(q, k, v, None, (("softcap", vals["cap"]),), scale=1.0)
    assert out[0, 0, 0, 0] == pytest.approx(vals["out"], rel=1e-14)
    assert lse[0, 0, 0] == pytest.approx(vals["lse"], rel=1e-14)


def test_softcap_huge_cap_is_identity():
    q, k, v = _rand((1, 1, 16, 8), 25), _rand((1, 1, 16, 8), 26), _rand((1, 1, 16, 8), 27)
    a, la = oa.flex_attention(q, k, v, ("causal",), (("softcap", 1e30),))
    b, lb = oa.flex_attention(q, k, v, ("causal",), ())
    np.testing.assert_allclose(a, b, rtol=1e-12)
    np.testing.assert_allclose(la, lb, rtol=1e-12)


def test_score_mod_order():
    # softcap then alibi differs from alibi then softcap; order follows the list
    q, k, v = _rand((1, 1, 16, 8), 28), _rand((1, 1, 16, 8), 29), _rand((1, 1, 16, 8), 30)
    s = np.array([0.7], np.float32)
    a, _ = oa.flex_attention(q, k, v, ("causal",), (("softcap", 2.0), ("alibi", s)), scale=1.0)
    b, _ = oa.flex_attention(q, k, v, ("causal",), (("alibi", s), ("softcap", 2.0)), scale=1.0)
    assert not np.allclose(a, b)


def test_document_mask_equals_sdpa_block_diag():
    lengths = [5, 11, 4]
    ids = np.repeat(np.arange(3), lengths).astype(np.int32)
    n = ids.size
    q, k, v = _rand((1, 1, n, 8), 31), _rand((1, 1, n, 8), 32), _rand((1, 1, n, 8), 33)
    out, _ = oa.flex_attention(q, k, v, ("and", ("document", ids[None], ids[None]), ("causal",)), (),
                               scale=0.4)
    blocks = [torch.ones(L, L, dtype=torch.bool).tril() for L in lengths]
    ref = F.scaled_dot_product_attention(q, k, v, attn_mask=torch.block_diag(*blocks),
                                         scale=float(np.float32(0.4)))
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_sampled_matches_full():
    q, k, v = _rand((2, 4, 40, 8), 34), _rand((2, 2, 50, 8), 35), _rand((2, 2, 50, 8), 36)
    tree = ("and", ("causal",), ("window", 7))
    mods = (("alibi", None),)
    out, lse = oa.flex_attention(q, k, v, tree, mods, enable_gqa=True)
    samples = [(0, 0, 0), (1, 3, 39), (0, 2, 17), (1, 1, 5)]
    so, sl = oa.flex_attention_sampled(q, k, v, samples, tree, mods, enable_gqa=True)
    for i, (b, h, r) in enumerate(samples):
        np.testing.assert_allclose(so[i], out[b, h, r], rtol=1e-13, atol=1e-14)
        assert sl[i] == pytest.approx(lse[b, h, r], rel=1e-13)


def _ids_from_cu(cu, total):
    ids = np.full(total, len(cu) - 1, np.int32)
    for i in range(len(cu) - 1):
        ids[cu[i]:cu[i + 1]] = i
    return ids


def test_varlen_equals_document_mask_and_sdpa():
    # L-GATr page: packed events attend within their event. The slicing
    # definition must equal the document-mask definition over the whole pack,
    # and each sequence must equal plain SDPA on its own tokens.
    rng = np.random.default_rng(5)
    Hq, Hkv, D = 4, 2, 16
    cu_q = [0, 37, 37, 120, 200]       # an empty sequence in the middle
    cu_k = [0, 50, 61, 150, 260]
    Mt, Nt = 210, 260                  # 10 q tokens past the last sequence
    q = torch.from_numpy(rng.standard_normal((Mt, Hq, D))).to(torch.bfloat16)
    k = torch.from_numpy(rng.standard_normal((Nt, Hkv, D))).to(torch.bfloat16)
    v = torch.from_numpy(rng.standard_normal((Nt, Hkv, D))).to(torch.bfloat16)
    out, lse = oa.flex_attention_varlen(q, k, v, cu_q, cu_k, False, (), None, True)
    qi, ki = _ids_from_cu(cu_q, Mt), _ids_from_cu(cu_k, Nt)
    tree = ("document", qi[None], ki[None])
    o2, l2 = oa.flex_attention(q.permute(1, 0, 2)[None], k.permute(1, 0, 2)[None], v.permute(1, 0, 2)[None],
                               tree, (), None, True)
    assert np.allclose(out, o2[0].transpose(1, 0, 2), atol=1e-12)
    assert np.array_equal(np.isneginf(lse), np.isneginf(l2[0]))
    fin = np.isfinite(lse)
    assert np.allclose(lse[fin], l2[0][fin], atol=1e-12)
    assert np.all(out[200:] == 0) and np.all(np.isneginf(lse[:, 200:]))
    for i in range(len(cu_q) - 1):
        q0, q1, k0, k1 = cu_q[i], cu_q[i + 1], cu_k[i], cu_k[i + 1]
        if q1 == q0:
            continue
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[q0:q1].double().permute(1, 0, 2), k[k0:k1].double().permute(1, 0, 2).repeat_interleave(2, 0),
            v[k0:k1].double().permute(1, 0, 2).repeat_interleave(2, 0))
        assert np.allclose(out[q0:q1], ref.permute(1, 0, 2).numpy(), atol=1e-10)


def test_varlen_causal_equals_document_and_causal():
    rng = np.random.default_rng(6)
    cu = [0, 70, 71, 200, 333]
    q = torch.from_numpy(rng.standard_normal((333, 2, 16))).to(torch.bfloat16)
    k = torch.from_numpy(rng.standard_normal((333, 2, 16))).to(torch.bfloat16)
    v = torch.from_numpy(rng.standard_normal((333, 2, 16))).to(torch.bfloat16)
    out, lse = oa.flex_attention_varlen(q, k, v, cu, cu, True)
    ids = _ids_from_cu(cu, 333)
    tree = ("and", ("document", ids[None], ids[None]), ("causal",))
    o2, l2 = oa.flex_attention(q.permute(1, 0, 2)[None], k.permute(1, 0, 2)[None], v.permute(1, 0, 2)[None], tree)
    assert np.allclose(out, o2[0].transpose(1, 0, 2), atol=1e-12)
    assert np.allclose(lse, l2[0], atol=1e-12)


def test_pool_rows_equal_the_oracle():
    # the spawned-pool runner of the GPU tests cuts slices into row ranges;
    # rows are independent, so it must reproduce the oracle itself
    from tests import oracle_pool
    import workloads
    q, k, v = workloads.random_inputs(90, 2, 4, 2, 300, 260, 64)
    dout = workloads.grad_output(91, 2, 4, 300, 64)
    tree = ("and", ("causal",), ("or", ("sink", 3), ("window", 70)))
    mods = (("softcap", 9.0), ("alibi", None))
    want_o, want_l = oa.flex_attention(q, k, v, tree, mods, None, True)
    tasks = oracle_pool.row_tasks([(0, 1), (1, 3)], 300, 128)
    got = oracle_pool.forward_rows(q, k, v, tasks, tree, mods, None, chunk=50)
    for (b, hq, r0, r1), (o, l) in zip(tasks, got):
        np.testing.assert_allclose(o, want_o[b, hq, r0:r1], rtol=0, atol=1e-12)
        np.testing.assert_allclose(l, want_l[b, hq, r0:r1], rtol=0, atol=1e-12)
    from oracle import backward as ob
    dq, dk, dv = ob.flex_attention_backward(q, k, v, dout, tree, mods, None, True)
    all_tasks = oracle_pool.row_tasks([(b, h) for b in range(2) for h in range(4)], 300, 100)
    res = oracle_pool.backward_rows(q, k, v, dout, all_tasks, tree, mods, None, want_kv=True, chunk=64)
    gk, gv = np.zeros_like(dk), np.zeros_like(dv)
    for (b, hq, r0, r1), (gq, pk, pv) in zip(all_tasks, res):
        np.testing.assert_allclose(gq, dq[b, hq, r0:r1], rtol=0, atol=1e-12)
        gk[b, hq // 2] += pk
        gv[b, hq // 2] += pv
    np.testing.assert_allclose(gk, dk, rtol=0, atol=1e-11)
    np.testing.assert_allclose(gv, dv, rtol=0, atol=1e-11)
