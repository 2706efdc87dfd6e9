"""GPU parity: packed variable-length attention (cu_seqlens) vs the fp64
oracle, including empty sequences, tokens past the last sequence, GQA,
causal and score mods."""
import numpy as np
import pytest
import torch

import block_sparse_masked_tile_b200 as bsmt
from oracle import attention as oa

pytestmark = pytest.mark.gpu


def packed(seed, Mt, Nt, Hq, Hkv, D):
    g = torch.Generator("cpu").manual_seed(seed)
    return tuple(torch.randn(shape, generator=g).to(torch.bfloat16)
                 for shape in ((Mt, Hq, D), (Nt, Hkv, D), (Nt, Hkv, D)))


def check(seed, cu_q, cu_k, Mt, Nt, Hq, Hkv, D, causal, mods=()):
    q, k, v = packed(seed, Mt, Nt, Hq, Hkv, D)
    cq = torch.tensor(cu_q, dtype=torch.int32).cuda()
    ck = cq if cu_k is cu_q else torch.tensor(cu_k, dtype=torch.int32).cuda()
    out, lse = bsmt.flex_attention_varlen(q.cuda(), k.cuda(), v.cuda(), cq, ck, causal=causal,
                                          score_mod=bsmt.score_mods_from_list(mods), enable_gqa=Hq != Hkv)
    bsmt.check_device_status()
    ro, rl = oa.flex_attention_varlen(q, k, v, cu_q, cu_k, causal, mods, None, Hq != Hkv)
    err = np.abs(out.float().cpu().numpy() - ro).max()
    assert err < 2e-2, err
    got_l = lse.cpu().numpy()
    assert np.array_equal(np.isneginf(got_l), np.isneginf(rl))
    fin = np.isfinite(rl)
    assert np.abs(got_l[fin] - rl[fin]).max() < 1e-2


@pytest.mark.parametrize("D", [64, 128])
def test_causal_shared_seqlens(D):
    cu = [0, 300, 301, 1000, 1500, 2600]
    check(1, cu, cu, 2600, 2600, 4, 2, D, True)


def test_non_causal_different_lengths_and_tail():
    cu_q = [0, 129, 129, 400, 700]
    cu_k = [0, 500, 777, 800, 1900]
    check(2, cu_q, cu_k, 760, 1900, 2, 2, 128, False)   # q tokens 700..759 belong to no sequence


def test_score_mods_and_many_sequences():
    rng = np.random.default_rng(3)
    lens = rng.integers(1, 300, size=40)
    cu = [0] + list(np.cumsum(lens))
    check(3, cu, cu, int(cu[-1]), int(cu[-1]), 4, 4, 64, True, (("softcap", 20.0),))
    check(4, cu, cu, int(cu[-1]), int(cu[-1]), 4, 1, 128, True, (("alibi", None),))


def test_unsorted_cu_seqlens_are_reported():
    cu = torch.tensor([0, 100, 50, 200], dtype=torch.int32).cuda()
    bsmt.seqlens_to_doc_ids(cu, 200)
    with pytest.raises(RuntimeError, match="DEVICE_PRECONDITION"):
        bsmt.check_device_status()


def test_alibi_needs_shared_seqlens():
    q, k, v = (t.cuda() for t in packed(5, 200, 300, 2, 2, 64))
    cq = torch.tensor([0, 100, 200], dtype=torch.int32).cuda()
    ck = torch.tensor([0, 150, 300], dtype=torch.int32).cuda()
    with pytest.raises(ValueError, match="share cu_seqlens"):
        bsmt.flex_attention_varlen(q, k, v, cq, ck, score_mod=bsmt.alibi())


# ------------------------------------------------------------------ backward
from oracle import backward as ob  # noqa: E402

GRAD_TOL = 2e-2  # per tensor: max |gpu - oracle| <= GRAD_TOL * max(1, max |oracle|)


def check_backward(seed, cu_q, cu_k, Mt, Nt, Hq, Hkv, D, causal, mods=()):
    q, k, v = packed(seed, Mt, Nt, Hq, Hkv, D)
    g = torch.Generator("cpu").manual_seed(seed + 500)
    dout = torch.randn((Mt, Hq, D), generator=g).to(torch.bfloat16)
    cq = torch.tensor(cu_q, dtype=torch.int32).cuda()
    ck = cq if cu_k is cu_q else torch.tensor(cu_k, dtype=torch.int32).cuda()
    sm = bsmt.score_mods_from_list(mods)
    gqa = Hq != Hkv
    qd, kd, vd, dd = (t.cuda() for t in (q, k, v, dout))
    out, lse = bsmt.flex_attention_varlen(qd, kd, vd, cq, ck, causal=causal, score_mod=sm, enable_gqa=gqa)
    got = bsmt.flex_attention_varlen_backward(qd, kd, vd, out, lse, dd, cq, ck, causal=causal, score_mod=sm,
                                              enable_gqa=gqa)
    bsmt.check_device_status()
    ref = ob.flex_attention_varlen_backward(q, k, v, dout, cu_q, cu_k, causal, mods, None, gqa)
    for name, a, r in zip(("dq", "dk", "dv"), got, ref):
        a = a.float().cpu().numpy()
        scale = max(1.0, float(np.abs(r).max(initial=0.0)))
        err = float(np.abs(a - r).max(initial=0.0))
        assert err <= GRAD_TOL * scale, (name, err, scale)
    # autograd through flex_attention_varlen gives the same bits
    qg, kg, vg = (t.clone().requires_grad_(True) for t in (qd, kd, vd))
    o2, _ = bsmt.flex_attention_varlen(qg, kg, vg, cq, ck, causal=causal, score_mod=sm, enable_gqa=gqa)
    (o2.float() * dd.float()).sum().backward()
    for a, b in zip((qg.grad, kg.grad, vg.grad), got):
        assert torch.equal(a, b)


@pytest.mark.parametrize("D", [64, 128])
def test_backward_causal_shared_seqlens(D):
    cu = [0, 300, 301, 1000, 1500, 2600]
    check_backward(11, cu, cu, 2600, 2600, 4, 2, D, True)


def test_backward_non_causal_different_lengths_and_tail():
    cu_q = [0, 129, 129, 400, 700]
    cu_k = [0, 500, 777, 800, 1900]
    check_backward(12, cu_q, cu_k, 760, 1900, 2, 2, 128, False)


def test_backward_score_mods_and_many_sequences():
    rng = np.random.default_rng(13)
    lens = rng.integers(1, 200, size=24)
    cu = [0] + list(np.cumsum(lens))
    check_backward(13, cu, cu, int(cu[-1]), int(cu[-1]), 4, 4, 64, True, (("softcap", 20.0),))
    check_backward(14, cu, cu, int(cu[-1]), int(cu[-1]), 4, 1, 128, True, (("alibi", None),))
