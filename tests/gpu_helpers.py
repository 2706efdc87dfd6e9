"""Shared helpers for the GPU parity tests (CUDA path vs the fp64 oracle)."""
import ctypes

import numpy as np
import torch

import block_sparse_masked_tile_b200 as bsmt

OUT_TOL = 2e-2   # max-abs on out (bf16 output, fp32 accumulation)
LSE_TOL = 1e-2   # max-abs on finite lse


def gpu_block_mask(tree, B, H, M, N):
    mm = bsmt.mask_from_tree(tree, device="cuda")
    bm = bsmt.create_block_mask(mm, B, H, M, N, device="cuda")
    bsmt.check_device_status()
    return bm


def block_mask_numpy(bm):
    return {k: getattr(bm, k).cpu().numpy() for k in
            ("kv_num_blocks", "kv_indices", "full_kv_num_blocks", "full_kv_indices")}


def assert_block_mask_equal(got: dict, want: dict):
    for key in ("kv_num_blocks", "kv_indices", "full_kv_num_blocks", "full_kv_indices"):
        g, w = got[key], want[key]
        assert g.shape == w.shape, (key, g.shape, w.shape)
        if not np.array_equal(g, w):
            bad = np.argwhere(g != w)[:5]
            raise AssertionError(f"{key} differs at {bad.tolist()}: got {[g[tuple(i)] for i in bad]}, "
                                 f"want {[w[tuple(i)] for i in bad]}")


def gpu_attention(q, k, v, tree, mods, scale, gqa, mask_B=None, mask_H=None, use_block_mask=True):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    B, Hq, M, _ = q.shape
    N = k.shape[2]
    bm = None
    if use_block_mask:
        bm = gpu_block_mask(tree, B if mask_B is None else mask_B, Hq if mask_H is None else mask_H, M, N)
    out, lse = bsmt.flex_attention(qd, kd, vd, block_mask=bm, score_mod=bsmt.score_mods_from_list(mods),
                                   scale=scale, enable_gqa=gqa)
    bsmt.check_device_status()
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def assert_attention_close(out, lse, ref_out, ref_lse, what=""):
    neg_g, neg_r = np.isneginf(lse), np.isneginf(ref_lse)
    assert np.array_equal(neg_g, neg_r), f"{what}: -inf lse positions differ ({neg_g.sum()} vs {neg_r.sum()})"
    assert np.all(np.isfinite(out)), f"{what}: non-finite output"
    err = np.abs(out - ref_out)
    assert err.max(initial=0.0) <= OUT_TOL, f"{what}: out max-abs {err.max():.3e} at {np.unravel_index(err.argmax(), err.shape)}"
    fin = ~neg_r
    lerr = np.abs(lse[fin] - ref_lse[fin])
    assert lerr.max(initial=0.0) <= LSE_TOL, f"{what}: lse max-abs {lerr.max():.3e}"
    assert np.all(out[neg_r] == 0.0), f"{what}: fully masked rows must be 0"
    return float(err.max(initial=0.0)), float(lerr.max(initial=0.0))


def within_dnf_limits(tree) -> bool:
    """Whether the library takes this mask program: its node count and its
    alternatives after the library's own simplification fit the limits. A
    host-only check (a block mask with no rows launches nothing)."""
    if tree is None:
        return True
    mm = bsmt.mask_from_tree(tree)
    if len(mm.nodes) > bsmt.MAX_NODES:
        return False
    spec, keep = mm._spec(torch.device("cpu"), 1)
    out = bsmt._BlockMask()
    st = bsmt._lib.bsmt_create_block_mask(ctypes.byref(spec), max(1, spec.doc_batch), 1, 0, 0, 128, 128,
                                          ctypes.byref(out), None)
    del keep
    return st == 0
