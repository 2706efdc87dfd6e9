"""Host logic: the library's simplification of mask programs.

The library distributes AND over OR and simplifies after every AND and OR
node: within an alternative, leaves of one kind collapse to the strictest
(one CAUSAL, one DOCUMENT, the smallest WINDOW, PREFIX_LM and SINK
arguments), repeated alternatives merge, and an alternative that another one
contains is dropped (bsmt.h, masks). A small model of those rules, written
here from that statement, predicts the number of alternatives a program
ends with. The library must accept exactly the programs of at most 16 and,
for the others, report the model's count. Host-only: a block mask with no
rows launches nothing.
"""
import ctypes
import re

import numpy as np
import torch

import block_sparse_masked_tile_b200 as bsmt
import workloads

LIMIT = 16          # BSMT_MAX_MASK_TERMS
WORK_LIMIT = 1024   # alternatives held while a program is evaluated


def _leaf(kind, arg):
    t = {"causal": False, "doc": False, "w": None, "p": None, "s": None}
    if kind == bsmt.MASK_CAUSAL:
        t["causal"] = True
    elif kind == bsmt.MASK_DOCUMENT:
        t["doc"] = True
    elif kind == bsmt.MASK_WINDOW:
        t["w"] = arg
    elif kind == bsmt.MASK_PREFIX_LM:
        t["p"] = arg
    elif kind == bsmt.MASK_SINK:
        t["s"] = arg
    return t


def _and(a, b):
    def smaller(x, y):
        return y if x is None else x if y is None else min(x, y)
    return {"causal": a["causal"] or b["causal"], "doc": a["doc"] or b["doc"],
            "w": smaller(a["w"], b["w"]), "p": smaller(a["p"], b["p"]), "s": smaller(a["s"], b["s"])}


def _within(inner, outer):
    if outer["causal"] and not inner["causal"]:
        return False
    if outer["doc"] and not inner["doc"]:
        return False
    for k in ("w", "p", "s"):
        if outer[k] is not None and (inner[k] is None or inner[k] > outer[k]):
            return False
    return True


def _simplify(terms):
    uniq = []
    for t in terms:
        if t not in uniq:
            uniq.append(t)
    return [t for i, t in enumerate(uniq) if not any(j != i and _within(t, o) for j, o in enumerate(uniq))]


def model_count(nodes):
    """Alternatives after simplification, or None when more than WORK_LIMIT
    are held while evaluating."""
    stack = []
    for kind, arg in nodes:
        if kind in (bsmt.MASK_AND, bsmt.MASK_OR):
            ops = stack[-arg:]
            del stack[-arg:]
            if kind == bsmt.MASK_OR:
                res = _simplify([t for d in ops for t in d])
            else:
                res = [_leaf(bsmt.MASK_NOOP, 0)]
                for d in ops:
                    res = _simplify([_and(a, b) for a in res for b in d])
                    if len(res) > WORK_LIMIT:
                        return None
            if len(res) > WORK_LIMIT:
                return None
            stack.append(res)
        else:
            stack.append([_leaf(kind, arg)])
    assert len(stack) == 1
    return len(stack[0])


def library_answer(mm):
    spec, keep = mm._spec(torch.device("cpu"), 1)
    out = bsmt._BlockMask()
    st = bsmt._lib.bsmt_create_block_mask(ctypes.byref(spec), max(1, spec.doc_batch), 1, 0, 0, 128, 128,
                                          ctypes.byref(out), None)
    msg = bsmt._lib.bsmt_last_error().decode() if st != 0 else ""
    del keep
    return st, msg


def check(tree):
    mm = bsmt.mask_from_tree(tree)
    if len(mm.nodes) > bsmt.MAX_NODES:
        return None
    want = model_count(mm.nodes)
    st, msg = library_answer(mm)
    if want is not None and want <= LIMIT:
        assert st == 0, (tree, want, msg)
    else:
        assert st == 3, (tree, want, st)  # BSMT_ERR_UNSUPPORTED
        if want is not None:
            got = int(re.search(r"(\d+) alternatives after", msg).group(1))
            assert got == want, (tree, got, want)
    return want


def test_random_programs_match_the_model():
    rng = np.random.default_rng(2024)
    counts = []
    for _ in range(400):
        depth = int(rng.integers(2, 6))
        tree = workloads.random_mask_tree(rng, 1, 300, 300, depth=depth)
        c = check(tree)
        if c is not None:
            counts.append(c)
    # the draw includes single alternatives and several of them
    assert min(counts) == 1 and max(counts) > 4


def test_handmade_programs():
    ids = np.zeros((1, 10), np.int32)
    cases = [
        # contained alternatives fold away
        (("or", ("causal",), ("and", ("causal",), ("window", 5))), 1),
        (("or", ("and", ("window", 3), ("sink", 2)), ("and", ("window", 4), ("sink", 2))), 1),
        # incomparable alternatives stay
        (("or", ("and", ("window", 3), ("sink", 4)), ("and", ("window", 4), ("sink", 2))), 2),
        # same-kind leaves collapse to the strictest
        (("and", ("window", 9), ("window", 4), ("prefix_lm", 7), ("prefix_lm", 3)), 1),
        # NOOP contains everything
        (("or", ("noop",), ("causal",), ("document", ids, ids)), 1),
        # 32 raw alternatives -> 2
        (("and",) + tuple(("or", ("causal",), ("sink", 2)) for _ in range(5)), 2),
        # document alternatives differ from causal ones
        (("or", ("and", ("document", ids, ids), ("causal",)), ("causal",), ("document", ids, ids)), 2),
        # 17 incomparable alternatives: over the limit, and reported as 17
        (("or",) + tuple(("and", ("window", 10 + i), ("sink", 100 - i)) for i in range(17)), 17),
    ]
    for tree, want in cases:
        assert check(tree) == want, tree
    # an AND of ORs whose arguments all differ: the model decides the side
    tree = ("and",) + tuple(("or", ("window", 10 + 7 * i), ("sink", 90 - 5 * i), ("prefix_lm", 50 + i))
                            for i in range(4))
    assert check(tree) is not None
