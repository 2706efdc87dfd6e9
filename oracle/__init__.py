"""fp64 CPU oracle for block-sparse masked attention (test infrastructure).

THIS PACKAGE IS TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT. Only three
places may import, call or execute it:

* ``tests/``;
* ``__graft_entry__.smoke()``;
* the ``cpu_baseline`` and ``--impl reference`` legs of ``bench.py``.

The CUDA path in ``block_sparse_masked_tile_b200`` neither imports it nor
shares any code, table or helper with it. The two sides share only the
seeded input generators in ``workloads``.

What it computes is the plain definition of each operation:

* ``masks.dense_mask`` evaluates a mask tree element by element.
  Sources: the tensorplay.nn.attention page (create_block_mask mask_mod,
  noop_mask, and_masks, or_masks, causal example), the L-GATr page
  ("Why care about Attention Kernels?": block-diagonal, sliding window,
  PrefixLM) and the transformerlab page (registry table: "sink").
* ``block_mask.create_block_mask`` classifies each 128x128 tile by counting
  allowed in-range elements (tensorplay.nn.attention page, BlockMask
  "Basics" and "Details" items 1-2).
* ``attention.flex_attention`` builds the full score matrix in fp64. It
  applies score_mod before the softmax (attention-gym page, "A gallery that
  grew into a toolkit"), sets masked scores to -inf and takes the softmax.
  A row with no allowed key gives output 0 and lse = -inf.
* ``backward.flex_attention_backward`` takes the gradients of
  sum(out * dout) with respect to q, k and v through the same steps in fp64
  (FlagAttention page, "Operator overview": forward and backward with GQA;
  tensorplay.nn.attention page, BlockMask "Details" items 3-4: dK and dV walk
  the mask along the query dimension).

Parity: every function here is pinned by tests in ``tests/test_oracle_*.py``
against closed forms, library routines on special cases and invariants. The
score_mod values are pinned only by closed-form cases (ALiBi on a constant
key, a soft-cap worked example built on tanh(1)).
"""
from . import attention, block_mask, masks  # noqa: F401
