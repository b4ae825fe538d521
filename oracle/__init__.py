"""fp64 CPU oracle for cube-routed block-sparse attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code with
the CUDA library and imports nothing from it; the two meet only through the
seeded inputs drawn by ``synth``.

Every function is a plain restatement of the method as the pages define it, in
float64, with numpy matmuls and sorts as the only library steps:

* cube layout .......... VSA page, "Cube Partitioning and Token Re-Indexing";
                         VSA2 page, section 2.2 "Permutation" and "Kernel Implementation" (padding)
* pooling, block scores  SpargeAttention2 page, "Block-Pooled Attention for Efficient
                         Mask Construction", steps 2-3
* Top-k / Top-p / union  SpargeAttention2 page, "The Hybrid Top-k+Top-p Masking Rule",
                         equation 9 and "Definition of the two component selectors"
* index lists .......... VSA page, "Kernel Implementation" (coarse-stage kernel writes
                         contiguous arrays of block indices)
* masked attention ..... SpargeAttention2 page, "Kernel Implementation of the Hybrid-Masked
                         Block-Sparse Attention" (the oracle computes the same softmax
                         non-online, two-pass); VSA2 page section 2.1 (softmax(S + M) V)
* backward ............. textbook derivative of softmax(S + M) V with the mask M held
                         constant (VSA2 page section 2.1: the router output M carries
                         no gradient)
* error decomposition .. SpargeAttention2 page, equation 8
* parity rule ......... tie rows at the k / p boundary (module ``parity``)
* coarse branch, gate .. VSA page, "Big-Picture Architecture" and "Gated Combination";
                         VSA2 page section 2.2, "Coarse Branch" and the gate equation
                         (module ``coarse``)

Parity pinning: every function here is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_*.py`` against worked numbers printed on the pages, closed
forms, brute force and independent library routines (torch SDPA in float64).
"""
from .attention import (  # noqa: F401
    CubeLayout, cube_layout, tile, untile, pool_cubes, block_scores, row_softmax,
    descending_order, topk_ids, topp_count, topp_ids, hybrid_ids, route_head, RouterTrace,
    attention_forward_head, attention_backward_head, dense_attention_head,
    e4m3_decode, dequantize_rows, eq8_error_terms, block_grid_shape, vsa_sparsity,
    topk_from_fraction,
)
from . import blocks128, parity, rope, vsa2_router  # noqa: F401
from .coarse import (  # noqa: F401
    coarse_forward_head, repeat_cubes, gated_forward_head, gated_backward_head,
)
