"""Oracle for Recursive Sparse Attention (RecSA): a plain, slow, float64 CPU
restatement of what the method computes.

This package is TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference leg of ``bench.py`` may import it. The product
path (the CUDA library and its Python binding) never imports, calls or links it,
and it shares no code, table or constant with that path.

Sources (web pages, cited by title and section):
  * "Recursive Sparse Attention: Million-Token Length Extrapolation at
    Logarithmic Cost", abstract -- the method statement: a tree over the KV
    cache, one key and one mean-pooled value per node, one pooler per layer
    shared by all levels, at most k candidates kept per level, summaries of
    unselected candidates in one softmax with the exact tokens, RoPE position =
    index among the candidates of the level.
  * "Subquadratic Attention with a Hierarchical Tree-Structured Indexer" (ZHA),
    Figure 3 caption (recursive pooling against reference queries, top-down
    descent) and Table VIII (only full nodes exist: n_l = floor(T / C^l)).
    Its routing variant (top-p expansion, attention over the reached leaves)
    is in ``zha.py``; its Table IX convention of a selection per KV group is
    applied to RecSA in ``group.py``; several reference queries per pooler
    (Figure 3 caption) are in ``multiref.py``; low-precision router keys
    (Figure 16 caption) in ``lowprec.py``.
  * "Efficient Sequence Modeling, Issue 13", highlights and editor's note on
    RecSA (normalisation shared with exact tokens; one pooler for selection and
    summary keys).

Parity status of each function is stated in its docstring. The one part with
no external pin is marked "parity unpinned" in ``recsa.py``.
"""

from .recsa import (  # noqa: F401
    Geometry,
    level_counts,
    visible_counts,
    pool_keys,
    build_tree,
    node_summary,
    LazyTree,
    FullTree,
    rope_cos_sin,
    rope_rotate,
    traverse_and_attend,
    closed_form_counts,
)
from .dense import dense_causal_attention  # noqa: F401
from .zha import top_p_prefix, zha_route_and_attend  # noqa: F401
from .group import group_select, group_traverse_and_attend  # noqa: F401
from .multiref import LazyMultiTree, MultiTree, build_tree_multi  # noqa: F401
from .lowprec import (build_tree_fp8, build_tree_fp8_multi, dequantize_row,  # noqa: F401
                      e4m3_decode, e4m3_round, near_rounding_boundary, quantize_row,
                      e2m1_decode, e2m1_round, quantize_row_nvfp4, build_tree_nvfp4_multi)
