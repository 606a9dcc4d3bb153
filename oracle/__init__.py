"""CPU oracle for the tree-verify hot path -- TEST INFRASTRUCTURE, not part of the product.

Plain, slow, obviously correct numpy code in float64 that restates what the JetFlow/JetSpec pages
define: tree-causal attention over a paged KV cache (``tree_attention``), best-first tree
construction by cumulative draft log-probability under a budget (``build_tree``), the greedy
acceptance walk (``accept``), the commit of the accepted path's K/V into the cache
(``commit_kv``), the write of the tree tokens' rotated K/V into the cache (``tree_kv_append``),
tree attention over an 8-bit E4M3 cache (``tree_attention_fp8``), and the round-by-round best-first
expansion from per-node (path-conditioned) draft logits (``expand_frontier``, ``grow_tree``).  It shares no code with the CUDA library and never imports it.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py`` may import this package.  The product path (the ``libjf.so`` C-ABI and its Python
binding) never calls it and fails loudly when the CUDA library is missing.

Sources (page titles; the pages print no code):
  [JF]  "JetFlow: Breaking the Scaling Ceiling of Speculative Decoding with Parallel Tree Drafting"
        (gist.science explainer, Chinese and French versions), technical summary sections 1-5.
  [JS]  "JetSpec" paper page (Hugging Face mirror), abstract.

Pin status: every function here is pinned by tests under ``tests/test_oracle_*.py`` against closed
forms, library routines or brute force (see each module's header).
"""
from .tree_attention import ancestor_sets, visible_slots, tree_attention  # noqa: F401
from .build_tree import row_stats, topk_tokens, build_tree  # noqa: F401
from .accept import accept  # noqa: F401
from .commit_kv import commit_kv  # noqa: F401
from .kv_append import rope, tree_kv_append  # noqa: F401
from .fp8_kv import e4m3_decode, e4m3_encode, quantize_cache, tree_attention_fp8  # noqa: F401
from .frontier import FrontierState, expand_frontier, grow_tree, start_tree  # noqa: F401
