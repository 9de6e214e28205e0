"""fp64 CPU oracle for the separator-sparse attention path and the SepCache decode step.

TEST INFRASTRUCTURE ONLY. This package is the checker that the CUDA library is
compared against. Only `tests/`, `__graft_entry__.smoke()` and the CPU-baseline
leg of `bench.py` may import it. It shares no code with the CUDA library
(`kv_cache_compression_sep_b200/`) and imports nothing from it; the library never
imports this package.

Sources (web pages about SepLLM, cited by page title and section):

* [AS] "SepLLM: Accelerate Large Language Models by Compressing One Segment into
  One Separator" (atlas.scime.ai summary), sections "Approach", "Key results",
  "Measured effects reported in the paper".
* [BD] "How SepLLM reorchestrates the language model for speed and efficiency"
  (beiduofen.top article), sections "SepLLM's Architecture: Composing Efficiency"
  (the four cache blocks and the formula O = M(A, V, M_b)) and "The Mechanics of
  Compression: Why Separators Work" (training-from-scratch setting).
* [SP] SepLLM project card (sourcepulse.org), section "Limitations & Caveats"
  (positional-encoding shifting in streaming).

Every function is pinned by a `-m "not gpu"` test in `tests/test_oracle_*.py`
against something other than itself (hand-derived worked examples under
`tests/golden/`, closed forms, library routines on special cases, brute force,
finite differences). No function here is "parity unpinned".
"""

from .sepattn_ref import (  # noqa: F401
    anchor_flags,
    keep_mask,
    keep_block,
    tile_class,
    kept_pairs,
    kept_pairs_closed_form,
    mask_build,
    attn_fwd,
    attn_bwd,
    kept_index_set,
    attn_fwd_rows,
    attn_bwd_sampled,
)
from .sepcache_ref import (  # noqa: F401
    SepCacheSim,
    rope_rotate,
    decode_attention,
)
