"""fp64 CPU oracle for LongGen sparse causal attention -- TEST INFRASTRUCTURE.

This package is the checker, not the product. Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it. The product path
(``attention_sink_long_b200``) never imports it, and it imports nothing from
the product: the two share no code, no constants and no helpers. The only
thing both sides use is the seeded input generator in ``synthetic_inputs``,
which holds none of the method's arithmetic.

Source: "A Little Goes a Long Way: Efficient Long Context Training and
Inference with Partial Contexts" (LongGen, arXiv 2410.01485).
  * Abstract, insight 1: the sparse layers keep the initial tokens (attention
    sink), the recent tokens (window attention) and strided token blocks
    (blockwise sparse attention).
  * Abstract, insight 2, and the atlas.scime.ai summary, "Approach": 1/3 of the
    layers keep full attention -- the all-blocks causal special case.
  * atlas.scime.ai summary, "Approach": the sparse patterns use static,
    block-wise access, and the kernel is FlashAttention-2-based, i.e. exact
    softmax attention restricted to that static mask.

The method is exact attention under a static mask, so the oracle is the plain
definition of masked causal softmax attention and its analytic gradient,
evaluated in float64. Every function is pinned by ``tests/test_oracle.py``
against closed forms, library routines (torch SDPA / autograd in float64) or
finite differences; see the pin list in that file.
"""

from .attention import (  # noqa: F401
    INT32_MAX,
    Pattern,
    allowed,
    token_mask,
    block_lists,
    block_lists_t,
    pair_count,
    attention_forward,
    attention_backward,
    attention_rows,
    attention_backward_rows,
    attention_backward_kv_rows,
    decode,
    reduced_cache_rows,
    reduced_cache,
    merge_partials,
)
