"""Oracle for blockwise packed causal RoPE attention (fp64, CPU).

TEST INFRASTRUCTURE ONLY. This package is the slow, obviously-correct
definition that the CUDA path is checked against. Only the test suite
(``tests/``), ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import it. The CUDA path
(``long_context_blockwise_causal_b200``) never imports it, and it never
imports the CUDA path: the two share no code.

What it computes, and where the pages fix it (page titles abbreviated as
in the design notes):

* causal autoregression over text and vision tokens --
  "LWM：突破 100 万 Token 的开源大模型", 概述; "Inside Large World Model",
  Core Architecture;
* masked sequence packing: a token attends only inside its own packed
  example -- "LWM：突破 100 万 Token 的开源大模型", 概述 contribution (b);
  "[论文解读] World Model on Million-Length Video And Language With Blockwise
  RingAttention", 提出的方法;
* RoPE whose theta is scaled with the context length -- "[论文解读] World
  Model on Million-Length Video ...", 提出的方法; the theta values in
  "LWM：突破 100 万 Token 的开源大模型", 脚本运行说明;
* blockwise attention with an online softmax as an exact re-organisation of
  dense attention -- "LWM：突破 100 万 Token 的开源大模型", 配置参数
  (scan_attention, query/key chunk sizes); "开源巨兽LWM：如何用RingAttention
  撬动百万Token多模态世界", 3.1 and 3.2; "Inside Large World Model", Stage I.

Readings where the pages are silent (softmax scale 1/sqrt(D), interleaved
RoPE pairs, theta^(-2k/D) frequencies in fp64, causal mask on token index,
natural-log logsumexp) are listed in the module docstrings that use them.

Modules:
  rope       -- RoPE frequencies, angles and rotation (interleaved pairs and
                the rotate-half layout, with the permutation between them).
  attention  -- dense fp64 forward/backward (row-blocked), sampled rows.
  blockwise  -- CPU online-softmax restatement in ring order (invariance pin).
  ring       -- partial attention over a key block, the log-sum-exp merge and
                a P-device ring run in order (RingAttention).
  classify   -- tile classification (brute force and a counting form).
  ffn        -- the blockwise (chunked) SwiGLU feed-forward network.
"""

from .rope import (  # noqa: F401
    rope_inv_freq, rope_angles, rope_rotate, rope_rotate_half,
    half_to_interleaved, interleaved_to_half,
)
from .attention import (  # noqa: F401
    allowed_mask, attn_fwd, attn_fwd_rows, attn_bwd, attn_bwd_rows,
    attn_bwd_cols, SOFTMAX_SCALE_RULE,
)
from .blockwise import blockwise_fwd  # noqa: F401
from .ring import (  # noqa: F401
    attn_fwd_partial, merge_partials, ring_chunks, ring_fwd, bwd_delta,
    attn_bwd_partial, ring_bwd,
)
from .ffn import (  # noqa: F401
    silu, swiglu_intermediate, swiglu_mlp, blockwise_mlp, silu_grad,
    swiglu_mlp_bwd,
)
from .classify import (  # noqa: F401
    classify_bruteforce, classify_count, classify_cross, visible_key_ranges,
    visible_query_ranges, TILE_EMPTY, TILE_PARTIAL, TILE_FULL,
)
