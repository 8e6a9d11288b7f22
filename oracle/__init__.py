"""CPU oracle for the sink + window chunk-attention path, the MoBA mask and its backward.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, fp64 restatement of
what the method computes.  Only the test suite, the package smoke check and
the benchmark's CPU-baseline leg may import it; the product path (the C-ABI
library and its Python binding) never does, and the oracle imports nothing of
the product path.  It shares no code with the CUDA side: the only common
module is the seeded input generator (``kv_cache_chunk_ring_b200.workloads``),
which holds no arithmetic of the method.

Sources (web pages; cited by title and section):
  [LWI]  "LingBot-World-Infinity: The Open-Source World Model That Refuses to
         Forget" (repo-explainer.com) -- "The trick: treat video like a causal
         stream" (anchor tokens + recent context, evict old tokens, keep
         anchors) and "How the cache keeps the world alive" (sliding KV cache,
         sink tokens kept at the front, old tokens discarded).
  [IW]   "Infinite Worlds with Versatile Interactions" (agihunt.info) --
         causal-pretraining paragraph (frames conditioned only on the past;
         MoBA = teacher-forcing mask + appended fully bidirectional block;
         causal chunk-wise cross-attention mask) and deployment paragraph
         (dynamic KV-cache scheduler adapting retained history).
  [MF]   "Mix Forcing: Causal Pre-Training via Mixture Attention for
         Interactive World Models" -- "Mix the training modes", "Condition
         each chunk".
  [WiW]  "Westlake AGI Lab's 'World in World' Steers Frozen Video Models" --
         second paragraph: 18 latent-frame slots = 6 anchors + 8 recent + 4
         current; initial observation + recently finalized outputs; temporary
         auxiliary attention blocks for the current chunk, removed once it is
         finalized.
  [RT]   kaarelkaarelson.com/lingbot (LingBot-World 2.0 in real time on one
         RTX 5090) -- setup paragraph (832x464, four denoising steps,
         16-frame chunks) and the step / kernel tables.

Parity status of each function is stated in its module header.  Every
function here is pinned by a CPU test against something other than itself
(closed forms, invariants, brute force on tiny inputs, worked examples).
"""

from .rope import rope3d, rope_positions, axis_of_pair, rope_pairs_default  # noqa: F401
from .cache import CacheModel, visible_frames_closed_form  # noqa: F401
from .attn import attention, masked_attention, attention_bruteforce  # noqa: F401
from .moba import (MobaLayout, block_of, moba_allowed, moba_mask, classify_tiles_mask,  # noqa: F401
                   classify_tiles_blocks, moba_attention_rows, TILE_EMPTY, TILE_PARTIAL,
                   TILE_FULL)
from .rollout import rollout, RolloutResult  # noqa: F401
from .moba_bwd import (attention_bwd_masked, moba_bwd_dense, moba_dq_rows,  # noqa: F401
                       moba_dkdv_keys)
