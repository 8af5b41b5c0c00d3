"""Float64 CPU oracle for EAGLE-3 tree verification.

TEST INFRASTRUCTURE.  Only the test suite, the smoke check in
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package.  The library under ``speculative_decoding_06_b200`` never does;
the two share no code.

What it computes, and where the pages fix it:

* greedy acceptance -- a draft token is accepted iff it equals the target's
  argmax at its parent; scan from the root and stop at the first mismatch;
  emit the accepted tokens plus the target's own token there
  ("EAGLE-3投机解码：树验证器方法", section 验证-接受语义);
* the chain example -- K=5 drafts with 4 right give 5 tokens, 1 right gives 2,
  0 right gives 1 (same page, section 问题);
* tree drafting with ancestor-only attention: the whole tree is verified by one
  target forward in which each token sees only its ancestors (same page,
  section 树draft vs 链draft);
* losslessness: the result equals running the target autoregressively (same
  page, sections 问题 and 验证-接受语义; the kuma.akvtc.cn summary of the
  EAGLE-3 paper, introduction);
* the draft-head feature path: low/mid/high features concatenated to 3k, an FC
  to k, concatenation with the next token's embedding, an FC to k, one
  decoder layer, the target's LM head (kuma.akvtc.cn summary, draft-stage
  description).

The transformer itself (RMSNorm, rotary embeddings, grouped-query attention,
SwiGLU MLP) is the standard Llama decoder, written out in float64.
"""

from .tree import tree_meta, accept_walk, ancestor_matrix, root_paths  # noqa: F401
from .model import (  # noqa: F401
    OracleModel, OracleSeq, oracle_prefill, oracle_tree_logits, oracle_verify,
    oracle_greedy_ar, causal_logits, top2_margin, argmax_fn_for_planting, causal_features, oracle_tree_features,
)
from .draft import OracleDraftHead  # noqa: F401
