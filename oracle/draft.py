"""Float64 EAGLE-3 draft-head step over a draft tree (test infrastructure).

Follows the draft-stage description of the kuma.akvtc.cn summary of "EAGLE-3:
Scaling up Inference Acceleration of Large Language Models via Training-Time
Test": the target's low, mid and high features l, m, h (k each) are
concatenated to 3k and reduced by one FC layer to the fused feature g (k); g is
concatenated with the embedding e of the token one step ahead and reduced by a
second FC layer to k; one decoder layer turns that into a; the target's LM
head maps a to the draft distribution.  Readings where the page is silent:
concatenation orders [l|m|h] and [g|e]; e comes from the target's embedding
table; the decoder layer is a pre-norm Llama layer of the target's shape with
its own prefix K/V; a final RMSNorm precedes the LM head; the tree nodes
attend to the draft prefix and to their ancestors, as in verification.

Parity unpinned by the pages beyond these definitions: the pages give no
numbers for the draft head.
"""

from __future__ import annotations

import dataclasses
from typing import List, Sequence

import numpy as np

from .model import OracleModel, rms_norm, to_f64
from .tree import ancestor_matrix, tree_meta


@dataclasses.dataclass
class DraftSeq:
    k: np.ndarray  # [len][Hkv][hd]
    v: np.ndarray

    @property
    def length(self) -> int:
        return int(self.k.shape[0])


def top_k_rows(logits: np.ndarray, k: int):
    """Top-k per row ordered by (value descending, index ascending)."""
    idx = np.empty((logits.shape[0], k), np.int64)
    val = np.empty((logits.shape[0], k), np.float64)
    cols = np.arange(logits.shape[1])
    for r in range(logits.shape[0]):
        order = np.lexsort((cols, -logits[r]))[:k]
        idx[r] = order
        val[r] = logits[r, order]
    return idx, val


class OracleDraftHead:
    def __init__(self, dims, target_weights: dict, draft_weights: dict):
        self.d = dims
        # a one-layer model that reuses the generic decoder layer; its embed / lm_head
        # entries are the target's (the draft head has no table of its own)
        self.layer_model = OracleModel(dims, {
            "embed": target_weights["embed"],
            "lm_head": target_weights["lm_head"],
            "final_norm": draft_weights["final_norm"],
            "layers": [draft_weights["layer"]],
        })
        self.fc_fuse = draft_weights["fc_fuse"]
        self.fc_in = draft_weights["fc_in"]

    def input_rows(self, feats: np.ndarray, tokens: Sequence[int]) -> np.ndarray:
        """feats [n][3][k] (storage format) and tokens [n] -> decoder input [n][k]."""
        n = feats.shape[0]
        lmh = to_f64(feats).reshape(n, 3 * self.d.hidden)      # [l|m|h]
        g = lmh @ to_f64(self.fc_fuse).T                        # fused feature g
        e = self.layer_model.embed(tokens)                      # embedding of the token one step ahead
        return np.concatenate([g, e], axis=1) @ to_f64(self.fc_in).T

    def prefill(self, feats: np.ndarray, tokens: Sequence[int]) -> DraftSeq:
        T = feats.shape[0]
        x = self.input_rows(feats, tokens)
        vis = np.tril(np.ones((T, T), bool))
        _, k, v = self.layer_model.layer_forward(0, x, np.arange(T), None, None, vis)
        return DraftSeq(k, v)

    def step_logits(self, seq: DraftSeq, feats: np.ndarray, tokens: Sequence[int], parents: Sequence[int]):
        depth, _ = tree_meta(parents)
        P = seq.length
        x = self.input_rows(feats, tokens)
        a, _, _ = self.layer_model.layer_forward(0, x, P + depth, seq.k, seq.v, ancestor_matrix(parents))
        return self.layer_model.lm_logits(a)

    def step_topk(self, seq: DraftSeq, feats, tokens, parents, k: int = 10):
        logits = self.step_logits(seq, feats, tokens, parents)
        idx, val = top_k_rows(logits, k)
        return idx, val, logits
