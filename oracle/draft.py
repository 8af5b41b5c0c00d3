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

Reduced draft vocabulary (VocabTrim / FR-Spec / SpecVocab in the aitangshan.cn
walkthrough, sections 1 and 3.2: the draft model's output covers a trimmed
vocabulary, which shrinks its search space and LM head): with `vocab_ids` the
draft head's LM head is the target's rows at those token ids (ascending), the
draft distribution is the softmax over that subset, and every drafted token is
one of them.  Verification is unchanged, so the output is still the target's.
Which tokens to keep is a property of a training corpus the pages do not give;
the subset is an input here.

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
    def __init__(self, dims, target_weights: dict, draft_weights: dict, vocab_ids=None):
        """vocab_ids: ascending token ids of a reduced draft vocabulary (None: the whole vocabulary)."""
        self.d = dims
        lm = target_weights["lm_head"]
        self.vocab_ids = None
        if vocab_ids is not None:
            ids = np.asarray(vocab_ids, dtype=np.int64)
            if ids.ndim != 1 or ids.size < 2 or np.any(np.diff(ids) <= 0) or ids[0] < 0 or ids[-1] >= lm.shape[0]:
                raise ValueError("vocab_ids must be strictly increasing token ids")
            self.vocab_ids = ids
            lm = lm[ids]  # the target's LM-head rows of the kept tokens
        # a one-layer model that reuses the generic decoder layer; its embed / lm_head
        # entries are the target's (the draft head has no table of its own)
        self.layer_model = OracleModel(dims, {
            "embed": target_weights["embed"],
            "lm_head": lm,
            "final_norm": draft_weights["final_norm"],
            "layers": [draft_weights["layer"]],
        })
        self.fc_fuse = draft_weights["fc_fuse"]
        self.fc_in = draft_weights["fc_in"]

    def token_of(self, idx):
        """Token ids of draft-vocabulary indices (identity without a reduced vocabulary)."""
        idx = np.asarray(idx, dtype=np.int64)
        return idx if self.vocab_ids is None else self.vocab_ids[idx]

    def fuse(self, feats: np.ndarray) -> np.ndarray:
        """feats [n][3][k] (storage format) -> fused feature g [n][k]."""
        n = feats.shape[0]
        lmh = to_f64(feats).reshape(n, 3 * self.d.hidden)      # [l|m|h]
        return lmh @ to_f64(self.fc_fuse).T

    def rows_from_g(self, g: np.ndarray, tokens: Sequence[int]) -> np.ndarray:
        """feature rows g [n][k] (fused target features, or the draft's own outputs a) and
        tokens [n] -> decoder input [n][k]."""
        e = self.layer_model.embed(tokens)                      # embedding of the token one step ahead
        return np.concatenate([to_f64(g), e], axis=1) @ to_f64(self.fc_in).T

    def input_rows(self, feats: np.ndarray, tokens: Sequence[int]) -> np.ndarray:
        """feats [n][3][k] (storage format) and tokens [n] -> decoder input [n][k]."""
        return self.rows_from_g(self.fuse(feats), tokens)

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

    def step_g(self, seq: DraftSeq, g: np.ndarray, tokens: Sequence[int], parents: Sequence[int]):
        """One step over a tree whose rows carry their feature g directly (fused target
        features or earlier draft outputs).  Returns (logits [n][V], a [n][k]), a being the
        decoder layer's output that the LM head reads (after the final norm) and that later
        steps take in place of g."""
        depth, _ = tree_meta(parents)
        P = seq.length
        x = self.rows_from_g(g, tokens)
        a, _, _ = self.layer_model.layer_forward(0, x, P + depth, seq.k, seq.v, ancestor_matrix(parents))
        return self.layer_model.lm_logits(a), a

    def step_topk(self, seq: DraftSeq, feats, tokens, parents, k: int = 10):
        """Top-k per node as token ids; logits over the draft vocabulary."""
        logits = self.step_logits(seq, feats, tokens, parents)
        idx, val = top_k_rows(logits, k)
        return self.token_of(idx), val, logits


# ---------------------------------------------------------------------------
# multi-step drafting and the dynamic draft tree
# ---------------------------------------------------------------------------

def log_softmax_rows(logits: np.ndarray):
    """(log-probabilities, log-sum-exp) of each row, float64."""
    m = logits.max(axis=1, keepdims=True)
    lse = m[:, 0] + np.log(np.exp(logits - m).sum(axis=1))
    return logits - lse[:, None], lse


def greedy_draft_chain(head: OracleDraftHead, seq: DraftSeq, g_root: np.ndarray, root_token: int, n: int):
    """Greedy multi-step drafting written out as a causal recompute (no tree machinery).

    The draft-stage description's worked example: the first step feeds the target
    feature of the last verified position with the embedding of the token after it;
    from the second step on the draft's own output a of the previous row replaces the
    target feature ("a_I" with "e_do", then "a_do" with "e_it").  Each new token is the
    argmax of the draft distribution at the last row.  Returns the n drafted tokens."""
    P = seq.length
    toks = [int(root_token)]
    gs = [np.asarray(g_root, np.float64)]
    out = []
    for _ in range(n):
        T = len(toks)
        x = head.rows_from_g(np.stack(gs), toks)
        vis = np.tril(np.ones((T, T), bool))
        a, _, _ = head.layer_model.layer_forward(0, x, P + np.arange(T), seq.k, seq.v, vis)
        logits = head.layer_model.lm_logits(a[-1:])
        t = int(head.token_of(np.argmax(logits[0])))
        out.append(t)
        toks.append(t)
        gs.append(a[-1])
    return out


@dataclasses.dataclass
class DraftTree:
    tokens: np.ndarray   # [total + 1], root first, ordered by depth then rank
    parents: np.ndarray  # [total + 1], parents[0] = -1, parents[i] < i
    values: np.ndarray   # [total + 1] cumulative log-probability of each node (root 0)
    offered: list        # every candidate offered: (value, depth, order, parent node, token)


def build_draft_tree(head: OracleDraftHead, seq: DraftSeq, g_root: np.ndarray, root_token: int,
                     steps: int = 8, topk: int = 10, total: int = 60) -> DraftTree:
    """Dynamic draft tree from the draft head's own confidence.

    The pages: EAGLE-2 takes the draft model's confidence as an estimate of the
    acceptance rate and shapes the draft tree with it; EAGLE-3 drafts several steps,
    feeding its own output a in place of the target feature from the second step on;
    the evaluated setting uses 8 drafting steps, 60 draft tokens and top-k 10.
    Reading taken for the steps they leave open:

    * a node's value is the sum of the log-probabilities (full-vocabulary softmax of the
      draft logits at its parent) along its root path; the root's value is 0;
    * step t runs the draft head over the tree built so far: the root's feature is the
      fused target feature g_root, every other node's the output a of its parent (every
      parent joined, and had its a computed, in an earlier step); each node that joined
      last (the root at t = 0) offers its top-k tokens as children; the top-k offers by
      value, ties to the earlier offer, join the tree;
    * after the last step every offer competes, joined or not: the `total` best by value,
      ties to the lower depth and then to the earlier offer, form the tree with the root.
      A chosen node's ancestors have values at least as high and lower depths, so the
      chosen set is closed under ancestors.
    """
    tok, par, val, dep = [int(root_token)], [-1], [0.0], [0]
    frontier = [0]
    a_of = {}
    offered = []
    order = 0
    node_of_offer = {}
    for _ in range(steps):
        n = len(tok)
        g = np.stack([np.asarray(g_root, np.float64) if i == 0 else a_of[par[i]] for i in range(n)])
        logits, a = head.step_g(seq, g, tok, par)
        for i in range(n):
            a_of.setdefault(i, a[i])
        lp, _ = log_softmax_rows(logits)
        offers = []
        for f in frontier:
            idx, _ = top_k_rows(logits[f:f + 1], topk)
            for t in idx[0]:
                offers.append((val[f] + lp[f, t], dep[f] + 1, order, f, int(head.token_of(t))))
                order += 1
        offered.extend(offers)
        frontier = []
        for v, d_, o, f, t in sorted(offers, key=lambda c: (-c[0], c[2]))[:topk]:
            tok.append(t)
            par.append(f)
            val.append(v)
            dep.append(d_)
            frontier.append(len(tok) - 1)
            node_of_offer[o] = len(tok) - 1
    best = sorted(offered, key=lambda c: (-c[0], c[1], c[2]))[:total]
    best.sort(key=lambda c: (c[1], -c[0], c[2]))  # by depth, so parents come first
    out_tok, out_par, out_val = [tok[0]], [-1], [0.0]
    pos = {0: 0}  # joined node -> output index
    for v, d_, o, f, t in best:
        if f not in pos:
            raise AssertionError("a chosen offer whose parent was not chosen")
        out_tok.append(t)
        out_par.append(pos[f])
        out_val.append(v)
        if o in node_of_offer:
            pos[node_of_offer[o]] = len(out_tok) - 1
    return DraftTree(np.array(out_tok, np.int64), np.array(out_par, np.int64), np.array(out_val), offered)
