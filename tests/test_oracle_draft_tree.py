"""Pins of the oracle's multi-step drafting and dynamic draft tree.

* The worked example of the draft-stage description ("EAGLE-3: Scaling up
  Inference Acceleration of Large Language Models via Training-Time Test"):
  step 1 feeds the fused target feature with the embedding of the next token,
  later steps feed the draft's own output a of the previous row.  Written out
  as a causal recompute (greedy_draft_chain), it must equal the tree builder
  with top-k 1 (the tree degenerates to a chain).
* One step: the tree is the root's top-k.
* Brute force: with top-k equal to the vocabulary every path of depth <= 2 is
  offered; the chosen nodes must be the `total` best paths by the sum of
  log-probabilities computed path by path with greedy_draft_chain's recompute.
* Invariants of any build: parents before children, values non-increasing along
  paths, and no offer left out with a value above a chosen one.
"""

import dataclasses

import numpy as np
import pytest

import synth
from oracle import OracleModel
from oracle.draft import (OracleDraftHead, build_draft_tree, greedy_draft_chain, log_softmax_rows, top_k_rows)

DIMS = synth.ModelDims(1, 64, 2, 1, 32, 96, 16, 1e-5, 10000.0, "f32")


def _host(t):
    return synth.tensor_to_host(t)


@pytest.fixture(scope="module")
def head():
    tw = synth.weights_to_host(synth.model_weights(DIMS, seed=0))
    tw["lm_head"] = (tw["lm_head"] * 60.0).astype(np.float32)  # peaky draft distributions: no near-ties
    dw = synth.draft_head_weights(DIMS, seed=6)
    dh = {"fc_fuse": _host(dw["fc_fuse"]), "fc_in": _host(dw["fc_in"]), "final_norm": _host(dw["final_norm"]),
          "layer": {k: _host(v) for k, v in dw["layer"].items()}}
    h = OracleDraftHead(DIMS, tw, dh)
    rng = np.random.default_rng(3)
    P = 9
    feats = rng.normal(size=(P, 3, DIMS.hidden)).astype(np.float32)
    seq = h.prefill(feats, rng.integers(0, DIMS.vocab, size=P))
    g_root = h.fuse(rng.normal(size=(1, 3, DIMS.hidden)).astype(np.float32))[0]
    return h, seq, g_root


def _path_logprob(h, seq, g_root, root, path_tokens):
    """Sum of draft log-probabilities of path_tokens after the root, by causal recompute."""
    P = seq.length
    toks = [root]
    gs = [g_root]
    total = 0.0
    for t in path_tokens:
        T = len(toks)
        x = h.rows_from_g(np.stack(gs), toks)
        a, _, _ = h.layer_model.layer_forward(0, x, P + np.arange(T), seq.k, seq.v, np.tril(np.ones((T, T), bool)))
        lp, _ = log_softmax_rows(h.layer_model.lm_logits(a[-1:]))
        total += lp[0, t]
        toks.append(int(t))
        gs.append(a[-1])
    return total


def test_top1_tree_is_the_greedy_draft_chain(head):
    h, seq, g_root = head
    chain = greedy_draft_chain(h, seq, g_root, 5, 6)
    tree = build_draft_tree(h, seq, g_root, 5, steps=6, topk=1, total=6)
    assert list(tree.tokens[1:]) == chain
    assert list(tree.parents) == [-1, 0, 1, 2, 3, 4, 5]


def test_one_step_gives_the_root_top_k(head):
    h, seq, g_root = head
    tree = build_draft_tree(h, seq, g_root, 7, steps=1, topk=5, total=5)
    logits, _ = h.step_g(seq, g_root[None, :], [7], [-1])
    idx, _ = top_k_rows(logits, 5)
    assert list(tree.tokens[1:]) == list(idx[0]) and list(tree.parents[1:]) == [0] * 5


def test_exhaustive_two_levels_match_brute_force(head):
    h, seq, g_root = head
    V = DIMS.vocab
    tree = build_draft_tree(h, seq, g_root, 3, steps=2, topk=V, total=20)
    paths = [(a,) for a in range(V)] + [(a, b) for a in range(V) for b in range(V)]
    vals = {p: _path_logprob(h, seq, g_root, 3, p) for p in paths}
    # the tree's chosen paths and their values
    chosen = {}
    for i in range(1, len(tree.tokens)):
        p, j = [], i
        while j > 0:
            p.append(int(tree.tokens[j]))
            j = int(tree.parents[j])
        chosen[tuple(reversed(p))] = tree.values[i]
    ranked = sorted(paths, key=lambda p: (-vals[p], len(p)))
    assert set(chosen) == set(ranked[:20])
    for p, v in chosen.items():
        assert abs(v - vals[p]) < 1e-9


def test_invariants_of_a_build(head):
    h, seq, g_root = head
    tree = build_draft_tree(h, seq, g_root, 11, steps=4, topk=4, total=12)
    n = len(tree.tokens)
    assert n == 13 and tree.parents[0] == -1
    for i in range(1, n):
        assert 0 <= tree.parents[i] < i
        assert tree.values[i] <= tree.values[tree.parents[i]] + 1e-12
    # no offer left out beats a chosen node
    cut = min(tree.values[1:])
    n_above = sum(1 for c in tree.offered if c[0] > cut + 1e-12)
    assert n_above <= n - 2
    # each value is the sum of log-probabilities along the node's path (causal recompute)
    for i in range(1, n):
        p, j = [], i
        while j > 0:
            p.append(int(tree.tokens[j]))
            j = int(tree.parents[j])
        np.testing.assert_allclose(tree.values[i], _path_logprob(h, seq, g_root, 11, list(reversed(p))),
                                   rtol=0, atol=1e-9)
