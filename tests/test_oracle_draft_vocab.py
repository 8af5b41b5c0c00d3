"""Pins of the oracle's reduced draft vocabulary (VocabTrim / FR-Spec / SpecVocab,
aitangshan.cn walkthrough sections 1 and 3.2): the draft head's LM head keeps
the target's rows of a token subset, its distribution is the softmax over that
subset, and every drafted token belongs to it.

* restriction: the reduced head's logits are the full head's logits at the kept
  columns;
* top-k: the reduced top-k equals brute force over the full logits restricted
  to the subset, as token ids;
* the whole vocabulary as the subset reproduces the full head exactly;
* draft tree: every node's token is in the subset, and a depth-1 node's value
  is the log-softmax over the subset (not over the whole vocabulary) of the
  root's draft logits at its token; a mutation that normalises over the whole
  vocabulary fails this.
"""

import numpy as np
import pytest

import synth
from oracle import OracleDraftHead
from oracle import draft as D
from oracle.draft import top_k_rows


@pytest.fixture(scope="module")
def setup():
    d = synth.SMALL_BF16
    host = synth.weights_to_host(synth.model_weights(d, seed=0))
    dw = synth.draft_head_weights(d, seed=6)
    dhost = {"fc_fuse": synth.tensor_to_host(dw["fc_fuse"]), "fc_in": synth.tensor_to_host(dw["fc_in"]),
             "final_norm": synth.tensor_to_host(dw["final_norm"]),
             "layer": {k: synth.tensor_to_host(v) for k, v in dw["layer"].items()}}
    ids = synth.draft_vocab_ids(d.vocab, 1500)
    full = OracleDraftHead(d, host, dhost)
    red = OracleDraftHead(d, host, dhost, vocab_ids=ids)
    P = 40
    feats = synth.tensor_to_host(synth.draft_features(P, d.hidden, seed=31))
    toks = synth.prefix_tokens(d.vocab, P, stream=31)
    seq = full.prefill(feats, toks)
    return d, host, dhost, ids, full, red, seq


def _step(head, seq, d):
    shape = synth.tree_from_widths((4, 3, 2), stream=2)
    nf = synth.tensor_to_host(synth.draft_features(shape.n, d.hidden, seed=32))
    nt = synth.prefix_tokens(d.vocab, shape.n, stream=32)
    return head.step_topk(seq, nf, nt, shape.parents, k=10)


def test_reduced_logits_are_the_full_logits_at_the_kept_columns(setup):
    d, host, dhost, ids, full, red, seq = setup
    _, _, lf = _step(full, seq, d)
    _, _, lr = _step(red, seq, d)
    assert lr.shape == (lf.shape[0], len(ids))
    np.testing.assert_allclose(lr, lf[:, ids], rtol=0, atol=1e-12)


def test_reduced_topk_is_brute_force_over_the_subset(setup):
    d, host, dhost, ids, full, red, seq = setup
    ti, tv, _ = _step(red, seq, d)
    _, _, lf = _step(full, seq, d)
    for r in range(lf.shape[0]):
        sub = lf[r, ids]
        order = sorted(range(len(ids)), key=lambda j: (-sub[j], ids[j]))[:10]
        assert list(ti[r]) == [int(ids[j]) for j in order]
        np.testing.assert_allclose(tv[r], sub[order], atol=1e-12)
    assert np.all(np.isin(ti, ids))


def test_whole_vocabulary_subset_is_the_full_head(setup):
    d, host, dhost, ids, full, red, seq = setup
    same = OracleDraftHead(d, host, dhost, vocab_ids=np.arange(d.vocab))
    a = _step(same, seq, d)
    b = _step(full, seq, d)
    assert np.array_equal(a[0], b[0]) and np.allclose(a[1], b[1], atol=0) and np.allclose(a[2], b[2], atol=0)


def _root_values(head, seq, d, lse_fn):
    g = synth.tensor_to_host(synth.draft_features(1, d.hidden, seed=33))
    g_root = head.fuse(g)[0]
    tree = D.build_draft_tree(head, seq, g_root, 17, steps=2, topk=4, total=6)
    logits, _ = head.step_g(seq, g_root[None, :], [17], [-1])
    lsm = logits[0] - lse_fn(logits)[1][0]
    return tree, lsm


def test_draft_tree_over_the_subset(setup):
    d, host, dhost, ids, full, red, seq = setup
    tree, lsm = _root_values(red, seq, d, D.log_softmax_rows)
    assert np.all(np.isin(tree.tokens[1:], ids))
    pos = {int(t): j for j, t in enumerate(ids)}
    depth1 = [i for i in range(1, len(tree.parents)) if tree.parents[i] == 0]
    assert depth1
    for i in depth1:
        assert abs(tree.values[i] - lsm[pos[int(tree.tokens[i])]]) < 1e-12


def test_mutation_full_vocabulary_normalisation_is_caught(setup):
    d, host, dhost, ids, full, red, seq = setup
    tree, lsm = _root_values(red, seq, d, D.log_softmax_rows)
    # the same tree's values normalised over the whole vocabulary instead of the subset
    _, _, lf = _step(full, seq, d)
    g = synth.tensor_to_host(synth.draft_features(1, d.hidden, seed=33))
    g_root = full.fuse(g)[0]
    logits_full, _ = full.step_g(seq, g_root[None, :], [17], [-1])
    wrong = logits_full[0] - D.log_softmax_rows(logits_full)[1][0]
    i = [i for i in range(1, len(tree.parents)) if tree.parents[i] == 0][0]
    assert abs(tree.values[i] - wrong[int(tree.tokens[i])]) > 1e-6
