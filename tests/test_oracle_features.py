"""Pins of the oracle's feature tap: the residual stream between decoder
blocks that EAGLE-3 feeds to its draft head ("EAGLE-3: Scaling up Inference
Acceleration of Large Language Models via Training-Time Test", draft-stage
description: low-, mid- and high-level features of every position, recorded in
prefill and in each verification step).

* against an independent implementation: Hugging Face transformers' Llama
  (float64, eager) returns the same hidden states after 1 and 2 layers, and
  after the last layer its (final-normed) hidden state equals the final
  RMSNorm of the oracle's last tap;
* tree = chain: a tree node's features equal those of a plain causal forward
  over the prefix and the node's root path (ancestor-only attention);
* the verification step returns the features of the root and the accepted
  nodes in path order, and the last tap reproduces those nodes' logits.
"""

import dataclasses

import numpy as np
import pytest
import torch

import synth
from oracle import OracleModel, oracle_prefill, oracle_verify, root_paths
from oracle.model import causal_features, oracle_tree_features, rms_norm, to_f64
from test_oracle_pins import GQA_TINY, HF_ATOL, HF_RTOL, hf_model

GQA3 = dataclasses.replace(GQA_TINY, n_layers=3)


@pytest.fixture(scope="module")
def gqa3():
    w = synth.model_weights(GQA3, seed=0)
    return w, OracleModel(GQA3, synth.weights_to_host(w))


def test_features_match_hf_hidden_states(gqa3):
    w, om = gqa3
    m = hf_model(GQA3, w)
    toks = synth.prefix_tokens(GQA3.vocab, 29, stream=6)
    feats = causal_features(om, toks, (1, 2, 3))
    with torch.no_grad():
        hs = m(torch.tensor([list(toks)]), output_hidden_states=True).hidden_states
    for f, j in enumerate((1, 2)):
        np.testing.assert_allclose(feats[:, f], hs[j][0].numpy(), rtol=HF_RTOL, atol=HF_ATOL)
    final = rms_norm(feats[:, 2], to_f64(om.w["final_norm"]), GQA3.rms_eps)
    np.testing.assert_allclose(final, hs[3][0].numpy(), rtol=HF_RTOL, atol=HF_ATOL)
    # a tap one layer off differs at the library's own precision by orders of magnitude
    assert np.max(np.abs(feats[:, 0] - hs[2][0].numpy())) > 1e3 * HF_ATOL


def test_tree_features_equal_chain_features(gqa3):
    _, om = gqa3
    prompt = synth.prefix_tokens(GQA3.vocab, 18, stream=7)
    seq, _ = oracle_prefill(om, prompt)
    shape = synth.tree_from_widths((3, 3, 2, 2), stream=3)
    rng = np.random.default_rng(8)
    tokens = rng.integers(0, GQA3.vocab, size=shape.n)
    tokens[0] = seq.pending
    _, _, feats = oracle_tree_features(om, seq, tokens, shape.parents, (1, 2, 3))
    for i, path in enumerate(root_paths(shape.parents)):
        ref = causal_features(om, list(prompt) + [int(tokens[j]) for j in path], (1, 2, 3))[-1]
        np.testing.assert_allclose(feats[i], ref, rtol=1e-10, atol=1e-12)


def test_verify_returns_path_features(gqa3):
    _, om = gqa3
    prompt = synth.prefix_tokens(GQA3.vocab, 21, stream=8)
    seq, _ = oracle_prefill(om, prompt)
    shape = synth.tree_from_widths((2, 3, 2), stream=4)
    from oracle import argmax_fn_for_planting
    draws = synth.plant_draws(shape.n, GQA3.vocab, stream=5)
    tokens = synth.plant_tree(shape, seq.pending, 1.0, draws, argmax_fn_for_planting(om, seq))
    _, _, all_feats = oracle_tree_features(om, seq, tokens, shape.parents, (1, 3, 2))
    r = oracle_verify(om, seq, tokens, shape.parents, taps=(1, 3, 2))
    keep = [0] + r["accepted_nodes"]
    assert r["accepted_len"] >= 1
    assert r["features"].shape == (len(keep), 3, GQA3.hidden)
    np.testing.assert_array_equal(r["features"], all_feats[keep])
    np.testing.assert_allclose(om.lm_logits(r["features"][:, 1]), r["logits"][keep], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("bad", [0, 4, -1])
def test_tap_outside_the_layers_is_rejected(gqa3, bad):
    _, om = gqa3
    with pytest.raises(ValueError):
        causal_features(om, [1, 2, 3], (1, bad, 2))
